"""fp64 CPU oracle of the fused MoE forward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The product path (the CUDA
library and its Python binding) never imports it, and it imports nothing
from the product.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, OpenMP
over independent tokens); this module only compiles it with gcc, loads it
with ctypes and converts numpy arrays.  See the header of ``moe_oracle.c``
for what each function computes and which page it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIBS: dict[int, ctypes.CDLL] = {}


def lib_path(mutation: int = 0) -> str:
    name = "liboracle.so" if mutation == 0 else f"liboracle_mut{mutation}.so"
    return os.path.join(_BUILD, name)


def build(mutation: int = 0, force: bool = False) -> str:
    """Compile moe_oracle.c (optionally with a planted mistake) with gcc."""
    out = lib_path(mutation)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
        return out
    os.makedirs(_BUILD, exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
           f"-DORACLE_MUTATION={int(mutation)}", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _load(mutation: int = 0) -> ctypes.CDLL:
    if mutation in _LIBS:
        return _LIBS[mutation]
    lib = ctypes.CDLL(build(mutation))
    P = ctypes.c_void_p
    i64, i32 = ctypes.c_int64, ctypes.c_int
    lib.oracle_route.argtypes = [P, i64, i32, i32, i32, P, P]
    lib.oracle_permute.argtypes = [P, i64, i32, P, P]
    lib.oracle_moe_token_loop.argtypes = [P, P, P, P, P, i64, i64, i64, i32, i32, P, i64, P]
    lib.oracle_moe_expert_loop.argtypes = [P, P, P, P, P, i64, i64, i64, i32, i32, P]
    lib.oracle_moe_token_loop_ex.argtypes = [P, P, P, P, P, i32, P, P, i64, i64, i64, i32, i32,
                                             P, i64, P]
    lib.oracle_moe_expert_loop_ex.argtypes = [P, P, P, P, P, i32, P, P, i64, i64, i64, i32, i32,
                                              P]
    lib.oracle_moe_token_loop_fp8.argtypes = [P, P, P, P, P, i64, P, P, i64, i64, i64, i32, i32,
                                              P, i64, P]
    lib.oracle_moe_expert_loop_fp8.argtypes = [P, P, P, P, P, i64, P, P, i64, i64, i64, i32,
                                               i32, P]
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_double.restype = ctypes.c_double
    for f in ("oracle_route", "oracle_permute", "oracle_moe_token_loop",
              "oracle_moe_expert_loop", "oracle_moe_token_loop_ex", "oracle_moe_expert_loop_ex",
              "oracle_moe_token_loop_fp8", "oracle_moe_expert_loop_fp8",
              "oracle_max_threads", "oracle_mutation"):
        getattr(lib, f).restype = ctypes.c_int
    lib.oracle_set_threads.argtypes = [i32]
    lib.oracle_set_threads.restype = None
    _LIBS[mutation] = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _bf16_bits(a) -> np.ndarray:
    """Accept a torch bf16 tensor or a uint16 array of bf16 bit patterns."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        a = a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns (uint16) or a torch bf16 tensor")
    return a


def max_threads(mutation: int = 0) -> int:
    return _load(mutation).oracle_max_threads()


def set_threads(n: int, mutation: int = 0) -> None:
    _load(mutation).oracle_set_threads(int(n))


def route(logits, k: int, renorm: bool, mutation: int = 0):
    """Softmax + top-k (+ renormalisation) of fp32 logits [T, E].

    Returns (ids int32 [T, k], weights float64 [T, k])."""
    lg = np.ascontiguousarray(np.asarray(logits, dtype=np.float32))
    T, E = lg.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    rc = _load(mutation).oracle_route(_ptr(lg), T, E, k, int(bool(renorm)), _ptr(ids), _ptr(w))
    if rc != 0:
        raise ValueError(f"oracle_route rejected T={T} E={E} k={k}")
    return ids, w


def permute(ids, E: int, mutation: int = 0):
    """Stable counting sort of the flat (token, slot) indices by expert.

    Returns (sorted_rows int32 [n] with -1 past offsets[E], offsets int32 [E+1])."""
    flat = np.ascontiguousarray(np.asarray(ids, dtype=np.int32).reshape(-1))
    n = flat.shape[0]
    rows = np.empty(max(n, 1), np.int32)
    offs = np.empty(E + 1, np.int32)
    rc = _load(mutation).oracle_permute(_ptr(flat), n, E, _ptr(rows), _ptr(offs))
    if rc != 0:
        raise ValueError("oracle_permute rejected its arguments")
    return rows[:n], offs


def _forward_args(hidden, w1, w2, topk_w, ids):
    hb, w1b, w2b = _bf16_bits(hidden), _bf16_bits(w1), _bf16_bits(w2)
    T, H = hb.shape
    E, twoI, H1 = w1b.shape
    I = twoI // 2
    if H1 != H or twoI != 2 * I or w2b.shape != (E, H, I):
        raise ValueError("shape mismatch between hidden, w1 [E,2I,H] and w2 [E,H,I]")
    tw = np.ascontiguousarray(np.asarray(topk_w, dtype=np.float64))
    ti = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    k = ti.shape[1] if ti.ndim == 2 else 1
    if tw.shape != (T, k) or ti.shape != (T, k):
        raise ValueError("topk weights/ids must both be [T, k]")
    return hb, w1b, w2b, tw, ti, T, H, I, E, k


# activations of the 0.13.2 page's activation_fn
ACTS = {"silu": 0, "gelu": 1, "swigluoai": 2}


def _variant_args(act, b1, b2, E, H, I):
    if act not in ACTS:
        raise ValueError(f"unknown activation {act!r}")
    b1a = b2a = None
    if b1 is not None:
        b1a = np.ascontiguousarray(np.asarray(b1, dtype=np.float32).reshape(E, 2 * I))
    if b2 is not None:
        b2a = np.ascontiguousarray(np.asarray(b2, dtype=np.float32).reshape(E, H))
    return ACTS[act], b1a, b2a


def moe_token_loop(hidden, w1, w2, topk_w, ids, rows=None, mutation: int = 0,
                   act: str = "silu", b1=None, b2=None):
    """Formulation A (per-token loop).  Returns float64 [T, H], or
    [len(rows), H] for the listed tokens only.  act: "silu", "gelu" (tanh
    form) or "swigluoai"; b1 fp32 [E, 2I] (gate then up), b2 fp32 [E, H]."""
    hb, w1b, w2b, tw, ti, T, H, I, E, k = _forward_args(hidden, w1, w2, topk_w, ids)
    a, b1a, b2a = _variant_args(act, b1, b2, E, H, I)
    if rows is None:
        rr, nrows, n = None, -1, T
    else:
        rr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = n = rr.shape[0]
    out = np.empty((max(n, 1), H), np.float64)
    rc = _load(mutation).oracle_moe_token_loop_ex(
        _ptr(hb), _ptr(w1b), _ptr(w2b), None if b1a is None else _ptr(b1a),
        None if b2a is None else _ptr(b2a), a, _ptr(tw), _ptr(ti), T, H, I, E, k,
        None if rr is None else _ptr(rr), nrows, _ptr(out))
    if rc != 0:
        raise RuntimeError("oracle_moe_token_loop failed")
    return out[:n]


def moe_expert_loop(hidden, w1, w2, topk_w, ids, mutation: int = 0,
                    act: str = "silu", b1=None, b2=None):
    """Formulation B (per-expert mask loop).  Returns float64 [T, H]."""
    hb, w1b, w2b, tw, ti, T, H, I, E, k = _forward_args(hidden, w1, w2, topk_w, ids)
    a, b1a, b2a = _variant_args(act, b1, b2, E, H, I)
    out = np.empty((max(T, 1), H), np.float64)
    rc = _load(mutation).oracle_moe_expert_loop_ex(
        _ptr(hb), _ptr(w1b), _ptr(w2b), None if b1a is None else _ptr(b1a),
        None if b2a is None else _ptr(b2a), a, _ptr(tw), _ptr(ti), T, H, I, E, k, _ptr(out))
    if rc != 0:
        raise RuntimeError("oracle_moe_expert_loop failed")
    return out[:T]


# ------------------------------------------------------------ FP8 weights
def e4m3_to_double(code: int, mutation: int = 0) -> float:
    """The value of one OCP FP8 E4M3 ("e4m3fn") code."""
    return _load(mutation).oracle_e4m3_to_double(int(code) & 0xFF)


def _fp8_args(hidden, q1, s1, q2, s2, block, topk_w, ids):
    hb = _bf16_bits(hidden)
    T, H = hb.shape
    q1a = np.ascontiguousarray(np.asarray(q1, dtype=np.uint8))
    q2a = np.ascontiguousarray(np.asarray(q2, dtype=np.uint8))
    E, twoI, H1 = q1a.shape
    I = twoI // 2
    block = int(block)
    if H1 != H or twoI != 2 * I or q2a.shape != (E, H, I):
        raise ValueError("shape mismatch between hidden, q1 [E,2I,H] and q2 [E,H,I]")
    if block < 1 or H % block or I % block:
        raise ValueError("block must divide H and I")
    s1a = np.ascontiguousarray(np.asarray(s1, dtype=np.float32).reshape(E, 2 * I, H // block))
    s2a = np.ascontiguousarray(np.asarray(s2, dtype=np.float32).reshape(E, H, I // block))
    tw = np.ascontiguousarray(np.asarray(topk_w, dtype=np.float64))
    ti = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    k = ti.shape[1] if ti.ndim == 2 else 1
    if tw.shape != (T, k) or ti.shape != (T, k):
        raise ValueError("topk weights/ids must both be [T, k]")
    return hb, q1a, s1a, q2a, s2a, block, tw, ti, T, H, I, E, k


def moe_token_loop_fp8(hidden, q1, s1, q2, s2, block, topk_w, ids, rows=None,
                       mutation: int = 0):
    """Formulation A on FP8 E4M3 weights (uint8 codes q1 [E,2I,H], q2
    [E,H,I]) with fp32 scales per row and block of `block` contraction
    elements (s1 [E,2I,H/block], s2 [E,H,I/block]); silu, no biases."""
    hb, q1a, s1a, q2a, s2a, block, tw, ti, T, H, I, E, k = _fp8_args(
        hidden, q1, s1, q2, s2, block, topk_w, ids)
    if rows is None:
        rr, nrows, n = None, -1, T
    else:
        rr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = n = rr.shape[0]
    out = np.empty((max(n, 1), H), np.float64)
    rc = _load(mutation).oracle_moe_token_loop_fp8(
        _ptr(hb), _ptr(q1a), _ptr(s1a), _ptr(q2a), _ptr(s2a), block, _ptr(tw), _ptr(ti), T, H,
        I, E, k, None if rr is None else _ptr(rr), nrows, _ptr(out))
    if rc != 0:
        raise RuntimeError("oracle_moe_token_loop_fp8 failed")
    return out[:n]


def moe_expert_loop_fp8(hidden, q1, s1, q2, s2, block, topk_w, ids, mutation: int = 0):
    """Formulation B on FP8 E4M3 weights (arguments as moe_token_loop_fp8)."""
    hb, q1a, s1a, q2a, s2a, block, tw, ti, T, H, I, E, k = _fp8_args(
        hidden, q1, s1, q2, s2, block, topk_w, ids)
    out = np.empty((max(T, 1), H), np.float64)
    rc = _load(mutation).oracle_moe_expert_loop_fp8(
        _ptr(hb), _ptr(q1a), _ptr(s1a), _ptr(q2a), _ptr(s2a), block, _ptr(tw), _ptr(ti), T, H,
        I, E, k, _ptr(out))
    if rc != 0:
        raise RuntimeError("oracle_moe_expert_loop_fp8 failed")
    return out[:T]
