"""Python binding of libmoe.so, the B200 (sm_100a) fused MoE forward.

Argument marshalling only: every function checks dtypes, shapes and devices
of torch tensors, passes raw device pointers, sizes and the current CUDA
stream to the C ABI of ``include/moe.h`` and raises ``MoEError`` on a
non-zero return code.  All arithmetic runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback, and importing this package fails if
libmoe.so has not been built (``python mixture_experts_expert_softmax_b200/build.py``).

    ids, w = moe_route(logits, k=8, renorm=True)          # [T,k] int32, fp32
    out = moe_forward(hidden, w1, w2, w, ids)              # [T,H] fp32
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_TIMEOUT = -4
MOE_ERR_NO_DEVICE = -5
MOE_ERR_OOM = -6
MOE_ERR_SCRATCH_LIMIT = -7
MOE_NOALLOC_MAX_T = 16
MOE_NOALLOC_MAX_ACT = 262144
MOE_STATUS_TIMEOUT = 0x1
MOE_STATUS_BAD_ID = 0x2
MOE_PERMUTE_AUTO = 0
MOE_PERMUTE_SINGLE = 1
MOE_PERMUTE_MULTI = 2
PERMUTE_KERNELS = {"auto": MOE_PERMUTE_AUTO, "single": MOE_PERMUTE_SINGLE,
                   "multi": MOE_PERMUTE_MULTI}
MOE_ACT_SILU = 0
MOE_ACT_GELU_TANH = 1
MOE_ACT_SWIGLUOAI = 2
ACTS = {"silu": MOE_ACT_SILU, "gelu": MOE_ACT_GELU_TANH, "swigluoai": MOE_ACT_SWIGLUOAI}

# every symbol declared in include/moe.h
EXPORTED = (
    "moe_route", "moe_forward", "moe_permute", "moe_error_string",
    "moe_get_device_status", "moe_set_small_t_max", "moe_set_sync_each_stage",
    "moe_set_wait_limit_ns", "moe_last_failed_stage", "moe_debug_wait_timeout",
    "moe_profile_enable", "moe_profile_reset", "moe_profile_read",
    "moe_forward_small_noalloc", "moe_forward_ex", "moe_forward_fp8", "moe_permute_ex",
    "moe_timeline", "moe_ep_dispatch_plan", "moe_ep_pack", "moe_ep_return", "moe_ep_combine",
)


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} (code {code})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python mixture_experts_expert_softmax_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    sig = {
        "moe_route": ([P, I64, I32, I32, I32, P, P, P], I32),
        "moe_forward": ([P, P, P, P, P, P, I64, I32, I32, I32, I32, P], I32),
        "moe_permute": ([P, I64, I32, I32, P, P, P], I32),
        "moe_permute_ex": ([P, I64, I32, I32, P, P, P, P, I32, P, I32, P], I32),
        "moe_timeline": ([P, I64], I32),
        "moe_ep_dispatch_plan": ([P, I64, I32, I32, I32, P, P, P, P], I32),
        "moe_ep_pack": ([P, I32, P, I64, I32, I32, I32, P, P, P, P, P, P], I32),
        "moe_ep_return": ([P, I32, I32, P, P, P, P], I32),
        "moe_ep_combine": ([P, P, P, P, I64, I32, I32, P], I32),
        "moe_error_string": ([I32], ctypes.c_char_p),
        "moe_get_device_status": ([P, ctypes.POINTER(ctypes.c_uint32)], I32),
        "moe_set_small_t_max": ([I32], I32),
        "moe_set_sync_each_stage": ([I32], I32),
        "moe_set_wait_limit_ns": ([I64], I64),
        "moe_last_failed_stage": ([], ctypes.c_char_p),
        "moe_debug_wait_timeout": ([I64, P], I32),
        "moe_profile_enable": ([I32], I32),
        "moe_profile_reset": ([], I32),
        "moe_profile_read": ([I32, P, P, P], I32),
        "moe_forward_small_noalloc": ([P, P, P, P, P, P, I64, I32, I32, I32, I32, P], I32),
        "moe_forward_ex": ([P, P, P, P, P, I32, P, P, P, I64, I32, I32, I32, I32, P], I32),
        "moe_forward_fp8": ([P, P, P, P, P, I32, P, P, P, I64, I32, I32, I32, I32, P], I32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def error_string(code: int) -> str:
    return _lib.moe_error_string(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != MOE_OK:
        raise MoEError(code, where)


def _stream(stream) -> int | None:
    if stream is None:
        if not torch.cuda.is_available():
            return None  # legacy default stream; the library reports the missing device
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def moe_route(logits: torch.Tensor, k: int, renorm: bool = True,
              topk_ids: torch.Tensor | None = None,
              topk_weights: torch.Tensor | None = None, stream=None):
    """Softmax over [T, E] fp32 logits, top-k (lowest index on ties),
    optional renormalisation.  Returns (topk_ids int32 [T,k], topk_weights fp32 [T,k])."""
    _need(logits, "logits", torch.float32)
    T, E = logits.shape
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if topk_weights is None:
        topk_weights = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _need(topk_ids, "topk_ids", torch.int32, (T, k))
    _need(topk_weights, "topk_weights", torch.float32, (T, k))
    _check(_lib.moe_route(logits.data_ptr(), T, E, int(k), int(bool(renorm)),
                          topk_ids.data_ptr(), topk_weights.data_ptr(), _stream(stream)),
           "moe_route")
    return topk_ids, topk_weights


def moe_forward(hidden: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor,
                topk_weights: torch.Tensor, topk_ids: torch.Tensor,
                out: torch.Tensor | None = None, stream=None, *, act: str = "silu",
                b1: torch.Tensor | None = None, b2: torch.Tensor | None = None) -> torch.Tensor:
    """Fused MoE forward: hidden [T,H] bf16, w1 [E,2I,H] bf16, w2 [E,H,I] bf16,
    topk_weights [T,k] fp32, topk_ids [T,k] int32 -> out [T,H] fp32.

    act ("silu", "gelu" (tanh form) or "swigluoai") and the optional fp32
    biases b1 [E,2I] and b2 [E,H] select the expert-FFN variant; anything
    but the default goes through moe_forward_ex."""
    if act not in ACTS:
        raise ValueError(f"act must be one of {sorted(ACTS)}, got {act!r}")
    _need(hidden, "hidden", torch.bfloat16)
    T, H = hidden.shape
    _need(w1, "w1", torch.bfloat16)
    E, twoI, _ = w1.shape
    I = twoI // 2
    _need(w1, "w1", torch.bfloat16, (E, 2 * I, H))
    _need(w2, "w2", torch.bfloat16, (E, H, I))
    k = topk_ids.shape[1] if topk_ids.dim() == 2 else 0
    _need(topk_ids, "topk_ids", torch.int32, (T, k))
    _need(topk_weights, "topk_weights", torch.float32, (T, k))
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32, device=hidden.device)
    _need(out, "out", torch.float32, (T, H))
    if act == "silu" and b1 is None and b2 is None:
        _check(_lib.moe_forward(hidden.data_ptr(), w1.data_ptr(), w2.data_ptr(),
                                topk_weights.data_ptr(), topk_ids.data_ptr(), out.data_ptr(),
                                T, H, I, E, k, _stream(stream)), "moe_forward")
        return out
    if b1 is not None:
        _need(b1, "b1", torch.float32, (E, 2 * I))
    if b2 is not None:
        _need(b2, "b2", torch.float32, (E, H))
    _check(_lib.moe_forward_ex(hidden.data_ptr(), w1.data_ptr(), w2.data_ptr(),
                               None if b1 is None else b1.data_ptr(),
                               None if b2 is None else b2.data_ptr(), ACTS[act],
                               topk_weights.data_ptr(), topk_ids.data_ptr(), out.data_ptr(),
                               T, H, I, E, k, _stream(stream)), "moe_forward_ex")
    return out


def moe_forward_fp8(hidden: torch.Tensor, w1: torch.Tensor, w1_scale: torch.Tensor,
                    w2: torch.Tensor, w2_scale: torch.Tensor, block: int,
                    topk_weights: torch.Tensor, topk_ids: torch.Tensor,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Fused MoE forward on FP8 E4M3 expert weights: w1 [E,2I,H] and w2
    [E,H,I] uint8 codes, w1_scale [E,2I,H/block] and w2_scale [E,H,I/block]
    fp32 scales (one per row and block of `block` contraction elements)."""
    _need(hidden, "hidden", torch.bfloat16)
    T, H = hidden.shape
    _need(w1, "w1", torch.uint8)
    E, twoI, _ = w1.shape
    I = twoI // 2
    block = int(block)
    if block < 1 or H % block or I % block:
        raise ValueError(f"block must be positive and divide H={H} and I={I}")
    _need(w1, "w1", torch.uint8, (E, 2 * I, H))
    _need(w2, "w2", torch.uint8, (E, H, I))
    _need(w1_scale, "w1_scale", torch.float32, (E, 2 * I, H // block))
    _need(w2_scale, "w2_scale", torch.float32, (E, H, I // block))
    k = topk_ids.shape[1] if topk_ids.dim() == 2 else 0
    _need(topk_ids, "topk_ids", torch.int32, (T, k))
    _need(topk_weights, "topk_weights", torch.float32, (T, k))
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32, device=hidden.device)
    _need(out, "out", torch.float32, (T, H))
    _check(_lib.moe_forward_fp8(hidden.data_ptr(), w1.data_ptr(), w1_scale.data_ptr(),
                                w2.data_ptr(), w2_scale.data_ptr(), block,
                                topk_weights.data_ptr(), topk_ids.data_ptr(), out.data_ptr(),
                                T, H, I, E, k, _stream(stream)), "moe_forward_fp8")
    return out


def moe_forward_small_noalloc(hidden: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor,
                              topk_weights: torch.Tensor, topk_ids: torch.Tensor,
                              out: torch.Tensor, stream=None) -> torch.Tensor:
    """Small-batch forward that allocates nothing on the device: for callers
    that reserve all device memory up front.  `out` must be given; limits
    T <= MOE_NOALLOC_MAX_T and T*k*I <= MOE_NOALLOC_MAX_ACT."""
    _need(hidden, "hidden", torch.bfloat16)
    T, H = hidden.shape
    E, twoI, _ = w1.shape
    I = twoI // 2
    _need(w1, "w1", torch.bfloat16, (E, 2 * I, H))
    _need(w2, "w2", torch.bfloat16, (E, H, I))
    k = topk_ids.shape[1] if topk_ids.dim() == 2 else 0
    _need(topk_ids, "topk_ids", torch.int32, (T, k))
    _need(topk_weights, "topk_weights", torch.float32, (T, k))
    _need(out, "out", torch.float32, (T, H))
    _check(_lib.moe_forward_small_noalloc(hidden.data_ptr(), w1.data_ptr(), w2.data_ptr(),
                                          topk_weights.data_ptr(), topk_ids.data_ptr(),
                                          out.data_ptr(), T, H, I, E, k, _stream(stream)),
           "moe_forward_small_noalloc")
    return out


def moe_permute(topk_ids: torch.Tensor, E: int, sorted_rows: torch.Tensor | None = None,
                expert_offsets: torch.Tensor | None = None, stream=None):
    """Stable grouping of the flat (token, slot) indices by expert.
    Returns (sorted_rows int32 [T*k], expert_offsets int32 [E+1])."""
    _need(topk_ids, "topk_ids", torch.int32)
    T, k = topk_ids.shape
    if sorted_rows is None:
        sorted_rows = torch.full((T * k,), -1, dtype=torch.int32, device=topk_ids.device)
    if expert_offsets is None:
        expert_offsets = torch.empty((E + 1,), dtype=torch.int32, device=topk_ids.device)
    _need(sorted_rows, "sorted_rows", torch.int32, (T * k,))
    _need(expert_offsets, "expert_offsets", torch.int32, (E + 1,))
    _check(_lib.moe_permute(topk_ids.data_ptr(), T, k, int(E), sorted_rows.data_ptr(),
                            expert_offsets.data_ptr(), _stream(stream)), "moe_permute")
    return sorted_rows, expert_offsets


def moe_permute_ex(topk_ids: torch.Tensor, E: int, kernel: str = "auto",
                   hidden: torch.Tensor | None = None, stream=None):
    """Everything the grouping stage of moe_forward produces, with a choice
    of grouping kernel ("auto", "single" or "multi").  Returns (sorted_rows
    int32 [T*k], expert_offsets int32 [E+1], inv int32 [T*k], xs) where xs
    is the expert-sorted copy of the bf16 hidden rows [T*k, H] when hidden
    is given (rows past expert_offsets[E] stay zero), else None."""
    _need(topk_ids, "topk_ids", torch.int32)
    if kernel not in PERMUTE_KERNELS:
        raise ValueError(f"kernel must be one of {sorted(PERMUTE_KERNELS)}, got {kernel!r}")
    T, k = topk_ids.shape
    dev = topk_ids.device
    sorted_rows = torch.full((T * k,), -1, dtype=torch.int32, device=dev)
    expert_offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    inv = torch.full((T * k,), -2, dtype=torch.int32, device=dev)
    xs, H = None, 0
    if hidden is not None:
        _need(hidden, "hidden", torch.bfloat16)
        if hidden.shape[0] != T:
            raise ValueError(f"hidden must have {T} rows, got {hidden.shape[0]}")
        H = hidden.shape[1]
        xs = torch.zeros((T * k, H), dtype=torch.bfloat16, device=dev)
    _check(_lib.moe_permute_ex(topk_ids.data_ptr(), T, k, int(E), sorted_rows.data_ptr(),
                               expert_offsets.data_ptr(), inv.data_ptr(),
                               None if hidden is None else hidden.data_ptr(), H,
                               None if xs is None else xs.data_ptr(),
                               PERMUTE_KERNELS[kernel], _stream(stream)), "moe_permute_ex")
    return sorted_rows, expert_offsets, inv, xs


TIMELINE_KINDS = {1: "gemm1", 2: "gemm2", 3: "gemm_fused", 4: "small_t"}
TIMELINE_ROLES = {0: "producer", 1: "mma", 2: "epilogue", 3: "phase1", 4: "barrier",
                  5: "act_load", 6: "w2_wait", 7: "phase2", 8: "phase2_dots"}
_timeline_buf = None


def timeline_start(capacity: int = 1 << 16, device=None) -> None:
    """Record the kernels' per-tile / per-phase timeline (moe_timeline) into
    a fresh device buffer until timeline_stop()."""
    global _timeline_buf
    _timeline_buf = torch.zeros(4 + 4 * int(capacity), dtype=torch.int64,
                                device=device or torch.device("cuda"))
    _check(_lib.moe_timeline(_timeline_buf.data_ptr(), int(capacity)), "moe_timeline")


def timeline_stop() -> list[dict]:
    """Stop recording; synchronise and return the records as dicts
    {kind, role, cta, sub, id, t0, t1} (nanoseconds of %globaltimer)."""
    global _timeline_buf
    _check(_lib.moe_timeline(None, 0), "moe_timeline")
    if _timeline_buf is None:
        return []
    torch.cuda.synchronize()
    raw = _timeline_buf.cpu()
    _timeline_buf = None
    n = (raw.numel() - 4) // 4
    rec = raw[4:4 + 4 * n].view(n, 4)
    rec = rec[rec[:, 0] != 0].tolist()  # slots nobody wrote
    out = []
    for tag, ident, t0, t1 in rec:
        tag &= (1 << 64) - 1
        out.append({"kind": TIMELINE_KINDS.get(tag >> 56, str(tag >> 56)),
                    "role": TIMELINE_ROLES.get((tag >> 48) & 0xff, str((tag >> 48) & 0xff)),
                    "cta": (tag >> 16) & 0xffffffff, "sub": tag & 0xffff, "id": ident,
                    "t0": t0 & ((1 << 64) - 1), "t1": t1 & ((1 << 64) - 1)})
    return out


def timeline_summary(records: list[dict]) -> dict:
    """Per (kind, role): record count, mean and max duration (us), and the
    span from the earliest t0 to the latest t1 (us).  Per GEMM kind also:
    the MMA records binned by their start (10 us bins from the first MMA:
    tiles started and their mean duration), each CTA's summed MMA time
    (min / median / max), and the median gap between consecutive tiles of
    one CTA's MMA thread."""
    import collections
    out: dict = {}
    by = collections.defaultdict(list)
    for r in records:
        by[(r["kind"], r["role"])].append(r)
    for (kind, role), rs in sorted(by.items()):
        d = [(r["t1"] - r["t0"]) / 1e3 for r in rs]
        out[f"{kind}/{role}"] = {
            "n": len(rs), "mean_us": round(sum(d) / len(d), 3), "max_us": round(max(d), 3),
            "span_us": round((max(r["t1"] for r in rs) - min(r["t0"] for r in rs)) / 1e3, 3)}
        if role != "mma":
            continue
        t0 = min(r["t0"] for r in rs)
        bins = collections.defaultdict(list)
        per_cta = collections.defaultdict(list)
        for r in rs:
            bins[int((r["t0"] - t0) / 1e4) * 10].append((r["t1"] - r["t0"]) / 1e3)
            per_cta[r["cta"]].append(r)
        busy = sorted(sum(r["t1"] - r["t0"] for r in v) / 1e3 for v in per_cta.values())
        gaps = sorted((b["t0"] - a["t1"]) / 1e3 for v in per_cta.values()
                      for a, b in zip(sorted(v, key=lambda r: r["t0"]),
                                      sorted(v, key=lambda r: r["t0"])[1:]))
        out[f"{kind}/mma"].update({
            "by_start_10us": {k: [len(v), round(sum(v) / len(v), 2)]
                              for k, v in sorted(bins.items())},
            "cta_mma_us_min_med_max": [round(busy[0], 1), round(busy[len(busy) // 2], 1),
                                       round(busy[-1], 1)],
            "tile_gap_us_median": round(gaps[len(gaps) // 2], 3) if gaps else None})
    return out


def get_device_status(stream=None) -> int:
    """Synchronise, return and clear the OR of MOE_STATUS_* bits."""
    v = ctypes.c_uint32(0)
    _check(_lib.moe_get_device_status(_stream(stream), ctypes.byref(v)), "moe_get_device_status")
    return int(v.value)


def set_small_t_max(n: int) -> int:
    return int(_lib.moe_set_small_t_max(int(n)))


def set_sync_each_stage(on: bool) -> int:
    return int(_lib.moe_set_sync_each_stage(int(bool(on))))


def set_wait_limit_ns(ns: int) -> int:
    return int(_lib.moe_set_wait_limit_ns(int(ns)))


def last_failed_stage() -> str:
    return _lib.moe_last_failed_stage().decode()


def debug_wait_timeout(limit_ns: int, stream=None) -> int:
    """Run the never-signalled bounded wait; returns the raw MOE_* code."""
    return int(_lib.moe_debug_wait_timeout(int(limit_ns), _stream(stream)))


def profile_enable(on: bool) -> bool:
    return bool(_lib.moe_profile_enable(int(bool(on))))


def profile_reset() -> None:
    _lib.moe_profile_reset()


def profile_read() -> dict[str, tuple[int, float]]:
    """Synchronise and return {kernel name: (launches, total ms)}."""
    n = _lib.moe_profile_read(0, None, None, None)
    if n <= 0:
        return {}
    names = (ctypes.c_char * 64 * n)()
    launches = (ctypes.c_int64 * n)()
    ms = (ctypes.c_double * n)()
    n = _lib.moe_profile_read(n, names, launches, ms)
    return {bytes(names[i]).split(b"\0", 1)[0].decode(): (int(launches[i]), float(ms[i]))
            for i in range(n)}


__all__ = [
    "moe_route", "moe_forward", "moe_forward_fp8", "moe_forward_small_noalloc", "moe_permute",
    "moe_permute_ex", "get_device_status", "set_small_t_max",
    "set_sync_each_stage", "set_wait_limit_ns", "last_failed_stage", "debug_wait_timeout",
    "profile_enable", "profile_reset", "profile_read", "error_string", "MoEError",
    "timeline_start", "timeline_stop", "timeline_summary",
    "LIB_PATH", "EXPORTED", "ACTS",
]
