"""Pins of the fp64 CPU oracle against things other than itself.

Each check compares the oracle with a value that the pages or mathematics fix
independently: hand-derived closed forms (tests/golden/), brute force over all
expert subsets, library routines (torch.topk, scipy softmax/expit, numpy and
torch fp64 matmul, numpy stable argsort) and invariants of the definition
(relabelling, linearity, zero token, duplicate ids).  The last test plants each
plausible mistake in a rebuilt oracle and checks that some pin catches it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from moe_inputs import make_inputs

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def to64(t):
    return t.float().double().numpy()


def dense_numpy(hidden, w1, w2, topk_w, ids):
    """Third formulation, for pins: run every expert on every token with numpy
    fp64 matmuls and weight it by the summed top-k weight (0 if unselected)."""
    X, W1, W2 = to64(hidden), to64(w1), to64(w2)
    T = X.shape[0]
    E, twoI, _ = W1.shape
    I = twoI // 2
    out = np.zeros((T, W2.shape[1]))
    ids = np.asarray(ids)
    for e in range(E):
        wd = np.where(ids == e, np.asarray(topk_w, np.float64), 0.0).sum(axis=1)
        G = X @ W1[e, :I].T
        U = X @ W1[e, I:].T
        A = G * scipy.special.expit(G) * U
        out += wd[:, None] * (A @ W2[e].T)
    return out


def close(a, b, rel=1e-12):
    a, b = np.asarray(a), np.asarray(b)
    scale = max(np.abs(b).max(), 1e-300)
    return np.abs(a - b).max() <= rel * scale


# ---------------------------------------------------------------- pin checks
# Each returns True when the (possibly mutated) oracle passes the pin.

def pin_golden_route(golden_dir, mutation=0):
    g = json.load(open(os.path.join(golden_dir, "worked_example.json")))
    lg = np.array(g["logits"], np.float32)
    ok = True
    ids, w = oracle.route(lg, 2, True, mutation=mutation)
    ok &= (ids.tolist() == g["expected_ids"])
    ok &= np.abs(w - np.array(g["expected_weights_renorm"])).max() <= g["tolerance_abs"]
    ids, w = oracle.route(lg, 2, False, mutation=mutation)
    ok &= (ids.tolist() == g["expected_ids"])
    ok &= np.abs(w - np.array(g["expected_weights_raw"])).max() <= g["tolerance_abs"]
    return bool(ok)


def pin_golden_forward(golden_dir, mutation=0):
    g = json.load(open(os.path.join(golden_dir, "worked_example.json")))
    hidden, w1, w2 = bf16(g["hidden"]), bf16(g["w1"]), bf16(g["w2"])
    ids = np.array(g["expected_ids"], np.int32)
    w = np.array(g["expected_weights_renorm"])
    exp = np.array(g["expected_out_renorm"])
    a = oracle.moe_token_loop(hidden, w1, w2, w, ids, mutation=mutation)
    b = oracle.moe_expert_loop(hidden, w1, w2, w, ids, mutation=mutation)
    tol = g["tolerance_abs"]
    return bool(np.abs(a - exp).max() <= tol and np.abs(b - exp).max() <= tol)


def pin_golden_permute(golden_dir, mutation=0):
    g = json.load(open(os.path.join(golden_dir, "permute_example.json")))
    rows, offs = oracle.permute(np.array(g["ids"], np.int32), g["E"], mutation=mutation)
    return rows.tolist() == g["expected_sorted_rows"] and offs.tolist() == g["expected_offsets"]


def pin_route_bruteforce(mutation=0, seed=1):
    """The chosen set maximises the sum of logits over all C(E,k) subsets, and
    among equal sums is the lexicographically smallest; the order is logit
    descending with lower index first.  Logits come from a small integer set
    so that ties are frequent."""
    rng = np.random.default_rng(seed)
    for E in (1, 2, 3, 5, 8):
        for k in range(1, E + 1):
            lg = rng.integers(-2, 3, size=(24, E)).astype(np.float32)
            ids, _ = oracle.route(lg, k, False, mutation=mutation)
            for t in range(lg.shape[0]):
                best = max(itertools.combinations(range(E), k),
                           key=lambda s: (sum(float(lg[t, e]) for e in s), [-e for e in s]))
                if sorted(ids[t].tolist()) != list(best):
                    return False
                order = sorted(best, key=lambda e: (-float(lg[t, e]), e))
                if ids[t].tolist() != order:
                    return False
    return True


def pin_route_library(mutation=0, seed=2):
    """Against torch.topk of the fp64 softmax (rows of continuous logits have
    no ties) and scipy's softmax for the weights."""
    rng = np.random.default_rng(seed)
    ok = True
    for E, k in ((8, 2), (128, 8), (64, 6), (5, 5)):
        lg = rng.standard_normal((50, E)).astype(np.float32)
        p = scipy.special.softmax(lg.astype(np.float64), axis=-1)
        tv, ti = torch.topk(torch.tensor(p), k, dim=-1)
        ids, w = oracle.route(lg, k, False, mutation=mutation)
        ok &= np.array_equal(ids, ti.numpy().astype(np.int32))
        ok &= close(w, tv.numpy(), 1e-13)
        ids_r, w_r = oracle.route(lg, k, True, mutation=mutation)
        ok &= np.array_equal(ids_r, ids)
        ok &= close(w_r, tv.numpy() / tv.numpy().sum(-1, keepdims=True), 1e-13)
    return bool(ok)


def pin_permute_library(mutation=0, seed=3):
    """Against numpy's stable argsort and bincount, with invalid ids mixed in."""
    rng = np.random.default_rng(seed)
    for n, E in ((0, 4), (1, 1), (37, 3), (1000, 8), (4096, 128), (777, 1024)):
        ids = rng.integers(-2, E + 2, size=n).astype(np.int32)
        rows, offs = oracle.permute(ids, E, mutation=mutation)
        valid = (ids >= 0) & (ids < E)
        idx = np.nonzero(valid)[0]
        ref_rows = idx[np.argsort(ids[idx], kind="stable")]
        ref_offs = np.concatenate([[0], np.cumsum(np.bincount(ids[idx], minlength=E))])
        if not np.array_equal(offs, ref_offs):
            return False
        nv = int(valid.sum())
        if not np.array_equal(rows[:nv], ref_rows) or not np.all(rows[nv:] == -1):
            return False
    return True


def pin_forward_dense(mutation=0, seed=4, H=64, I=32):
    """Both formulations against the dense numpy fp64 formulation."""
    ok = True
    for T, E, k in ((9, 4, 2), (16, 8, 3), (5, 1, 1), (12, 6, 6)):
        hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=seed)
        ids, w = oracle.route(logits.numpy(), k, True)
        ref = dense_numpy(hidden, w1, w2, w, ids)
        a = oracle.moe_token_loop(hidden, w1, w2, w, ids, mutation=mutation)
        b = oracle.moe_expert_loop(hidden, w1, w2, w, ids, mutation=mutation)
        ok &= close(a, ref) and close(b, ref)
    return bool(ok)


# ------------------------------------------- pins of the epilogue variants
# (activation_fn, swigluoai and the b1/b2 biases of the 0.13.2 TPU page)


def _dense_mlp(act, hidden, w1e, w2e):
    """One expert on every token with torch fp64 library routines."""
    X = torch.tensor(to64(hidden))
    W1, W2 = torch.tensor(to64(w1e)), torch.tensor(to64(w2e))
    I = W1.shape[0] // 2
    G = X @ W1[:I].T
    U = X @ W1[I:].T
    if act == "gelu":
        A = torch.nn.functional.gelu(G, approximate="tanh") * U
    elif act == "swigluoai":
        # unclamped range only: g * sigmoid(1.702 g) = silu(1.702 g) / 1.702
        assert G.max() < 7 and U.abs().max() < 7
        A = (U + 1.0) * torch.nn.functional.silu(1.702 * G) / 1.702
    else:
        A = torch.nn.functional.silu(G) * U
    return (A @ W2.T).numpy()


def pin_activation_library(mutation=0, seed=21):
    """E = k = 1 with weight 1 is one expert's MLP: gelu (tanh form) and
    swigluoai (in its unclamped range) against torch fp64."""
    ok = True
    for act in ("gelu", "swigluoai", "silu"):
        hidden, w1, w2, _ = make_inputs(11, 64, 32, 1, seed=seed)
        ids = np.zeros((11, 1), np.int32)
        w = np.ones((11, 1))
        ref = _dense_mlp(act, hidden, w1[0], w2[0])
        a = oracle.moe_token_loop(hidden, w1, w2, w, ids, mutation=mutation, act=act)
        b = oracle.moe_expert_loop(hidden, w1, w2, w, ids, mutation=mutation, act=act)
        ok &= close(a, ref) and close(b, ref)
    return bool(ok)


def pin_swigluoai_clamped(mutation=0):
    """All gate values 8 and up values -8 or 9: both clip, so every
    activation is (clip(u) + 1) * 7 * sigmoid(11.914), and doubling w1
    changes nothing."""
    H, I, E = 64, 32, 2
    hidden = bf16(np.ones((3, H)))
    w1 = np.zeros((E, 2 * I, H), np.float32)
    w1[:, :I, :] = 0.125                       # g = 8
    w1[0, I:, :] = -0.125                      # u = -8 -> -7
    w1[1, I:, :] = 9.0 / 64                    # u = 9 -> 7
    w2 = np.random.default_rng(3).standard_normal((E, H, I)).astype(np.float32) * 0.1
    ids = np.array([[0, 1], [1, 0], [1, 1]], np.int32)
    w = np.array([[0.25, 0.75], [0.5, 0.5], [0.1, 0.9]])
    sig = scipy.special.expit(1.702 * 7.0)
    acts = np.stack([np.full(I, (-7.0 + 1.0) * 7.0 * sig), np.full(I, (7.0 + 1.0) * 7.0 * sig)])
    W2 = to64(bf16(w2.reshape(-1)).reshape(E, H, I))
    y = np.einsum("ehi,ei->eh", W2, acts)
    ref = np.stack([sum(w[t, j] * y[ids[t, j]] for j in range(2)) for t in range(3)])
    ok = True
    for scale in (1.0, 2.0):
        a = oracle.moe_token_loop(hidden, bf16(w1 * scale), bf16(w2), w, ids,
                                  mutation=mutation, act="swigluoai")
        ok &= close(a, ref, 1e-12)
    return bool(ok)


def pin_b1_with_zero_w1(mutation=0):
    """w1 = 0: the projections are the biases alone, so
    act = silu(b1_gate) * b1_up per expert, the same for every token."""
    T, H, I, E, k = 5, 48, 16, 3, 2
    hidden, _, w2, logits = make_inputs(T, H, I, E, seed=22)
    w1 = bf16(np.zeros((E, 2 * I, H)))
    b1 = np.random.default_rng(5).standard_normal((E, 2 * I)).astype(np.float32)
    ids, w = oracle.route(logits.numpy(), k, True)
    G, U = b1[:, :I].astype(np.float64), b1[:, I:].astype(np.float64)
    A = G * scipy.special.expit(G) * U
    y = np.einsum("ehi,ei->eh", to64(w2), A)
    ref = np.stack([sum(w[t, j] * y[ids[t, j]] for j in range(k)) for t in range(T)])
    a = oracle.moe_token_loop(hidden, w1, w2, w, ids, mutation=mutation, b1=b1)
    b = oracle.moe_expert_loop(hidden, w1, w2, w, ids, mutation=mutation, b1=b1)
    return bool(close(a, ref) and close(b, ref))


def pin_b2_with_zero_w2(mutation=0):
    """w2 = 0: each expert's output is its bias b2[e], so
    out[t] = sum_j w[t, j] * b2[ids[t, j]] exactly."""
    T, H, I, E, k = 6, 32, 16, 4, 3
    hidden, w1, _, logits = make_inputs(T, H, I, E, seed=23)
    w2 = bf16(np.zeros((E, H, I)))
    b2 = np.random.default_rng(6).standard_normal((E, H)).astype(np.float32)
    ids, w = oracle.route(logits.numpy(), k, False)
    ref = np.stack([sum(w[t, j] * b2[ids[t, j]].astype(np.float64) for j in range(k))
                    for t in range(T)])
    a = oracle.moe_token_loop(hidden, w1, w2, w, ids, mutation=mutation, b2=b2)
    b = oracle.moe_expert_loop(hidden, w1, w2, w, ids, mutation=mutation, b2=b2)
    return bool(close(a, ref) and close(b, ref))


def pin_variants_formulations_agree(mutation=0):
    ok = True
    for act in ("silu", "gelu", "swigluoai"):
        hidden, w1, w2, logits = make_inputs(13, 64, 32, 5, seed=24)
        rng = np.random.default_rng(7)
        b1 = rng.standard_normal((5, 64)).astype(np.float32) * 0.1
        b2 = rng.standard_normal((5, 64)).astype(np.float32) * 0.1
        ids, w = oracle.route(logits.numpy(), 2, True)
        a = oracle.moe_token_loop(hidden, w1, w2, w, ids, mutation=mutation, act=act, b1=b1, b2=b2)
        b = oracle.moe_expert_loop(hidden, w1, w2, w, ids, mutation=mutation, act=act, b1=b1,
                                   b2=b2)
        ok &= close(a, b)
    return bool(ok)


# ------------------------------------------------ pins of the FP8 weights
# (w1_scale / w2_scale / subc_quant_wsz of the 0.13.2 TPU page's ref_moe)


def pin_e4m3_decoder(mutation=0):
    """Every one of the 256 E4M3 codes against torch's float8_e4m3fn."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_to_double(c, mutation=mutation) for c in codes])
    nan = np.isnan(ref)
    return bool(np.array_equal(nan, np.isnan(got)) and np.array_equal(ref[~nan], got[~nan]))


def _fp8_case(T=9, H=512, I=256, E=4, k=2, block=128, seed=31):
    """Codes and power-of-two scales that differ per block: the dequantised
    weights are then exact in bf16, so the bf16 forward applies to them."""
    rng = np.random.default_rng(seed)
    hidden, _, _, logits = make_inputs(T, H, I, E, seed=seed)
    q1 = rng.integers(0, 256, (E, 2 * I, H), dtype=np.uint8)
    q2 = rng.integers(0, 256, (E, H, I), dtype=np.uint8)
    q1[(q1 & 0x7F) == 0x7F] = 0  # no NaN codes
    q2[(q2 & 0x7F) == 0x7F] = 0
    s1 = np.exp2(rng.integers(-14, -8, (E, 2 * I, H // block))).astype(np.float32)
    s2 = np.exp2(rng.integers(-14, -8, (E, H, I // block))).astype(np.float32)
    ids, w = oracle.route(logits.numpy(), k, True)
    return hidden, q1, s1, q2, s2, block, w, ids


def _dequant_bf16(q, s, block):
    """torch's E4M3 conversion times each block's scale (np.repeat spreads a
    block's scale over its elements, as ref_moe's jnp.repeat does), as bf16."""
    v = torch.from_numpy(q).view(torch.float8_e4m3fn).double()
    v = v * torch.from_numpy(np.repeat(s.astype(np.float64), block, axis=-1))
    bf = v.to(torch.bfloat16)
    assert torch.equal(bf.double(), v)  # exact: power-of-two scales
    return bf


def pin_fp8_equals_bf16_of_dequantised(mutation=0):
    hidden, q1, s1, q2, s2, block, w, ids = _fp8_case()
    w1 = _dequant_bf16(q1, s1, block)
    w2 = _dequant_bf16(q2, s2, block)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    a = oracle.moe_token_loop_fp8(hidden, q1, s1, q2, s2, block, w, ids, mutation=mutation)
    b = oracle.moe_expert_loop_fp8(hidden, q1, s1, q2, s2, block, w, ids, mutation=mutation)
    return bool(close(a, ref, 1e-12) and close(b, ref, 1e-12))


def pin_fp8_w2_scale_linearity(mutation=0):
    """Every w2 scale times 2 doubles the output exactly."""
    hidden, q1, s1, q2, s2, block, w, ids = _fp8_case(seed=32)
    a = oracle.moe_token_loop_fp8(hidden, q1, s1, q2, s2, block, w, ids, mutation=mutation)
    b = oracle.moe_token_loop_fp8(hidden, q1, s1, q2, 2 * s2, block, w, ids, mutation=mutation)
    return bool(np.array_equal(2 * a, b))


# ---------------------------------------------------------------- tests

def test_golden_route(golden_dir):
    assert pin_golden_route(golden_dir)


def test_golden_forward(golden_dir):
    assert pin_golden_forward(golden_dir)


def test_golden_permute(golden_dir):
    assert pin_golden_permute(golden_dir)


def test_route_bruteforce():
    assert pin_route_bruteforce()


def test_route_library():
    assert pin_route_library()


def test_route_renorm_sum_and_k1():
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((200, 64)).astype(np.float32)
    _, w = oracle.route(lg, 7, True)
    assert np.abs(w.sum(-1) - 1.0).max() <= 1e-12
    _, w1 = oracle.route(lg, 1, True)
    assert np.all(w1 == 1.0)


def test_route_k_equals_e_is_full_softmax():
    """k = E without renormalisation returns the whole softmax (scipy)."""
    rng = np.random.default_rng(6)
    lg = (3 * rng.standard_normal((40, 16))).astype(np.float32)
    ids, w = oracle.route(lg, 16, False)
    p = scipy.special.softmax(lg.astype(np.float64), axis=-1)
    assert close(w, np.take_along_axis(p, ids.astype(np.int64), -1), 1e-13)
    assert np.all(np.sort(ids, -1) == np.arange(16))


def test_route_neg_inf():
    """-inf logits get weight 0 and fill the leftover slots lowest index first."""
    lg = np.array([[-np.inf, 3.0, -np.inf, -np.inf],
                   [0.5, -np.inf, 0.5, -np.inf]], np.float32)
    ids, w = oracle.route(lg, 3, False)
    assert ids.tolist() == [[1, 0, 2], [0, 2, 1]]
    assert w[0].tolist() == [1.0, 0.0, 0.0]
    assert w[1].tolist() == [0.5, 0.5, 0.0]


def test_route_rejects_bad_k():
    with pytest.raises(ValueError):
        oracle.route(np.zeros((2, 4), np.float32), 5, True)
    with pytest.raises(ValueError):
        oracle.route(np.zeros((2, 4), np.float32), 0, True)


def test_permute_library():
    assert pin_permute_library()


def test_forward_dense_numpy():
    assert pin_forward_dense()


def test_forward_dense_square():
    assert pin_forward_dense(H=48, I=48)


def test_forward_single_expert_is_dense_swiglu_mlp():
    """E = 1, k = 1, w = 1: a dense SwiGLU MLP (torch fp64 F.linear / F.silu)."""
    hidden, w1, w2, _ = make_inputs(7, 128, 64, 1, seed=7)
    ids = np.zeros((7, 1), np.int32)
    w = np.ones((7, 1))
    x = hidden.double()
    h = torch.nn.functional.linear(x, w1[0].double())
    ref = torch.nn.functional.linear(torch.nn.functional.silu(h[:, :64]) * h[:, 64:],
                                     w2[0].double()).numpy()
    assert close(oracle.moe_token_loop(hidden, w1, w2, w, ids), ref)
    assert close(oracle.moe_expert_loop(hidden, w1, w2, w, ids), ref)


def test_forward_formulations_agree():
    hidden, w1, w2, logits = make_inputs(33, 96, 64, 8, seed=8)
    ids, w = oracle.route(logits.numpy(), 3, True)
    a = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    b = oracle.moe_expert_loop(hidden, w1, w2, w, ids)
    assert close(a, b)


def test_forward_zero_token_gives_zero_row():
    hidden, w1, w2, logits = make_inputs(6, 64, 32, 4, seed=9)
    hidden[2] = 0
    ids, w = oracle.route(logits.numpy(), 2, True)
    for out in (oracle.moe_token_loop(hidden, w1, w2, w, ids),
                oracle.moe_expert_loop(hidden, w1, w2, w, ids)):
        assert np.all(out[2] == 0.0)
        assert np.abs(out[[0, 1, 3]]).max() > 0


def test_forward_relabel_experts():
    """Permuting the expert slices of w1/w2 together with the ids leaves the
    output unchanged."""
    hidden, w1, w2, logits = make_inputs(20, 64, 32, 6, seed=10)
    ids, w = oracle.route(logits.numpy(), 2, True)
    perm = np.array([3, 5, 0, 1, 4, 2])
    inv = np.argsort(perm)
    w1p, w2p = w1[torch.tensor(inv)], w2[torch.tensor(inv)]
    ids_p = perm[ids].astype(np.int32)
    a = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    b = oracle.moe_token_loop(hidden, w1p, w2p, w, ids_p)
    assert close(a, b)


def test_forward_linear_in_weights():
    hidden, w1, w2, logits = make_inputs(10, 64, 32, 4, seed=11)
    ids, w = oracle.route(logits.numpy(), 2, True)
    a = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    b = oracle.moe_token_loop(hidden, w1, w2, 2.5 * w, ids)
    assert close(b, 2.5 * a)


def test_forward_duplicate_ids_sum_weights():
    """A token routed twice to one expert gets the summed weight, as in the
    per-expert loop of atrex-bench #009 reference.py."""
    hidden, w1, w2, _ = make_inputs(4, 64, 32, 3, seed=12)
    ids2 = np.array([[1, 1], [0, 2], [2, 2], [0, 0]], np.int32)
    w2v = np.array([[0.25, 0.5], [0.5, 0.5], [1.0, 2.0], [0.1, 0.2]])
    ids1 = ids2[:, :1].copy()
    ids1[1, 0] = -1                       # row 1 is checked separately
    w1v = w2v.sum(1, keepdims=True)
    a = oracle.moe_token_loop(hidden, w1, w2, w2v, ids2)
    b = oracle.moe_expert_loop(hidden, w1, w2, w2v, ids2)
    c = oracle.moe_token_loop(hidden, w1, w2, w1v, ids1)
    rows = [0, 2, 3]
    assert close(a[rows], c[rows]) and close(b[rows], c[rows])


def test_activation_variants_against_torch():
    assert pin_activation_library()


def test_swigluoai_clamps():
    assert pin_swigluoai_clamped()


def test_b1_with_zero_w1_is_closed_form():
    assert pin_b1_with_zero_w1()


def test_b2_with_zero_w2_is_weighted_bias_sum():
    assert pin_b2_with_zero_w2()


def test_variant_formulations_agree():
    assert pin_variants_formulations_agree()


def test_e4m3_decoder_golden_values(golden_dir):
    """Hand-derived E4M3 values (tests/golden/e4m3_codes.json)."""
    with open(os.path.join(golden_dir, "e4m3_codes.json")) as f:
        doc = json.load(f)
    for code, want, why in doc["cases"]:
        got = oracle.e4m3_to_double(int(code, 16))
        if want == "nan":
            assert math.isnan(got), (code, why)
        else:
            assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), \
                (code, got, want, why)


def test_e4m3_decoder_matches_torch():
    assert pin_e4m3_decoder()


def test_fp8_forward_equals_bf16_forward_of_dequantised_weights():
    assert pin_fp8_equals_bf16_of_dequantised()


def test_fp8_w2_scale_linearity():
    assert pin_fp8_w2_scale_linearity()


def test_fp8_block_must_divide():
    hidden, q1, s1, q2, s2, block, w, ids = _fp8_case(T=2)
    with pytest.raises(ValueError):
        oracle.moe_token_loop_fp8(hidden, q1, s1, q2, s2, 96, w, ids)


def test_unknown_activation_rejected():
    hidden, w1, w2, logits = make_inputs(2, 64, 32, 2, seed=25)
    ids, w = oracle.route(logits.numpy(), 1, True)
    with pytest.raises(ValueError):
        oracle.moe_token_loop(hidden, w1, w2, w, ids, act="relu")


def test_forward_invalid_ids_skipped():
    hidden, w1, w2, _ = make_inputs(3, 64, 32, 4, seed=13)
    ids = np.array([[1, 9], [-1, 2], [-5, 4]], np.int32)
    w = np.array([[0.5, 0.5], [0.3, 0.7], [0.5, 0.5]])
    a = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    b = oracle.moe_expert_loop(hidden, w1, w2, w, ids)
    ref = dense_numpy(hidden, w1, w2, np.where((ids >= 0) & (ids < 4), w, 0.0),
                      np.clip(ids, 0, 3))
    assert close(a, ref) and close(b, ref)
    assert np.all(a[2] == 0.0)


def test_forward_row_sampling_matches_full():
    hidden, w1, w2, logits = make_inputs(17, 64, 32, 5, seed=14)
    ids, w = oracle.route(logits.numpy(), 2, True)
    full = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    rows = [16, 0, 5, 5]
    part = oracle.moe_token_loop(hidden, w1, w2, w, ids, rows=rows)
    assert np.array_equal(part, full[rows])


def test_forward_empty_batch():
    hidden, w1, w2, logits = make_inputs(0, 64, 32, 4, seed=15)
    ids = np.zeros((0, 2), np.int32)
    w = np.zeros((0, 2))
    assert oracle.moe_token_loop(hidden, w1, w2, w, ids).shape == (0, 64)
    assert oracle.moe_expert_loop(hidden, w1, w2, w, ids).shape == (0, 64)
    rows, offs = oracle.permute(ids, 4)
    assert rows.shape == (0,) and offs.tolist() == [0, 0, 0, 0, 0]


# Each planted mistake and the pins expected to catch it (at least one must).
MUTATIONS = {
    1: "gate and up rows of w1 swapped",
    2: "w2 read as [I, H] instead of [H, I]",
    3: "renormalisation dropped",
    4: "ties broken towards the highest index",
    5: "permutation visits indices from the back (unstable)",
    6: "gate and up biases of b1 swapped",
    7: "b2 added once per expert after the top-k weighting",
    8: "gelu in its erf form instead of the tanh form",
    9: "FP8 scale block chosen by the index modulo the block count",
    10: "E4M3 exponent bias 8 instead of 7",
}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(mutation, golden_dir):
    oracle.build(mutation)
    results = {
        "golden_route": pin_golden_route(golden_dir, mutation),
        "golden_forward": pin_golden_forward(golden_dir, mutation),
        "golden_permute": pin_golden_permute(golden_dir, mutation),
        "route_bruteforce": pin_route_bruteforce(mutation),
        "route_library": pin_route_library(mutation),
        "permute_library": pin_permute_library(mutation),
        "forward_dense": pin_forward_dense(mutation) and pin_forward_dense(mutation, H=48, I=48),
        "activation_library": pin_activation_library(mutation),
        "swigluoai_clamped": pin_swigluoai_clamped(mutation),
        "b1_zero_w1": pin_b1_with_zero_w1(mutation),
        "b2_zero_w2": pin_b2_with_zero_w2(mutation),
        "variants_agree": pin_variants_formulations_agree(mutation),
        "e4m3_decoder": pin_e4m3_decoder(mutation),
        "fp8_dequantised": pin_fp8_equals_bf16_of_dequantised(mutation),
        "fp8_w2_linearity": pin_fp8_w2_scale_linearity(mutation),
    }
    assert oracle._load(mutation).oracle_mutation() == mutation
    caught = [k for k, v in results.items() if not v]
    assert caught, f"planted mistake {MUTATIONS[mutation]!r} passed every pin"
