"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Gates: routing ids, permutation indices and expert offsets bit-exact;
routing weights within 1e-6 + 1e-5*|w|; forward output within
1e-2 + 1e-2*|ref| elementwise plus the diagnostic gates of moe_testutil.
Shapes span several 128-row tiles with ragged tails, empty experts, the
small-T path and both GEMM paths; the five named workloads run at full size
(all tokens for the tiny and decode workloads, sampled tokens that the
oracle computes one by one for the three prefill workloads).
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_softmax_b200 as moe
import oracle
from moe_inputs import SHAPES, TABLE_SHAPES, make_biases, make_inputs, make_shape_inputs
from moe_testutil import assert_output_close, assert_weights_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    # every batch of up to 16 tokens takes the small-T path unless a test
    # forces the GEMM path (the default threshold is lower)
    prev = moe.set_small_t_max(16)
    yield
    moe.set_small_t_max(prev)


def gpu_route(logits_cpu, k, renorm=True):
    ids, w = moe.moe_route(logits_cpu.cuda(), k, renorm)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


def gpu_forward(hidden, w1, w2, w, ids, act="silu", b1=None, b2=None):
    """Inputs may live on CPU or GPU; routing comes in as numpy."""
    dev = torch.device("cuda")
    # NaN-filled: every element of out must be written by the call
    out = torch.full((hidden.shape[0], hidden.shape[1]), float("nan"), device=dev)
    out = moe.moe_forward(hidden.to(dev), w1.to(dev), w2.to(dev),
                          torch.as_tensor(np.asarray(w, np.float32)).to(dev),
                          torch.as_tensor(np.asarray(ids, np.int32)).to(dev), out=out, act=act,
                          b1=None if b1 is None else b1.to(dev),
                          b2=None if b2 is None else b2.to(dev))
    torch.cuda.synchronize()
    return out.cpu().numpy()


def check_status_clean():
    assert moe.get_device_status() == 0


# ------------------------------------------------------------------ routing
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_route_workloads(name):
    s = SHAPES[name]
    logits = torch.randn(s.T, s.E, generator=torch.Generator().manual_seed(0))
    for renorm in (True, False):
        ids_r, w_r = oracle.route(logits.numpy(), s.k, renorm)
        ids_g, w_g = gpu_route(logits, s.k, renorm)
        assert np.array_equal(ids_g, ids_r)
        assert_weights_close(w_g, w_r, name)


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (3, 2, 2), (257, 37, 5), (100, 100, 16),
                                   (64, 256, 8), (33, 512, 3), (17, 1024, 16), (9, 8, 8)])
def test_route_shapes(T, E, k):
    g = torch.Generator().manual_seed(T * 1000 + E)
    logits = torch.randn(T, E, generator=g)
    ids_r, w_r = oracle.route(logits.numpy(), k, True)
    ids_g, w_g = gpu_route(logits, k, True)
    assert np.array_equal(ids_g, ids_r)
    assert_weights_close(w_g, w_r)


def test_route_ties_and_neg_inf():
    g = torch.Generator().manual_seed(5)
    logits = torch.randint(-2, 3, (300, 40), generator=g).float()
    logits[::7, 3:30] = -float("inf")
    logits[1, :] = 0.0
    for k in (1, 4, 40):
        ids_r, w_r = oracle.route(logits.numpy(), k, False)
        ids_g, w_g = gpu_route(logits, k, False)
        assert np.array_equal(ids_g, ids_r)
        assert_weights_close(w_g, w_r)


def test_route_empty():
    ids, w = moe.moe_route(torch.empty(0, 8, device="cuda"), 2)
    assert ids.shape == (0, 2)


# ------------------------------------------------------------------ permutation
def _perm_ids(kind, T, k, E, seed):
    """Expert ids for the grouping tests: uniform with ids outside [0, E)
    mixed in, routed (softmax top-k of randn logits, distinct per token),
    every id on one expert, or a heavily skewed mix."""
    g = torch.Generator().manual_seed(seed)
    if kind == "uniform_invalid":
        return torch.randint(-1, E + 1, (T, k), generator=g, dtype=torch.int32).numpy()
    if kind == "routed":
        ids, _ = oracle.route(torch.randn(T, E, generator=g).numpy(), k, True)
        return ids
    if kind == "one_expert":
        return np.full((T, k), E - 1, np.int32)
    if kind == "skewed":
        # three quarters of the ids on expert 0, the rest spread, a few invalid
        ids = torch.randint(0, E, (T, k), generator=g, dtype=torch.int32).numpy()
        u = torch.rand(T, k, generator=g).numpy()
        ids[u < 0.75] = 0
        ids[u > 0.995] = -5
        return ids
    raise ValueError(kind)


def _oracle_inverse(rows_r, nv, n):
    """inv[i] = position of flat index i among the nv grouped entries, -1
    for an entry whose id is outside [0, E)."""
    inv = np.full(n, -1, np.int64)
    inv[rows_r[:nv]] = np.arange(nv)
    return inv


PERMUTE_CASES = [
    # (ids kind, T, k, E)
    ("uniform_invalid", 1, 1, 1),
    ("uniform_invalid", 5, 2, 3),
    ("uniform_invalid", 1024, 2, 8),
    ("uniform_invalid", 1025, 2, 8),
    ("routed", 64, 2, 8),             # the tiny workload's routing
    ("routed", 1979, 2, 8),           # the 8-expert prefill's routing
    ("routed", 1024, 8, 128),         # exactly 8192 entries
    ("uniform_invalid", 4096, 2, 8),  # exactly 8192 entries, invalid ids
    ("one_expert", 4096, 2, 8),       # every entry on one expert
    ("one_expert", 1, 16, 1024),
    ("skewed", 2000, 4, 64),
    ("uniform_invalid", 512, 16, 1024),  # E = 1024, 8192 entries
    ("uniform_invalid", 4097, 2, 8),  # 8194 entries: only the three-kernel grouping
    ("routed", 8192, 8, 128),         # the thin prefill's routing
    ("uniform_invalid", 3000, 7, 1024),
    ("skewed", 15381, 2, 8),
    ("uniform_invalid", 100, 16, 1000),
]


@pytest.mark.parametrize("kind,T,k,E", PERMUTE_CASES)
def test_permute_bit_exact_both_kernels(kind, T, k, E):
    """sorted_rows, expert_offsets and the inverse permutation bit for bit
    against the oracle's stable counting sort, from the kernel moe_forward
    uses (auto) and from each grouping kernel that can take this size."""
    ids = _perm_ids(kind, T, k, E, seed=T + 7 * E + k)
    n = T * k
    rows_r, offs_r = oracle.permute(ids, E)
    nv = int(offs_r[-1])
    inv_r = _oracle_inverse(rows_r, nv, n)
    kernels = ["auto", "multi"] + (["single"] if n <= 8192 else [])
    ids_d = torch.as_tensor(ids).cuda()
    for kern in kernels:
        rows_g, offs_g, inv_g, _ = moe.moe_permute_ex(ids_d, E, kernel=kern)
        torch.cuda.synchronize()
        assert np.array_equal(offs_g.cpu().numpy(), offs_r), kern
        rows_g = rows_g.cpu().numpy()
        assert np.array_equal(rows_g[:nv], rows_r[:nv]), kern
        assert np.all(rows_g[nv:] == -1), kern  # positions past the valid ids untouched
        assert np.array_equal(inv_g.cpu().numpy(), inv_r), kern
    # the plain export runs the same grouping
    rows_p, offs_p = moe.moe_permute(ids_d, E)
    torch.cuda.synchronize()
    assert np.array_equal(offs_p.cpu().numpy(), offs_r)
    assert np.array_equal(rows_p.cpu().numpy()[:nv], rows_r[:nv])


@pytest.mark.parametrize("kind,T,k,E,H", [
    ("routed", 64, 2, 8, 256),
    ("routed", 1979, 2, 8, 2048),
    ("uniform_invalid", 4096, 2, 8, 128),   # 8192 entries: one kernel, many CTAs
    ("routed", 4097, 2, 8, 256),            # three kernels and the separate row copy
    ("one_expert", 300, 1, 4, 384),
])
def test_permute_sorted_row_copy(kind, T, k, E, H):
    """The expert-sorted copy of the hidden rows the top-k <= 2 GEMM path
    loads (xs[r] = hidden[sorted_rows[r] // k]), bit for bit, from every
    grouping kernel that can take this size."""
    ids = _perm_ids(kind, T, k, E, seed=3 * T + H)
    hidden = (torch.randn(T, H, generator=torch.Generator().manual_seed(T)) * 0.1).to(torch.bfloat16)
    rows_r, offs_r = oracle.permute(ids, E)
    nv = int(offs_r[-1])
    want = hidden[torch.as_tensor(rows_r[:nv] // k, dtype=torch.long)]
    kernels = ["auto", "multi"] + (["single"] if T * k <= 8192 else [])
    for kern in kernels:
        _, offs_g, _, xs = moe.moe_permute_ex(torch.as_tensor(ids).cuda(), E, kernel=kern,
                                              hidden=hidden.cuda())
        torch.cuda.synchronize()
        assert np.array_equal(offs_g.cpu().numpy(), offs_r), kern
        xs = xs.cpu()
        assert torch.equal(xs[:nv].view(torch.int16), want.view(torch.int16)), kern
        assert torch.all(xs[nv:].view(torch.int16) == 0), kern


# ------------------------------------------------------------------ forward
CASES = [
    # (T, H, I, E, k)            what it covers
    (64, 256, 128, 8, 2),      # the tiny workload
    (300, 512, 256, 8, 2),     # several m-tiles per expert, ragged tails
    (333, 384, 384, 16, 4),    # H = 3*128: GEMM2's last n-tile is half valid
    (100, 256, 128, 128, 8),   # most experts hold < 1 tile, many empty
    (17, 256, 256, 4, 4),      # k = E
    (129, 128, 128, 1, 1),     # one expert, one slot
    (257, 640, 512, 32, 6),    # odd k, E not a power of two multiple of tiles
]


@pytest.mark.parametrize("T,H,I,E,k", CASES)
@pytest.mark.parametrize("path", ["auto", "gemm"])
def test_forward_parity(T, H, I, E, k, path):
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=T + H)
    ids, w = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    prev = moe.set_small_t_max(0 if path == "gemm" else 16)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids)
    finally:
        moe.set_small_t_max(prev)
    assert_output_close(out, ref, f"T={T} H={H} I={I} E={E} k={k} {path}")
    check_status_clean()


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8, 16])
@pytest.mark.parametrize("path", ["small_t", "gemm"])
def test_forward_small_batches(T, path):
    H, I, E, k = 2048, 768, 128, 8
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=40 + T)
    ids, w = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    prev = moe.set_small_t_max(16 if path == "small_t" else 0)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids)
    finally:
        moe.set_small_t_max(prev)
    assert_output_close(out, ref, f"T={T} {path}")
    check_status_clean()


@pytest.mark.parametrize("T", [1, 3])
def test_forward_small_batches_wide_hidden(T):
    """The GEMV path at H = 4096, I = 384 (the thin experts): 28 output rows
    per CTA, the last CTAs with a partial slice or none."""
    H, I, E, k = 4096, 384, 128, 8
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=70 + T)
    ids, w = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    out = gpu_forward(hidden, w1, w2, w, ids)
    assert_output_close(out, ref, f"T={T} H={H} I={I}")
    check_status_clean()


def test_forward_small_t_shared_and_duplicate_experts():
    """Several tokens on one expert, and one token routed twice to an expert."""
    T, H, I, E, k = 6, 512, 256, 4, 3
    hidden, w1, w2, _ = make_inputs(T, H, I, E, seed=3)
    ids = np.array([[0, 1, 2], [0, 1, 2], [2, 2, 0], [3, 3, 3], [1, 0, 3], [0, 0, 1]], np.int32)
    w = np.random.default_rng(0).uniform(0.1, 1.0, (T, k))
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    for small in (16, 0):
        prev = moe.set_small_t_max(small)
        try:
            out = gpu_forward(hidden, w1, w2, w, ids)
        finally:
            moe.set_small_t_max(prev)
        assert_output_close(out, ref, f"small_t_max={small}")


@pytest.mark.parametrize("small,k", [(16, 2), (0, 2), (0, 4)])
def test_forward_invalid_ids_are_skipped_and_flagged(small, k):
    """k = 2 on the GEMM path flags bad ids in the grouping (GEMM2 adds into
    out); k = 4 also goes through the separate combine."""
    T, H, I, E = 12, 256, 128, 8
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=11)
    ids, w = oracle.route(logits.numpy(), k, True)
    ids[3, 1] = -1
    ids[7, 0] = E
    ids[9, :] = 99  # no valid slot -> zero row
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    moe.get_device_status()
    prev = moe.set_small_t_max(small)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids)
    finally:
        moe.set_small_t_max(prev)
    assert_output_close(out, ref)
    assert np.all(out[9] == 0.0)
    assert moe.get_device_status() & moe.MOE_STATUS_BAD_ID


@pytest.mark.parametrize("small", [16, 0])
def test_forward_zero_token_gives_zero_row(small):
    T, H, I, E, k = 20, 256, 128, 8, 2
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=12)
    hidden[4] = 0
    ids, w = oracle.route(logits.numpy(), k, True)
    prev = moe.set_small_t_max(small)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids)
    finally:
        moe.set_small_t_max(prev)
    assert np.all(out[4] == 0.0)


@pytest.mark.parametrize("T,H,I,E,k", [(64, 256, 128, 8, 2), (600, 512, 256, 8, 2),
                                        (600, 512, 256, 8, 1), (300, 384, 256, 16, 4)])
def test_forward_deterministic(T, H, I, E, k):
    """Identical bits on repeated calls: with k <= 2 GEMM2 adds two rounded
    products onto zero in whatever order the tiles finish (a commutative
    sum), with k > 2 the combine sums in fixed order."""
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=5)
    ids, w = oracle.route(logits.numpy(), k, True)
    prev = moe.set_small_t_max(0)
    try:
        a = gpu_forward(hidden, w1, w2, w, ids)
        b = gpu_forward(hidden, w1, w2, w, ids)
        c = gpu_forward(hidden, w1, w2, w, ids)
    finally:
        moe.set_small_t_max(prev)
    assert np.array_equal(a, b) and np.array_equal(a, c)


@pytest.mark.parametrize("T,H,I,E,k", [(1979, 2048, 2048, 8, 2), (2000, 1024, 384, 64, 8)])
def test_forward_beside_other_work(T, H, I, E, k):
    """The forward while another stream keeps the SMs busy with matrix
    products (finite work: CTAs it holds back start when it ends, well
    inside the wait limit): the result is bit-identical to the forward run
    alone and no bounded wait runs out (which would raise the timeout bit)."""
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=31)
    ids, w = oracle.route(logits.numpy(), k, True)
    dev = torch.device("cuda")
    args = [hidden.to(dev), w1.to(dev), w2.to(dev),
            torch.as_tensor(w.astype(np.float32)).to(dev), torch.as_tensor(ids).to(dev)]
    prev = moe.set_small_t_max(0)
    try:
        alone = moe.moe_forward(*args)
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        a = torch.randn(4096, 4096, device=dev, dtype=torch.bfloat16)
        outs = []
        for _ in range(3):
            with torch.cuda.stream(side):
                for _ in range(20):
                    a = (a @ a).clamp_(-1, 1)
            outs.append(moe.moe_forward(*args))
        torch.cuda.synchronize()
    finally:
        moe.set_small_t_max(prev)
    check_status_clean()
    for o in outs:
        assert torch.equal(o, alone)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids, rows=np.arange(0, T, 7))
    assert_output_close(alone.cpu().numpy()[::7], ref, f"T={T} k={k}")


def test_forward_gemm_duplicate_slots_top2():
    """A token routed twice to one expert: two rows of that expert's group
    added into the same output row (summed weight in atrex-bench #009)."""
    T, H, I, E, k = 40, 256, 256, 4, 2
    hidden, w1, w2, _ = make_inputs(T, H, I, E, seed=21)
    rng = np.random.default_rng(1)
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    ids[::3, 1] = ids[::3, 0]
    w = rng.uniform(0.1, 1.0, (T, k))
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    prev = moe.set_small_t_max(0)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids)
    finally:
        moe.set_small_t_max(prev)
    assert_output_close(out, ref)
    check_status_clean()


def test_forward_empty_batch():
    out = moe.moe_forward(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"),
                          torch.zeros(8, 256, 256, dtype=torch.bfloat16, device="cuda"),
                          torch.zeros(8, 256, 128, dtype=torch.bfloat16, device="cuda"),
                          torch.empty(0, 2, device="cuda"),
                          torch.empty(0, 2, dtype=torch.int32, device="cuda"))
    assert out.shape == (0, 256)


def test_end_to_end_route_then_forward():
    """GPU routing feeds the GPU forward; the oracle routes for itself."""
    for name in ("tiny",):
        s = SHAPES[name]
        hidden, w1, w2, logits = make_shape_inputs(s)
        ids_r, w_r = oracle.route(logits.numpy(), s.k, True)
        ref = oracle.moe_token_loop(hidden, w1, w2, w_r, ids_r)
        ids_g, w_g = moe.moe_route(logits.cuda(), s.k, True)
        out = moe.moe_forward(hidden.cuda(), w1.cuda(), w2.cuda(), w_g, ids_g)
        torch.cuda.synchronize()
        assert np.array_equal(ids_g.cpu().numpy(), ids_r)
        assert_output_close(out.cpu().numpy(), ref, name)


# ------------------------------------------------------------------ epilogue variants
VARIANT_CASES = [
    (64, 256, 128, 8, 2),      # tiny: one-kernel grouping, both GEMMs in one launch
    (333, 384, 384, 16, 4),    # k > 2: separate GEMM launches, fp32 P, combine
    (100, 256, 128, 128, 8),   # many experts below one tile
]


def _biases(which, E, H, I, seed):
    b1, b2 = make_biases(E, H, I, seed=seed)
    return (b1 if which in ("b1", "both") else None), (b2 if which in ("b2", "both") else None)


@pytest.mark.parametrize("T,H,I,E,k", VARIANT_CASES)
@pytest.mark.parametrize("act", ["silu", "gelu", "swigluoai"])
@pytest.mark.parametrize("bias", ["none", "b1", "b2", "both"])
def test_forward_variants(T, H, I, E, k, act, bias):
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=T + 7)
    b1, b2 = _biases(bias, E, H, I, seed=T)
    ids, w = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids, act=act, b1=b1, b2=b2)
    prev = moe.set_small_t_max(0)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids, act, b1, b2)
    finally:
        moe.set_small_t_max(prev)
    assert_output_close(out, ref, f"T={T} E={E} k={k} act={act} bias={bias}")
    check_status_clean()


@pytest.mark.parametrize("T", [1, 4])
@pytest.mark.parametrize("act", ["silu", "gelu", "swigluoai"])
def test_forward_variants_small_t(T, act):
    H, I, E, k = 2048, 768, 128, 8
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=50 + T)
    b1, b2 = make_biases(E, H, I, seed=T)
    ids, w = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids, act=act, b1=b1, b2=b2)
    for bb1, bb2 in ((b1, b2), (None, None)):
        r = ref if bb1 is not None else oracle.moe_token_loop(hidden, w1, w2, w, ids, act=act)
        out = gpu_forward(hidden, w1, w2, w, ids, act, bb1, bb2)
        assert_output_close(out, r, f"T={T} act={act} bias={bb1 is not None}")
    check_status_clean()


@pytest.mark.parametrize("small", [16, 0])
def test_forward_swigluoai_clamps(small):
    """Projections of a few units: many gate values above 7 and up values
    beyond +-7, so both clips of swigluoai decide the result.  w2 is scaled
    by 2^-7 (exact in bf16) so that the output, and with it the rounding of
    the bf16 intermediate of the GEMM path (activations up to 56), stays at
    the size the absolute tolerance was derived for."""
    T, H, I, E, k = 12, 256, 128, 8, 2
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=13, hidden_scale=12.0)
    w2 = w2 * 2.0 ** -7
    ids, w = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids, act="swigluoai")
    g = hidden.double() @ w1[0, :I].double().T
    assert (g > 7).float().mean() > 0.15  # the clip is really exercised
    prev = moe.set_small_t_max(small)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids, "swigluoai")
    finally:
        moe.set_small_t_max(prev)
    assert_output_close(out, ref, f"small_t_max={small}")


def test_forward_ex_default_equals_forward():
    """moe_forward_ex with silu and no biases is moe_forward, bit for bit."""
    T, H, I, E, k = 300, 512, 256, 8, 2
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=17)
    ids, w = oracle.route(logits.numpy(), k, True)
    dev = torch.device("cuda")
    args = [hidden.to(dev), w1.to(dev), w2.to(dev),
            torch.as_tensor(w.astype(np.float32)).to(dev), torch.as_tensor(ids).to(dev)]
    a = moe.moe_forward(*args)
    b = torch.empty_like(a)
    rc = moe._lib.moe_forward_ex(args[0].data_ptr(), args[1].data_ptr(), args[2].data_ptr(),
                                 None, None, moe.MOE_ACT_SILU, args[3].data_ptr(),
                                 args[4].data_ptr(), b.data_ptr(), T, H, I, E, k,
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == moe.MOE_OK
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ------------------------------------------------------------------ FP8 weights
def gpu_forward_fp8(hidden, q1, s1, q2, s2, block, w, ids):
    dev = torch.device("cuda")
    out = torch.full((hidden.shape[0], hidden.shape[1]), float("nan"), device=dev)
    out = moe.moe_forward_fp8(hidden.to(dev), q1.to(dev), s1.to(dev), q2.to(dev), s2.to(dev),
                              block, torch.as_tensor(np.asarray(w, np.float32)).to(dev),
                              torch.as_tensor(np.asarray(ids, np.int32)).to(dev), out=out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("T,H,I,E,k,block,path", [
    (1, 2048, 768, 128, 8, 256, "small_t"),    # decode
    (4, 2048, 768, 128, 8, 128, "small_t"),    # several tokens, blocks of 128
    (3, 512, 256, 4, 2, 256, "small_t"),       # tokens sharing experts
    (4, 2048, 768, 128, 8, 256, "gemm"),
    (64, 256, 128, 8, 2, 128, "gemm"),         # tiny: one-launch GEMMs
    (100, 384, 384, 16, 4, 128, "gemm"),       # k > 2: P and combine, half n-tile
])
def test_forward_fp8(T, H, I, E, k, block, path):
    from moe_inputs import make_fp8_weights
    hidden, _, _, logits = make_inputs(T, H, I, E, seed=60 + T)
    q1, s1, q2, s2 = make_fp8_weights(E, H, I, block, seed=T)
    ids, w = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop_fp8(hidden, q1, s1, q2, s2, block, w, ids)
    prev = moe.set_small_t_max(16 if path == "small_t" else 0)
    try:
        out = gpu_forward_fp8(hidden, q1, s1, q2, s2, block, w, ids)
    finally:
        moe.set_small_t_max(prev)
    assert_output_close(out, ref, f"T={T} H={H} I={I} E={E} k={k} block={block} {path}")
    check_status_clean()


@pytest.mark.parametrize("name,block", [("decode", 256), ("prefill_8e", 256),
                                        ("prefill_thin", 128)])
def test_forward_fp8_full_size(name, block):
    from moe_inputs import make_fp8_weights
    s = SHAPES[name]
    hidden, _, _, logits = make_shape_inputs(s, device="cuda")
    q1, s1, q2, s2 = make_fp8_weights(s.E, s.H, s.I, block, seed=5, device="cuda")
    ids_r, w_r = oracle.route(logits.cpu().numpy(), s.k, True)
    out = moe.moe_forward_fp8(hidden, q1, s1, q2, s2, block,
                              torch.as_tensor(w_r.astype(np.float32)).cuda(),
                              torch.as_tensor(ids_r).cuda())
    torch.cuda.synchronize()
    rows = np.arange(s.T) if s.T <= 64 else _sample_rows(s.T, 6, 7)
    ref = oracle.moe_token_loop_fp8(hidden.cpu(), q1.cpu(), s1.cpu(), q2.cpu(), s2.cpu(), block,
                                    w_r, ids_r, rows=rows)
    assert_output_close(out.cpu().numpy()[rows], ref, f"{name} fp8")
    check_status_clean()
    assert torch.isfinite(out).all()


# ------------------------------------------------------------------ full-size workloads
def _sample_rows(T, n, seed):
    rng = np.random.default_rng(seed)
    rows = {0, T - 1} | set(rng.choice(T, size=min(n, T), replace=False).tolist())
    return np.array(sorted(rows), np.int64)


def _tail_tile_tokens(ids, E, k, tile=256):
    """Tokens of every row in each expert's last, partial m-tile of the
    expert-sorted order (where the GEMM epilogues mask rows)."""
    rows_r, offs_r = oracle.permute(ids, E)
    toks = set()
    for e in range(E):
        lo, hi = int(offs_r[e]), int(offs_r[e + 1])
        full = lo + (hi - lo) // tile * tile
        toks.update((rows_r[full:hi] // k).tolist())
    return toks


def full_size_rows(s, ids):
    """Rows of a full-size workload compared with the oracle: every row up
    to the thin prefill (8192 tokens, ~30 s of oracle time on 16 cores);
    for the large prefill every token in an expert's last partial m-tile,
    the first and last token, and 2000 random tokens."""
    if s.T <= 8192:
        return np.arange(s.T)
    rng = np.random.default_rng(11)
    toks = _tail_tile_tokens(ids, s.E, s.k) | {0, s.T - 1}
    toks |= set(rng.choice(s.T, size=2000, replace=False).tolist())
    return np.array(sorted(toks), np.int64)


@pytest.mark.parametrize("name", ["decode", "prefill_8e", "prefill_thin", "prefill_big"])
def test_forward_full_size_workloads(name):
    s = SHAPES[name]
    hidden, w1, w2, logits = make_shape_inputs(s, device="cuda")
    logits_c = logits.cpu()
    ids_r, w_r = oracle.route(logits_c.numpy(), s.k, True)
    ids_g, w_g = moe.moe_route(logits, s.k, True)
    torch.cuda.synchronize()
    assert np.array_equal(ids_g.cpu().numpy(), ids_r)
    # the forward takes the oracle's routing so both sides compute the same sum
    out = moe.moe_forward(hidden, w1, w2, torch.as_tensor(w_r.astype(np.float32)).cuda(),
                          torch.as_tensor(ids_r).cuda())
    torch.cuda.synchronize()
    rows = full_size_rows(s, ids_r)
    print(f"{name}: {rows.size} of {s.T} rows compared with the oracle")
    ref = oracle.moe_token_loop(hidden.cpu(), w1.cpu(), w2.cpu(), w_r, ids_r, rows=rows)
    assert_output_close(out.cpu().numpy()[rows], ref, name)
    check_status_clean()
    # properties that hold at any size: every row written and finite
    assert torch.isfinite(out).all()


TABLE_ONLY = [n for n, s in TABLE_SHAPES.items()
              if (s.T, s.H, s.I, s.E, s.k) not in
              {(w.T, w.H, w.I, w.E, w.k) for w in SHAPES.values()}]


@pytest.mark.parametrize("name", TABLE_ONLY)
def test_forward_table_rows(name):
    """The other rows of the page's shapes table (and a two-token decode) at
    full size: routing bit-exact, sampled tokens against the oracle."""
    s = TABLE_SHAPES[name]
    hidden, w1, w2, logits = make_shape_inputs(s, seed=1, device="cuda")
    ids_r, w_r = oracle.route(logits.cpu().numpy(), s.k, True)
    ids_g, w_g = moe.moe_route(logits, s.k, True)
    out = moe.moe_forward(hidden, w1, w2, torch.as_tensor(w_r.astype(np.float32)).cuda(),
                          torch.as_tensor(ids_r).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(ids_g.cpu().numpy(), ids_r)
    rows = np.arange(s.T) if s.T <= 16 else _sample_rows(s.T, 6, 4)
    ref = oracle.moe_token_loop(hidden.cpu(), w1.cpu(), w2.cpu(), w_r, ids_r, rows=rows)
    assert_output_close(out.cpu().numpy()[rows], ref, name)
    check_status_clean()
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("name,act", [("decode", "gelu"), ("prefill_8e", "swigluoai"),
                                      ("prefill_thin", "gelu"), ("prefill_big", "swigluoai")])
def test_forward_full_size_variants(name, act):
    """The variant epilogues in the launch configuration of each workload
    (prefill_big: GEMM1 and GEMM2 as two launches), on sampled tokens."""
    s = SHAPES[name]
    hidden, w1, w2, logits = make_shape_inputs(s, device="cuda")
    b1, b2 = make_biases(s.E, s.H, s.I, seed=2, device="cuda")
    ids_r, w_r = oracle.route(logits.cpu().numpy(), s.k, True)
    out = moe.moe_forward(hidden, w1, w2, torch.as_tensor(w_r.astype(np.float32)).cuda(),
                          torch.as_tensor(ids_r).cuda(), act=act, b1=b1, b2=b2)
    torch.cuda.synchronize()
    rows = np.arange(s.T) if s.T <= 64 else _sample_rows(s.T, 10, 3)
    ref = oracle.moe_token_loop(hidden.cpu(), w1.cpu(), w2.cpu(), w_r, ids_r, rows=rows, act=act,
                                b1=b1.cpu(), b2=b2.cpu())
    assert_output_close(out.cpu().numpy()[rows], ref, f"{name} {act}")
    check_status_clean()
    assert torch.isfinite(out).all()


# ------------------------------------------------------------------ failure paths
def test_bounded_wait_times_out_without_hanging():
    moe.get_device_status()
    assert moe.debug_wait_timeout(2_000_000) == moe.MOE_ERR_TIMEOUT  # 2 ms
    assert moe.get_device_status() & moe.MOE_STATUS_TIMEOUT
    # the context is still usable afterwards
    test_forward_deterministic(64, 256, 128, 8, 2)
    check_status_clean()


@pytest.mark.parametrize("T,k,kinds", [(300, 2, {"gemm_fused"}), (300, 4, {"gemm1", "gemm2"}),
                                       (1, 8, {"small_t"})])
def test_timeline_records(T, k, kinds):
    """The debug timeline: every tile of the GEMM launches (or every CTA of
    the small-batch kernel) leaves its records, t0 <= t1, and the forward's
    result is the same with it on."""
    H, I, E = 512, 256, 16
    hidden, w1, w2, logits = [t.cuda() for t in make_inputs(T, H, I, E, seed=4)]
    ids, w = moe.moe_route(logits, k, True)
    ref = moe.moe_forward(hidden, w1, w2, w, ids)
    moe.timeline_start(1 << 14)
    try:
        out = moe.moe_forward(hidden, w1, w2, w, ids)
    finally:
        recs = moe.timeline_stop()
    assert torch.equal(out, ref)
    assert recs and {r["kind"] for r in recs} == kinds
    assert all(r["t0"] <= r["t1"] for r in recs)
    if "small_t" in kinds:
        ctas = {r["id"] for r in recs if r["role"] == "phase2"}
        assert len(ctas) == torch.cuda.get_device_properties(0).multi_processor_count
    else:
        for kind in kinds:  # each launch numbers its tiles from 0
            prod = [r for r in recs if r["kind"] == kind and r["role"] == "producer"
                    and r["sub"] == 0]
            assert len({r["id"] for r in prod}) == len(prod)  # each tile claimed once
            mma = {r["id"] for r in recs if r["kind"] == kind and r["role"] == "mma"}
            assert mma == {r["id"] for r in prod}
    summary = moe.timeline_summary(recs)
    assert all(v["n"] > 0 for v in summary.values())
    moe.moe_forward(hidden, w1, w2, w, ids)  # off again: nothing recorded, nothing breaks
    torch.cuda.synchronize()


def test_sync_each_stage_mode_and_profiler():
    s = SHAPES["tiny"]
    hidden, w1, w2, logits = make_shape_inputs(s)
    ids, w = oracle.route(logits.numpy(), s.k, True)
    prev = moe.set_sync_each_stage(True)
    moe.profile_reset()
    moe.profile_enable(True)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids)
    finally:
        moe.profile_enable(False)
        moe.set_sync_each_stage(prev)
    prof = moe.profile_read()
    # top-2: hidden rows copied into expert order, both GEMMs in one launch
    # that also adds into out, no separate combine
    for kname in ("group_gather", "gemm_fused"):
        assert prof[kname][0] == 1 and prof[kname][1] > 0
    assert "combine" not in prof and "gemm2" not in prof
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    assert_output_close(out, ref)

    T, H, I, E, k = 64, 256, 128, 8, 4
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=8)
    ids, w = oracle.route(logits.numpy(), k, True)
    prev = moe.set_sync_each_stage(True)
    moe.profile_reset()
    moe.profile_enable(True)
    try:
        out = gpu_forward(hidden, w1, w2, w, ids)
    finally:
        moe.profile_enable(False)
        moe.set_sync_each_stage(prev)
    prof = moe.profile_read()
    for kname in ("permute", "gemm1_swiglu", "gemm2", "combine"):
        assert prof[kname][0] == 1 and prof[kname][1] > 0
    assert_output_close(out, oracle.moe_token_loop(hidden, w1, w2, w, ids))
