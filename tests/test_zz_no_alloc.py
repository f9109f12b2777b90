"""The no-allocation small-batch entry point (moe_forward_small_noalloc).

It serves callers that reserve all device memory when they start and cannot
allocate later (or cannot afford the device-wide synchronisation of
cudaFree).  Called here through the C ABI, twice in a row: it runs the same
kernel as moe_forward's small-batch path, so its output must equal that of
moe_forward bit for bit, and both must pass the oracle's tolerance gates.
Kept in a file that pytest collects last.
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_softmax_b200 as moe
import oracle
from moe_inputs import make_inputs
from moe_testutil import assert_output_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _call_noalloc(hidden, w1, w2, w, ids, out):
    T, H = hidden.shape
    E, twoI, _ = w1.shape
    return moe._lib.moe_forward_small_noalloc(
        hidden.data_ptr(), w1.data_ptr(), w2.data_ptr(), w.data_ptr(), ids.data_ptr(),
        out.data_ptr(), T, H, twoI // 2, E, ids.shape[1], torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("T,H,I,E,k", [(1, 2048, 768, 128, 8), (5, 1024, 512, 16, 4),
                                       (16, 512, 256, 8, 2)])
def test_noalloc_matches_moe_forward_on_two_calls(T, H, I, E, k):
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=77 + T)
    ids_r, w_r = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop(hidden, w1, w2, w_r, ids_r)
    hidden, w1, w2 = hidden.cuda(), w1.cuda(), w2.cuda()
    ids = torch.as_tensor(ids_r).cuda()
    w = torch.as_tensor(w_r.astype(np.float32)).cuda()
    prev = moe.set_small_t_max(16)
    try:
        want = moe.moe_forward(hidden, w1, w2, w, ids)
    finally:
        moe.set_small_t_max(prev)
    torch.cuda.synchronize()
    want = want.cpu().numpy()
    assert_output_close(want, ref, f"moe_forward T={T}")
    for _ in range(2):
        out = torch.full((T, H), float("nan"), device="cuda")
        assert _call_noalloc(hidden, w1, w2, w, ids, out) == moe.MOE_OK
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        # the same kernel on the same inputs: identical bits
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
        assert_output_close(got, ref, f"noalloc T={T}")


def test_noalloc_rejects_requests_beyond_its_scratch():
    H, I, E = 256, 4096, 8
    hidden, w1, w2, logits = [t.cuda() for t in make_inputs(17, H, I, E, seed=1)]
    ids, w = moe.moe_route(logits, 2, True)
    out = torch.empty(17, H, device="cuda")
    assert _call_noalloc(hidden, w1, w2, w, ids, out) == moe.MOE_ERR_SCRATCH_LIMIT  # T > 16
    ids9, w9 = ids[:9].contiguous(), w[:9].contiguous()
    # 9 * 2 * 4096 = 73728 fits; with k = 8 it would not (9 * 8 * 4096 > 262144)
    assert _call_noalloc(hidden[:9].contiguous(), w1, w2, w9, ids9, out[:9]) == moe.MOE_OK
    ids8, w8 = moe.moe_route(logits[:9].contiguous(), 8, True)
    assert _call_noalloc(hidden[:9].contiguous(), w1, w2, w8, ids8, out[:9]) == \
        moe.MOE_ERR_SCRATCH_LIMIT
    assert "scratch" in moe.error_string(moe.MOE_ERR_SCRATCH_LIMIT)
