"""The output gates reject plausible wrong outputs (negative controls, CPU)."""
import numpy as np
import torch

import oracle
from moe_inputs import make_inputs
from moe_testutil import gate_report, passes


def _case(T=64, H=256, I=128, E=8, k=2, seed=0):
    hidden, w1, w2, logits = make_inputs(T, H, I, E, seed=seed)
    ids, w = oracle.route(logits.numpy(), k, True)
    ref = oracle.moe_token_loop(hidden, w1, w2, w, ids)
    return hidden, w1, w2, ids, w, ref


def test_exact_passes():
    *_, ref = _case()
    assert passes(ref, ref)


def test_bf16_rounded_intermediate_passes():
    """Rounding act to bf16 (what the GPU path may do) stays inside the gates."""
    hidden, w1, w2, ids, w, ref = _case()
    X, W1, W2 = hidden.double(), w1.double(), w2.double()
    out = np.zeros_like(ref)
    for t in range(X.shape[0]):
        for j in range(ids.shape[1]):
            e = ids[t, j]
            h = W1[e] @ X[t]
            a = torch.nn.functional.silu(h[:128]) * h[128:]
            a = a.to(torch.bfloat16).double()
            out[t] += w[t, j] * (W2[e] @ a).numpy()
    assert passes(out.astype(np.float32), ref), gate_report(out, ref)


def test_zero_output_fails():
    *_, ref = _case()
    assert not passes(np.zeros_like(ref), ref)
    # and on the many-thin-experts shape family, where the elementwise gate alone would pass
    *_, ref2 = _case(T=16, H=2048, I=256, E=128, k=8, seed=1)
    r = gate_report(np.zeros_like(ref2), ref2)
    assert not passes(np.zeros_like(ref2), ref2), r


def test_swapped_expert_weights_fail():
    hidden, w1, w2, ids, w, ref = _case()
    w1s = w1.clone()
    w1s[[0, 1]] = w1[[1, 0]]
    bad = oracle.moe_token_loop(hidden, w1s, w2, w, ids)
    assert not passes(bad, ref)


def test_dropped_renorm_fails():
    hidden, w1, w2, ids, w, ref = _case()
    _, w_raw = oracle.route(make_inputs(64, 256, 128, 8, seed=0)[3].numpy(), 2, False)
    bad = oracle.moe_token_loop(hidden, w1, w2, w_raw, ids)
    assert not passes(bad, ref)
