"""Shared helpers of the tests: tolerance gates and tensor conversion.

Acceptance (the gate every parity test applies): routing ids, permutation
indices and expert offsets bit-exact; routing weights within
1e-6 + 1e-5*|w|; the fp32 forward output elementwise within
1e-2 + 1e-2*|ref| of the fp64 oracle.

Because the outputs of these workloads are small (|out| ~ 1e-3..1e-2), the
elementwise gate alone would accept an all-zero output on some shapes, so
two diagnostic gates derived from the arithmetic are applied as well:
  * relative Frobenius error <= 5e-3.  Rounding the SwiGLU intermediate to
    bf16 (relative error <= 2^-9 per element, random sign) gives about
    2^-9/sqrt(3) ~ 1.1e-3 on a sum of many terms, fp32 accumulation adds
    far less; 5e-3 leaves a 4x margin.
  * |gpu - ref| <= 5e-2 * RMS(ref) + 1e-2 * |ref| elementwise.
An all-zero output, or one computed with two experts' weights swapped,
fails both (checked on the CPU in test_tolerance_gates.py).
"""
from __future__ import annotations

import numpy as np

ATOL_OUT = 1e-2
RTOL_OUT = 1e-2
FROB_MAX = 5e-3
RMS_FRAC = 5e-2
W_ATOL = 1e-6
W_RTOL = 1e-5


def gate_report(out, ref) -> dict:
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.abs(out - ref)
    nref = np.linalg.norm(ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    return {
        "elementwise": bool(np.all(d <= ATOL_OUT + RTOL_OUT * np.abs(ref))),
        "frobenius": float(np.linalg.norm(out - ref) / nref) if nref > 0 else float(np.linalg.norm(out)),
        "rms_gate": bool(np.all(d <= RMS_FRAC * rms + RTOL_OUT * np.abs(ref))),
        "max_abs": float(d.max()) if d.size else 0.0,
    }


def passes(out, ref) -> bool:
    r = gate_report(out, ref)
    return r["elementwise"] and r["frobenius"] <= FROB_MAX and r["rms_gate"]


def assert_output_close(out, ref, what: str = "") -> dict:
    r = gate_report(out, ref)
    assert r["elementwise"], f"{what}: elementwise gate failed {r}"
    assert r["frobenius"] <= FROB_MAX, f"{what}: Frobenius gate failed {r}"
    assert r["rms_gate"], f"{what}: RMS gate failed {r}"
    return r


def assert_weights_close(w_gpu, w_ref, what: str = "") -> None:
    w_gpu = np.asarray(w_gpu, np.float64)
    w_ref = np.asarray(w_ref, np.float64)
    bad = np.abs(w_gpu - w_ref) > W_ATOL + W_RTOL * np.abs(w_ref)
    assert not bad.any(), f"{what}: {int(bad.sum())} weights off, max {np.abs(w_gpu - w_ref).max()}"
