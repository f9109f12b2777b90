"""The roofline arithmetic of bench.py (CPU only): algorithmic bytes and the
roofline time of the workloads against hand-computed values."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from moe_inputs import SHAPES  # noqa: E402

PEAKS = {"hbm_gbs": 6532.2, "bf16_tflops": 1648.5}


def test_decode_bytes_and_bound():
    s = SHAPES["decode"]
    # 8 active experts x 3 x 2048 x 768 bf16 weights + hidden + ids/weights + out
    want = 8 * 3 * 2048 * 768 * 2 + 2048 * 2 + 8 * 8 + 2048 * 4
    assert bench.algorithmic_bytes(s, 8) == want
    t, bound = bench.roofline_us(s, 8, PEAKS)
    assert bound == "hbm" and t == pytest.approx(want / 6532.2e9 * 1e6)


def test_fp8_bytes_count_codes_and_scales():
    s = SHAPES["decode"]
    n_w = 8 * 3 * 2048 * 768
    want = n_w + n_w / 128 * 4 + 2048 * 2 + 8 * 8 + 2048 * 4
    assert bench.algorithmic_bytes(s, 8, fp8_block=128) == pytest.approx(want)


def test_prefill_is_tensor_bound():
    s = SHAPES["prefill_8e"]
    t, bound = bench.roofline_us(s, 8, PEAKS)
    assert bound == "tensor"
    assert t == pytest.approx(6 * 1979 * 2 * 2048 * 2048 / 1648.5e12 * 1e6)
    assert 60.0 < t < 61.0
