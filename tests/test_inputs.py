"""The seeded input module: the workloads are rows of the page's shapes
table, and the draws are reproducible (CPU only)."""
import torch

from moe_inputs import PAGE_TABLE, SHAPES, TABLE_SHAPES, make_biases, make_inputs


def test_workloads_are_rows_of_the_shapes_table():
    rows = {r: (T, H, I, E, k) for r, T, H, I, E, k, _ in PAGE_TABLE}
    for name, r in (("prefill_8e", 4), ("decode", 8), ("prefill_thin", 19), ("prefill_big", 22)):
        s = SHAPES[name]
        assert (s.T, s.H, s.I, s.E, s.k) == rows[r]


def test_table_is_complete_and_well_formed():
    assert [r for r, *_ in PAGE_TABLE] == list(range(23))
    assert len(TABLE_SHAPES) == 24
    for s in TABLE_SHAPES.values():
        # the alignment the TPU wrapper checks, which the kernels rely on too
        assert s.H % 128 == 0 and s.I % 128 == 0 and 1 <= s.k <= s.E


def test_draws_are_seeded():
    a = make_inputs(3, 128, 128, 2, seed=9)
    b = make_inputs(3, 128, 128, 2, seed=9)
    c = make_inputs(3, 128, 128, 2, seed=10)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not torch.equal(a[0], c[0])
    b1, b2 = make_biases(2, 128, 128, seed=1)
    assert b1.shape == (2, 256) and b2.shape == (2, 128) and b1.dtype == torch.float32


def test_fp8_weights_shapes_and_range():
    from moe_inputs import make_fp8_weights
    q1, s1, q2, s2 = make_fp8_weights(2, 256, 128, 128, seed=3)
    assert q1.dtype == torch.uint8 and q1.shape == (2, 256, 256)
    assert s1.shape == (2, 256, 2) and s2.shape == (2, 256, 1)
    assert q2.shape == (2, 256, 128) and s1.dtype == torch.float32
    # no NaN codes, and every block uses the top of the E4M3 range
    v = q1.view(torch.float8_e4m3fn).float()
    assert not torch.isnan(v).any()
    assert torch.allclose(v.abs().reshape(2, 256, 2, 128).amax(-1), torch.full((2, 256, 2), 448.0))
