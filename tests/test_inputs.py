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
