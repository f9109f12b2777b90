"""Seeded synthetic inputs for the fused MoE forward.

This module is shared by the tests, the benchmark and the oracle's callers.
It holds no part of the method's arithmetic: it only draws random tensors
with the shapes and distributions of the atrex-bench #009 "fused_moe"
workload (its input.py, ``_make_inputs``): hidden ``randn * 0.1`` in bf16,
w1 ``randn * H**-0.5`` and w2 ``randn * I**-0.5`` in bf16, and fp32 ``randn``
router logits.  Routing (softmax / top-k / renormalisation) is NOT done here;
each side computes it from the logits with its own code.

The draws come from one seeded torch generator on the requested device (CPU
by default).  Both sides always see the same tensors: GPU draws are copied to
the host for the oracle, CPU draws are copied to the GPU for the kernels.
Large shapes draw on the GPU because the CPU generator needs tens of seconds
for the biggest weight sets.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class MoEShape:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int

    @property
    def flops(self) -> float:
        """Useful FLOPs of one forward: 2 GEMMs of 2*T*k*H*(2I) and 2*T*k*I*H."""
        return 6.0 * self.T * self.k * self.H * self.I

    def describe(self) -> dict:
        return {"workload": self.name, "T": self.T, "H": self.H, "I": self.I,
                "E": self.E, "top_k": self.k}


# The five workloads: a tiny case, and rows 4, 8, 19 and 22 of the
# atrex-bench #009 shapes table.
SHAPES = {
    "tiny": MoEShape("tiny fused MoE T=64 H=256 I=128 E=8 k=2", 64, 256, 128, 8, 2),
    "prefill_8e": MoEShape("prefill, few large experts T=1979 H=2048 I=2048 E=8 k=2",
                           1979, 2048, 2048, 8, 2),
    "decode": MoEShape("decode, many small experts T=1 H=2048 I=768 E=128 k=8",
                       1, 2048, 768, 128, 8),
    "prefill_thin": MoEShape("prefill, many thin experts T=8192 H=4096 I=384 E=128 k=8",
                             8192, 4096, 384, 128, 8),
    "prefill_big": MoEShape("large prefill, big experts T=15381 H=4096 I=4096 E=8 k=2",
                            15381, 4096, 4096, 8, 2),
}


# The "Shapes" table of atrex-bench #009: (row, T, H, I, E, top-k, T_Prod in
# microseconds of the production op on the page's "XPU-A" hardware, context
# only).  Rows 4, 8, 19 and 22 are four of the workloads above.
PAGE_TABLE = (
    (0, 135, 2048, 2048, 8, 2, 232.70),
    (1, 277, 2048, 2048, 8, 2, 249.80),
    (2, 668, 2048, 2048, 8, 2, 477.10),
    (3, 1023, 2048, 2048, 8, 2, 539.00),
    (4, 1979, 2048, 2048, 8, 2, 772.50),
    (5, 4195, 2048, 2048, 8, 2, 1600.0),
    (6, 7689, 2048, 2048, 8, 2, 2680.0),
    (7, 15809, 2048, 2048, 8, 2, 5370.0),
    (8, 1, 2048, 768, 128, 8, 116.90),
    (9, 2400, 2048, 768, 128, 8, 2160.0),
    (10, 4195, 2048, 768, 128, 8, 2980.0),
    (11, 8192, 2048, 768, 128, 8, 4990.0),
    (12, 15809, 2048, 768, 128, 8, 9090.0),
    (13, 25632, 2048, 768, 128, 8, 14480.0),
    (14, 45936, 2048, 768, 128, 8, 25710.0),
    (15, 520, 4096, 384, 128, 8, 595.80),
    (16, 1019, 4096, 384, 128, 8, 882.90),
    (17, 2044, 4096, 384, 128, 8, 1610.0),
    (18, 3936, 4096, 384, 128, 8, 2800.0),
    (19, 8192, 4096, 384, 128, 8, 5690.0),
    (20, 4098, 4096, 4096, 8, 2, 5330.0),
    (21, 8179, 4096, 4096, 8, 2, 10100.0),
    (22, 15381, 4096, 4096, 8, 2, 18640.0),
)

# Every row of the table as a shape, plus a two-token decode (the batch of
# two rows that the Rust page's decode kernels process).
TABLE_SHAPES = {
    f"row{r:02d}": MoEShape(f"atrex-bench #009 shapes row {r}: T={T} H={H} I={I} E={E} k={k}",
                            T, H, I, E, k)
    for r, T, H, I, E, k, _ in PAGE_TABLE
}
TABLE_SHAPES["decode_t2"] = MoEShape("decode, two tokens T=2 H=2048 I=768 E=128 k=8",
                                     2, 2048, 768, 128, 8)
PAGE_T_PROD_US = {f"row{r:02d}": t for r, *_, t in PAGE_TABLE}


def make_inputs(T: int, H: int, I: int, E: int, seed: int = 0,
                hidden_scale: float = 0.1, device: str = "cpu"):
    """Draw (hidden [T,H] bf16, w1 [E,2I,H] bf16, w2 [E,H,I] bf16,
    logits [T,E] fp32) on `device`, in that order, from one seeded generator."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    kw = dict(generator=g, device=device)
    hidden = torch.randn(T, H, dtype=torch.bfloat16, **kw) * hidden_scale
    w1 = torch.randn(E, 2 * I, H, dtype=torch.bfloat16, **kw) * (H ** -0.5)
    w2 = torch.randn(E, H, I, dtype=torch.bfloat16, **kw) * (I ** -0.5)
    logits = torch.randn(T, E, dtype=torch.float32, **kw)
    return hidden, w1, w2, logits


def make_biases(E: int, H: int, I: int, seed: int = 0, b1_scale: float = 0.1,
                b2_scale: float = 0.005, device: str = "cpu"):
    """Draw fp32 expert biases (b1 [E,2I], b2 [E,H]) for the variant forward
    of the 0.13.2 TPU page, ``randn`` times a scale comparable to the
    projections (b1) and to an expert's output (b2) of make_inputs."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    kw = dict(generator=g, device=device)
    b1 = torch.randn(E, 2 * I, dtype=torch.float32, **kw) * b1_scale
    b2 = torch.randn(E, H, dtype=torch.float32, **kw) * b2_scale
    return b1, b2


def make_fp8_weights(E: int, H: int, I: int, block: int, seed: int = 0, device: str = "cpu"):
    """Sub-channel-quantised expert weights for the FP8 forward: randn
    weights with the fan-in scaling of make_inputs, cut into blocks of
    `block` consecutive contraction elements per output row; each block gets
    the fp32 scale max|w| / 448 (the largest E4M3 value) and its codes are
    torch's float8_e4m3fn conversion of w / scale.  Returns (q1 uint8
    [E,2I,H], s1 fp32 [E,2I,H/block], q2 uint8 [E,H,I], s2 fp32
    [E,H,I/block]).  This only prepares inputs (a checkpoint would hold
    them); the forward reads codes and scales as given."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    kw = dict(generator=g, device=device)

    def quant(w):
        K = w.shape[-1]
        wb = w.reshape(*w.shape[:-1], K // block, block)
        sc = (wb.abs().amax(-1) / 448.0).clamp_min(1e-30)
        q = (wb / sc.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
        return q.reshape(w.shape).contiguous(), sc.float().contiguous()

    q1, s1 = quant(torch.randn(E, 2 * I, H, dtype=torch.float32, **kw) * (H ** -0.5))
    q2, s2 = quant(torch.randn(E, H, I, dtype=torch.float32, **kw) * (I ** -0.5))
    return q1, s1, q2, s2


def make_shape_inputs(shape: MoEShape, seed: int = 0, device: str = "cpu"):
    return make_inputs(shape.T, shape.H, shape.I, shape.E, seed=seed, device=device)
