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


def make_shape_inputs(shape: MoEShape, seed: int = 0, device: str = "cpu"):
    return make_inputs(shape.T, shape.H, shape.I, shape.E, seed=seed, device=device)
