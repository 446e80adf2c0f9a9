"""Seeded synthetic inputs for the WTConv layer.

Shared by the tests, the benchmark and the smoke check.  This module draws
random tensors and nothing else: it holds none of the layer's arithmetic, and
it imports neither the oracle nor the CUDA binding.

Every tensor is drawn on the CPU from a ``torch.Generator`` in float32, so the
GPU path and the oracle see the same bits; bf16 storage rounds the float32
draw to nearest-even.  Draw order is fixed: x, dy, base_w, base_b, wt_w,
wt_scale (base_scale is a constant unless a case asks for it to be random).

Workloads (the evaluation of the WTConvNeXt configuration across levels and
tensor shapes in "Fast and Memory-Efficient Wavelet Convolutions via I/O-Aware
Reformulation", Abstract; the pages give no shapes, so the stage shapes of a
ConvNeXt-T-like network stand in):

  tiny        B=1,  C=4,   16x16, k=5, L=2, fp32, seed 0, forward only
  stage1      B=32, C=96,  56x56, k=5, L=3, fp32, seed 1
  stage2      B=32, C=192, 28x28, k=5, L=2, fp32, seed 2
  train_bf16  B=64, C=96,  56x56, k=5, L=3, bf16 storage, seed 3,
              wt_scale ~ U(0.05, 0.2)
  sweep       C in {64,128,256,512} x H=W in {32,64,128,256} x L in {1..4}
              x k in {3,5}; B = round(2^28 / (4 C H^2)) so x is ~256 MiB;
              seed 1000 + point index

Distributions: x, dy ~ N(0,1); base_w, wt_w ~ N(0, 0.1^2);
base_b ~ N(0, 0.01^2); base_scale = 1; wt_scale = 0.1 unless stated.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Case:
    name: str
    B: int
    C: int
    H: int
    W: int
    k: int
    L: int
    dtype: str = "f32"          # activation storage: "f32" or "bf16"
    seed: int = 0
    wt_scale: str = "const"      # "const" (0.1), "uniform" (U(0.05,0.2)) or "normal" (N(0,1))
    base_scale: str = "one"      # "one" or "normal" (N(1, 0.5^2))
    calls: tuple = field(default=("fwd", "bwd_in", "bwd_w"))

    @property
    def numel(self) -> int:
        return self.B * self.C * self.H * self.W

    @property
    def esize(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def with_(self, **kw) -> "Case":
        return replace(self, **kw)


TINY = Case("tiny", 1, 4, 16, 16, 5, 2, "f32", 0, calls=("fwd",))
STAGE1 = Case("stage1", 32, 96, 56, 56, 5, 3, "f32", 1)
STAGE2 = Case("stage2", 32, 192, 28, 28, 5, 2, "f32", 2)
TRAIN_BF16 = Case("train_bf16", 64, 96, 56, 56, 5, 3, "bf16", 3, wt_scale="uniform")

NAMED = {c.name: c for c in (TINY, STAGE1, STAGE2, TRAIN_BF16)}


def sweep_cases() -> list[Case]:
    """The 128-point shape/level sweep, in a fixed order."""
    out = []
    i = 0
    for C in (64, 128, 256, 512):
        for H in (32, 64, 128, 256):
            for L in (1, 2, 3, 4):
                for k in (3, 5):
                    B = max(1, round(2 ** 28 / (4 * C * H * H)))
                    out.append(Case(f"sweep{i:03d}_C{C}_H{H}_L{L}_k{k}", B, C, H, H, k, L, "f32", 1000 + i))
                    i += 1
    return out


def make_inputs(case: Case, with_dy: bool = True) -> dict:
    """Draw the case's tensors on the CPU.

    Returns float32 parameters and activations stored in the case's dtype
    (float32 or bfloat16).  ``dy`` is drawn even when unused so that the
    parameters do not depend on ``with_dy``; pass ``with_dy=False`` only to
    skip returning it.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(case.seed)
    shape = (case.B, case.C, case.H, case.W)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    dy = torch.randn(shape, generator=g, dtype=torch.float32)
    k, C, L = case.k, case.C, case.L
    base_w = 0.1 * torch.randn((C, k, k), generator=g, dtype=torch.float32)
    base_b = 0.01 * torch.randn((C,), generator=g, dtype=torch.float32)
    wt_w = 0.1 * torch.randn((L, C, 4, k, k), generator=g, dtype=torch.float32)
    if case.wt_scale == "const":
        wt_scale = torch.full((L, C, 4), 0.1, dtype=torch.float32)
    elif case.wt_scale == "uniform":
        wt_scale = 0.05 + 0.15 * torch.rand((L, C, 4), generator=g, dtype=torch.float32)
    elif case.wt_scale == "normal":
        wt_scale = torch.randn((L, C, 4), generator=g, dtype=torch.float32)
    else:
        raise ValueError(case.wt_scale)
    if case.base_scale == "one":
        base_scale = torch.ones((C,), dtype=torch.float32)
    elif case.base_scale == "normal":
        base_scale = 1.0 + 0.5 * torch.randn((C,), generator=g, dtype=torch.float32)
    else:
        raise ValueError(case.base_scale)
    if case.dtype == "bf16":
        x = x.to(torch.bfloat16)
        dy = dy.to(torch.bfloat16)
    out = dict(x=x, base_w=base_w, base_b=base_b, base_scale=base_scale, wt_w=wt_w, wt_scale=wt_scale)
    if with_dy:
        out["dy"] = dy
    return out
