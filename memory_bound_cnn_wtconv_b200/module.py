"""Autograd function and ``nn.Module`` over the C ABI (binding layer only).

The forward saves only its input x and the parameters, not the wavelet
subbands: the backward recomputes every subband on chip (the Abstract of
"Fast and Memory-Efficient Wavelet Convolutions via I/O-Aware
Reformulation", arXiv 2608.10805, credits this with about half the peak
memory of the unfused layer in training).  Every step runs in the CUDA
kernels of ``libwtconv_b200.so``; there is no CPU fallback.
"""
from __future__ import annotations

import math

import torch

from . import backward, backward_input, backward_weight, forward

__all__ = ["WTConvFunction", "WTConv2d", "wtconv"]

_PARAMS = ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")


class WTConvFunction(torch.autograd.Function):
    """y = WTConv(x).  Backward: the input- and weight-gradient passes, or
    with ``one_pass`` the one-pass kernel ``wtconv_backward_one_pass`` (same
    results; it moves a quarter fewer bytes but was measured no faster on
    B200, its larger on-chip footprint allowing one CTA per SM instead of
    two; planes split into cluster strips have no one-pass plan and raise)."""

    @staticmethod
    def forward(ctx, x, base_w, base_b, base_scale, wt_w, wt_scale, L: int, one_pass: bool = False):
        # Channels-last inputs stay NHWC (the kernels read either layout).
        x = x if x.dim() == 4 and x.is_contiguous(memory_format=torch.channels_last) else x.contiguous()
        y = forward(x, base_w, base_b, base_scale, wt_w, wt_scale, L)
        ctx.save_for_backward(x, base_w, base_b, base_scale, wt_w, wt_scale)
        ctx.L = L
        ctx.one_pass = bool(one_pass)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, base_w, base_b, base_scale, wt_w, wt_scale = ctx.saved_tensors
        L = ctx.L
        fmt = torch.contiguous_format if x.is_contiguous() else torch.channels_last
        dy = dy.to(x.dtype).contiguous(memory_format=fmt)
        need = ctx.needs_input_grad
        dx, g = None, {}
        if ctx.one_pass and need[0] and any(need[1:6]):
            dx, g = backward(x, dy, base_w, base_b, base_scale, wt_w, wt_scale, L, one_pass=True)
        else:
            if need[0]:
                dx = backward_input(dy, base_w, base_scale, wt_w, wt_scale, L)
            if any(need[1:6]):
                g = backward_weight(x, dy, base_w, base_b, base_scale, wt_w, wt_scale, L)
        out = [g.get(k) if need[1 + i] else None for i, k in enumerate(_PARAMS)]
        if L == 0 and out[3] is not None:  # no wavelet parameters: empty gradients of the right shape
            out[3] = torch.zeros_like(wt_w)
            out[4] = torch.zeros_like(wt_scale)
        return (dx, *out, None, None)


def wtconv(x, base_w, base_b, base_scale, wt_w, wt_scale, L: int, one_pass: bool = False):
    """Functional form with autograd support."""
    return WTConvFunction.apply(x, base_w, base_b, base_scale, wt_w, wt_scale, L, one_pass)


class WTConv2d(torch.nn.Module):
    """Depthwise wavelet convolution layer on ``channels`` NCHW channels.

    Parameters (float32): base_w [C,k,k], base_b [C], base_scale [C],
    wt_w [L,C,4,k,k], wt_scale [L,C,4].  Initialisation (the pages give none):
    base_w and wt_w uniform in +-1/k like a depthwise ``nn.Conv2d``, base_b 0,
    base_scale 1, wt_scale 0.1.  Inputs: float32 or bfloat16 CUDA tensors,
    W a multiple of 4 (8 for bfloat16 when H or W is not a multiple of
    2^levels; such planes are zero-padded on chip and cropped).
    """

    def __init__(self, channels: int, kernel_size: int = 5, levels: int = 1, device=None):
        super().__init__()
        if kernel_size not in (1, 3, 5, 7):
            raise ValueError("kernel_size must be 1, 3, 5 or 7")
        C, k, L = int(channels), int(kernel_size), int(levels)
        self.channels, self.kernel_size, self.levels = C, k, L
        f = dict(device=device, dtype=torch.float32)
        self.base_w = torch.nn.Parameter(torch.empty((C, k, k), **f))
        self.base_b = torch.nn.Parameter(torch.zeros((C,), **f))
        self.base_scale = torch.nn.Parameter(torch.ones((C,), **f))
        self.wt_w = torch.nn.Parameter(torch.empty((L, C, 4, k, k), **f))
        self.wt_scale = torch.nn.Parameter(torch.full((L, C, 4), 0.1, **f))
        self.reset_parameters()

    def reset_parameters(self):
        bound = 1.0 / math.sqrt(self.kernel_size * self.kernel_size)
        with torch.no_grad():
            self.base_w.uniform_(-bound, bound)
            self.wt_w.uniform_(-bound, bound)

    def forward(self, x):
        return WTConvFunction.apply(x, self.base_w, self.base_b, self.base_scale, self.wt_w, self.wt_scale,
                                    self.levels, False)

    def extra_repr(self) -> str:
        return f"channels={self.channels}, kernel_size={self.kernel_size}, levels={self.levels}"
