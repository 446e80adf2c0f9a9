"""Planes whose H or W is not a multiple of 2^L (oracle, CPU).

The oracle zero-pads to multiples of 2^L, applies the layer and crops.  These
tests pin that reading against an independent formulation that pads each
level's LL by one row / column only where it is odd and crops every level's
reconstruction back to that level's size before adding it (PyTorch ops,
float64), and check the input gradient is the adjoint of the cropped map.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import bench
from wtconv_inputs import Case, make_inputs

NAMES = ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")


def per_level_padded(x, base_w, base_b, base_scale, wt_w, wt_scale, L):
    B, C, H, W = x.shape
    k = base_w.shape[-1]
    p = k // 2
    y = F.conv2d(x, base_w.unsqueeze(1), base_b, padding=p, groups=C) * base_scale.view(1, C, 1, 1)
    if L == 0:
        return y
    filt = bench.haar_filters(C, x.dtype, x.device)
    ll, shat, shapes = x, [], []
    for l in range(L):
        h, w = ll.shape[-2:]
        shapes.append((h, w))
        ll = F.pad(ll, (0, w % 2, 0, h % 2))
        s = F.conv2d(ll, filt, stride=2, groups=C)
        hs, ws = s.shape[-2:]
        z = F.conv2d(s, wt_w[l].reshape(4 * C, 1, k, k), padding=p, groups=4 * C)
        shat.append(z * wt_scale[l].reshape(1, 4 * C, 1, 1))
        ll = s.view(B, C, 4, hs, ws)[:, :, 0]
    zc = None
    for l in range(L - 1, -1, -1):
        z = shat[l]
        hs, ws = z.shape[-2:]
        if zc is not None:
            z4 = z.view(B, C, 4, hs, ws)
            z = torch.cat([z4[:, :, :1] + zc.unsqueeze(2), z4[:, :, 1:]], dim=2).view(B, 4 * C, hs, ws)
        zc = F.conv_transpose2d(z, filt, stride=2, groups=C)
        h, w = shapes[l]
        zc = zc[..., :h, :w]
    return y + zc


CASES = [
    Case("odd_both", 2, 3, 13, 11, 5, 2, "f32", 60, "normal", "normal"),
    Case("rows_only", 1, 2, 20, 16, 3, 3, "f32", 61, "normal", "normal"),
    Case("cols_only", 1, 2, 16, 12, 5, 3, "f32", 62, "normal", "normal"),
    Case("tiny_L4", 1, 1, 9, 7, 7, 4, "f32", 63, "normal", "normal"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_pad_crop_matches_per_level_padding(oracle, case):
    d = {k: v.double() for k, v in make_inputs(case).items()}
    ref = per_level_padded(d["x"], *(d[k] for k in NAMES), case.L).numpy()
    got = oracle.forward(d["x"].numpy(), *(d[k].numpy() for k in NAMES), case.L)
    assert got.shape == ref.shape
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_padded_gradients_match_autograd(oracle, case):
    d = {k: v.double() for k, v in make_inputs(case).items()}
    x = d["x"].clone().requires_grad_(True)
    p = {k: d[k].clone().requires_grad_(True) for k in NAMES}
    per_level_padded(x, *(p[k] for k in NAMES), case.L).backward(d["dy"])
    dx = oracle.backward_input(d["dy"].numpy(), d["base_w"].numpy(), d["base_scale"].numpy(), d["wt_w"].numpy(),
                               d["wt_scale"].numpy(), case.L)
    assert np.abs(dx - x.grad.numpy()).max() <= 1e-12 * np.abs(dx).max()
    g = oracle.backward_weight(d["x"].numpy(), d["dy"].numpy(), *(d[k].numpy() for k in NAMES), case.L)
    for k in NAMES:
        assert np.abs(g[k] - p[k].grad.numpy()).max() <= 1e-11 * np.abs(g[k]).max(), k
