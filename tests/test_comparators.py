"""The unfused PyTorch comparator against the oracle (CPU, float64).

bench.unfused_wtconv restates the layer as PyTorch library ops (stride-2
grouped convs for the Haar analysis, grouped convs per subband, transposed
convs for the synthesis); it shares nothing with the oracle.  Agreement of its
forward, and of its autograd gradients with the oracle's adjoint and
weight-gradient sums, pins both to the layer's definition from a second,
independent direction.
"""
import numpy as np
import pytest
import torch

import bench
from wtconv_inputs import Case, make_inputs

CASES = [
    Case("tiny", 1, 4, 16, 16, 5, 2, "f32", 0, "const", "one"),
    Case("L0", 2, 3, 12, 8, 5, 0, "f32", 1, "normal", "normal"),
    Case("k3_L3_rect", 2, 2, 24, 16, 3, 3, "f32", 2, "uniform", "normal"),
    Case("k7_L4", 1, 2, 16, 16, 7, 4, "f32", 3, "normal", "normal"),
    Case("k1_L1", 1, 2, 8, 4, 1, 1, "f32", 4, "normal", "normal"),
]
NAMES = ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")


def _f64(inp):
    return {k: v.double() for k, v in inp.items()}


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_unfused_forward_matches_oracle(oracle, case):
    d = _f64(make_inputs(case))
    y = bench.unfused_wtconv(d["x"], d["base_w"], d["base_b"], d["base_scale"], d["wt_w"], d["wt_scale"], case.L)
    r = oracle.forward(d["x"].numpy(), *(d[k].numpy() for k in NAMES), case.L)
    assert np.abs(y.numpy() - r).max() <= 1e-12 * np.abs(r).max()


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_unfused_autograd_matches_oracle_backward(oracle, case):
    d = _f64(make_inputs(case))
    x = d["x"].clone().requires_grad_(True)
    p = {k: d[k].clone().requires_grad_(True) for k in NAMES}
    y = bench.unfused_wtconv(x, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
    y.backward(d["dy"])
    dy = d["dy"].numpy()
    dx = oracle.backward_input(dy, p["base_w"].detach().numpy(), p["base_scale"].detach().numpy(),
                               p["wt_w"].detach().numpy(), p["wt_scale"].detach().numpy(), case.L)
    assert np.abs(x.grad.numpy() - dx).max() <= 1e-12 * np.abs(dx).max()
    ref = oracle.backward_weight(d["x"].numpy(), dy, *(p[k].detach().numpy() for k in NAMES), case.L)
    for k in NAMES:
        if case.L == 0 and k in ("wt_w", "wt_scale"):
            continue
        got = p[k].grad.numpy()
        assert np.abs(got - ref[k]).max() <= 1e-11 * max(np.abs(ref[k]).max(), 1e-300), k


def test_haar_filters_are_orthonormal():
    f = bench.haar_filters(1, torch.float64, "cpu").reshape(4, 4)
    assert torch.allclose(f @ f.T, torch.eye(4, dtype=torch.float64))
