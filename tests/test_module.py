"""Autograd function / nn.Module over the C ABI (GPU), against the oracle."""
import numpy as np
import pytest
import torch

import memory_bound_cnn_wtconv_b200 as wt
from oracle_pins import relerr
from wtconv_inputs import Case, make_inputs

NAMES = ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")


def _oracle_all(oracle, inp, L):
    d = {k: v.double().numpy() for k, v in inp.items()}
    y = oracle.forward(d["x"], *(d[k] for k in NAMES), L)
    dx = oracle.backward_input(d["dy"], d["base_w"], d["base_scale"], d["wt_w"], d["wt_scale"], L)
    g = oracle.backward_weight(d["x"], d["dy"], *(d[k] for k in NAMES), L)
    return y, dx, g


@pytest.mark.gpu
@pytest.mark.parametrize("case", [
    Case("mod_f32", 2, 3, 24, 16, 5, 2, "f32", 40, "normal", "normal"),
    Case("mod_bf16", 2, 3, 32, 32, 3, 3, "bf16", 41, "uniform", "normal"),
    Case("mod_L0", 1, 2, 8, 8, 5, 0, "f32", 42, "normal", "normal"),
], ids=lambda c: c.name)
@pytest.mark.parametrize("one_pass", [False, True], ids=["two_pass", "one_pass"])
def test_autograd_matches_oracle(oracle, case, one_pass):
    inp = make_inputs(case)
    dev = torch.device("cuda", 0)
    dt = torch.bfloat16 if case.dtype == "bf16" else torch.float32
    x = inp["x"].to(dev, dt).requires_grad_(True)
    p = {k: inp[k].to(dev).requires_grad_(True) for k in NAMES}
    y = wt.wtconv(x, *(p[k] for k in NAMES), case.L, one_pass)
    y.backward(inp["dy"].to(dev, dt))
    torch.cuda.synchronize()
    ry, rdx, rg = _oracle_all(oracle, inp, case.L)
    tol = 2e-2 if case.dtype == "bf16" else 1e-5
    assert relerr(y.detach().double().cpu().numpy(), ry) <= tol
    assert relerr(x.grad.double().cpu().numpy(), rdx) <= tol
    for k in NAMES:
        if case.L == 0 and k in ("wt_w", "wt_scale"):
            assert p[k].grad is None or not p[k].grad.any()
            continue
        assert relerr(p[k].grad.double().cpu().numpy(), rg[k]) <= tol, k


@pytest.mark.gpu
def test_module_runs_and_only_requested_grads():
    dev = torch.device("cuda", 0)
    m = wt.WTConv2d(8, 5, 2, device=dev)
    x = torch.randn(2, 8, 16, 16, device=dev)
    y = m(x)
    assert y.shape == x.shape and torch.isfinite(y).all()
    y.sum().backward()
    assert all(q.grad is not None and torch.isfinite(q.grad).all() for q in m.parameters())
    m.zero_grad()
    for q in m.parameters():
        q.requires_grad_(False)
    x2 = x.clone().requires_grad_(True)
    m(x2).sum().backward()
    assert x2.grad is not None and all(q.grad is None for q in m.parameters())


@pytest.mark.gpu
def test_training_step_peak_memory_below_unfused():
    # The fused layer saves only x; the unfused PyTorch layer keeps every
    # level's subbands and conv outputs for its backward.
    import bench
    dev = torch.device("cuda", 0)
    case = Case("peak", 8, 32, 64, 64, 5, 3, "f32", 43, "normal", "normal")
    inp = make_inputs(case)
    peaks = {}
    for name in ("fused", "unfused"):
        x = inp["x"].to(dev).requires_grad_(True)
        p = {k: inp[k].to(dev).requires_grad_(True) for k in NAMES}
        fn = wt.wtconv if name == "fused" else bench.unfused_wtconv
        dy = inp["dy"].to(dev)
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        fn(x, *(p[k] for k in NAMES), case.L).backward(dy)
        torch.cuda.synchronize()
        peaks[name] = torch.cuda.max_memory_allocated(dev) - base
        del x, p, dy
    assert peaks["fused"] < 0.75 * peaks["unfused"], peaks
