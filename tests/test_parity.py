"""CUDA path vs. the oracle, through the C ABI (needs a B200).

Metric (per output tensor): normwise relative error max|g - r| / max|r|, with
r the float64 oracle on the same inputs (float32 or bf16 values widened
exactly).  Bounds: 1e-5 for float32 storage, 2e-2 for bf16 storage.

Small cases run the oracle on every plane; they span several tiles per plane,
ragged tile edges, odd batch sizes, rectangular planes, L = 0, k = 1, kernels
larger than the coarsest subband (1x1 and 2x2 coarsest subbands) and random
(signed) scales.  Full-size workloads run exactly as the benchmark launches
them and compare sampled planes (forward / input gradient: planes are
independent) and sampled channels (weight gradient: the oracle sums that
channel over the whole batch).
"""
import numpy as np
import pytest
import torch

import memory_bound_cnn_wtconv_b200 as wt
from oracle_pins import relerr
from wtconv_inputs import NAMED, STAGE1, STAGE2, TINY, TRAIN_BF16, Case, make_inputs, sweep_cases

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}
PARAMS = ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def gpu_inputs(inp, nhwc=False):
    """The case's tensors on the GPU; with nhwc the activations channels-last
    (the same logical NCHW values, stored NHWC)."""
    g = {k: v.cuda() for k, v in inp.items()}
    if nhwc:
        for k in ("x", "dy"):
            g[k] = g[k].contiguous(memory_format=torch.channels_last)
    return g


def run_gpu(case: Case, g, calls, fused_bwd=False):
    out = {}
    if "fwd" in calls:
        out["y"] = wt.forward(g["x"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], case.L)
    if fused_bwd:
        # dx and the parameter gradients from one backward call: the path
        # the library picks ("auto") or the one-pass kernel ("one_pass").
        out["dx"], out["grads"] = wt.backward(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"],
                                              g["wt_scale"], case.L, one_pass=fused_bwd == "one_pass")
    else:
        if "bwd_in" in calls:
            out["dx"] = wt.backward_input(g["dy"], g["base_w"], g["base_scale"], g["wt_w"], g["wt_scale"], case.L)
        if "bwd_w" in calls:
            out["grads"] = wt.backward_weight(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"],
                                              g["wt_scale"], case.L)
    torch.cuda.synchronize()
    for k in ("y", "dx"):
        if k in out:
            assert out[k].is_contiguous(memory_format=torch.channels_last) == g["x"].is_contiguous(
                memory_format=torch.channels_last), f"{k} does not keep the input's layout"
            out[k] = out[k].contiguous()
    return out


def oracle_params(inp, c=None):
    p = {k: f64(inp[k]) for k in PARAMS}
    if c is not None:
        p["base_w"], p["base_b"], p["base_scale"] = p["base_w"][c:c + 1], p["base_b"][c:c + 1], p["base_scale"][c:c + 1]
        p["wt_w"], p["wt_scale"] = p["wt_w"][:, c:c + 1], p["wt_scale"][:, c:c + 1]
    return p


def check_full(oracle, case: Case, calls=("fwd", "bwd_in", "bwd_w"), fused_bwd=False, nhwc=False):
    inp = make_inputs(case)
    out = run_gpu(case, gpu_inputs(inp, nhwc), calls, fused_bwd)
    p = oracle_params(inp)
    x, dy = f64(inp["x"]), f64(inp["dy"])
    tol = TOL[case.dtype]
    errs = {}
    if "fwd" in calls:
        ref = oracle.forward(x, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
        errs["y"] = relerr(f64(out["y"]), ref)
    if "bwd_in" in calls:
        ref = oracle.backward_input(dy, p["base_w"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
        errs["dx"] = relerr(f64(out["dx"]), ref)
    if "bwd_w" in calls:
        ref = oracle.backward_weight(x, dy, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"],
                                     case.L)
        for k in PARAMS:
            if case.L == 0 and k.startswith("wt_"):
                continue
            errs["d_" + k] = relerr(f64(out["grads"][k]), ref[k])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"{case}: {errs}"
    return errs


def check_sampled(oracle, case: Case, calls=("fwd", "bwd_in", "bwd_w"), nplanes=6, nchannels=3, seed=0,
                  fused_bwd=False, nhwc=False):
    inp = make_inputs(case)
    out = run_gpu(case, gpu_inputs(inp, nhwc), calls, fused_bwd)
    rng = np.random.default_rng(seed)
    planes = {(0, 0), (case.B - 1, case.C - 1)}
    while len(planes) < min(nplanes, case.B * case.C):
        planes.add((int(rng.integers(case.B)), int(rng.integers(case.C))))
    chans = sorted({0, case.C - 1, *map(int, rng.integers(0, case.C, max(0, nchannels - 2)))})
    tol = TOL[case.dtype]
    errs = {}
    for name, src, call in (("y", "x", "fwd"), ("dx", "dy", "bwd_in")):
        if call not in calls:
            continue
        g_all, r_all = [], []
        for b, c in sorted(planes):
            p = oracle_params(inp, c)
            a = f64(inp[src][b:b + 1, c:c + 1])
            if call == "fwd":
                r = oracle.forward(a, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
            else:
                r = oracle.backward_input(a, p["base_w"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
            g_all.append(f64(out[name][b, c]))
            r_all.append(r[0, 0])
        errs[name] = relerr(np.stack(g_all), np.stack(r_all))
    if "bwd_w" in calls:
        # Normwise per gradient tensor over its sampled channels, as the
        # outputs above are over their sampled planes.
        got, want = {}, {}
        for c in chans:
            p = oracle_params(inp, c)
            ref = oracle.backward_weight(f64(inp["x"][:, c:c + 1]), f64(inp["dy"][:, c:c + 1]), p["base_w"],
                                         p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
            g = out["grads"]
            pairs = {"base_w": (g["base_w"][c], ref["base_w"][0]), "base_b": (g["base_b"][c], ref["base_b"][0]),
                     "base_scale": (g["base_scale"][c], ref["base_scale"][0])}
            if case.L > 0:
                pairs["wt_w"] = (g["wt_w"][:, c], ref["wt_w"][:, 0])
                pairs["wt_scale"] = (g["wt_scale"][:, c], ref["wt_scale"][:, 0])
            for k, (gv, rv) in pairs.items():
                got.setdefault(k, []).append(f64(gv))
                want.setdefault(k, []).append(np.asarray(rv))
        for k in got:
            errs[f"d_{k}[c in {chans}]"] = relerr(np.stack(got[k]), np.stack(want[k]))
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"{case}: {errs}"
    return errs


SMALL = [
    TINY.with_(calls=("fwd", "bwd_in", "bwd_w")),
    Case("odd_batch_stage1_plane", 3, 5, 56, 56, 5, 3, "f32", 11, "normal", "normal"),
    Case("stage2_plane", 2, 4, 28, 28, 5, 2, "f32", 12, "normal", "normal"),
    Case("k3_L4", 2, 3, 32, 32, 3, 4, "f32", 13, "normal", "normal"),
    Case("k7_coarsest_1x1", 1, 2, 16, 16, 7, 4, "f32", 14, "normal", "normal"),
    Case("k5_coarsest_1x1", 2, 2, 8, 8, 5, 3, "f32", 15, "normal", "normal"),
    Case("rect_24x40", 2, 3, 24, 40, 3, 3, "f32", 16, "normal", "normal"),
    Case("rect_64x4", 1, 2, 64, 4, 7, 2, "f32", 17, "normal", "normal"),
    Case("L0", 2, 3, 12, 8, 5, 0, "f32", 18, "normal", "normal"),
    Case("k1", 1, 2, 16, 16, 1, 2, "f32", 19, "normal", "normal"),
    Case("L1_2x4", 1, 1, 2, 4, 3, 1, "f32", 20, "normal", "normal"),
    Case("L6_64", 1, 1, 64, 64, 7, 6, "f32", 21, "normal", "normal"),
    Case("plane64_L4", 1, 2, 64, 64, 5, 4, "f32", 22, "normal", "normal"),
    Case("bf16_stage1_plane", 3, 2, 56, 56, 5, 3, "bf16", 23, "uniform", "normal"),
    Case("bf16_rect", 5, 3, 20, 12, 5, 2, "bf16", 24, "normal", "normal"),
    # Two tiles per thread in the weight gradient (more tiles than threads).
    Case("plane64_L2_two_tiles", 2, 2, 64, 64, 5, 2, "f32", 25, "normal", "normal"),
    # Planes split into row strips across a thread-block cluster (halo rows
    # exchanged through distributed shared memory).
    Case("strips_128_L4", 2, 2, 128, 128, 5, 4, "f32", 26, "normal", "normal"),
    Case("strips_128_L1_k3", 1, 3, 128, 128, 3, 1, "f32", 27, "normal", "normal"),
    Case("strips_256_L4", 1, 1, 256, 256, 5, 4, "f32", 28, "normal", "normal"),
    Case("strips_256_L3_k3", 2, 1, 256, 256, 3, 3, "f32", 29, "normal", "normal"),
    Case("strips_256_L2_bf16", 1, 2, 256, 256, 5, 2, "bf16", 30, "normal", "normal"),
    # H or W not a multiple of 2^L: zero-padded on chip, real outputs only.
    Case("pad_13x12_L2", 2, 3, 13, 12, 5, 2, "f32", 31, "normal", "normal"),
    Case("pad_20x16_k3_L3", 2, 3, 20, 16, 3, 3, "f32", 32, "normal", "normal"),
    Case("pad_9x8_k7_L4", 1, 2, 9, 8, 7, 4, "f32", 33, "normal", "normal"),
    Case("pad_17x8_k3_L1", 2, 3, 17, 8, 3, 1, "f32", 34, "normal", "normal"),
    Case("pad_bf16_13x16", 2, 3, 13, 16, 5, 2, "bf16", 35, "uniform", "normal"),
    Case("pad_strips_250x248", 1, 1, 250, 248, 5, 4, "f32", 36, "normal", "normal"),
    # strips of L = 0 planes and of planes with levels past the one-pass pyramid (L = 5, 6)
    Case("strips_256_L0", 1, 2, 256, 256, 5, 0, "f32", 42, "normal", "normal"),
    Case("strips_256_L5", 1, 1, 256, 256, 5, 5, "f32", 43, "normal", "normal"),
    Case("strips_512x64_L6_bf16", 1, 1, 512, 64, 5, 6, "bf16", 44, "normal", "normal"),
    # deepest levels, bf16 with k = 7, and one channel over many batch elements
    Case("L5_32_k3", 1, 2, 32, 32, 3, 5, "f32", 37, "normal", "normal"),
    Case("bf16_k7_L3", 2, 2, 24, 24, 7, 3, "bf16", 38, "uniform", "normal"),
    Case("one_channel_130_planes", 130, 1, 16, 16, 5, 2, "f32", 39, "normal", "normal"),
    Case("pad_40x36_L6", 1, 2, 40, 36, 5, 6, "f32", 40, "normal", "normal"),
    Case("pad_60x64_k3_L6", 2, 1, 60, 64, 3, 6, "f32", 41, "normal", "normal"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_case_all_outputs(oracle, case):
    check_full(oracle, case, case.calls)


def _one_pass_plan_exists(case: Case, nhwc: bool = False) -> bool:
    """Whether wtconv_backward_one_pass plans this case (whole planes only);
    asked through the call itself with an empty workspace, which returns
    WTCONV_ERR_WORKSPACE (7) after planning and before any launch."""
    import ctypes
    lib = wt.load_library()
    d = wt.Desc(case.B, case.C, case.H, case.W, case.k, case.L, 1 if case.dtype == "bf16" else 0, int(nhwc))
    fake = ctypes.c_void_p(0x10000)
    rc = lib.wtconv_backward_one_pass(ctypes.byref(d), *([fake] * 13), ctypes.c_void_p(0), ctypes.c_size_t(0), None)
    assert rc in (7, 8), rc
    return rc == 7


@pytest.mark.parametrize("mode", ["auto", "one_pass"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_case_fused_backward(oracle, case, mode):
    if mode == "one_pass" and not _one_pass_plan_exists(case):
        pytest.skip("planes split into cluster strips have no one-pass plan")
    check_full(oracle, case, ("bwd_in", "bwd_w"), fused_bwd=mode)


@pytest.mark.parametrize("mode", ["auto", "one_pass"])
@pytest.mark.parametrize("case", [STAGE1, STAGE2, TRAIN_BF16], ids=lambda c: c.name)
def test_full_size_fused_backward_sampled(oracle, case, mode):
    check_sampled(oracle, case, ("bwd_in", "bwd_w"), fused_bwd=mode)


@pytest.mark.parametrize("one_pass", [False, True], ids=["auto", "one_pass"])
def test_fused_backward_is_deterministic(one_pass):
    case = STAGE1
    g = gpu_inputs(make_inputs(case))
    args = (g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], case.L)
    dx_a, ga = wt.backward(*args, one_pass=one_pass)
    dx_a, ga = dx_a.clone(), {k: v.clone() for k, v in ga.items()}
    dx_b, gb = wt.backward(*args, one_pass=one_pass)
    torch.cuda.synchronize()
    assert torch.equal(dx_a, dx_b)
    for k in PARAMS:
        assert torch.equal(ga[k], gb[k]), k


def test_tiny_config_forward(oracle):
    check_full(oracle, TINY, ("fwd",))


@pytest.mark.parametrize("case", [STAGE1, STAGE2, TRAIN_BF16], ids=lambda c: c.name)
def test_full_size_workloads_sampled(oracle, case):
    check_sampled(oracle, case)


def _supported(case: Case) -> bool:
    d = wt.Desc(case.B, case.C, case.H, case.W, case.k, case.L, 0)
    import ctypes
    return wt.load_library().wtconv_workspace_bytes(ctypes.byref(d)) > 0


def _one_point_per_geometry() -> list:
    """One sweep point for each of the sweep's 32 plane geometries (H, L, k),
    the channel count rotating through all four values.  The plan (strip
    count, tile height, dy read from its staging, threads) depends on the
    geometry only, so these points run every plan the sweep uses."""
    cases = sweep_cases()
    picks = []
    for hi in range(4):
        for li in range(4):
            for ki in range(2):
                ci = (hi + li + ki) % 4
                picks.append(((ci * 4 + hi) * 4 + li) * 2 + ki)
    assert len({(cases[i].H, cases[i].L, cases[i].k) for i in picks}) == 32
    return sorted(picks)


SWEEP_PICK = _one_point_per_geometry()


@pytest.mark.parametrize("idx", SWEEP_PICK)
def test_sweep_points_sampled(oracle, idx):
    case = sweep_cases()[idx]
    assert _supported(case), f"{case.name}: no on-chip plan"
    check_sampled(oracle, case, nplanes=4, nchannels=2)


@pytest.mark.parametrize("idx", [i for i in SWEEP_PICK if sweep_cases()[i].H <= 64])
def test_sweep_points_one_pass_backward_sampled(oracle, idx):
    # Whole planes (H <= 64) have a one-pass plan; larger ones are strips.
    case = sweep_cases()[idx]
    check_sampled(oracle, case, ("bwd_in", "bwd_w"), nplanes=4, nchannels=2, fused_bwd="one_pass")


def _sweep_batch(C: int, H: int) -> int:
    return max(1, round(2 ** 28 / (4 * C * H * H)))


# Plans the sweep's shapes never pick, at the sweep's channel counts and
# batch rule (x of about 256 Mi elements): clusters of 4 and 16 strips, the
# weight gradient reading dy from its staging at 4 strips, and bf16 strips.
PLAN_VARIANTS = [
    Case("strips4_dy_from_staging_H192_L1_k5", _sweep_batch(128, 192), 128, 192, 192, 5, 1, "f32", 2001),
    Case("strips4_dy_from_staging_H192_L4_k3", _sweep_batch(256, 192), 256, 192, 192, 3, 4, "f32", 2002),
    Case("strips4_bf16_H192_L1_k7", _sweep_batch(64, 192), 64, 192, 192, 7, 1, "bf16", 2003, "uniform"),
    Case("strips16_H320_L1_k3", _sweep_batch(64, 320), 64, 320, 320, 3, 1, "f32", 2004),
    Case("strips16_bf16_H320_L1_k5", _sweep_batch(512, 320), 512, 320, 320, 5, 1, "bf16", 2005, "uniform"),
]


@pytest.mark.parametrize("case", PLAN_VARIANTS, ids=lambda c: c.name)
def test_plan_variants_at_sweep_sizes_sampled(oracle, case):
    assert _supported(case), f"{case.name}: no on-chip plan"
    check_sampled(oracle, case, nplanes=4, nchannels=2)


def test_weight_gradient_is_deterministic():
    case = STAGE1
    g = gpu_inputs(make_inputs(case))
    a = wt.backward_weight(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"],
                           case.L)
    a = {k: v.clone() for k, v in a.items()}
    b = wt.backward_weight(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"],
                           case.L)
    torch.cuda.synchronize()
    for k in PARAMS:
        assert torch.equal(a[k], b[k]), k


def test_outputs_do_not_depend_on_stale_memory(oracle):
    # Outputs and gradients are overwritten: pre-filled garbage must not leak.
    case = SMALL[1]
    inp = make_inputs(case)
    g = gpu_inputs(inp)
    y = torch.full_like(g["x"], float("nan"))
    wt.forward(g["x"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], case.L, y=y)
    grads = {k: torch.full_like(g[k], float("nan")) for k in PARAMS}
    wt.backward_weight(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], case.L,
                       grads=grads)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    for k in PARAMS:
        assert torch.isfinite(grads[k]).all(), k


# NHWC (channels-last) activations: the same layer on the same logical
# values, gathered and scattered element by element.  Shapes cover whole
# planes, strips (2, 8 and 16 CTAs), planes padded on chip, L = 0, k = 1 and
# 7, bf16, and rows that are not whole 16-byte chunks (allowed in NHWC only).
NHWC_SMALL = [
    Case("nhwc_odd_batch_stage1_plane", 3, 5, 56, 56, 5, 3, "f32", 51, "normal", "normal"),
    Case("nhwc_rect_24x40", 2, 3, 24, 40, 3, 3, "f32", 52, "normal", "normal"),
    Case("nhwc_L0", 2, 3, 12, 8, 5, 0, "f32", 53, "normal", "normal"),
    Case("nhwc_k1", 1, 2, 16, 16, 1, 2, "f32", 54, "normal", "normal"),
    Case("nhwc_k7_L4", 2, 3, 32, 32, 7, 4, "f32", 55, "normal", "normal"),
    Case("nhwc_bf16_stage1_plane", 3, 4, 56, 56, 5, 3, "bf16", 56, "uniform", "normal"),
    Case("nhwc_bf16_pad_13x12", 2, 3, 13, 12, 5, 2, "bf16", 57, "normal", "normal"),
    Case("nhwc_pad_30x28_L3", 3, 2, 30, 28, 5, 3, "f32", 58, "normal", "normal"),
    Case("nhwc_strips_128_L2", 1, 3, 128, 128, 5, 2, "f32", 59, "normal", "normal"),
    Case("nhwc_strips_256_L3_bf16", 1, 2, 256, 256, 3, 3, "bf16", 60, "normal", "normal"),
    Case("nhwc_pad_strips_250x248", 1, 1, 250, 248, 5, 4, "f32", 61, "normal", "normal"),
    # C a multiple of 8 on whole planes of a multiple of 32 pixels: the forward and input gradient
    # run as clusters of 8 CTAs over channel octets (odd unit counts per cluster, bf16, L = 0,
    # k = 1 and 7, a 64x64 plane at one CTA per SM)
    Case("nhwc_octets_stage1_plane", 3, 16, 56, 56, 5, 3, "f32", 63, "normal", "normal"),
    Case("nhwc_octets_bf16_32", 2, 8, 32, 32, 3, 2, "bf16", 64, "uniform", "normal"),
    Case("nhwc_octets_L0_k7", 2, 16, 56, 56, 7, 0, "f32", 65, "normal", "normal"),
    Case("nhwc_octets_k1_bf16", 5, 8, 16, 16, 1, 2, "bf16", 66, "normal", "normal"),
    Case("nhwc_octets_64_L4", 1, 24, 64, 64, 5, 4, "f32", 67, "normal", "normal"),
    # runs of an even number of pixels that is not a multiple of 4 (98 at 28x28, 30 at 20x12)
    Case("nhwc_octets_28_stage2_plane", 3, 16, 28, 28, 5, 2, "f32", 69, "normal", "normal"),
    Case("nhwc_octets_28_bf16_L0", 2, 8, 28, 28, 3, 0, "bf16", 70, "normal", "normal"),
    Case("nhwc_octets_20x12_bf16", 5, 8, 20, 12, 3, 1, "bf16", 71, "uniform", "normal"),
    # levels past the pyramid (L = 5: CTA barriers inside the analysis of an octet walk)
    Case("nhwc_octets_64_L5", 2, 8, 64, 64, 3, 5, "f32", 73, "normal", "normal"),
    Case("nhwc_octets_32_L5_bf16", 2, 16, 32, 32, 5, 5, "bf16", 74, "normal", "normal"),
]
NHWC_OCTETS = [c for c in NHWC_SMALL if c.name.startswith("nhwc_octets")]


@pytest.mark.parametrize("case", NHWC_SMALL, ids=lambda c: c.name)
def test_nhwc_small_case_all_outputs(oracle, case):
    check_full(oracle, case, case.calls, nhwc=True)


@pytest.mark.parametrize("mode", ["auto", "one_pass"])
@pytest.mark.parametrize("case", NHWC_SMALL[:8] + NHWC_OCTETS[:2] + NHWC_OCTETS[-4:], ids=lambda c: c.name)
def test_nhwc_small_case_fused_backward(oracle, case, mode):
    if mode == "one_pass" and not _one_pass_plan_exists(case, nhwc=True):
        pytest.skip("planes split into cluster strips have no one-pass plan")
    check_full(oracle, case, ("bwd_in", "bwd_w"), fused_bwd=mode, nhwc=True)


@pytest.mark.parametrize("case", [STAGE1, STAGE2, TRAIN_BF16], ids=lambda c: c.name)
def test_nhwc_full_size_workloads_sampled(oracle, case):
    check_sampled(oracle, case, nhwc=True)


@pytest.mark.parametrize("case", [
    Case("nhwc_vs_nchw", 4, 6, 40, 36, 5, 3, "f32", 62, "normal", "normal"),
    Case("nhwc_vs_nchw_octets", 3, 16, 32, 32, 5, 3, "f32", 68, "normal", "normal"),
    Case("nhwc_vs_nchw_octets_28", 3, 16, 28, 28, 5, 2, "f32", 72, "normal", "normal"),
], ids=lambda c: c.name)
def test_nhwc_matches_nchw_bitwise(case):
    # Same on-chip arithmetic in the same order: the layouts must agree bit for bit
    # (element-by-element gather, and channel octets).
    inp = make_inputs(case)
    a = run_gpu(case, gpu_inputs(inp), ("fwd", "bwd_in", "bwd_w"))
    b = run_gpu(case, gpu_inputs(inp, nhwc=True), ("fwd", "bwd_in", "bwd_w"))
    assert torch.equal(a["y"], b["y"]) and torch.equal(a["dx"], b["dx"])
    for k in PARAMS:
        assert torch.equal(a["grads"][k], b["grads"][k]), k
