"""wtconv_backward_weight_noalloc against wtconv_backward_weight (needs a B200).

Some callers cannot allocate device memory: code running under a fixed
memory budget, inside an allocator hook, or while a stream is being captured
into a graph (where cudaMalloc is not allowed).  For them the library offers
wtconv_backward_weight_noalloc, which keeps the weight gradient's partial
sums in a fixed array inside the library instead of a caller workspace.  This
test calls it through the C ABI twice in a row, on two different problems, and
checks each result against the workspace entry point on the same inputs.  The
file is named to be collected last, and it stands alone: it builds what it
needs and shares no state with the other tests.
"""
import ctypes

import pytest
import torch

import memory_bound_cnn_wtconv_b200 as wt
from wtconv_inputs import Case, make_inputs

pytestmark = pytest.mark.gpu

PARAMS = ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")
CASES = [
    Case("noalloc_stage1_like", 8, 12, 56, 56, 5, 3, "f32", 41, "normal", "normal"),
    Case("noalloc_bf16_rect", 6, 5, 32, 24, 3, 2, "bf16", 42, "normal", "normal"),
]


def _noalloc(lib, case, g, grads, stream):
    fn = lib.wtconv_backward_weight_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(wt.Desc)] + [vp] * 13
    fn.restype = ctypes.c_int
    d = wt.make_desc(g["x"], case.k, case.L)
    p = lambda t: vp(t.data_ptr())
    return fn(ctypes.byref(d), p(g["x"]), p(g["dy"]), p(g["base_w"]), p(g["base_b"]), p(g["base_scale"]),
              p(g["wt_w"]), p(g["wt_scale"]), p(grads["base_w"]), p(grads["base_b"]), p(grads["base_scale"]),
              p(grads["wt_w"]), p(grads["wt_scale"]), vp(stream.cuda_stream))


def test_noalloc_matches_workspace_entry_point_twice(cuda_lib):
    stream = torch.cuda.current_stream()
    for case in CASES:  # two calls in a row; the second sees the first one's leftovers
        g = {k: v.cuda() for k, v in make_inputs(case).items()}
        ref = wt.backward_weight(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"],
                                 g["wt_scale"], case.L)
        ref = {k: v.clone() for k, v in ref.items()}
        out = {k: torch.full_like(ref[k], float("nan")) for k in PARAMS}
        rc = _noalloc(cuda_lib, case, g, out, stream)
        assert rc == 0, wt.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        for k in PARAMS:
            r, o = ref[k].double(), out[k].double()
            err = float((o - r).abs().max() / r.abs().max().clamp_min(1e-30))
            assert err <= 1e-5, (case.name, k, err)


def test_noalloc_refuses_oversize_plans_and_leaves_outputs_untouched(cuda_lib):
    # Partials beyond the fixed 4 MiB array: WTCONV_ERR_WORKSPACE, nothing enqueued.
    case = Case("noalloc_oversize", 2, 4096, 16, 16, 7, 2, "f32", 43, "normal", "normal")
    g = {k: v.cuda() for k, v in make_inputs(case).items()}
    out = {k: torch.full_like(g[k], float("nan")) for k in PARAMS}
    rc = _noalloc(cuda_lib, case, g, out, torch.cuda.current_stream())
    assert rc == 7, wt.STATUS.get(rc, rc)
    torch.cuda.synchronize()
    for k in PARAMS:
        assert torch.isnan(out[k]).all(), k
