"""C ABI checks that need no GPU.

The library must load and export every function declared in include/wtconv.h,
and argument validation (done on the host before any CUDA call) must return
the documented status codes.  Pointers passed here are never dereferenced:
each case fails validation before any launch.
"""
import ctypes
import os
import re

import pytest

import memory_bound_cnn_wtconv_b200 as w

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wtconv.h")

OK, NULLPTR, BAD_SHAPE, BAD_K, BAD_L, MISALIGNED, DTYPE, WORKSPACE, UNSUPPORTED, CUDA, LAYOUT = range(11)
FAKE = 0x10000  # 16-byte aligned, never dereferenced


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(wtconv_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_api():
    names = declared_functions()
    for n in ("wtconv_forward", "wtconv_backward_input", "wtconv_backward_weight", "wtconv_workspace_bytes",
              "wtconv_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(cuda_lib):
    for name in declared_functions():
        assert hasattr(cuda_lib, name), name


def _desc(B=2, C=3, H=16, W=16, k=5, L=2, dtype=0, layout=0):
    return w.Desc(B, C, H, W, k, L, dtype, layout)


def _fwd(lib, d, x=FAKE, y=FAKE, ww=FAKE, ws=FAKE):
    p = ctypes.c_void_p
    return lib.wtconv_forward(ctypes.byref(d) if d is not None else None, p(x), p(FAKE), p(FAKE), p(FAKE),
                              p(ww), p(ws), p(y), None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), BAD_SHAPE), (dict(C=-1), BAD_SHAPE), (dict(H=0), BAD_SHAPE),
    (dict(k=4), BAD_K), (dict(k=9), BAD_K), (dict(k=0), BAD_K),
    (dict(L=-1), BAD_L), (dict(L=7), BAD_L),
    (dict(W=6, L=1), BAD_SHAPE), (dict(H=12, W=12, L=3, dtype=1), BAD_SHAPE),
    (dict(dtype=2), DTYPE), (dict(layout=2), LAYOUT), (dict(layout=-1), LAYOUT),
    # NHWC gathers element by element, so bf16 rows need not be whole 16-byte chunks
    (dict(H=12, W=12, L=3, dtype=1, layout=1), OK),
])
def test_forward_validation(cuda_lib, kw, code):
    if code == OK:  # valid: planned without launching (the workspace query plans every pass)
        assert cuda_lib.wtconv_workspace_bytes(ctypes.byref(_desc(**kw))) > 0
        return
    assert _fwd(cuda_lib, _desc(**kw)) == code


@pytest.mark.parametrize("kw", [dict(H=12, L=3), dict(W=20, L=3), dict(H=13, W=12, L=2), dict(H=9, W=16, L=4, dtype=1)])
def test_sizes_not_multiples_of_2L_are_planned(cuda_lib, kw):
    # Zero-padded on chip (host planning only; nothing is launched here).
    assert cuda_lib.wtconv_workspace_bytes(ctypes.byref(_desc(**kw))) > 0


@pytest.mark.parametrize("shape,k,L,dtype", [
    ((32, 96, 56, 56), 5, 3, 0), ((64, 96, 56, 56), 5, 3, 1), ((32, 192, 28, 28), 5, 2, 0),
    ((256, 64, 32, 32), 3, 1, 0), ((64, 16, 56, 56), 7, 0, 0), ((1024, 64, 32, 32), 3, 1, 0),
    ((2, 5, 56, 56), 5, 3, 0), ((4, 192, 28, 28), 5, 2, 0), ((6, 192, 32, 32), 3, 1, 1),
])
def test_nhwc_workspace_equals_nchw(cuda_lib, shape, k, L, dtype):
    # The weight gradient's batch groups are chosen without the channel-octet buffer, so both
    # layouts of a shape need the same workspace; the binding's query takes the layout.
    import torch
    B, C, H, W = shape
    nchw = cuda_lib.wtconv_workspace_bytes(ctypes.byref(_desc(B, C, H, W, k, L, dtype, 0)))
    nhwc = cuda_lib.wtconv_workspace_bytes(ctypes.byref(_desc(B, C, H, W, k, L, dtype, 1)))
    assert 0 < nhwc == nchw
    tdt = torch.bfloat16 if dtype else torch.float32
    assert w.workspace_bytes(shape, k, L, tdt, channels_last=True) == nhwc
    assert w.workspace_bytes(shape, k, L, tdt) == nchw


def test_null_and_alignment(cuda_lib):
    assert _fwd(cuda_lib, None) == NULLPTR
    assert _fwd(cuda_lib, _desc(), x=0) == NULLPTR
    assert _fwd(cuda_lib, _desc(), ww=0) == NULLPTR
    assert _fwd(cuda_lib, _desc(), x=FAKE + 4) == MISALIGNED
    assert _fwd(cuda_lib, _desc(), y=FAKE + 8) == MISALIGNED


def test_unsupported_plane(cuda_lib):
    # Planes up to 256 x 256 are split into cluster strips; a 64-row strip of
    # a 1024 x 1024 plane still does not fit on one SM.
    assert _fwd(cuda_lib, _desc(H=1024, W=1024, L=4)) == UNSUPPORTED
    assert _fwd(cuda_lib, _desc(H=256, W=256, L=4)) != UNSUPPORTED


def test_backward_input_validation(cuda_lib):
    p = ctypes.c_void_p
    d = _desc(k=2)
    assert cuda_lib.wtconv_backward_input(ctypes.byref(d), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE),
                                          None) == BAD_K
    d = _desc()
    assert cuda_lib.wtconv_backward_input(ctypes.byref(d), p(0), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE),
                                          None) == NULLPTR


def test_backward_weight_workspace(cuda_lib):
    p = ctypes.c_void_p
    d = _desc()
    need = cuda_lib.wtconv_workspace_bytes(ctypes.byref(d))
    assert need > 0
    args = [p(FAKE)] * 12
    assert cuda_lib.wtconv_backward_weight(ctypes.byref(d), *args, p(FAKE), ctypes.c_size_t(need - 4),
                                           None) == WORKSPACE
    assert cuda_lib.wtconv_backward_weight(ctypes.byref(d), *args, p(0), ctypes.c_size_t(need), None) == WORKSPACE
    bad = _desc(L=9)
    assert cuda_lib.wtconv_workspace_bytes(ctypes.byref(bad)) == 0


def test_status_strings(cuda_lib):
    for code in range(11):
        s = cuda_lib.wtconv_status_string(code)
        assert s and len(s) > 1
    assert cuda_lib.wtconv_status_string(999) == b"unknown status"


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(w, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(w, "_lib", None)
    with pytest.raises(w.WTConvLibraryMissing):
        w.load_library()


def test_product_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "memory_bound_cnn_wtconv_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "wtconv_oracle" not in text and "liboracle" not in text, f


def test_backward_validation(cuda_lib):
    p = ctypes.c_void_p
    d = _desc()
    need = cuda_lib.wtconv_workspace_bytes(ctypes.byref(d))
    args = [p(FAKE)] * 7  # x, dy, base_w, base_b, base_scale, wt_w, wt_scale
    grads = [p(FAKE)] * 5
    assert cuda_lib.wtconv_backward(ctypes.byref(d), *args, p(0), *grads, p(FAKE), ctypes.c_size_t(need),
                                    None) == NULLPTR
    assert cuda_lib.wtconv_backward(ctypes.byref(d), *args, p(FAKE), *grads, p(FAKE), ctypes.c_size_t(need - 4),
                                    None) == WORKSPACE
    assert cuda_lib.wtconv_backward(ctypes.byref(_desc(k=4)), *args, p(FAKE), *grads, p(FAKE),
                                    ctypes.c_size_t(need), None) == BAD_K


def test_backward_one_pass_validation(cuda_lib):
    p = ctypes.c_void_p
    args = [p(FAKE)] * 7
    grads = [p(FAKE)] * 5
    d = _desc(H=32, W=32, L=2)
    need = cuda_lib.wtconv_workspace_bytes(ctypes.byref(d))
    fn = cuda_lib.wtconv_backward_one_pass
    assert fn(ctypes.byref(d), *args, p(0), *grads, p(FAKE), ctypes.c_size_t(need), None) == NULLPTR
    assert fn(ctypes.byref(d), *args, p(FAKE + 4), *grads, p(FAKE), ctypes.c_size_t(need), None) == MISALIGNED
    assert fn(ctypes.byref(d), *args, p(FAKE), *grads, p(FAKE), ctypes.c_size_t(need - 4), None) == WORKSPACE
    # A 256 x 256 plane is held as cluster strips: no one-pass plan.  The
    # library-picked backward still plans it (as the two passes).
    big = _desc(H=256, W=256, L=4)
    need_big = cuda_lib.wtconv_workspace_bytes(ctypes.byref(big))
    assert need_big > 0
    assert fn(ctypes.byref(big), *args, p(FAKE), *grads, p(FAKE), ctypes.c_size_t(need_big), None) == UNSUPPORTED
    assert cuda_lib.wtconv_backward(ctypes.byref(big), *args, p(FAKE), *grads, p(FAKE),
                                    ctypes.c_size_t(need_big - 4), None) == WORKSPACE


def test_backward_checks_the_workspace_before_any_pass(cuda_lib):
    # Whichever path the library picks, a short workspace is refused before
    # the input-gradient pass could write dx (dx is a never-dereferenced fake).
    p = ctypes.c_void_p
    for kw in (dict(), dict(B=32, C=96, H=56, W=56, k=5, L=3), dict(H=128, W=128, L=3)):
        d = _desc(**kw)
        need = cuda_lib.wtconv_workspace_bytes(ctypes.byref(d))
        assert need > 0
        rc = cuda_lib.wtconv_backward(ctypes.byref(d), *([p(FAKE)] * 14), ctypes.c_size_t(need - 4), None)
        assert rc == WORKSPACE, kw


def test_noalloc_rejects_plans_beyond_its_array(cuda_lib):
    # The fixed array holds 2^20 floats of partial sums and counters; a plan
    # that needs more is refused after planning, before any CUDA call.
    p = ctypes.c_void_p
    d = _desc(B=4, C=4096, H=16, W=16, k=7, L=2)
    assert cuda_lib.wtconv_workspace_bytes(ctypes.byref(d)) > 4 << 20
    fn = cuda_lib.wtconv_backward_weight_noalloc
    fn.argtypes = [ctypes.POINTER(w.Desc)] + [p] * 13
    fn.restype = ctypes.c_int
    assert fn(ctypes.byref(d), *([p(FAKE)] * 12), None) == WORKSPACE
