"""B200-native fused WTConv: Python binding of the C ABI in ``include/wtconv.h``.

Argument marshalling only.  Every step of the layer runs in the CUDA kernels
of ``libwtconv_b200.so``; there is no CPU or PyTorch fallback.  If the
library is missing, importing works but every call raises
``WTConvLibraryMissing``.  Build it with ``python -m memory_bound_cnn_wtconv_b200.build``.

The layer ("Fast and Memory-Efficient Wavelet Convolutions via I/O-Aware
Reformulation", arXiv 2608.10805, Abstract): a depthwise k x k base conv with
per-channel scale and bias, plus an L-level orthonormal Haar wavelet branch
with one scaled depthwise conv per subband, recombined by the inverse Haar
synthesis.  Parameter layouts: base_w [C,k,k], base_b [C], base_scale [C],
wt_w [L,C,4,k,k], wt_scale [L,C,4] (float32); activations float32 or bfloat16
on one CUDA device, either contiguous (NCHW) or channels-last contiguous
(NHWC, ``torch.channels_last``); a call's activations share the layout.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "forward", "backward_input", "backward_weight", "backward", "workspace_bytes", "WTConvError",
    "WTConvLibraryMissing", "library_path", "load_library", "Desc", "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libwtconv_b200.so")
_lib = None

STATUS = {
    0: "WTCONV_OK", 1: "WTCONV_ERR_NULLPTR", 2: "WTCONV_ERR_BAD_SHAPE", 3: "WTCONV_ERR_BAD_K",
    4: "WTCONV_ERR_BAD_L", 5: "WTCONV_ERR_MISALIGNED", 6: "WTCONV_ERR_DTYPE", 7: "WTCONV_ERR_WORKSPACE",
    8: "WTCONV_ERR_UNSUPPORTED", 9: "WTCONV_ERR_CUDA", 10: "WTCONV_ERR_LAYOUT",
}
F32, BF16 = 0, 1
NCHW, NHWC = 0, 1


class WTConvError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({status_string(code)})")


class WTConvLibraryMissing(RuntimeError):
    pass


class Desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("C", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("k", ctypes.c_int), ("L", ctypes.c_int), ("dtype", ctypes.c_int), ("layout", ctypes.c_int)]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load ``libwtconv_b200.so`` (raises WTConvLibraryMissing if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise WTConvLibraryMissing(
            f"{_LIB_PATH} is missing; build it with `python -m memory_bound_cnn_wtconv_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
    dp = ctypes.POINTER(Desc)
    lib.wtconv_status_string.argtypes = [ctypes.c_int]
    lib.wtconv_status_string.restype = ctypes.c_char_p
    lib.wtconv_workspace_bytes.argtypes = [dp]
    lib.wtconv_workspace_bytes.restype = sz
    lib.wtconv_forward.argtypes = [dp, vp, fp, fp, fp, fp, fp, vp, vp]
    lib.wtconv_forward.restype = ctypes.c_int
    lib.wtconv_backward_input.argtypes = [dp, vp, fp, fp, fp, fp, vp, vp]
    lib.wtconv_backward_input.restype = ctypes.c_int
    lib.wtconv_backward_weight.argtypes = [dp, vp, vp, fp, fp, fp, fp, fp, fp, fp, fp, fp, fp, vp, sz, vp]
    lib.wtconv_backward_weight.restype = ctypes.c_int
    lib.wtconv_backward.argtypes = [dp, vp, vp, fp, fp, fp, fp, fp, vp, fp, fp, fp, fp, fp, vp, sz, vp]
    lib.wtconv_backward.restype = ctypes.c_int
    lib.wtconv_backward_one_pass.argtypes = lib.wtconv_backward.argtypes
    lib.wtconv_backward_one_pass.restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(code: int) -> str:
    try:
        return load_library().wtconv_status_string(int(code)).decode()
    except WTConvLibraryMissing:
        return STATUS.get(code, "unknown")


def _check(code: int, what: str) -> None:
    if code != 0:
        raise WTConvError(code, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")


def layout_of(t: torch.Tensor) -> int:
    """NCHW (0) for a contiguous tensor, NHWC (1) for a channels-last
    contiguous one (a tensor that is both reads the same either way)."""
    if t.dim() == 4 and t.is_contiguous():
        return NCHW
    if t.dim() == 4 and t.is_contiguous(memory_format=torch.channels_last):
        return NHWC
    raise ValueError("activations must be 4-D and contiguous (NCHW) or channels-last contiguous (NHWC)")


def _act(t: torch.Tensor, name: str, layout=None) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if layout is None:
        layout_of(t)
    elif not t.is_contiguous(memory_format=torch.channels_last if layout == NHWC else torch.contiguous_format):
        raise ValueError(f"{name} must have the layout of the input ({'NHWC' if layout == NHWC else 'NCHW'})")
    return t


def _param(t, name: str, device, shape):
    if t is None:
        return None
    if t.dtype != torch.float32 or t.device != device or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous float32 tensor on {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def make_desc(x: torch.Tensor, k: int, L: int) -> Desc:
    B, C, H, W = x.shape
    return Desc(B, C, H, W, int(k), int(L), _dtype_code(x), layout_of(x))


def _params(x, base_w, base_b, base_scale, wt_w, wt_scale, L):
    dev = x.device
    C = x.shape[1]
    k = base_w.shape[-1]
    _param(base_w, "base_w", dev, (C, k, k))
    if base_b is not None:
        _param(base_b, "base_b", dev, (C,))
    _param(base_scale, "base_scale", dev, (C,))
    if L > 0:
        _param(wt_w, "wt_w", dev, (L, C, 4, k, k))
        _param(wt_scale, "wt_scale", dev, (L, C, 4))
    return k


def workspace_bytes(x_shape, k: int, L: int, dtype=torch.float32, channels_last: bool = False) -> int:
    """Workspace of ``backward_weight`` / ``backward`` for activations of this
    shape (NCHW), dtype and layout (``channels_last``: NHWC; both layouts of a
    shape need the same size)."""
    B, C, H, W = x_shape
    d = Desc(B, C, H, W, int(k), int(L), F32 if dtype == torch.float32 else BF16,
             NHWC if channels_last else NCHW)
    return int(load_library().wtconv_workspace_bytes(ctypes.byref(d)))


def forward(x, base_w, base_b, base_scale, wt_w, wt_scale, L: int, y=None, stream=None):
    """y = WTConv(x) via ``wtconv_forward``; returns y (allocated if not given)."""
    lib = load_library()
    _act(x, "x")
    k = _params(x, base_w, base_b, base_scale, wt_w, wt_scale, L)
    if y is None:
        y = torch.empty_like(x)
    _act(y, "y", layout_of(x))
    d = make_desc(x, k, L)
    _check(lib.wtconv_forward(ctypes.byref(d), _ptr(x), _ptr(base_w), _ptr(base_b), _ptr(base_scale),
                              _ptr(wt_w if L > 0 else None), _ptr(wt_scale if L > 0 else None), _ptr(y),
                              _stream(x.device, stream)), "wtconv_forward")
    return y


def backward_input(dy, base_w, base_scale, wt_w, wt_scale, L: int, dx=None, stream=None):
    """dx = J^T dy via ``wtconv_backward_input``; returns dx."""
    lib = load_library()
    _act(dy, "dy")
    k = _params(dy, base_w, None, base_scale, wt_w, wt_scale, L)
    if dx is None:
        dx = torch.empty_like(dy)
    _act(dx, "dx", layout_of(dy))
    d = make_desc(dy, k, L)
    _check(lib.wtconv_backward_input(ctypes.byref(d), _ptr(dy), _ptr(base_w), _ptr(base_scale),
                                     _ptr(wt_w if L > 0 else None), _ptr(wt_scale if L > 0 else None), _ptr(dx),
                                     _stream(dy.device, stream)), "wtconv_backward_input")
    return dx


def backward_weight(x, dy, base_w, base_b, base_scale, wt_w, wt_scale, L: int, grads=None, workspace=None,
                    stream=None):
    """Parameter gradients via ``wtconv_backward_weight``.

    Returns a dict with keys base_w, base_b, base_scale, wt_w, wt_scale
    (float32, overwritten).  ``workspace`` is a uint8 CUDA tensor of at least
    ``workspace_bytes`` bytes; allocated here if not given.
    """
    lib = load_library()
    _act(x, "x")
    _act(dy, "dy", layout_of(x))
    if dy.shape != x.shape or dy.dtype != x.dtype or dy.device != x.device:
        raise ValueError("x and dy must have the same shape, dtype and device")
    k = _params(x, base_w, base_b, base_scale, wt_w, wt_scale, L)
    B, C, H, W = x.shape
    dev = x.device
    if grads is None:
        grads = dict(base_w=torch.empty((C, k, k), device=dev), base_b=torch.empty((C,), device=dev),
                     base_scale=torch.empty((C,), device=dev),
                     wt_w=torch.empty((L, C, 4, k, k), device=dev), wt_scale=torch.empty((L, C, 4), device=dev))
    d = make_desc(x, k, L)
    nbytes = int(lib.wtconv_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=dev)
    _check(lib.wtconv_backward_weight(
        ctypes.byref(d), _ptr(x), _ptr(dy), _ptr(base_w), _ptr(base_b), _ptr(base_scale),
        _ptr(wt_w if L > 0 else None), _ptr(wt_scale if L > 0 else None),
        _ptr(grads["base_w"]), _ptr(grads["base_b"]), _ptr(grads["base_scale"]),
        _ptr(grads["wt_w"] if L > 0 else None), _ptr(grads["wt_scale"] if L > 0 else None),
        _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        _stream(dev, stream)), "wtconv_backward_weight")
    return grads


def backward(x, dy, base_w, base_b, base_scale, wt_w, wt_scale, L: int, dx=None, grads=None, workspace=None,
             stream=None, one_pass: bool = False):
    """dx and the parameter gradients via ``wtconv_backward`` (the library
    picks the one-pass kernel or the two passes), or with ``one_pass`` via
    ``wtconv_backward_one_pass`` (raises WTConvError WTCONV_ERR_UNSUPPORTED
    for planes split into cluster strips).

    Returns (dx, grads) with grads as for ``backward_weight``.
    """
    lib = load_library()
    _act(x, "x")
    _act(dy, "dy", layout_of(x))
    if dy.shape != x.shape or dy.dtype != x.dtype or dy.device != x.device:
        raise ValueError("x and dy must have the same shape, dtype and device")
    k = _params(x, base_w, base_b, base_scale, wt_w, wt_scale, L)
    B, C, H, W = x.shape
    dev = x.device
    if dx is None:
        dx = torch.empty_like(dy)
    _act(dx, "dx", layout_of(dy))
    if grads is None:
        grads = dict(base_w=torch.empty((C, k, k), device=dev), base_b=torch.empty((C,), device=dev),
                     base_scale=torch.empty((C,), device=dev),
                     wt_w=torch.empty((L, C, 4, k, k), device=dev), wt_scale=torch.empty((L, C, 4), device=dev))
    d = make_desc(x, k, L)
    nbytes = int(lib.wtconv_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=dev)
    fn, name = ((lib.wtconv_backward_one_pass, "wtconv_backward_one_pass") if one_pass
                else (lib.wtconv_backward, "wtconv_backward"))
    _check(fn(
        ctypes.byref(d), _ptr(x), _ptr(dy), _ptr(base_w), _ptr(base_b), _ptr(base_scale),
        _ptr(wt_w if L > 0 else None), _ptr(wt_scale if L > 0 else None), _ptr(dx),
        _ptr(grads["base_w"]), _ptr(grads["base_b"]), _ptr(grads["base_scale"]),
        _ptr(grads["wt_w"] if L > 0 else None), _ptr(grads["wt_scale"] if L > 0 else None),
        _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        _stream(dev, stream)), name)
    return dx, grads


# Autograd function and module (defined after the calls they wrap).
from .module import WTConv2d, WTConvFunction, wtconv  # noqa: E402

__all__ += ["WTConv2d", "WTConvFunction", "wtconv"]
