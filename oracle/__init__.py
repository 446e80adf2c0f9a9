"""WTConv oracle -- TEST INFRASTRUCTURE ONLY.

Python access (ctypes + numpy, float64) to the plain C restatement of the
WTConv layer in ``wtconv_oracle.c``.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this package; the CUDA library and its
binding never do, and this package imports nothing from them.

The layer (arXiv 2608.10805, "Fast and Memory-Efficient Wavelet Convolutions
via I/O-Aware Reformulation", Abstract) is computed literally: depthwise base
conv with per-channel scale and bias, an L-level orthonormal 2-D Haar analysis
recursing on the raw LL subband, a scaled depthwise conv per subband, and the
inverse Haar synthesis cascade.  See ``wtconv_oracle.c`` for the formulas and
the subband convention.

Planes whose H or W is not a multiple of 2^L: the pages fix no rule for them.
The plainest reading, taken here: zero-pad the plane at the bottom and right
to the next multiples of 2^L, apply the layer, crop the output back.  Its
adjoint (input gradient) crops the adjoint applied to the zero-padded dy, and
the weight gradient is taken on the zero-padded x and dy.  (The same result
follows from padding each level's LL by one row / column when odd and
cropping each level's reconstruction; a test checks the two agree.)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wtconv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_wtconv.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)


def compile_oracle(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle C file into a shared library with gcc and OpenMP."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", *extra_flags, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    return out


def build() -> str:
    """Build the oracle library if it is missing or older than its source."""
    with _lock:
        if (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
            compile_oracle()
    return _LIB_PATH


def _bind(lib):
    i = ctypes.c_int
    lib.orc_dwt2.argtypes = [_D, i, i, _D]
    lib.orc_iwt2.argtypes = [_D, i, i, _D]
    lib.orc_dwconv.argtypes = [_D, i, i, _D, i, _D]
    lib.orc_dwconv_adj.argtypes = [_D, i, i, _D, i, _D]
    lib.orc_forward.argtypes = [i] * 6 + [_D] * 7
    lib.orc_backward_input.argtypes = [i] * 6 + [_D] * 6
    lib.orc_backward_weight.argtypes = [i] * 6 + [_D] * 12
    for f in (lib.orc_forward, lib.orc_backward_input, lib.orc_backward_weight, lib.orc_num_threads):
        f.restype = ctypes.c_int
    for f in (lib.orc_dwt2, lib.orc_iwt2, lib.orc_dwconv, lib.orc_dwconv_adj):
        f.restype = None
    return lib


def load_library(path: str | None = None):
    """Load (building if needed) the oracle library; ``path`` loads a variant."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _f64(a) -> np.ndarray:
    return np.array(a, dtype=np.float64, copy=True, order="C")


def _p(a: np.ndarray):
    return a.ctypes.data_as(_D)


class Oracle:
    """Thin numpy front end over one loaded oracle library."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load_library()

    def num_threads(self) -> int:
        return int(self.lib.orc_num_threads())

    # -- single-plane primitives --
    def dwt2(self, X):
        X = _f64(X)
        nh, nw = X.shape
        S = np.empty((4, nh // 2, nw // 2))
        self.lib.orc_dwt2(_p(X), nh, nw, _p(S))
        return S

    def iwt2(self, S):
        S = _f64(S)
        _, mh, mw = S.shape
        X = np.empty((2 * mh, 2 * mw))
        self.lib.orc_iwt2(_p(S), mh, mw, _p(X))
        return X

    def dwconv(self, X, w):
        X, w = _f64(X), _f64(w)
        Y = np.empty_like(X)
        self.lib.orc_dwconv(_p(X), X.shape[0], X.shape[1], _p(w), w.shape[0], _p(Y))
        return Y

    def dwconv_adj(self, Y, w):
        Y, w = _f64(Y), _f64(w)
        X = np.empty_like(Y)
        self.lib.orc_dwconv_adj(_p(Y), Y.shape[0], Y.shape[1], _p(w), w.shape[0], _p(X))
        return X

    # -- the layer --
    @staticmethod
    def _dims(x, base_w, L):
        B, C, H, W = x.shape
        k = base_w.shape[-1]
        return B, C, H, W, k, L

    @staticmethod
    def _wt(wt_w, wt_scale, L, C, k):
        if L == 0:
            return np.zeros((1,)), np.zeros((1,))
        return _f64(wt_w).reshape(L, C, 4, k, k), _f64(wt_scale).reshape(L, C, 4)

    @staticmethod
    def _pad(a, L):
        """a zero-padded at the bottom / right to multiples of 2^L (a itself if already)."""
        m = 1 << L
        H, W = a.shape[-2:]
        Hp, Wp = -(-H // m) * m, -(-W // m) * m
        if (Hp, Wp) == (H, W):
            return a
        out = np.zeros(a.shape[:-2] + (Hp, Wp))
        out[..., :H, :W] = a
        return out

    def forward(self, x, base_w, base_b, base_scale, wt_w, wt_scale, L):
        x, base_w, base_b, base_scale = map(_f64, (x, base_w, base_b, base_scale))
        xp = self._pad(x, L)
        if xp is not x:
            H, W = x.shape[-2:]
            return self.forward(xp, base_w, base_b, base_scale, wt_w, wt_scale, L)[..., :H, :W].copy()
        B, C, H, W, k, L = self._dims(x, base_w, L)
        wt_w, wt_scale = self._wt(wt_w, wt_scale, L, C, k)
        y = np.empty_like(x)
        rc = self.lib.orc_forward(B, C, H, W, k, L, _p(x), _p(base_w), _p(base_b), _p(base_scale),
                                  _p(wt_w), _p(wt_scale), _p(y))
        if rc != 0:
            raise ValueError(f"oracle forward rejected its arguments (code {rc})")
        return y

    def backward_input(self, dy, base_w, base_scale, wt_w, wt_scale, L):
        dy, base_w, base_scale = map(_f64, (dy, base_w, base_scale))
        dyp = self._pad(dy, L)
        if dyp is not dy:
            H, W = dy.shape[-2:]
            return self.backward_input(dyp, base_w, base_scale, wt_w, wt_scale, L)[..., :H, :W].copy()
        B, C, H, W, k, L = self._dims(dy, base_w, L)
        wt_w, wt_scale = self._wt(wt_w, wt_scale, L, C, k)
        dx = np.empty_like(dy)
        rc = self.lib.orc_backward_input(B, C, H, W, k, L, _p(dy), _p(base_w), _p(base_scale),
                                         _p(wt_w), _p(wt_scale), _p(dx))
        if rc != 0:
            raise ValueError(f"oracle backward_input rejected its arguments (code {rc})")
        return dx

    def backward_weight(self, x, dy, base_w, base_b, base_scale, wt_w, wt_scale, L):
        x, dy, base_w, base_b, base_scale = map(_f64, (x, dy, base_w, base_b, base_scale))
        xp = self._pad(x, L)
        if xp is not x:
            return self.backward_weight(xp, self._pad(dy, L), base_w, base_b, base_scale, wt_w, wt_scale, L)
        B, C, H, W, k, L = self._dims(x, base_w, L)
        wt_w, wt_scale = self._wt(wt_w, wt_scale, L, C, k)
        d_base_w = np.empty((C, k, k))
        d_base_b = np.empty((C,))
        d_base_scale = np.empty((C,))
        d_wt_w = np.empty((max(L, 1), C, 4, k, k))
        d_wt_scale = np.empty((max(L, 1), C, 4))
        rc = self.lib.orc_backward_weight(B, C, H, W, k, L, _p(x), _p(dy), _p(base_w), _p(base_b),
                                          _p(base_scale), _p(wt_w), _p(wt_scale), _p(d_base_w),
                                          _p(d_base_b), _p(d_base_scale), _p(d_wt_w), _p(d_wt_scale))
        if rc != 0:
            raise ValueError(f"oracle backward_weight rejected its arguments (code {rc})")
        if L == 0:
            d_wt_w = np.zeros((0, C, 4, k, k))
            d_wt_scale = np.zeros((0, C, 4))
        return dict(base_w=d_base_w, base_b=d_base_b, base_scale=d_base_scale,
                    wt_w=d_wt_w, wt_scale=d_wt_scale)


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
