"""Pins for the oracle: checks against facts that do not come from the oracle.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
if the oracle disagrees with:
  * hand-derived values of one Haar step (the definition: a 2x2 block maps to
    its sum and differences divided by 2 -- "SETAREH ... Haar wavelet"
    (kongchang.com), section on the Haar transform);
  * invariants of an orthogonal transform (perfect reconstruction with the
    transpose as inverse, Parseval, inner-product preservation -- same page,
    inner-product section);
  * a library routine (torch.nn.functional.conv2d in float64);
  * closed forms derived here from the layer's definition ("Fast and
    Memory-Efficient Wavelet Convolutions via I/O-Aware Reformulation",
    Abstract): the closed-form analysis and the closed-form, coordinate-bit
    indexed synthesis, special cases of scales and delta kernels;
  * calculus: the adjoint (dense operator) and central finite differences.

The same functions run against deliberately broken oracle builds in
test_oracle_mutants.py, which checks that every planted mistake is caught.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

RNG_SEED = 12345


# ---------------------------------------------------------------------------
# Independent closed forms (numpy / torch), written from the definition.
# ---------------------------------------------------------------------------
def sigma(s: int, a, b):
    """Sign of subband s for the bit pair (a, b): LL +, LH by row bit, HL by column bit, HH both."""
    a = np.asarray(a)
    b = np.asarray(b)
    if s == 0:
        return np.ones(np.broadcast(a, b).shape)
    if s == 1:
        return (-1.0) ** a * np.ones_like(b)
    if s == 2:
        return np.ones_like(a) * (-1.0) ** b
    return (-1.0) ** (a + b)


def closed_analysis(x: np.ndarray, l: int) -> np.ndarray:
    """S_{l,s}[i,j] = 2^-(l+1) sum over the 2^(l+1) block of sigma_s(bit_l dh, bit_l dw) x."""
    bs = 2 ** (l + 1)
    H, W = x.shape
    xr = x.reshape(H // bs, bs, W // bs, bs)
    bit = (np.arange(bs) >> l) & 1
    out = []
    for s in range(4):
        sg = sigma(s, bit[:, None], bit[None, :])
        out.append(np.einsum("iajb,ab->ij", xr, sg) / 2 ** (l + 1))
    return np.stack(out)


def closed_synthesis(hats, H: int, W: int) -> np.ndarray:
    """y[h,w] = sum_l 2^-(l+1) sum_s sigma_s(bit_l h, bit_l w) hat_{l,s}[h>>(l+1), w>>(l+1)]."""
    y = np.zeros((H, W))
    h = np.arange(H)[:, None]
    w = np.arange(W)[None, :]
    for l, hat in enumerate(hats):
        a = (h >> l) & 1
        b = (w >> l) & 1
        for s in range(4):
            y += 2.0 ** -(l + 1) * sigma(s, a, b) * hat[s][h >> (l + 1), w >> (l + 1)]
    return y


def torch_conv(X: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Cross-correlation, 'same' zero padding, float64 library routine."""
    k = w.shape[0]
    t = F.conv2d(torch.from_numpy(np.array(X, dtype=np.float64, copy=True))[None, None],
                 torch.from_numpy(np.array(w, dtype=np.float64, copy=True))[None, None], padding=k // 2)
    return t[0, 0].numpy()


def closed_forward(x, base_w, base_b, base_scale, wt_w, wt_scale, L):
    B, C, H, W = x.shape
    y = np.empty((B, C, H, W))
    for b in range(B):
        for c in range(C):
            yb = base_scale[c] * (torch_conv(x[b, c], base_w[c]) + base_b[c])
            hats = []
            for l in range(L):
                S = closed_analysis(x[b, c], l)
                hats.append(np.stack([wt_scale[l, c, s] * torch_conv(S[s], wt_w[l, c, s]) for s in range(4)]))
            y[b, c] = yb + closed_synthesis(hats, H, W)
    return y


def rand_params(rng, C, k, L, scales="random"):
    p = dict(
        base_w=rng.normal(0, 0.3, (C, k, k)),
        base_b=rng.normal(0, 0.5, (C,)),
        base_scale=rng.normal(1.0, 0.5, (C,)) if scales == "random" else np.ones(C),
        wt_w=rng.normal(0, 0.3, (L, C, 4, k, k)),
        wt_scale=rng.normal(0, 1.0, (L, C, 4)) if scales == "random" else np.full((L, C, 4), 0.1),
    )
    return p


def relerr(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (den if den > 0 else 1.0))


# ---------------------------------------------------------------------------
# Pins.
# ---------------------------------------------------------------------------
def pin_haar_worked_block(orc):
    # block (a b / c d) = (1 2 / 3 4): sum 10, row difference (1+2)-(3+4) = -4,
    # column difference (1+3)-(2+4) = -2, diagonal (1+4)-(2+3) = 0; all / 2.
    S = orc.dwt2(np.array([[1.0, 2.0], [3.0, 4.0]]))
    assert np.array_equal(S[:, 0, 0], [5.0, -2.0, -1.0, 0.0]), S[:, 0, 0]
    X = orc.iwt2(np.array([5.0, -2.0, -1.0, 0.0]).reshape(4, 1, 1))
    assert np.array_equal(X, [[1.0, 2.0], [3.0, 4.0]]), X


def pin_haar_reconstruction_and_energy(orc):
    rng = np.random.default_rng(RNG_SEED)
    for shape in [(2, 2), (8, 12), (16, 6)]:
        X = rng.normal(size=shape)
        Y = rng.normal(size=shape)
        S, T = orc.dwt2(X), orc.dwt2(Y)
        assert np.max(np.abs(orc.iwt2(S) - X)) < 1e-14
        assert abs(np.sum(S * S) - np.sum(X * X)) < 1e-12 * np.sum(X * X)
        assert abs(np.sum(S * T) - np.sum(X * Y)) < 1e-12 * (np.linalg.norm(X) * np.linalg.norm(Y))
        Z = rng.normal(size=S.shape)  # iwt2 is the transpose of dwt2: <dwt2 X, Z> = <X, iwt2 Z>
        assert abs(np.sum(S * Z) - np.sum(X * orc.iwt2(Z))) < 1e-12 * np.linalg.norm(X) * np.linalg.norm(Z)


def pin_haar_constant_and_closed_form(orc):
    S = orc.dwt2(np.full((4, 6), 3.0))
    assert np.allclose(S[0], 6.0) and np.allclose(S[1:], 0.0)
    rng = np.random.default_rng(RNG_SEED + 1)
    x = rng.normal(size=(16, 24))
    cur = x
    for l in range(3):  # the recursive cascade on the raw LL equals the closed-form analysis
        S = orc.dwt2(cur)
        assert np.max(np.abs(S - closed_analysis(x, l))) < 1e-13
        cur = S[0]


def pin_pyramid_parseval(orc):
    rng = np.random.default_rng(RNG_SEED + 2)
    x = rng.normal(size=(32, 16))
    e, cur = 0.0, x
    for _ in range(4):
        S = orc.dwt2(cur)
        e += np.sum(S[1:] ** 2)
        cur = S[0]
    e += np.sum(cur ** 2)
    assert abs(e - np.sum(x ** 2)) < 1e-12 * np.sum(x ** 2)


def pin_dwconv_library(orc):
    rng = np.random.default_rng(RNG_SEED + 3)
    for k in (1, 3, 5, 7):
        for shape in [(9, 7), (2, 2), (1, 1), (4, 12)]:
            X = rng.normal(size=shape)
            w = rng.normal(size=(k, k))
            assert np.max(np.abs(orc.dwconv(X, w) - torch_conv(X, w))) < 1e-12
            Y = rng.normal(size=shape)  # adjoint: <dwconv X, Y> = <X, dwconv_adj Y>
            lhs = np.sum(orc.dwconv(X, w) * Y)
            rhs = np.sum(X * orc.dwconv_adj(Y, w))
            assert abs(lhs - rhs) < 1e-11 * (1 + abs(lhs))
            assert np.max(np.abs(orc.dwconv_adj(Y, w) - torch_conv(Y, w[::-1, ::-1]))) < 1e-12


def pin_level0_is_depthwise_conv(orc):
    rng = np.random.default_rng(RNG_SEED + 4)
    B, C, H, W, k = 2, 3, 8, 12, 5
    x = rng.normal(size=(B, C, H, W))
    p = rand_params(rng, C, k, 0)
    y = orc.forward(x, p["base_w"], p["base_b"], p["base_scale"], None, None, 0)
    ref = F.conv2d(torch.from_numpy(x), torch.from_numpy(p["base_w"][:, None]), torch.from_numpy(p["base_b"]),
                   padding=k // 2, groups=C).numpy() * p["base_scale"][None, :, None, None]
    assert np.max(np.abs(y - ref)) < 1e-12


def pin_delta_identity(orc):
    # Delta kernels; detail scales 1 at every level, LL scale 1 at the coarsest
    # level and 0 at the finer ones; base scale 0: analysis then synthesis is
    # the identity, so y == x.
    rng = np.random.default_rng(RNG_SEED + 5)
    for (H, W, k, L) in [(16, 16, 5, 2), (8, 24, 3, 3), (4, 4, 7, 2)]:
        C = 2
        x = rng.normal(size=(1, C, H, W))
        delta = np.zeros((k, k))
        delta[k // 2, k // 2] = 1.0
        wt_w = np.broadcast_to(delta, (L, C, 4, k, k)).copy()
        wt_scale = np.ones((L, C, 4))
        wt_scale[: L - 1, :, 0] = 0.0
        y = orc.forward(x, rng.normal(size=(C, k, k)), rng.normal(size=C), np.zeros(C), wt_w, wt_scale, L)
        assert np.max(np.abs(y - x)) < 1e-12


def pin_delta_block_averages(orc):
    # Delta kernels, all wavelet scales 1, base scale 0:  y = sum_{l<L} P_{2^l} x,
    # P_m = average over aligned m x m blocks (P_1 = identity).
    rng = np.random.default_rng(RNG_SEED + 6)
    H, W, k, L, C = 16, 8, 3, 3, 1
    x = rng.normal(size=(1, C, H, W))
    delta = np.zeros((k, k))
    delta[k // 2, k // 2] = 1.0
    y = orc.forward(x, np.zeros((C, k, k)), np.zeros(C), np.zeros(C),
                    np.broadcast_to(delta, (L, C, 4, k, k)).copy(), np.ones((L, C, 4)), L)
    ref = np.zeros((H, W))
    for l in range(L):
        m = 2 ** l
        blk = x[0, 0].reshape(H // m, m, W // m, m).mean(axis=(1, 3))
        ref += np.repeat(np.repeat(blk, m, axis=0), m, axis=1)
    assert np.max(np.abs(y[0, 0] - ref)) < 1e-12


def pin_closed_form_forward(orc):
    rng = np.random.default_rng(RNG_SEED + 7)
    for (B, C, H, W, k, L) in [(1, 2, 16, 16, 5, 2), (2, 1, 8, 24, 3, 3), (1, 1, 8, 8, 7, 3), (1, 1, 4, 4, 5, 2),
                               (1, 2, 32, 16, 1, 4)]:
        x = rng.normal(size=(B, C, H, W))
        p = rand_params(rng, C, k, L)
        y = orc.forward(x, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], L)
        ref = closed_forward(x, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], L)
        assert np.max(np.abs(y - ref)) < 1e-11 * max(1.0, np.max(np.abs(ref)))


def _dense_operator(orc, p, C, H, W, L):
    n = C * H * W
    zero = np.zeros((1, C, H, W))
    y0 = orc.forward(zero, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], L).ravel()
    M = np.empty((n, n))
    for i in range(n):
        e = np.zeros(n)
        e[i] = 1.0
        M[:, i] = orc.forward(e.reshape(1, C, H, W), p["base_w"], p["base_b"], p["base_scale"], p["wt_w"],
                              p["wt_scale"], L).ravel() - y0
    return M, y0


def pin_dense_operator_adjoint(orc):
    rng = np.random.default_rng(RNG_SEED + 8)
    for (C, H, W, k, L) in [(1, 8, 8, 3, 2), (1, 4, 4, 5, 2), (2, 4, 8, 3, 1)]:
        p = rand_params(rng, C, k, L)
        M, y0 = _dense_operator(orc, p, C, H, W, L)
        x = rng.normal(size=(1, C, H, W))
        y = orc.forward(x, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], L).ravel()
        assert np.max(np.abs((y - y0) - M @ x.ravel())) < 1e-11  # affine in x
        dy = rng.normal(size=(1, C, H, W))
        dx = orc.backward_input(dy, p["base_w"], p["base_scale"], p["wt_w"], p["wt_scale"], L).ravel()
        assert np.max(np.abs(dx - M.T @ dy.ravel())) < 1e-11


def pin_backward_input_is_rotated_forward(orc):
    rng = np.random.default_rng(RNG_SEED + 9)
    B, C, H, W, k, L = 2, 2, 16, 8, 5, 3
    p = rand_params(rng, C, k, L)
    dy = rng.normal(size=(B, C, H, W))
    dx = orc.backward_input(dy, p["base_w"], p["base_scale"], p["wt_w"], p["wt_scale"], L)
    ref = orc.forward(dy, p["base_w"][:, ::-1, ::-1], np.zeros(C), p["base_scale"], p["wt_w"][..., ::-1, ::-1],
                      p["wt_scale"], L)
    assert np.max(np.abs(dx - ref)) < 1e-12 * max(1.0, np.max(np.abs(ref)))


def pin_finite_differences(orc):
    # loss = <dy, y>; y is affine in every single parameter, so a central
    # difference with step 1 is exact up to rounding.
    rng = np.random.default_rng(RNG_SEED + 10)
    B, C, H, W, k, L = 2, 2, 8, 8, 3, 2
    x = rng.normal(size=(B, C, H, W))
    dy = rng.normal(size=(B, C, H, W))
    p = rand_params(rng, C, k, L)
    g = orc.backward_weight(x, dy, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], L)

    def loss(q):
        return float(np.sum(dy * orc.forward(x, q["base_w"], q["base_b"], q["base_scale"], q["wt_w"],
                                             q["wt_scale"], L)))

    for name in ("base_w", "base_b", "base_scale", "wt_w", "wt_scale"):
        fd = np.empty_like(p[name])
        for idx in np.ndindex(p[name].shape):
            qp = {kk: v.copy() for kk, v in p.items()}
            qm = {kk: v.copy() for kk, v in p.items()}
            qp[name][idx] += 1.0
            qm[name][idx] -= 1.0
            fd[idx] = (loss(qp) - loss(qm)) / 2.0
        assert np.max(np.abs(g[name] - fd)) < 1e-9 * max(1.0, np.max(np.abs(fd))), name
    # d wt_scale = sum_t wt_w[t] * (d wt_w[t] / wt_scale)
    ident = np.sum(p["wt_w"] * (g["wt_w"] / p["wt_scale"][..., None, None]), axis=(-1, -2))
    assert np.max(np.abs(ident - g["wt_scale"])) < 1e-10 * max(1.0, np.max(np.abs(g["wt_scale"])))


def pin_shift_equivariance(orc):
    rng = np.random.default_rng(RNG_SEED + 11)
    H = W = 64
    L, k, C = 2, 3, 1
    x = np.zeros((1, C, H, W))
    x[0, 0, 16:40, 20:44] = rng.normal(size=(24, 24))
    p = rand_params(rng, C, k, L)
    p["base_b"][:] = 0.0
    y = orc.forward(x, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], L)
    s = 2 ** L
    xs = np.roll(x, (s, s), axis=(2, 3))
    ys = orc.forward(xs, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], L)
    assert np.max(np.abs(ys - np.roll(y, (s, s), axis=(2, 3)))) < 1e-12
    # an odd shift is not an equivariance of the wavelet branch
    x1 = np.roll(x, (1, 0), axis=(2, 3))
    y1 = orc.forward(x1, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], L)
    assert np.max(np.abs(y1 - np.roll(y, (1, 0), axis=(2, 3)))) > 1e-6


ALL_PINS = [
    pin_haar_worked_block, pin_haar_reconstruction_and_energy, pin_haar_constant_and_closed_form,
    pin_pyramid_parseval, pin_dwconv_library, pin_level0_is_depthwise_conv, pin_delta_identity,
    pin_delta_block_averages, pin_closed_form_forward, pin_dense_operator_adjoint,
    pin_backward_input_is_rotated_forward, pin_finite_differences, pin_shift_equivariance,
]
