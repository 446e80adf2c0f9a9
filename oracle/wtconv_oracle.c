/*
 * WTConv oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, literal CPU restatement of the wavelet-convolution (WTConv)
 * layer, in double precision, used to check the CUDA library.  Only the test
 * suite, the smoke check and the CPU-baseline leg of the benchmark may load
 * it; the library never does.  It shares no code, header, table or helper
 * with the CUDA sources.
 *
 * What it follows ("Fast and Memory-Efficient Wavelet Convolutions via I/O-
 * Aware Reformulation", arXiv 2608.10805, Abstract): the layer is a depthwise
 * convolution plus a multi-level Haar wavelet branch; the fused method only
 * reorganises the same arithmetic (recomputed analysis, closed-form synthesis,
 * folded scales), so the oracle is the plain definition run level by level:
 *
 *   base branch   yb = base_scale[c] * (dwconv(x, base_w[c]) + base_b[c])
 *   analysis      S_l = dwt2(LL_{l-1}),  LL_{-1} = x,  LL_l = S_{l,LL}  (raw)
 *   subband conv  Shat_{l,s} = wt_scale[l,c,s] * dwconv(S_{l,s}, wt_w[l,c,s])
 *   synthesis     Z_L = 0;  Z_l = iwt2(Shat_{l,LL} + Z_{l+1}, Shat_{l,LH..HH})
 *   output        y = yb + Z_0
 *
 * The Haar step is the 2-D orthonormal one: each 2x2 block (a b / c d) maps
 * to (sum, row-difference, column-difference, diagonal) divided by 2, the 2-D
 * form of the sum/difference pairing with orthogonal transform matrix
 * described on "SETAREH ... Haar wavelet" (kongchang.com), section on the
 * Haar transform; its inverse is its transpose (same page, same section), and
 * inner products are preserved under it (same page, inner-product section).
 * Subband order: 0 = LL, 1 = LH (high-pass along H), 2 = HL (high-pass along
 * W), 3 = HH.  dwconv is cross-correlation with "same" zero padding,
 * p = k / 2, applied at each subband's own resolution.
 *
 * Layouts (row-major, all double):
 *   x, y, dy, dx   [B][C][H][W]
 *   base_w [C][k][k], base_b [C], base_scale [C]
 *   wt_w [L][C][4][k][k], wt_scale [L][C][4]
 *
 * Parity status: every function here is pinned by tests in
 * tests/test_oracle.py (perfect reconstruction, Parseval, L = 0 against a
 * library convolution, the delta-kernel identity, the block-average closed
 * form, the brute-force closed-form synthesis, the dense-operator adjoint and
 * central finite differences).
 */
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- one orthonormal 2-D Haar step ------------------------------------ */

/* X is nh x nw (both even).  S receives 4 planes of (nh/2) x (nw/2) in the
 * order LL, LH, HL, HH. */
void orc_dwt2(const double *X, int nh, int nw, double *S)
{
    int mh = nh / 2, mw = nw / 2;
    size_t m = (size_t)mh * mw;
    for (int i = 0; i < mh; ++i) {
        for (int j = 0; j < mw; ++j) {
            double a = X[(size_t)(2 * i) * nw + 2 * j];
            double b = X[(size_t)(2 * i) * nw + 2 * j + 1];
            double c = X[(size_t)(2 * i + 1) * nw + 2 * j];
            double d = X[(size_t)(2 * i + 1) * nw + 2 * j + 1];
            size_t o = (size_t)i * mw + j;
            S[0 * m + o] = (a + b + c + d) / 2.0;
            S[1 * m + o] = (a + b - c - d) / 2.0;
            S[2 * m + o] = (a - b + c - d) / 2.0;
            S[3 * m + o] = (a - b - c + d) / 2.0;
        }
    }
}

/* Inverse (= transpose) of orc_dwt2.  S holds 4 planes of mh x mw; X
 * receives (2 mh) x (2 mw). */
void orc_iwt2(const double *S, int mh, int mw, double *X)
{
    int nw = 2 * mw;
    size_t m = (size_t)mh * mw;
    for (int i = 0; i < mh; ++i) {
        for (int j = 0; j < mw; ++j) {
            size_t o = (size_t)i * mw + j;
            double ll = S[0 * m + o], lh = S[1 * m + o];
            double hl = S[2 * m + o], hh = S[3 * m + o];
            X[(size_t)(2 * i) * nw + 2 * j] = (ll + lh + hl + hh) / 2.0;
            X[(size_t)(2 * i) * nw + 2 * j + 1] = (ll + lh - hl - hh) / 2.0;
            X[(size_t)(2 * i + 1) * nw + 2 * j] = (ll - lh + hl - hh) / 2.0;
            X[(size_t)(2 * i + 1) * nw + 2 * j + 1] = (ll - lh - hl + hh) / 2.0;
        }
    }
}

/* ---- depthwise convolution (one plane) --------------------------------- */

/* Y[i][j] = sum_{u,v<k} w[u][v] * X[i+u-p][j+v-p], X = 0 outside. */
void orc_dwconv(const double *X, int nh, int nw, const double *w, int k, double *Y)
{
    int p = k / 2;
    for (int i = 0; i < nh; ++i) {
        for (int j = 0; j < nw; ++j) {
            double acc = 0.0;
            for (int u = 0; u < k; ++u) {
                int r = i + u - p;
                if (r < 0 || r >= nh) continue;
                for (int v = 0; v < k; ++v) {
                    int q = j + v - p;
                    if (q < 0 || q >= nw) continue;
                    acc += w[u * k + v] * X[(size_t)r * nw + q];
                }
            }
            Y[(size_t)i * nw + j] = acc;
        }
    }
}

/* Adjoint of orc_dwconv: X[i][j] = sum_{u,v} w[u][v] * Y[i-u+p][j-v+p]. */
void orc_dwconv_adj(const double *Y, int nh, int nw, const double *w, int k, double *X)
{
    int p = k / 2;
    for (int i = 0; i < nh; ++i) {
        for (int j = 0; j < nw; ++j) {
            double acc = 0.0;
            for (int u = 0; u < k; ++u) {
                int r = i - u + p;
                if (r < 0 || r >= nh) continue;
                for (int v = 0; v < k; ++v) {
                    int q = j - v + p;
                    if (q < 0 || q >= nw) continue;
                    acc += w[u * k + v] * Y[(size_t)r * nw + q];
                }
            }
            X[(size_t)i * nw + j] = acc;
        }
    }
}

/* ---- argument check ---------------------------------------------------- */

static int orc_check(int B, int C, int H, int W, int k, int L)
{
    if (B <= 0 || C <= 0 || H <= 0 || W <= 0) return -1;
    if (k < 1 || (k % 2) == 0) return -2;
    if (L < 0 || L > 16) return -3;
    if ((H % (1 << L)) != 0 || (W % (1 << L)) != 0) return -4;
    return 0;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Offsets of level l's pyramid planes inside one contiguous scratch block:
 * level l holds 4 planes of (H >> (l+1)) x (W >> (l+1)). */
static size_t orc_level_offset(int H, int W, int l)
{
    size_t off = 0;
    for (int t = 0; t < l; ++t) off += 4 * (size_t)(H >> (t + 1)) * (size_t)(W >> (t + 1));
    return off;
}

/* Literal level-by-level analysis of one plane: pyr receives, for each
 * level l, the 4 subbands of dwt2 applied to the previous level's raw LL. */
static void orc_analysis(const double *plane, int H, int W, int L, double *pyr)
{
    const double *cur = plane;
    for (int l = 0; l < L; ++l) {
        int nh = H >> l, nw = W >> l;
        double *S = pyr + orc_level_offset(H, W, l);
        orc_dwt2(cur, nh, nw, S);
        cur = S; /* S_{l,LL}: the raw approximation recurses */
    }
}

/* ---- forward ------------------------------------------------------------ */

int orc_forward(int B, int C, int H, int W, int k, int L,
                const double *x, const double *base_w, const double *base_b,
                const double *base_scale, const double *wt_w, const double *wt_scale,
                double *y)
{
    int rc = orc_check(B, C, H, W, k, L);
    if (rc) return rc;
    size_t plane = (size_t)H * W;
    size_t kk = (size_t)k * k;
    size_t pyr_sz = orc_level_offset(H, W, L) + 1;
    int np = B * C;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bc = 0; bc < np; ++bc) {
        int c = bc % C;
        const double *xp = x + (size_t)bc * plane;
        double *yp = y + (size_t)bc * plane;
        double *pyr = (double *)malloc(pyr_sz * sizeof(double));
        double *hat = (double *)malloc(pyr_sz * sizeof(double));
        double *z = (double *)malloc(plane * sizeof(double));
        double *tmp = (double *)malloc(plane * sizeof(double));
        if (!pyr || !hat || !z || !tmp) {
            free(pyr); free(hat); free(z); free(tmp);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        /* base branch: scale * (conv + bias) */
        orc_dwconv(xp, H, W, base_w + (size_t)c * kk, k, yp);
        for (size_t i = 0; i < plane; ++i) yp[i] = base_scale[c] * (yp[i] + base_b[c]);

        /* analysis, then per-subband conv and scale */
        orc_analysis(xp, H, W, L, pyr);
        for (int l = 0; l < L; ++l) {
            int mh = H >> (l + 1), mw = W >> (l + 1);
            size_t m = (size_t)mh * mw;
            size_t off = orc_level_offset(H, W, l);
            for (int s = 0; s < 4; ++s) {
                const double *wk = wt_w + (((size_t)l * C + c) * 4 + s) * kk;
                double a = wt_scale[((size_t)l * C + c) * 4 + s];
                double *dst = hat + off + s * m;
                orc_dwconv(pyr + off + s * m, mh, mw, wk, k, dst);
                for (size_t i = 0; i < m; ++i) dst[i] *= a;
            }
        }

        /* synthesis cascade, coarsest level first */
        if (L > 0) {
            int mh = H >> L, mw = W >> L;
            memset(z, 0, (size_t)mh * mw * sizeof(double));
            for (int l = L - 1; l >= 0; --l) {
                mh = H >> (l + 1); mw = W >> (l + 1);
                size_t m = (size_t)mh * mw;
                double *S = hat + orc_level_offset(H, W, l);
                for (size_t i = 0; i < m; ++i) S[i] += z[i]; /* coarser reconstruction into LL */
                orc_iwt2(S, mh, mw, tmp);
                memcpy(z, tmp, 4 * m * sizeof(double));
            }
            for (size_t i = 0; i < plane; ++i) yp[i] += z[i];
        }
        free(pyr); free(hat); free(z); free(tmp);
    }
    return failed ? -10 : 0;
}

/* ---- backward with respect to the input -------------------------------- */

/* The adjoint of each forward step, in reverse order: the adjoint of the
 * orthonormal iwt2 is dwt2 and vice versa, and the adjoint of dwconv is the
 * correlation with the kernel rotated by 180 degrees (orc_dwconv_adj). */
int orc_backward_input(int B, int C, int H, int W, int k, int L,
                       const double *dy, const double *base_w, const double *base_scale,
                       const double *wt_w, const double *wt_scale, double *dx)
{
    int rc = orc_check(B, C, H, W, k, L);
    if (rc) return rc;
    size_t plane = (size_t)H * W;
    size_t kk = (size_t)k * k;
    size_t pyr_sz = orc_level_offset(H, W, L) + 1;
    int np = B * C;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bc = 0; bc < np; ++bc) {
        int c = bc % C;
        const double *gp = dy + (size_t)bc * plane;
        double *dxp = dx + (size_t)bc * plane;
        double *D = (double *)malloc(pyr_sz * sizeof(double));
        double *dS = (double *)malloc(pyr_sz * sizeof(double));
        double *g = (double *)malloc(plane * sizeof(double));
        double *tmp = (double *)malloc(plane * sizeof(double));
        if (!D || !dS || !g || !tmp) {
            free(D); free(dS); free(g); free(tmp);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        /* adjoint of the synthesis cascade: D_l = dwt2 of the gradient that
         * reached level l's reconstruction; its LL part flows to level l+1. */
        orc_analysis(gp, H, W, L, D);
        /* adjoint of scale * dwconv for every subband */
        for (int l = 0; l < L; ++l) {
            int mh = H >> (l + 1), mw = W >> (l + 1);
            size_t m = (size_t)mh * mw;
            size_t off = orc_level_offset(H, W, l);
            for (int s = 0; s < 4; ++s) {
                const double *wk = wt_w + (((size_t)l * C + c) * 4 + s) * kk;
                double a = wt_scale[((size_t)l * C + c) * 4 + s];
                double *dst = dS + off + s * m;
                orc_dwconv_adj(D + off + s * m, mh, mw, wk, k, dst);
                for (size_t i = 0; i < m; ++i) dst[i] *= a;
            }
        }
        /* adjoint of the analysis cascade, coarsest level first */
        orc_dwconv_adj(gp, H, W, base_w + (size_t)c * kk, k, dxp);
        for (size_t i = 0; i < plane; ++i) dxp[i] *= base_scale[c];
        if (L > 0) {
            int mh = H >> L, mw = W >> L;
            memset(g, 0, (size_t)mh * mw * sizeof(double));
            for (int l = L - 1; l >= 0; --l) {
                mh = H >> (l + 1); mw = W >> (l + 1);
                size_t m = (size_t)mh * mw;
                double *S = dS + orc_level_offset(H, W, l);
                for (size_t i = 0; i < m; ++i) S[i] += g[i];
                orc_iwt2(S, mh, mw, tmp);
                memcpy(g, tmp, 4 * m * sizeof(double));
            }
            for (size_t i = 0; i < plane; ++i) dxp[i] += g[i];
        }
        free(D); free(dS); free(g); free(tmp);
    }
    return failed ? -10 : 0;
}

/* ---- backward with respect to the parameters --------------------------- */

/* Sums over the batch and every position, per channel:
 *   d wt_w[l,c,s][u][v] = wt_scale * sum D_{l,s}[i,j] * S_{l,s}[i+u-p, j+v-p]
 *   d wt_scale[l,c,s]   = sum D_{l,s} * dwconv(S_{l,s}, wt_w[l,c,s])
 *   d base_w[c][u][v]   = base_scale * sum dy[h,w] * x[h+u-p, w+v-p]
 *   d base_b[c]         = base_scale * sum dy
 *   d base_scale[c]     = sum dy * (dwconv(x, base_w[c]) + base_b[c])
 * where S = analysis of x and D = analysis of dy (the gradient reaching
 * every subband's scaled conv output).  Gradients are overwritten. */
int orc_backward_weight(int B, int C, int H, int W, int k, int L,
                        const double *x, const double *dy, const double *base_w,
                        const double *base_b, const double *base_scale,
                        const double *wt_w, const double *wt_scale,
                        double *d_base_w, double *d_base_b, double *d_base_scale,
                        double *d_wt_w, double *d_wt_scale)
{
    int rc = orc_check(B, C, H, W, k, L);
    if (rc) return rc;
    size_t plane = (size_t)H * W;
    size_t kk = (size_t)k * k;
    size_t pyr_sz = orc_level_offset(H, W, L) + 1;
    int p = k / 2;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int c = 0; c < C; ++c) {
        double *S = (double *)malloc(pyr_sz * sizeof(double));
        double *D = (double *)malloc(pyr_sz * sizeof(double));
        double *conv = (double *)malloc(plane * sizeof(double));
        double *gw = (double *)calloc((size_t)(L > 0 ? L : 1) * 4 * kk, sizeof(double));
        double *gs = (double *)calloc((size_t)(L > 0 ? L : 1) * 4, sizeof(double));
        double *gb = (double *)calloc(kk, sizeof(double));
        if (!S || !D || !conv || !gw || !gs || !gb) {
            free(S); free(D); free(conv); free(gw); free(gs); free(gb);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        double sdy = 0.0, dbs = 0.0;
        for (int b = 0; b < B; ++b) {
            const double *xp = x + ((size_t)b * C + c) * plane;
            const double *gp = dy + ((size_t)b * C + c) * plane;
            /* base branch */
            for (int u = 0; u < k; ++u)
                for (int v = 0; v < k; ++v) {
                    double acc = 0.0;
                    for (int h = 0; h < H; ++h) {
                        int r = h + u - p;
                        if (r < 0 || r >= H) continue;
                        for (int w = 0; w < W; ++w) {
                            int q = w + v - p;
                            if (q < 0 || q >= W) continue;
                            acc += gp[(size_t)h * W + w] * xp[(size_t)r * W + q];
                        }
                    }
                    gb[u * k + v] += acc;
                }
            orc_dwconv(xp, H, W, base_w + (size_t)c * kk, k, conv);
            for (size_t i = 0; i < plane; ++i) {
                sdy += gp[i];
                dbs += gp[i] * (conv[i] + base_b[c]);
            }
            /* wavelet branch */
            orc_analysis(xp, H, W, L, S);
            orc_analysis(gp, H, W, L, D);
            for (int l = 0; l < L; ++l) {
                int mh = H >> (l + 1), mw = W >> (l + 1);
                size_t m = (size_t)mh * mw;
                size_t off = orc_level_offset(H, W, l);
                for (int s = 0; s < 4; ++s) {
                    const double *Ss = S + off + s * m;
                    const double *Ds = D + off + s * m;
                    const double *wk = wt_w + (((size_t)l * C + c) * 4 + s) * kk;
                    for (int u = 0; u < k; ++u)
                        for (int v = 0; v < k; ++v) {
                            double acc = 0.0;
                            for (int i = 0; i < mh; ++i) {
                                int r = i + u - p;
                                if (r < 0 || r >= mh) continue;
                                for (int j = 0; j < mw; ++j) {
                                    int q = j + v - p;
                                    if (q < 0 || q >= mw) continue;
                                    acc += Ds[(size_t)i * mw + j] * Ss[(size_t)r * mw + q];
                                }
                            }
                            gw[((size_t)l * 4 + s) * kk + u * k + v] += acc;
                        }
                    orc_dwconv(Ss, mh, mw, wk, k, conv);
                    double acc = 0.0;
                    for (size_t i = 0; i < m; ++i) acc += Ds[i] * conv[i];
                    gs[l * 4 + s] += acc;
                }
            }
        }
        for (size_t t = 0; t < kk; ++t) d_base_w[(size_t)c * kk + t] = base_scale[c] * gb[t];
        d_base_b[c] = base_scale[c] * sdy;
        d_base_scale[c] = dbs;
        for (int l = 0; l < L; ++l)
            for (int s = 0; s < 4; ++s) {
                size_t pi = ((size_t)l * C + c) * 4 + s;
                for (size_t t = 0; t < kk; ++t)
                    d_wt_w[pi * kk + t] = wt_scale[pi] * gw[((size_t)l * 4 + s) * kk + t];
                d_wt_scale[pi] = gs[l * 4 + s];
            }
        free(S); free(D); free(conv); free(gw); free(gs); free(gb);
    }
    return failed ? -10 : 0;
}
