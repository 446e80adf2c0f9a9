// Host-only replay of every shared-memory and global-memory access made by
// the WTConv kernels, for one shape, against the plan the library builds.
//
//   plan_access_check B C H W k L dtype
//
// For each kernel (fused forward / input gradient, weight gradient) it walks
// the same loops as the device code, with the same index arithmetic, over a
// shadow tag per shared-memory float, and fails if
//   - an index leaves the dynamic shared-memory allocation or its buffer,
//   - a conv / correlation window reads something other than the plane it
//     belongs to (interior) or untouched zero (padding and tile slack),
//   - a synthesis read sees anything but the conv output it needs,
//   - a global load or store leaves its H x W plane.
// Prints "OK <summary>" and exits 0, or prints the first violation and exits 1.
#include <cstdio>
#include <cstdlib>
#include <string>
#include <vector>

#include "../memory_bound_cnn_wtconv_b200/csrc/wtconv_planner.h"

using namespace wtc;

namespace {

enum : int { ZERO = 0, WTS = 1, BIAS = 2, XT = 3, DYT = 4, ZT = 5 };
int s_tag(int l, int s) { return 100 + 4 * l + s; }
int q_tag(int l, int s) { return 200 + 4 * l + s; }

struct Shadow {
    std::vector<int> tag;
    const char* phase = "";
    explicit Shadow(int n) : tag(n, ZERO) {}
    [[noreturn]] void fail(const std::string& m, long long idx) {
        std::printf("FAIL [%s] %s (index %lld of %zu)\n", phase, m.c_str(), idx, tag.size());
        std::exit(1);
    }
    void in_bounds(long long i, long long lo, long long hi, const char* what) {
        if (i < 0 || i >= (long long)tag.size()) fail(std::string(what) + ": outside shared memory", i);
        if (i < lo || i >= hi) fail(std::string(what) + ": outside its buffer", i);
    }
    void write(long long i, long long lo, long long hi, int t, const char* what) {
        in_bounds(i, lo, hi, what);
        tag[i] = t;
    }
    void read(long long i, long long lo, long long hi, int expect, const char* what) {
        in_bounds(i, lo, hi, what);
        if (tag[i] != expect) fail(std::string(what) + ": expected tag " + std::to_string(expect) + ", found " +
                                       std::to_string(tag[i]), i);
    }
};

void check_global(long long idx, long long n, const char* what) {
    if (idx < 0 || idx >= n) {
        std::printf("FAIL global %s index %lld of %lld\n", what, idx, n);
        std::exit(1);
    }
}

// Replays load_plane: element (i, j) -> dst + i*stride + j.
void replay_load(Shadow& sh, const Plan& P, long long dst, int stride, long long lo, long long hi, int t) {
    for (int i = 0; i < P.H; ++i)
        for (int j = 0; j < P.W; j += 4) {
            check_global((long long)i * P.W + j + 3, (long long)P.H * P.W, "plane load");
            for (int e = 0; e < 4; ++e) sh.write(dst + (long long)i * stride + j + e, lo, hi, t, "plane store");
        }
}

// Replays haar_level.
void replay_haar(Shadow& sh, long long src, int ss, long long slo, long long shi, int stag, int n, int m,
                 long long dst, int ds, int dsub, long long dlo, long long dhi, int (*dtag)(int, int), int l) {
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < m; ++j) {
            const long long s0 = src + 2LL * i * ss + 2LL * j;
            sh.read(s0, slo, shi, stag, "haar src");
            sh.read(s0 + 1, slo, shi, stag, "haar src");
            sh.read(s0 + ss, slo, shi, stag, "haar src");
            sh.read(s0 + ss + 1, slo, shi, stag, "haar src");
        }
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < m; ++j)
            for (int s = 0; s < 4; ++s) {
                const long long d = dst + (long long)i * ds + j + (long long)s * dsub;
                sh.write(d, dlo + (long long)s * dsub, dlo + (long long)(s + 1) * dsub, dtag(l, s), "haar dst");
            }
    (void)dhi;
}

// Replays the window reads of conv_tile / corr_tile on a padded plane whose
// padded element (-p, -p) sits at `base`; interior n x m must carry `itag`.
void replay_window(Shadow& sh, const Plan& P, long long base, int stride, long long lo, long long hi, int n, int m,
                   int tr, int tc, int itag, const char* what) {
    const int K = P.k, p = P.p, TR = P.TR, TC = P.TC;
    const int WV4 = 4 * ((TC + K - 1 + 3) / 4);
    const long long win = base + (long long)tr * TR * stride + (long long)tc * TC;
    if (win % 4 != 0) sh.fail(std::string(what) + ": window not 16-byte aligned", win);
    if (stride % 4 != 0) sh.fail(std::string(what) + ": stride not a multiple of 4", stride);
    for (int r = 0; r < TR + K - 1; ++r)
        for (int c = 0; c < WV4; ++c) {
            const long long a = win + (long long)r * stride + c;
            if (c >= TC + K - 1) {  // loaded but unused
                sh.in_bounds(a, lo, hi, what);
                continue;
            }
            const int i = tr * TR + r - p, j = tc * TC + c - p;
            const bool interior = i >= 0 && i < n && j >= 0 && j < m;
            sh.read(a, lo, hi, interior ? itag : ZERO, what);
        }
}

// Replays the D-tile reads of corr_tile on an unpadded, tile-rounded plane.
void replay_dtile(Shadow& sh, const Plan& P, long long base, int stride, long long lo, long long hi, int n, int m,
                  int tr, int tc, int itag) {
    const int TR = P.TR, TC = P.TC;
    const long long dt = base + (long long)tr * TR * stride + (long long)tc * TC;
    if (dt % 4 != 0) sh.fail("D tile not 16-byte aligned", dt);
    for (int r = 0; r < TR; ++r)
        for (int c = 0; c < TC; ++c) {
            const int i = tr * TR + r, j = tc * TC + c;
            const bool interior = i < n && j < m;
            sh.read(dt + (long long)r * stride + c, lo, hi, interior ? itag : ZERO, "D tile");
        }
}

void check_fused(const wtconv_desc_t& d, Kind kind) {
    Plan P;
    const wtconv_status_t st = make_plan(&d, kind, &P);
    if (st == WTCONV_ERR_UNSUPPORTED) {
        std::printf("fused: unsupported (plane too large)\n");
        return;
    }
    if (st != WTCONV_OK) {
        std::printf("FAIL fused plan status %d\n", (int)st);
        std::exit(1);
    }
    const int K = P.k, KK = K * K, p = P.p, L = P.L, H = P.H, W = P.W, TR = P.TR, TC = P.TC;
    const int ncls = 1 + 4 * L;
    if (P.smem_floats % 4 || P.smem_floats * 4 > 227 * 1024) {
        std::printf("FAIL smem size\n");
        std::exit(1);
    }
    Shadow sh(P.smem_floats);
    const long long all = P.smem_floats;
    sh.phase = "weights";
    for (int cl = 0; cl < ncls; ++cl)
        for (int t = 0; t < KK; ++t)
            sh.write(P.wbase + (long long)cl * P.wcls + t, P.wbase, P.wbase + (long long)ncls * P.wcls, WTS, "weights");
    sh.write(P.bias, P.bias, P.bias + 1, BIAS, "bias");
    for (int cl = 0; cl < ncls; ++cl)
        if ((P.wbase + cl * P.wcls) % 4) sh.fail("weight class not 16-byte aligned", P.wbase + cl * P.wcls);

    const int xrows = P.ntr[kMaxL] * TR + 2 * p;
    const long long xlo = P.X.base, xhi = P.X.base + (long long)xrows * P.X.stride;
    sh.phase = "load";
    replay_load(sh, P, P.X.base + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi, XT);

    sh.phase = "analysis";
    for (int l = 0; l < L; ++l) {
        const int n = H >> (l + 1), m = W >> (l + 1);
        long long src, slo, shi;
        int ss, stag;
        if (l == 0) {
            src = P.X.base + (long long)p * P.X.stride + p; ss = P.X.stride; slo = xlo; shi = xhi; stag = XT;
        } else {
            const Buf& S = P.S[l - 1];
            src = S.base + (long long)p * S.stride + p; ss = S.stride; slo = S.base; shi = S.base + S.sub; stag = s_tag(l - 1, 0);
        }
        const Buf& S = P.S[l];
        replay_haar(sh, src, ss, slo, shi, stag, n, m, S.base + (long long)p * S.stride + p, S.stride, S.sub, S.base,
                    S.base + 4LL * S.sub, s_tag, l);
    }

    sh.phase = "subband convs";
    for (int cl = 1; cl < ncls; ++cl) {
        const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
        const int n = H >> (l + 1), m = W >> (l + 1);
        const int ntiles = P.sub_begin[cl] - P.sub_begin[cl - 1];
        if (ntiles != P.ntr[l] * P.ntc[l]) sh.fail("tile count", cl);
        for (int local = 0; local < ntiles; ++local) {
            const int tr = local / P.ntc[l], tc = local % P.ntc[l];
            for (int t = 0; t < KK; ++t) sh.read(P.wbase + (long long)cl * P.wcls + t, 0, all, WTS, "weights");
            const Buf& S = P.S[l];
            replay_window(sh, P, S.base + (long long)s * S.sub, S.stride, S.base + (long long)s * S.sub,
                          S.base + (long long)(s + 1) * S.sub, n, m, tr, tc, s_tag(l, s), "subband window");
            const Buf& Q = P.Q[l];
            const long long out = Q.base + (long long)s * Q.sub + (long long)tr * TR * Q.stride + (long long)tc * TC;
            if (out % 4) sh.fail("Q tile not 16-byte aligned", out);
            for (int o = 0; o < TR; ++o)
                for (int j = 0; j < TC; ++j)
                    sh.write(out + (long long)o * Q.stride + j, Q.base + (long long)s * Q.sub,
                             Q.base + (long long)(s + 1) * Q.sub, q_tag(l, s), "Q tile");
        }
    }

    const int n0 = H >> 1, m0 = W >> 1;
    if (L >= 2) {
        sh.phase = "coarse synthesis";
        std::vector<long long> zw;
        for (int i = 0; i < n0; ++i)
            for (int j = 0; j < m0; ++j) {
                for (int l = 1; l < L; ++l) {
                    const Buf& Q = P.Q[l];
                    if ((i >> l) >= (H >> (l + 1)) || (j >> l) >= (W >> (l + 1))) sh.fail("coarse index", l);
                    for (int s = 0; s < 4; ++s)
                        sh.read(Q.base + (long long)(i >> l) * Q.stride + (j >> l) + (long long)s * Q.sub,
                                Q.base + (long long)s * Q.sub, Q.base + (long long)(s + 1) * Q.sub, q_tag(l, s),
                                "coarse Q read");
                }
                zw.push_back(P.Z.base + (long long)i * P.Z.stride + j);
            }
        // Z overwrites dead S[0]; it must not touch X, weights, or any Q plane.
        for (long long a : zw) {
            sh.in_bounds(a, P.S[0].base, P.S[0].base + 4LL * P.S[0].sub, "Z write");
            sh.tag[a] = ZT;
        }
    }

    sh.phase = "base conv + synthesis";
    const int ntc = P.ntc[kMaxL];
    for (int t = 0; t < P.n_base_tiles; ++t) {
        const int tr = t / ntc, tc = t % ntc;
        for (int q = 0; q < KK; ++q) sh.read(P.wbase + q, 0, all, WTS, "base weights");
        sh.read(P.bias, 0, all, BIAS, "bias");
        replay_window(sh, P, P.X.base, P.X.stride, xlo, xhi, H, W, tr, tc, XT, "base window");
        for (int o = 0; o < TR; ++o) {
            const int h = tr * TR + o;
            if (h >= H) continue;
            const int w0 = tc * TC;
            if (L >= 1) {
                const Buf& Q = P.Q[0];
                const int i = h >> 1;
                for (int pos = 0; pos < TC / 2; ++pos) {
                    const int j = (w0 >> 1) + pos;
                    if (i >= n0 || j >= m0) sh.fail("level-0 synthesis index", j);
                    for (int s = 0; s < 4; ++s)
                        sh.read(Q.base + (long long)i * Q.stride + j + (long long)s * Q.sub, Q.base + (long long)s * Q.sub,
                                Q.base + (long long)(s + 1) * Q.sub, q_tag(0, s), "level-0 Q read");
                    if (L >= 2) sh.read(P.Z.base + (long long)i * P.Z.stride + j, 0, all, ZT, "Z read");
                }
            }
            for (int e = 0; e < TC; ++e) check_global((long long)h * W + w0 + e, (long long)H * W, "y store");
        }
    }
    std::printf("fused(kind %d): smem %d B, threads %d, TR %d, tiles %d+%d\n", (int)kind, P.smem_floats * 4,
                P.nthreads, TR, P.n_sub_tiles, P.n_base_tiles);
}

void check_bwdw(const wtconv_desc_t& d) {
    Plan P;
    const wtconv_status_t st = make_plan(&d, kBackwardWeight, &P);
    if (st == WTCONV_ERR_UNSUPPORTED) {
        std::printf("bwdw: unsupported (plane too large)\n");
        return;
    }
    if (st != WTCONV_OK) {
        std::printf("FAIL bwdw plan status %d\n", (int)st);
        std::exit(1);
    }
    const int K = P.k, KK = K * K, p = P.p, L = P.L, H = P.H, W = P.W, TR = P.TR;
    const int ncls = 1 + 4 * L;
    Shadow sh(P.smem_floats);
    const int xrows = P.ntr[kMaxL] * TR + 2 * p;
    const long long xlo = P.X.base, xhi = P.X.base + (long long)xrows * P.X.stride;
    const long long dlo = P.DY.base, dhi = P.DY.base + (long long)P.ntr[kMaxL] * TR * P.DY.stride;
    // Two planes in a row: the second must see the same zero padding.
    for (int plane = 0; plane < 2; ++plane) {
        sh.phase = "load";
        replay_load(sh, P, P.X.base + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi, XT);
        replay_load(sh, P, P.DY.base, P.DY.stride, dlo, dhi, DYT);
        sh.phase = "analysis";
        for (int l = 0; l < L; ++l) {
            const int n = H >> (l + 1), m = W >> (l + 1);
            {
                long long src, slo, shi;
                int ss, stag;
                if (l == 0) {
                    src = P.X.base + (long long)p * P.X.stride + p; ss = P.X.stride; slo = xlo; shi = xhi; stag = XT;
                } else {
                    const Buf& S = P.S[l - 1];
                    src = S.base + (long long)p * S.stride + p; ss = S.stride; slo = S.base; shi = S.base + S.sub;
                    stag = s_tag(l - 1, 0);
                }
                const Buf& S = P.S[l];
                replay_haar(sh, src, ss, slo, shi, stag, n, m, S.base + (long long)p * S.stride + p, S.stride, S.sub,
                            S.base, S.base + 4LL * S.sub, s_tag, l);
            }
            {
                long long src, slo, shi;
                int ss, stag;
                if (l == 0) {
                    src = P.DY.base; ss = P.DY.stride; slo = dlo; shi = dhi; stag = DYT;
                } else {
                    const Buf& Q = P.Q[l - 1];
                    src = Q.base; ss = Q.stride; slo = Q.base; shi = Q.base + Q.sub; stag = q_tag(l - 1, 0);
                }
                const Buf& Q = P.Q[l];
                replay_haar(sh, src, ss, slo, shi, stag, n, m, Q.base, Q.stride, Q.sub, Q.base, Q.base + 4LL * Q.sub,
                            q_tag, l);
            }
        }
        sh.phase = "correlation";
        for (int tid = 0; tid < P.n_all_tiles; ++tid) {
            int cl = 0;
            while (tid >= P.cls_begin[cl + 1]) ++cl;
            const int lvl = (cl == 0) ? kMaxL : ((cl - 1) >> 2);
            const int local = tid - P.cls_begin[cl];
            const int tr = local / P.ntc[lvl], tc = local % P.ntc[lvl];
            if (tr >= P.ntr[lvl]) sh.fail("tile row out of grid", tid);
            if (cl == 0) {
                replay_window(sh, P, P.X.base, P.X.stride, xlo, xhi, H, W, tr, tc, XT, "base S window");
                replay_dtile(sh, P, P.DY.base, P.DY.stride, dlo, dhi, H, W, tr, tc, DYT);
            } else {
                const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
                const int n = H >> (l + 1), m = W >> (l + 1);
                const Buf& S = P.S[l];
                const Buf& Q = P.Q[l];
                replay_window(sh, P, S.base + (long long)s * S.sub, S.stride, S.base + (long long)s * S.sub,
                              S.base + (long long)(s + 1) * S.sub, n, m, tr, tc, s_tag(l, s), "subband S window");
                replay_dtile(sh, P, Q.base + (long long)s * Q.sub, Q.stride, Q.base + (long long)s * Q.sub,
                             Q.base + (long long)(s + 1) * Q.sub, n, m, tr, tc, q_tag(l, s));
            }
        }
    }
    sh.phase = "reduction";
    const long long red_end = (long long)P.red + (long long)P.nthreads * KK + P.nthreads;
    if (red_end > P.smem_floats) sh.fail("reduction scratch", red_end);
    if (P.nthreads < P.n_all_tiles || P.nthreads > 512 || P.nthreads % 32) sh.fail("thread count", P.nthreads);
    if (P.B % P.groups) sh.fail("groups must divide B", P.groups);
    if (P.nv != ncls * KK + 1) sh.fail("partial vector length", P.nv);
    std::printf("bwdw: smem %d B, threads %d, TR %d, tiles %d, groups %d\n", P.smem_floats * 4, P.nthreads, TR,
                P.n_all_tiles, P.groups);
}

}  // namespace

int main(int argc, char** argv) {
    if (argc != 8) {
        std::printf("usage: plan_access_check B C H W k L dtype\n");
        return 2;
    }
    wtconv_desc_t d;
    d.B = std::atoi(argv[1]); d.C = std::atoi(argv[2]); d.H = std::atoi(argv[3]); d.W = std::atoi(argv[4]);
    d.k = std::atoi(argv[5]); d.L = std::atoi(argv[6]); d.dtype = std::atoi(argv[7]);
    if (validate(&d) != WTCONV_OK) {
        std::printf("invalid (status %d)\n", (int)validate(&d));
        return 3;
    }
    check_fused(d, kForward);
    check_fused(d, kBackwardInput);
    check_bwdw(d);
    std::printf("OK\n");
    return 0;
}
