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
//   - a global load or store leaves its H x W plane,
//   - two phases of the kernel race: the CTA barriers split the replay into
//     phases, and no float may be written by one work item and read or
//     written by another inside one phase.
// Prints "OK <summary>" and exits 0, or prints the first violation and exits 1.
#include <cstdio>
#include <cstdlib>
#include <string>
#include <vector>

#include "../memory_bound_cnn_wtconv_b200/csrc/wtconv_planner.h"

using namespace wtc;

namespace {

enum : int { ZERO = 0, WTS = 1, BIAS = 2, XT = 3, DYT = 4, ZT = 5, YT = 6, RED = 7 };
int g_rank = 0;  // strip of the CTA being replayed (the analysis replays read it)
int s_tag(int l, int s) { return 100 + 4 * l + s; }
int q_tag(int l, int s) { return 200 + 4 * l + s; }
int ss_tag(int l, int s) { return 300 + 4 * l + s; }

struct Shadow {
    std::vector<int> tag;
    std::vector<int> rd, wr;  // last phase that read / wrote each float
    int epoch = 1;            // current phase; a CTA barrier starts the next
    const char* phase = "";
    explicit Shadow(int n) : tag(n, ZERO), rd(n, 0), wr(n, 0) {}
    void barrier() { ++epoch; }
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
        if (rd[i] == epoch) fail(std::string(what) + ": written in the phase that reads it", i);
        if (wr[i] == epoch) fail(std::string(what) + ": written twice in one phase", i);
        wr[i] = epoch;
        tag[i] = t;
    }
    // A load whose value is not used (vector-load slack): bounds and races only.
    void touch(long long i, long long lo, long long hi, const char* what) {
        in_bounds(i, lo, hi, what);
        if (wr[i] == epoch) fail(std::string(what) + ": read in the phase that writes it", i);
        rd[i] = epoch;
    }
    void read(long long i, long long lo, long long hi, int expect, const char* what) {
        touch(i, lo, hi, what);
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

// Replays stage_plane: 16-byte chunk ch of this CTA's rows (strip `rank`) of
// the stored plane -> staging floats [stg + 4ch, stg + 4ch + 4).
// False while replaying an analysis whose plane copy the kernel skips (the
// weight gradient's dy when its tiles read the staging; COPY = false).
bool g_copy_plane = true;

int real_rows_host(const Plan& P, int rank) { return std::max(0, std::min(P.H, P.Hr - rank * P.H)); }

void replay_stage(Shadow& sh, const Plan& P, long long stg, int tag, int rank) {
    const long long strip_bytes = (long long)P.H * P.W * P.esize;
    const long long plane_bytes = (long long)P.Hr * P.Wr * P.esize;
    if (P.nhwc) {
        // Element by element: strip element e = r*Wr + col (plane element
        // rank*H*Wr + e) -> staging element r*W + col; a staging float holds
        // 4 / esize elements and is written once.
        if (stg % 4) sh.fail("staging not 16-byte aligned", stg);
        const int rows = real_rows_host(P, rank);
        const int per = 4 / P.esize;
        std::vector<char> hit((size_t)P.stg_floats, 0);
        for (long long e = 0; e < (long long)rows * P.Wr; ++e) {
            const int r = (int)fastdiv_host((uint32_t)e, P.div_wr), col = (int)e - r * P.Wr;
            if (r != e / P.Wr) sh.fail("element-row division", e);
            check_global((long long)rank * P.H * P.Wr + e, (long long)P.Hr * P.Wr, "staging source element");
            const long long f = ((long long)r * P.W + col) / per;
            if (f < 0 || f >= P.stg_floats) sh.fail("staging element outside the staging buffer", f);
            if (!hit[f]) {
                hit[f] = 1;
                sh.write(stg + f, stg, stg + P.stg_floats, tag, "staging");
            }
        }
        return;
    }
    if (P.plane_chunks * 16LL != strip_bytes) sh.fail("strip is not a whole number of 16-byte chunks", strip_bytes);
    if (stg % 4) sh.fail("staging not 16-byte aligned", stg);
    if (!P.padded) {
        if (P.Hr != P.Hp || P.Wr != P.W) sh.fail("unpadded plan with padded sizes", P.Hr);
        for (int ch = 0; ch < P.plane_chunks; ++ch) {
            check_global(rank * strip_bytes + 16LL * ch + 15, plane_bytes, "staging source");
            for (int e = 0; e < 4; ++e) sh.write(stg + 4LL * ch + e, stg, stg + P.stg_floats, tag, "staging");
        }
        return;
    }
    // Row by row: the real rows of this strip, Wr elements each, into staging rows of W.
    const int rows = real_rows_host(P, rank), rc = P.row_chunks;
    if ((long long)rc * 16 != (long long)P.Wr * P.esize) sh.fail("row chunks", rc);
    for (int ch = 0; ch < rows * rc; ++ch) {
        const int r = (int)fastdiv_host(ch, P.div_rowc), c = ch - r * rc;
        if (r != ch / rc) sh.fail("row-chunk division", ch);
        const long long src = ((long long)rank * P.H + r) * P.Wr * P.esize + 16LL * c;
        check_global(src + 15, plane_bytes, "staging source");
        const long long dst = stg + ((long long)r * P.W * P.esize + 16LL * c) / 4;
        for (int e = 0; e < 4; ++e) sh.write(dst + e, stg, stg + P.stg_floats, tag, "staging");
    }
}

// Tag a staged element (virtual row r, column col of this strip) must carry:
// the staging tag where the plane has data, zero in the on-chip padding.
int staged_tag(const Plan& P, int rank, int r, int col, int stag) {
    return (r < real_rows_host(P, rank) && col < P.Wr) ? stag : ZERO;
}

// Replays unpack_level0: staged element e (4 at a time) -> dst (element (0,0) at `dst`, row stride ds),
// and, if level0, the level-0 butterflies of rows 2i, 2i+1 / columns 4q..4q+3 -> the 4 subband planes.
void replay_unpack(Shadow& sh, const Plan& P, long long stg, int stag, long long dst, int ds, long long dlo,
                   long long dhi, int dtag, long long sb, int sbs, int sbsub, long long sblo, int (*sbtag)(int, int),
                   bool level0) {
    const int W = P.W;
    auto stage_read = [&](int e) {  // 4 elements at element index e
        if (e % 4) sh.fail("staged load not 4-element aligned", e);
        const long long f0 = stg + (long long)e * P.esize / 4;
        const int nf = P.esize;  // 4 elements = esize floats
        const int t = staged_tag(P, g_rank, e / W, e % W, stag);
        for (int q = 0; q < nf; ++q) sh.read(f0 + q, stg, stg + P.stg_floats, t, "staging read");
    };
    const int rows = level0 ? P.H / 2 : P.H;
    for (int i = 0; i < rows; ++i)
        for (int q = 0; q < W / 4; ++q) {
            const int nr = level0 ? 2 : 1;
            for (int rr = 0; rr < nr; ++rr) {
                const int r = level0 ? 2 * i + rr : i;
                stage_read(r * W + 4 * q);
                if (g_copy_plane)
                    for (int e = 0; e < 4; ++e) sh.write(dst + (long long)r * ds + 4 * q + e, dlo, dhi, dtag, "unpack store");
            }
            if (level0)
                for (int s = 0; s < 4; ++s)
                    for (int e = 0; e < 2; ++e)
                        sh.write(sb + (long long)s * sbsub + (long long)i * sbs + 2 * q + e, sblo + (long long)s * sbsub,
                                 sblo + (long long)(s + 1) * sbsub, sbtag(0, s), "level-0 store");
        }
}

void replay_haar(Shadow& sh, long long src, int ss, long long slo, long long shi, int stag, int n, int m,
                 long long dst, int ds, int dsub, long long dlo, long long dhi, int (*dtag)(int, int), int l);

// Replays analysis_pyramid: threads own 4x4 blocks (lane groups of G*G
// lanes per (4G)^2 region), write the block into the plane buffer, levels 0
// and 1 to their subband planes, and levels 2.. from the group leader.
void replay_pyramid(Shadow& sh, const Plan& P, long long stg, int stag, long long dst, int ds, long long dlo,
                    long long dhi, int dtag, const Buf* bufs, int pad, int (*sbtag)(int, int)) {
    const int H = P.H, W = P.W, lg = P.pyr_lg, G = 1 << lg, G2 = G * G;
    if ((4 * G) != (P.pyr_levels >= 2 ? (1 << P.pyr_levels) : 4)) sh.fail("pyramid region size", G);
    if (H % (4 * G) || W % (4 * G)) sh.fail("pyramid regions must tile the plane", G);
    if (32 % G2) sh.fail("pyramid lane group must divide a warp", G2);
    const int nreg_w = W >> (lg + 2);
    const int items = (H >> (lg + 2)) * nreg_w * G2;
    for (int item = 0; item < items; ++item) {
        const int r = item >> (2 * lg), o = item & (G2 - 1);
        const int by = o >> lg, bx = o & (G - 1);
        const int rrow = (int)fastdiv_host(r, P.div_rw), rcol = r - rrow * nreg_w;
        if (rrow != r / nreg_w) sh.fail("region row division", r);
        const int brow = rrow * G + by, bcol = rcol * G + bx;
        const int r0 = 4 * brow, c0 = 4 * bcol;
        for (int q = 0; q < 4; ++q) {
            const long long f0 = stg + (long long)((r0 + q) * W + c0) * P.esize / 4;
            const int t = staged_tag(P, g_rank, r0 + q, c0, stag);
            for (int e = 0; e < P.esize; ++e) sh.read(f0 + e, stg, stg + P.stg_floats, t, "pyramid staging read");
            if (g_copy_plane)
                for (int e = 0; e < 4; ++e) sh.write(dst + (long long)(r0 + q) * ds + c0 + e, dlo, dhi, dtag, "pyramid plane store");
        }
        auto lvl_store = [&](int l, int i, int j) {
            const Buf& b = bufs[l];
            if (i >= (H >> (l + 1)) || j >= (W >> (l + 1))) sh.fail("pyramid subband index", l);
            for (int s2 = 0; s2 < 4; ++s2)
                sh.write(b.base + (long long)s2 * b.sub + (long long)(i + pad) * b.stride + (j + pad), b.base + (long long)s2 * b.sub,
                         b.base + (long long)(s2 + 1) * b.sub, sbtag(l, s2), "pyramid subband store");
        };
        for (int pi = 0; pi < 2; ++pi)
            for (int pj = 0; pj < 2; ++pj) lvl_store(0, 2 * brow + pi, 2 * bcol + pj);
        if (P.pyr_levels >= 2) lvl_store(1, brow, bcol);
        for (int l = 2; l < P.pyr_levels; ++l) {
            const int sh2 = l - 2, m = (2 << sh2) - 1;
            if ((G << sh2) >= G2) sh.fail("shuffle partner outside the lane group", l);
            if ((by & m) == 0 && (bx & m) == 0) lvl_store(l, brow >> (l - 1), bcol >> (l - 1));
        }
    }
}

// Replays analyse_plane (pyramid or unpack + level 0, then the remaining levels one by one).
void replay_analyse(Shadow& sh, const Plan& P, long long stg, int stag, long long dst, int ds, long long dlo, long long dhi,
                    int dtag, const Buf* bufs, int pad, int (*sbtag)(int, int)) {
    int done;
    if (P.pyr) {
        replay_pyramid(sh, P, stg, stag, dst, ds, dlo, dhi, dtag, bufs, pad, sbtag);
        done = P.pyr_levels;
    } else {
        const Buf& b = bufs[0];
        replay_unpack(sh, P, stg, stag, dst, ds, dlo, dhi, dtag, P.L >= 1 ? b.base + (long long)pad * b.stride + pad : 0,
                      b.stride, b.sub, b.base, sbtag, P.L >= 1);
        done = P.L >= 1 ? 1 : 0;
    }
    for (int l = done; l < P.L; ++l) {
        sh.barrier();  // sync() before every level computed on its own
        const int n = P.H >> (l + 1), m = P.W >> (l + 1);
        const Buf& s0 = bufs[l - 1];
        const Buf& s1 = bufs[l];
        replay_haar(sh, s0.base + (long long)pad * s0.stride + pad, s0.stride, s0.base, s0.base + s0.sub, sbtag(l - 1, 0), n, m,
                    s1.base + (long long)pad * s1.stride + pad, s1.stride, s1.sub, s1.base, s1.base + 4LL * s1.sub, sbtag, l);
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
                   int tr, int tc, int itag, const char* what, int rank) {
    const int K = P.k, p = P.p, TR = P.TR, TC = P.TC;
    const int WV4 = 4 * ((TC + K - 1 + 3) / 4);
    const long long win = base + (long long)tr * TR * stride + (long long)tc * TC;
    if (win % 4 != 0) sh.fail(std::string(what) + ": window not 16-byte aligned", win);
    if (stride % 4 != 0) sh.fail(std::string(what) + ": stride not a multiple of 4", stride);
    for (int r = 0; r < TR + K - 1; ++r)
        for (int c = 0; c < WV4; ++c) {
            const long long a = win + (long long)r * stride + c;
            if (c >= TC + K - 1) {  // loaded but unused
                sh.touch(a, lo, hi, what);
                continue;
            }
            const int i = tr * TR + r - p, j = tc * TC + c - p;
            // Row i of this strip is plane row rank*n + i: its own rows and
            // the p halo rows on each side (copied from the neighbouring
            // strips) carry the data tag inside the plane and zero outside;
            // rows further down only feed tile-slack outputs and stay zero.
            const long long g = (long long)rank * n + i;
            const bool interior = i >= -p && i < n + p && g >= 0 && g < (long long)P.nstrips * n && j >= 0 && j < m;
            sh.read(a, lo, hi, interior ? itag : ZERO, what);
        }
}

// Replays the D-tile reads of corr_tile on an unpadded, tile-rounded plane.
void replay_dtile(Shadow& sh, const Plan& P, long long base, int stride, long long lo, long long hi, int n, int m,
                  int tr, int tc, int itag, int align = 4) {
    const int TR = P.TR, TC = P.TC;
    const long long dt = base + (long long)tr * TR * stride + (long long)tc * TC;
    if (dt % align != 0 || stride % align != 0) sh.fail("D tile misaligned for its loads", dt);
    for (int r = 0; r < TR; ++r)
        for (int c = 0; c < TC; ++c) {
            const int i = tr * TR + r, j = tc * TC + c;
            const bool interior = i < n && j < m;
            sh.read(dt + (long long)r * stride + c, lo, hi, interior ? itag : ZERO, "D tile");
        }
}

// The kernels compute n / d as fastdiv(n); check it exactly for every n the
// kernel can pass (0 <= n < nmax).
void check_div(FastDiv f, int d, long long nmax, const char* what) {
    for (long long n = 0; n < nmax; ++n)
        if ((long long)fastdiv_host((uint32_t)n, f) != n / d) {
            std::printf("FAIL fastdiv %s: %lld / %d\n", what, n, d);
            std::exit(1);
        }
}

void check_divs(const Plan& P) {
    check_div(P.div_q4, P.W / 4, (long long)P.H * (P.W / 4) + 1, "W/4");
    for (int l = 0; l < P.L; ++l)
        check_div(P.div_m[l], P.W >> (l + 1), (long long)(P.H >> (l + 1)) * (P.W >> (l + 1)) + 1, "level cols");
    for (int l = 0; l <= kMaxL; ++l) {
        if (l < kMaxL && l >= P.L) continue;
        check_div(P.div_ntc[l], P.ntc[l], (long long)P.ntr[l] * P.ntc[l] + 1, "tile cols");
    }
}

// Replays push_halos of every strip (all strips in the phase after their own
// CTA barrier that follows the analysis): strip r sends each of its rows that
// strip t = r + d holds as a halo row, whole (padding columns and the 16-byte
// rounding included), into t's padding row.  t may still be in its analysis
// phase when the store lands (no cluster barrier in between), so each float
// written must also be untouched in t's previous phase.
void replay_push(std::vector<Shadow>& shs, const Plan& P) {
    const int NS = (int)shs.size();
    auto one = [&](int rank, const Buf& b, int nsub_lg, int rows, int cols, int tagbase, bool per_sub_tag) {
        Shadow& me = shs[rank];
        const int pad = P.p;
        const int reach = (pad + rows - 1) / rows;
        const int nq = (cols + 2 * pad + 3) >> 2;
        const long long span = (long long)(1 << nsub_lg) * (b.sub ? b.sub : 0);
        const long long lo = b.base, hi = nsub_lg ? b.base + span : b.base + (long long)(rows + 2 * pad) * b.stride;
        if (b.base % 4 || b.stride % 4 || b.sub % 4) me.fail("halo rows not 16-byte aligned", b.base);
        if (4 * nq > b.stride) me.fail("padded row rounded to 16 bytes exceeds the stride", nq);
        for (int d = -reach; d <= reach; ++d) {
            const int t = rank + d;
            if (d == 0 || t < 0 || t >= NS) continue;
            int i0, n;
            if (d > 0) {
                i0 = std::max(-pad, -d * rows);
                n = std::min(0, (1 - d) * rows) - i0;
            } else {
                i0 = std::max(rows, -d * rows);
                n = std::min(rows + pad, (1 - d) * rows) - i0;
            }
            if (n <= 0) continue;
            const int total = (n << nsub_lg) * nq;
            for (int e = 0; e < total; ++e) {
                const int rest = e / nq, q = e - rest * nq;
                const int j = rest >> nsub_lg, s = rest - (j << nsub_lg);
                const int i = i0 + j;
                const int lr = d * rows + i;
                if (lr < 0 || lr >= rows) me.fail("halo source row outside the strip", lr);
                if (!(i < 0 || i >= rows)) me.fail("halo destination row inside the strip", i);
                const long long slo = nsub_lg ? b.base + (long long)s * b.sub : lo;
                const long long shi = nsub_lg ? b.base + (long long)(s + 1) * b.sub : hi;
                const int tag = per_sub_tag ? tagbase + s : tagbase;
                Shadow& tg = shs[t];
                for (int f = 0; f < 4; ++f) {
                    const int c = 4 * q + f - pad;  // interior column (negative or >= cols: padding, zero)
                    const long long at = b.base + (long long)s * b.sub + 4LL * q + f;
                    const long long src = at + (long long)(lr + pad) * b.stride;
                    const long long dst = at + (long long)(i + pad) * b.stride;
                    const int expect = (c >= 0 && c < cols) ? tag : ZERO;
                    me.read(src, slo, shi, expect, "halo source row");
                    tg.in_bounds(dst, slo, shi, "halo row");
                    if (tg.rd[dst] >= tg.epoch - 1 || tg.wr[dst] >= tg.epoch - 1)
                        tg.fail("halo row touched by its strip while the owner's store may land", dst);
                    tg.write(dst, slo, shi, expect, "halo row");
                }
            }
        }
    };
    // The planner's push constants against the kernel's formulas.
    {
        const int nw = P.nthreads / 32;
        int gbase = 0;
        for (int bi = 0; bi <= P.L; ++bi) {
            const int rows = bi == 0 ? P.H : P.H >> bi, cols = bi == 0 ? P.W : P.W >> bi;
            const int reach = (P.p + rows - 1) / rows;
            if (P.hal_nq[bi] != ((cols + 2 * P.p + 3) >> 2) || P.hal_reach[bi] != reach || P.hal_g0[bi] != gbase % nw)
                shs[0].fail("halo push constants", bi);
            gbase += (2 * reach) << (bi == 0 ? 0 : 2);
        }
    }
    for (int r = 0; r < NS; ++r) {
        shs[r].phase = "halo push";
        one(r, P.X, 0, P.H, P.W, XT, false);
        for (int l = 0; l < P.L; ++l) one(r, P.S[l], 2, P.H >> (l + 1), P.W >> (l + 1), s_tag(l, 0), true);
    }
}

void barrier_all(std::vector<Shadow>& shs) {
    for (auto& sh : shs) sh.barrier();
}

// NHWC channel octets.  The octet run of CTA r (pixels r*opix ..): 16-byte
// chunks of whole pixels, from the last octet of the last batch element
// (bounds), into the octet buffer once each.
const int OCT = 400;  // tag of octet-buffer floats
void replay_octet_load(Shadow& sh, const Plan& P, int r, long long tbuf = -1) {
    const int cpp = P.esize / 2, H = P.H, W = P.W;
    const long long total = (long long)P.B * H * W * P.C;  // NHWC elements
    const int o = P.C / 8 - 1, b = P.B - 1;
    if (tbuf < 0) tbuf = P.tbuf;
    if (tbuf % 4 || tbuf < P.stg) sh.fail("octet buffer", tbuf);
    for (int ch = 0; ch < P.opix * cpp; ++ch) {
        const int j = cpp == 2 ? ch >> 1 : ch, h = ch - j * cpp;
        const long long e0 = ((long long)b * H * W + (long long)r * P.opix + j) * P.C + 8LL * o + 8 / cpp * h;
        check_global(e0, total, "octet run first element");
        check_global(e0 + 16 / P.esize - 1, total, "octet run last element");
        if ((e0 * P.esize) % 16) sh.fail("octet chunk source not 16-byte aligned", e0);
        for (int f = 0; f < 4; ++f) sh.write(tbuf + 4LL * ch + f, tbuf, tbuf + P.stg_floats, OCT, "octet buffer");
    }
}

// Scatter of CTA r: its pixels' channel q into CTA q's staging at stg (tag
// stag), og pixels a step (og * esize bytes a channel, aligned to that).
void replay_octet_scatter(std::vector<Shadow>& shs, const Plan& P, int r, long long stg, int stag, long long tbuf = -1) {
    Shadow& me = shs[r];
    if (tbuf < 0) tbuf = P.tbuf;
    for (int f = 0; f < P.stg_floats; ++f) me.read(tbuf + f, tbuf, tbuf + P.stg_floats, OCT, "octet buffer");
    const int per = 4 / P.esize, og = P.og;  // elements a staging float; pixels a step
    if (stg % 4) me.fail("scattered staging not 16-byte aligned", stg);
    if (og != (P.opix % 4 == 0 ? 4 : 2) || P.opix % og) me.fail("octet step", og);
    for (int gq = 0; gq < P.opix / og; ++gq) {
        const long long e = (long long)r * P.opix + (long long)og * gq;
        if ((e * P.esize) % (og * P.esize)) me.fail("scatter store misaligned", e);
        for (int q = 0; q < 8; ++q)
            for (long long f = e / per; f < (e + og) / per; ++f)
                shs[q].write(stg + f, stg, stg + P.stg_floats, stag, "scattered staging");
    }
}

void check_fused(const wtconv_desc_t& d, Kind kind) {
    Plan P;
    const wtconv_status_t st = make_plan(&d, kind, kB200SMs, &P);
    if (st == WTCONV_ERR_UNSUPPORTED) {
        std::printf("fused: unsupported (plane too large)\n");
        return;
    }
    if (st != WTCONV_OK) {
        std::printf("FAIL fused plan status %d\n", (int)st);
        std::exit(1);
    }
    const int K = P.k, KK = K * K, p = P.p, L = P.L, H = P.H, W = P.W, TR = P.TR, TC = P.TC;
    const int ncls = 1 + 4 * L, NS = P.nstrips;
    check_divs(P);
    check_div(P.div_w, W, (long long)(2 * p * 4) * W + 1, "W");
    if (P.Hp != H * NS || NS < 1 || NS > kMaxStrips || (NS > 1 && (H % (1 << L) || H % 4))) {
        std::printf("FAIL strips: Hp %d H %d n %d\n", P.Hp, H, NS);
        std::exit(1);
    }
    if (P.nthreads % 32 || P.nthreads > (P.nstrips > 1 ? kStripMaxThreads : kFusedMaxThreads) || P.nthreads < 32) {
        std::printf("FAIL fused thread count %d\n", P.nthreads);
        std::exit(1);
    }
    if (P.base_tid0 < P.n_sub_tiles || P.tile_end != P.base_tid0 + P.n_base_tiles ||
        P.merged != (P.tile_end <= P.nthreads ? 1 : 0)) {
        std::printf("FAIL tile index space: sub %d base0 %d base %d end %d threads %d\n", P.n_sub_tiles, P.base_tid0,
                    P.n_base_tiles, P.tile_end, P.nthreads);
        std::exit(1);
    }
    if (P.n_fin != (L >= 1 ? (H / 2) * (W / 4) : 0) || P.fin_off < 0 || P.fin_off >= P.nthreads || P.fin_off % 32) {
        std::printf("FAIL synthesis items %d offset %d\n", P.n_fin, P.fin_off);
        std::exit(1);
    }
    if (P.smem_floats % 4 || P.smem_floats * 4 > 227 * 1024) {
        std::printf("FAIL smem size\n");
        std::exit(1);
    }
    // NHWC channel octets: 8 CTAs a cluster, each on whole planes (strip 0),
    // staging filled by the cluster's scatters from the octet buffers.
    const int NC = cluster_ctas(P);
    if (P.oct) {
        if (!P.nhwc || NS != 1 || P.padded || P.C % 8 || P.opix * 8LL != (long long)H * W || P.opix % 2 ||
            P.tbuf % 4 || P.tbuf < P.stg + P.stg_floats || P.tbuf + (long long)P.stg_floats > P.smem_floats ||
            (kind != kForward && kind != kBackwardInput)) {
            std::printf("FAIL octet plan: opix %d tbuf %d stg %d smem %d\n", P.opix, P.tbuf, P.stg, P.smem_floats);
            std::exit(1);
        }
    } else if (P.nhwc && kind != kBackward && NS == 1 && !P.padded && P.C % 8 == 0 && ((long long)H * W) % 16 == 0 &&
               P.smem_floats + (long long)P.stg_floats <= kSmemLimitFloats && (kind == kForward || kind == kBackwardInput)) {
        std::printf("FAIL octet plan not taken where it fits\n");
        std::exit(1);
    }
    std::vector<Shadow> shs(NC, Shadow(P.smem_floats));
    const long long all = P.smem_floats;
    if (P.grid < 1 || P.grid > (long long)P.B * P.C) shs[0].fail("grid", P.grid);
    auto octet_load = [&](Shadow& sh, int r) { replay_octet_load(sh, P, r); };
    auto octet_scatter = [&](int r) { replay_octet_scatter(shs, P, r, P.stg, XT + 10); };
    const int xrows = P.ntr[kMaxL] * TR + 2 * p;
    const long long xlo = P.X.base, xhi = P.X.base + (long long)xrows * P.X.stride;
    const long long ylo = P.Y.base, yhi = P.Y.base + (long long)P.ntr[kMaxL] * TR * P.Y.stride;
    for (int cl = 0; cl < ncls; ++cl)
        if ((P.wbase + cl * P.wcls) % 4) shs[0].fail("weight class not 16-byte aligned", P.wbase + cl * P.wcls);
    const int ntc = P.ntc[kMaxL];
    const long long plane = (long long)P.Hr * P.Wr;

    // Channel octets with a synthesis: outputs go to the owners' output octet
    // buffers ([8 channels][opix pixels], stored format; CTA r's channel row r).
    const int OUT = 401;
    const bool oct_out = P.oct && L >= 1;
    if (oct_out && (P.obuf % 4 || P.obuf < P.tbuf + P.stg_floats || P.obuf + (long long)P.stg_floats > P.smem_floats))
        shs[0].fail("output octet buffer", P.obuf);
    // Four outputs from pixel px (og = 2: two pixel pairs, each to its own owner).
    auto octet_out = [&](int r, int px4) {
        for (int px = px4; px < px4 + 4; px += P.og) {
            const int owner = (int)fastdiv_host((uint32_t)px, P.div_opix), j = px - owner * P.opix;
            if (owner != px / P.opix || owner < 0 || owner >= 8) shs[r].fail("output owner", px);
            if ((px + P.og - 1) / P.opix != owner) shs[r].fail("output store crosses a run", px);
            const long long e = (long long)r * P.opix + j;  // element of the owner's buffer
            if ((e * P.esize) % (P.og * P.esize)) shs[r].fail("output octet store misaligned", e);
            const int per = 4 / P.esize;
            for (long long f = e / per; f < (e + P.og) / per; ++f)
                shs[owner].write(P.obuf + f, P.obuf, P.obuf + P.stg_floats, OUT, "output octet buffer");
        }
    };
    // The owner's pass over its buffer: every float read, its pixels' 8
    // channels stored in y (last octet of the last batch element: bounds).
    auto octet_stream = [&](int r) {
        Shadow& me = shs[r];
        for (int f = 0; f < P.stg_floats; ++f) me.read(P.obuf + f, P.obuf, P.obuf + P.stg_floats, OUT, "output octet buffer");
        const long long total = (long long)P.B * H * W * P.C;
        for (int j = 0; j < P.opix; ++j) {
            const long long e0 = ((long long)(P.B - 1) * H * W + (long long)r * P.opix + j) * P.C + 8LL * (P.C / 8 - 1);
            check_global(e0, total, "octet output run");
            check_global(e0 + 7, total, "octet output run");
            if ((e0 * P.esize) % 16) me.fail("octet output run not 16-byte aligned", e0);
        }
    };

    // Phase A's synthesis of the previous plane: rows 2i, 2i+1 x columns 4q..4q+3.
    auto synthesis = [&](Shadow& sh, int rank, int crank) {
        for (int t = 0; t < P.n_fin; ++t) {
            const int i = (int)fastdiv_host(t, P.div_q4), q = t - i * (W / 4);
            if (i != t / (W / 4)) sh.fail("synthesis item division", t);
            const int j0 = 2 * q;
            for (int l = L - 1; l >= 1; --l) {
                const Buf& Q = P.Q[l];
                const int ri = i >> l, rj = j0 >> l;
                if (ri >= (H >> (l + 1)) || rj >= (W >> (l + 1))) sh.fail("coarse synthesis index", l);
                for (int s2 = 0; s2 < 4; ++s2)
                    sh.read(Q.base + (long long)s2 * Q.sub + (long long)ri * Q.stride + rj, Q.base + (long long)s2 * Q.sub,
                            Q.base + (long long)(s2 + 1) * Q.sub, q_tag(l, s2), "coarse Q read");
            }
            const Buf& Q = P.Q[0];
            if (j0 + 1 >= W / 2) sh.fail("level-0 synthesis column", j0);
            for (int s2 = 0; s2 < 4; ++s2) {
                const long long a = Q.base + (long long)s2 * Q.sub + (long long)i * Q.stride + j0;
                if (a % 2) sh.fail("level-0 pair load not 8-byte aligned", a);
                for (int e = 0; e < 2; ++e)
                    sh.read(a + e, Q.base + (long long)s2 * Q.sub, Q.base + (long long)(s2 + 1) * Q.sub, q_tag(0, s2),
                            "level-0 Q read");
            }
            for (int rr = 0; rr < 2; ++rr) {
                const long long a = P.Y.base + (long long)(2 * i + rr) * P.Y.stride + 4 * q;
                if (a % 4) sh.fail("Y load not 16-byte aligned", a);
                const bool store = 2 * i + rr < real_rows_host(P, rank) && 4 * q < P.Wr;
                for (int e = 0; e < 4; ++e) {
                    sh.read(a + e, ylo, yhi, YT, "Y read");
                    if (store && !oct_out) check_global((long long)(rank * H + 2 * i + rr) * P.Wr + 4 * q + e, plane, "y store");
                }
                if (oct_out) octet_out(crank, (2 * i + rr) * W + 4 * q);
            }
        }
    };

    // The persistent walk over two planes and the final synthesis, with the
    // kernel's barriers (cluster-wide with strips) as phase boundaries:
    //   stage(0) | A(0) | [strips: halo push(0)] | B(0): stage(1), tiles(0) | A(1) | ... | A(end)
    if (P.oct) {
        for (int r = 0; r < NC; ++r) {
            shs[r].phase = "initial octet run";
            octet_load(shs[r], r);
        }
        barrier_all(shs);
        for (int r = 0; r < NC; ++r) {
            shs[r].phase = "initial scatter";
            octet_scatter(r);
        }
    } else {
        for (int r = 0; r < NS; ++r) {
            shs[r].phase = "initial staging";
            replay_stage(shs[r], P, P.stg, XT + 10, r);
        }
    }
    for (int unit = 0; unit <= 2; ++unit) {
        barrier_all(shs);
        for (int r = 0; r < NC; ++r) {
            Shadow& sh = shs[r];
            if (unit < 2) {
                if (P.oct && unit + 1 < 2) {
                    sh.phase = "A: next octet run";
                    octet_load(sh, r);
                }
                sh.phase = "A: fold";
                for (int cl = 0; cl < ncls; ++cl)
                    for (int t = 0; t < KK; ++t)
                        sh.write(P.wbase + (long long)cl * P.wcls + t, P.wbase, P.wbase + (long long)ncls * P.wcls, WTS,
                                 "weights");
                sh.write(P.bias, P.bias, P.bias + 1, BIAS, "bias");
            }
        }
        if (unit < 2) {
            // The analysis may have its own CTA barriers (levels computed one
            // at a time); the synthesis runs after its last one.
            for (int r = 0; r < NC; ++r) {
                shs[r].phase = "A: analysis";
                g_rank = P.oct ? 0 : r;
                const int e0 = shs[r].epoch;
                replay_analyse(shs[r], P, P.stg, XT + 10, P.X.base + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi,
                               XT, P.S, p, s_tag);
                if (r + 1 < NC) shs[r].epoch = e0;  // replay the next strip from the same phase
                else for (int q = 0; q + 1 < NC; ++q) shs[q].epoch = shs[r].epoch;
            }
        }
        if (unit > 0 && L >= 1)
            for (int r = 0; r < NC; ++r) {
                shs[r].phase = "A: synthesis";
                synthesis(shs[r], P.oct ? 0 : r, r);
            }
        if (unit == 2) {
            if (oct_out) {
                barrier_all(shs);
                for (int r = 0; r < NC; ++r) {
                    shs[r].phase = "final output octets";
                    octet_stream(r);
                }
            }
            break;
        }
        // Strips: CTA barrier, halo push, then the cluster barrier.
        if (NS > 1) {
            barrier_all(shs);
            replay_push(shs, P);
        }
        barrier_all(shs);
        for (int r = 0; r < NC; ++r) {
            shs[r].phase = "B: staging";
            if (unit + 1 < 2) {
                if (P.oct) octet_scatter(r);
                else replay_stage(shs[r], P, P.stg, XT + 10, r);
            }
            if (oct_out && unit > 0) {
                shs[r].phase = "B: output octets";
                octet_stream(r);
            }
        }
        for (int rr = 0; rr < NC; ++rr) {
            Shadow& sh = shs[rr];
            const int r = P.oct ? 0 : rr;  // strip of the CTA
            sh.phase = "B: subband tiles";
            for (int cl = 1; cl < ncls; ++cl) {
                const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
                const int n = H >> (l + 1), m = W >> (l + 1);
                const int ntiles = P.sub_begin[cl] - P.sub_begin[cl - 1];
                if (ntiles != P.ntr[l] * P.ntc[l]) sh.fail("tile count", cl);
                for (int local = 0; local < ntiles; ++local) {
                    const int tr = (int)fastdiv_host(local, P.div_ntc[l]), tc = local - tr * P.ntc[l];
                    for (int t = 0; t < KK; ++t) sh.read(P.wbase + (long long)cl * P.wcls + t, 0, all, WTS, "weights");
                    const Buf& S = P.S[l];
                    replay_window(sh, P, S.base + (long long)s * S.sub, S.stride, S.base + (long long)s * S.sub,
                                  S.base + (long long)(s + 1) * S.sub, n, m, tr, tc, s_tag(l, s), "subband window", r);
                    const Buf& Q = P.Q[l];
                    const long long out = Q.base + (long long)s * Q.sub + (long long)tr * TR * Q.stride + (long long)tc * TC;
                    if (out % 4) sh.fail("Q tile not 16-byte aligned", out);
                    for (int o = 0; o < TR; ++o)
                        for (int j = 0; j < TC; ++j)
                            sh.write(out + (long long)o * Q.stride + j, Q.base + (long long)s * Q.sub,
                                     Q.base + (long long)(s + 1) * Q.sub, q_tag(l, s), "Q tile");
                }
            }
            sh.phase = "B: base tiles";
            for (int t = 0; t < P.n_base_tiles; ++t) {
                const int tr = (int)fastdiv_host(t, P.div_ntc[kMaxL]), tc = t - tr * ntc;
                for (int q = 0; q < KK; ++q) sh.read(P.wbase + q, 0, all, WTS, "base weights");
                sh.read(P.bias, 0, all, BIAS, "bias");
                replay_window(sh, P, P.X.base, P.X.stride, xlo, xhi, H, W, tr, tc, XT, "base window", r);
                if (L >= 1) {
                    const long long yo = P.Y.base + (long long)tr * TR * P.Y.stride + (long long)tc * TC;
                    if (yo % 4 || P.Y.stride % 4) sh.fail("Y tile not 16-byte aligned", yo);
                    for (int o = 0; o < TR; ++o)
                        for (int e = 0; e < TC; ++e) sh.write(yo + (long long)o * P.Y.stride + e, ylo, yhi, YT, "Y tile");
                } else {
                    for (int o = 0; o < TR; ++o) {
                        const int h = tr * TR + o;
                        if (h >= real_rows_host(P, r)) continue;
                        for (int e = 0; e < TC; ++e)
                            check_global((long long)(r * H + h) * P.Wr + tc * TC + e, plane, "y store");
                    }
                }
            }
        }
    }
    std::printf("fused(kind %d): smem %d B, threads %d, TR %d, tiles %d+%d, merged %d, strips %d%s\n", (int)kind,
                P.smem_floats * 4, P.nthreads, TR, P.n_sub_tiles, P.n_base_tiles, P.merged, NS,
                P.oct ? ", channel octets" : "");
}

void check_bwdw(const wtconv_desc_t& d) {
    Plan P;
    const wtconv_status_t st = make_plan(&d, kBackwardWeight, kB200SMs, &P);
    if (st == WTCONV_ERR_UNSUPPORTED) {
        std::printf("bwdw: unsupported (plane too large)\n");
        return;
    }
    if (st != WTCONV_OK) {
        std::printf("FAIL bwdw plan status %d\n", (int)st);
        std::exit(1);
    }
    const int K = P.k, KK = K * K, p = P.p, L = P.L, H = P.H, W = P.W, TR = P.TR;
    const int ncls = 1 + 4 * L, NS = P.nstrips;
    check_divs(P);
    check_div(P.div_w, W, (long long)(2 * p * 4) * W + 1, "W");
    // NHWC channel octets: 8 CTAs a cluster on whole planes; the x run and
    // then the dy run go through the one octet buffer.
    const int NC = cluster_ctas(P);
    if (P.oct && (!P.nhwc || NS != 1 || P.padded || P.dy_stg || P.C % 8 || P.opix * 8LL != (long long)H * W ||
                  P.opix % 2 || P.tbuf < P.stg + 2LL * P.stg_floats || P.tbuf + (long long)P.stg_floats > P.smem_floats)) {
        std::printf("FAIL weight-gradient octet plan\n");
        std::exit(1);
    }
    std::vector<Shadow> shs(NC, Shadow(P.smem_floats));
    const int xrows = P.ntr[kMaxL] * TR + 2 * p;
    const long long xlo = P.X.base, xhi = P.X.base + (long long)xrows * P.X.stride;
    // dys: DY is the dy staging itself (strips of fp32 planes of whole tile
    // rows); the dy analysis writes no plane copy and the next dy strip is
    // staged after the correlation tiles, behind a CTA barrier.
    const bool dys = P.dy_stg != 0;
    const long long dlo = dys ? (long long)P.stg + P.stg_floats : P.DY.base;
    const long long dhi = dys ? dlo + P.stg_floats : P.DY.base + (long long)P.ntr[kMaxL] * TR * P.DY.stride;
    const int dtile_tag = dys ? DYT + 10 : DYT;
    if (dys && (P.DY.base != dlo || P.DY.stride != W || P.ntr[kMaxL] * TR != H || P.esize != 4 || P.padded || NS < 2 ||
                (long long)H * W != P.stg_floats))
        shs[0].fail("dy read from staging needs fp32 strips of whole tile rows", P.DY.base);
    if (P.stg % 4 || P.stg_floats % 4) shs[0].fail("staging alignment", P.stg);
    // Two planes in a row (the second must see the same zero padding), with
    // the kernel's barriers (cluster-wide with strips) as phase boundaries:
    //   stage(0) | analysis(0) | [strips: halo push(0), stage(1)] | [whole planes: stage(1)], correlation(0) | analysis(1) | ... | reduction
    // Octets, per CTA r: x run | scatter x | dy run | scatter dy, each step
    // behind a barrier.
    auto octet_pair = [&](const char* what) {
        for (int r = 0; r < NC; ++r) { shs[r].phase = what; replay_octet_load(shs[r], P, r); }
        barrier_all(shs);
        for (int r = 0; r < NC; ++r) replay_octet_scatter(shs, P, r, P.stg, XT + 10);
        barrier_all(shs);
        for (int r = 0; r < NC; ++r) replay_octet_load(shs[r], P, r);
        barrier_all(shs);
        for (int r = 0; r < NC; ++r) replay_octet_scatter(shs, P, r, P.stg + P.stg_floats, DYT + 10);
    };
    if (P.oct) {
        octet_pair("initial octet runs");
    } else {
        for (int r = 0; r < NS; ++r) {
            shs[r].phase = "initial staging";
            replay_stage(shs[r], P, P.stg, XT + 10, r);
            replay_stage(shs[r], P, P.stg + P.stg_floats, DYT + 10, r);
        }
    }
    for (int plane = 0; plane < 2; ++plane) {
        barrier_all(shs);
        for (int r = 0; r < NC; ++r) {
            Shadow& sh = shs[r];
            if (P.oct && plane == 0) {
                sh.phase = "next x run";
                replay_octet_load(sh, P, r);
            }
            sh.phase = "analysis";
            g_rank = P.oct ? 0 : r;
            const int e0 = sh.epoch;
            replay_analyse(sh, P, P.stg, XT + 10, P.X.base + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi, XT, P.S,
                           p, s_tag);
            g_copy_plane = !dys;
            replay_analyse(sh, P, P.stg + P.stg_floats, DYT + 10, P.DY.base, P.DY.stride, dlo, dhi, DYT, P.Q, 0, q_tag);
            g_copy_plane = true;
            if (r + 1 < NC) sh.epoch = e0;
            else for (int q = 0; q + 1 < NC; ++q) shs[q].epoch = sh.epoch;
        }
        if (NS > 1) {
            barrier_all(shs);
            replay_push(shs, P);
        } else {
            barrier_all(shs);
        }
        if (P.oct) {
            // Scatter the x run; behind a CTA barrier, the dy run (its
            // scatter follows the correlation tiles).
            for (int r = 0; r < NC; ++r) {
                shs[r].phase = "x scatter";
                if (plane == 0) replay_octet_scatter(shs, P, r, P.stg, XT + 10);
            }
            barrier_all(shs);
            for (int r = 0; r < NC; ++r) {
                shs[r].phase = "next dy run";
                if (plane == 0) replay_octet_load(shs[r], P, r);
            }
        } else {
            for (int r = 0; r < NS; ++r) {
                shs[r].phase = "staging";
                if (plane == 0) {
                    replay_stage(shs[r], P, P.stg, XT + 10, r);
                    if (!dys) replay_stage(shs[r], P, P.stg + P.stg_floats, DYT + 10, r);
                }
            }
        }
        if (NS > 1) barrier_all(shs);
        for (int rr = 0; rr < NC; ++rr) {
            Shadow& sh = shs[rr];
            const int r = P.oct ? 0 : rr;  // strip of the CTA
            sh.phase = "correlation";
            int covered = 0;
            for (int tid = 0; tid < P.cls_thr[ncls]; ++tid)
              for (int k = 0; k < P.tpt; ++k) {
                int cl = 0;
                while (tid >= P.cls_thr[cl + 1]) ++cl;
                const int lvl = (cl == 0) ? kMaxL : ((cl - 1) >> 2);
                const int first = (tid - P.cls_thr[cl]) * P.tpt;
                const int cnt = std::min(P.tpt, P.cls_tiles[cl] - first);
                if (cnt < 1) sh.fail("thread without tiles", tid);
                if (k >= cnt) continue;
                const int local = first + k;
                ++covered;
                const int tr = (int)fastdiv_host(local, P.div_ntc[lvl]), tc = local - tr * P.ntc[lvl];
                if (tr >= P.ntr[lvl]) sh.fail("tile row out of grid", tid);
                if (cl == 0) {
                    replay_window(sh, P, P.X.base, P.X.stride, xlo, xhi, H, W, tr, tc, XT, "base S window", r);
                    replay_dtile(sh, P, P.DY.base, P.DY.stride, dlo, dhi, H, W, tr, tc, dtile_tag);
                } else {
                    const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
                    const int n = H >> (l + 1), m = W >> (l + 1);
                    const Buf& S = P.S[l];
                    const Buf& Q = P.Q[l];
                    replay_window(sh, P, S.base + (long long)s * S.sub, S.stride, S.base + (long long)s * S.sub,
                                  S.base + (long long)(s + 1) * S.sub, n, m, tr, tc, s_tag(l, s), "subband S window", r);
                    replay_dtile(sh, P, Q.base + (long long)s * Q.sub, Q.stride, Q.base + (long long)s * Q.sub,
                                 Q.base + (long long)(s + 1) * Q.sub, n, m, tr, tc, q_tag(l, s));
                }
              }
            if (covered != P.n_all_tiles) sh.fail("tiles covered", covered);
            if (dys) {
                sh.barrier();  // the CTA's dy tiles are all read
                sh.phase = "dy staging";
                if (plane == 0) replay_stage(sh, P, P.stg + P.stg_floats, DYT + 10, r);
            }
        }
        if (P.oct) {
            barrier_all(shs);
            for (int r = 0; r < NC; ++r) {
                shs[r].phase = "dy scatter";
                if (plane == 0) replay_octet_scatter(shs, P, r, P.stg + P.stg_floats, DYT + 10);
            }
        }
    }
    const long long red_end = (long long)P.red + (long long)P.nthreads * KK + P.nthreads;
    barrier_all(shs);
    for (int r = 0; r < NC; ++r) {
        Shadow& sh = shs[r];
        sh.phase = "reduction";
        if (red_end > P.smem_floats) sh.fail("reduction scratch", red_end);
        for (int tid = 0; tid < P.nthreads; ++tid)
            for (int t = 0; t < KK; ++t) sh.write(P.red + (long long)tid * KK + t, P.red, red_end, RED, "class sums");
        for (int w = 0; w < P.nthreads / 32; ++w)
            sh.write(P.red + (long long)P.nthreads * KK + w, P.red, red_end, RED, "warp dy sums");
    }
    barrier_all(shs);
    for (int r = 0; r < NC; ++r)
        for (int k2 = 0; k2 < ncls; ++k2)
            for (int th = P.cls_thr[k2]; th < P.cls_thr[k2 + 1]; ++th)
                for (int t = 0; t < KK; ++t)
                    shs[r].read(P.red + (long long)th * KK + t, P.red, red_end, RED, "class reduction");
    Shadow& sh = shs[0];
    if (P.nthreads < P.cls_thr[ncls] || P.nthreads > (NS > 1 ? kStripMaxThreads : kBwdwMaxThreads) || P.nthreads % 32)
        sh.fail("thread count", P.nthreads);
    for (int cl = 0; cl < ncls; ++cl) {
        const int lv = cl == 0 ? kMaxL : (cl - 1) >> 2;
        if (P.cls_tiles[cl] != P.ntr[lv] * P.ntc[lv]) sh.fail("class tiles", cl);
    }
    if (P.groups < 1 || P.groups > P.B) sh.fail("groups", P.groups);
    if (P.parts != P.groups * NS) sh.fail("partial vectors", P.parts);
    if ((long long)P.nthreads * KK + P.nthreads / 32 > P.smem_floats) sh.fail("sum-dy scratch", P.nthreads);
    if (P.nv != ncls * KK + 1) sh.fail("partial vector length", P.nv);
    if ((long long)P.nv + ncls * KK + 1 > P.smem_floats) sh.fail("final-step scratch", P.nv);
    std::printf("bwdw: smem %d B, threads %d, TR %d, tiles %d (<= %d per thread), groups %d, strips %d%s%s\n",
                P.smem_floats * 4, P.nthreads, TR, P.n_all_tiles, P.tpt, P.groups, NS, dys ? ", dy read from staging" : "",
                P.oct ? ", channel octets" : "");
}

// Fused backward: dx conv tiles (the input-gradient pass: dy in X / S, dx
// in Q / Y) and correlation tiles (x windows in XS / SS against dy tiles at
// the interior of X / S) in one walk.
// Fused backward on NHWC channel octets: the octet buffers (x run at tbuf,
// dy run after it, the dx output buffer at obuf) and the two stagings of the
// cluster's 8 CTAs, over two planes: every staging float written once a
// plane by the cluster's scatters, every output float once by the owners'
// synthesis items, no phase race on them, and the global runs in bounds.
// The rest of the walk is the whole-plane one, replayed by check_bwd.
void check_bwd_octets(const Plan& P) {
    const int H = P.H, W = P.W, L = P.L, per = 4 / P.esize;
    const long long T0 = P.tbuf, T1 = P.tbuf + P.stg_floats;
    std::vector<Shadow> shs(8, Shadow(P.smem_floats));
    if (P.tbuf < P.stg + 2LL * P.stg_floats || (L >= 1 && P.obuf != P.tbuf + 2LL * P.stg_floats) ||
        (L >= 1 ? P.obuf : T1) + (long long)P.stg_floats > P.smem_floats || P.opix * 8LL != (long long)H * W ||
        P.og != (P.opix % 4 == 0 ? 4 : 2) || P.opix % P.og)
        shs[0].fail("octet buffers of the fused backward", P.tbuf);
    const int OUTB = 402;
    auto loads = [&](const char* what) {
        for (int r = 0; r < 8; ++r) {
            shs[r].phase = what;
            replay_octet_load(shs[r], P, r, T0);
            replay_octet_load(shs[r], P, r, T1);
        }
    };
    auto scatters = [&]() {
        for (int r = 0; r < 8; ++r) {
            shs[r].phase = "scatter";
            replay_octet_scatter(shs, P, r, P.stg, XT + 10, T0);
            replay_octet_scatter(shs, P, r, P.stg + P.stg_floats, DYT + 10, T1);
        }
    };
    auto analyses = [&]() {  // every staging float read by the two analyses
        for (int r = 0; r < 8; ++r) {
            shs[r].phase = "analysis reads";
            for (int f = 0; f < P.stg_floats; ++f) {
                shs[r].read(P.stg + f, P.stg, P.stg + P.stg_floats, XT + 10, "x staging");
                shs[r].read(P.stg + P.stg_floats + f, P.stg + P.stg_floats, P.stg + 2LL * P.stg_floats, DYT + 10,
                            "dy staging");
            }
        }
    };
    auto outputs = [&]() {  // the synthesis items of every CTA into the owners' output buffers
        if (L < 1) return;
        for (int r = 0; r < 8; ++r) {
            shs[r].phase = "dx outputs";
            for (int t = 0; t < P.n_fin; ++t) {
                const int i = t / (W / 4), q = t - i * (W / 4);
                for (int rr = 0; rr < 2; ++rr)
                    for (int px = (2 * i + rr) * W + 4 * q; px < (2 * i + rr) * W + 4 * q + 4; px += P.og) {
                        const int owner = (int)fastdiv_host((uint32_t)px, P.div_opix), j = px - owner * P.opix;
                        if (owner != px / P.opix || owner >= 8 || (px + P.og - 1) / P.opix != owner)
                            shs[r].fail("dx output owner", px);
                        const long long e = (long long)r * P.opix + j;
                        for (long long f = e / per; f < (e + P.og) / per; ++f)
                            shs[owner].write(P.obuf + f, P.obuf, P.obuf + P.stg_floats, OUTB, "dx output buffer");
                    }
            }
        }
    };
    auto streams = [&]() {
        if (L < 1) return;
        const long long total = (long long)P.B * H * W * P.C;
        for (int r = 0; r < 8; ++r) {
            shs[r].phase = "dx write-out";
            for (int f = 0; f < P.stg_floats; ++f)
                shs[r].read(P.obuf + f, P.obuf, P.obuf + P.stg_floats, OUTB, "dx output buffer");
            for (int j = 0; j < P.opix; ++j) {
                const long long e0 = ((long long)(P.B - 1) * H * W + (long long)r * P.opix + j) * P.C + 8LL * (P.C / 8 - 1);
                check_global(e0 + 7, total, "dx output run");
            }
        }
    };
    // prologue: runs, cluster barrier, scatters; then per plane: [barrier] A:
    // next runs, analyses, outputs of the previous plane; [barrier] B:
    // scatters, write-out of the previous plane; the last outputs behind a
    // final barrier.
    loads("initial runs");
    barrier_all(shs);
    scatters();
    for (int plane = 0; plane <= 2; ++plane) {
        barrier_all(shs);
        if (plane < 2) {
            if (plane + 1 < 2) loads("next runs");
            analyses();
        }
        if (plane > 0) outputs();
        if (plane == 2) break;
        barrier_all(shs);
        if (plane + 1 < 2) scatters();
        if (plane > 0) streams();
    }
    barrier_all(shs);
    streams();
}

void check_bwd(const wtconv_desc_t& d) {
    Plan P;
    const wtconv_status_t st = make_plan(&d, kBackward, kB200SMs, &P);
    if (st == WTCONV_ERR_UNSUPPORTED) {
        std::printf("bwd: no one-pass plan (two passes)\n");
        return;
    }
    if (st != WTCONV_OK) {
        std::printf("FAIL bwd plan status %d\n", (int)st);
        std::exit(1);
    }
    const int K = P.k, KK = K * K, p = P.p, L = P.L, H = P.H, W = P.W, TR = P.TR, TC = P.TC;
    const int ncls = 1 + 4 * L;
    check_divs(P);
    Shadow sh(P.smem_floats);
    const long long all = P.smem_floats;
    if (P.nstrips != 1) sh.fail("strips in the fused backward", P.nstrips);
    if (P.oct) check_bwd_octets(P);
    if (P.nthreads > kBwdMaxThreads || P.nthreads % 32 || P.corr0 % 32 || P.corr0 < P.tile_end) sh.fail("threads", P.nthreads);
    const int ncorr = P.cls_thr[ncls];
    if (P.corr0 + ncorr > P.nthreads) sh.fail("correlation threads", ncorr);
    if (P.an_split % 32 || P.an_split <= 0 || P.an_split >= P.nthreads) sh.fail("analysis split", P.an_split);
    if (P.parts != P.groups || P.groups < 1 || P.groups > P.B) sh.fail("groups", P.groups);
    if (P.smem_floats * 4 > 227 * 1024) sh.fail("smem", P.smem_floats);
    const int xrows = P.ntr[kMaxL] * TR + 2 * p;
    const long long xlo = P.X.base, xhi = P.X.base + (long long)xrows * P.X.stride;
    const long long slo = P.XS.base, shi = P.XS.base + (long long)xrows * P.XS.stride;
    const long long ylo = P.Y.base, yhi = P.Y.base + (long long)P.ntr[kMaxL] * TR * P.Y.stride;
    const int align = (p % 2 == 0) ? 2 : 1;
    const long long plane = (long long)P.Hr * P.Wr;
    // Weights folded once (before the first barrier), then the first pair staged.
    sh.phase = "fold";
    for (int cl = 0; cl < ncls; ++cl)
        for (int t = 0; t < KK; ++t)
            sh.write(P.wbase + (long long)cl * P.wcls + t, P.wbase, P.wbase + (long long)ncls * P.wcls, WTS, "weights");
    sh.write(P.bias, P.bias, P.bias + 1, BIAS, "bias");
    sh.phase = "initial staging";
    replay_stage(sh, P, P.stg, XT + 10, 0);
    replay_stage(sh, P, P.stg + P.stg_floats, DYT + 10, 0);
    auto synthesis = [&]() {
        for (int t = 0; t < P.n_fin; ++t) {
            const int i = (int)fastdiv_host(t, P.div_q4), q = t - i * (W / 4);
            const int j0 = 2 * q;
            for (int l = L - 1; l >= 1; --l) {
                const Buf& Q = P.Q[l];
                for (int s2 = 0; s2 < 4; ++s2)
                    sh.read(Q.base + (long long)s2 * Q.sub + (long long)(i >> l) * Q.stride + (j0 >> l),
                            Q.base + (long long)s2 * Q.sub, Q.base + (long long)(s2 + 1) * Q.sub, q_tag(l, s2), "coarse Q");
            }
            const Buf& Q = P.Q[0];
            for (int s2 = 0; s2 < 4; ++s2)
                for (int e = 0; e < 2; ++e)
                    sh.read(Q.base + (long long)s2 * Q.sub + (long long)i * Q.stride + j0 + e, Q.base + (long long)s2 * Q.sub,
                            Q.base + (long long)(s2 + 1) * Q.sub, q_tag(0, s2), "level-0 Q");
            for (int rr = 0; rr < 2; ++rr)
                for (int e = 0; e < 4; ++e) {
                    sh.read(P.Y.base + (long long)(2 * i + rr) * P.Y.stride + 4 * q + e, ylo, yhi, YT, "Y");
                    if (2 * i + rr < P.Hr && 4 * q < P.Wr)
                        check_global((long long)(2 * i + rr) * P.Wr + 4 * q + e, plane, "dx store");
                }
        }
    };
    for (int plane_i = 0; plane_i <= 2; ++plane_i) {
        sh.barrier();
        if (plane_i < 2) {
            sh.phase = "A: analysis of x and dy";
            g_rank = 0;
            const int e0 = sh.epoch;
            replay_analyse(sh, P, P.stg, XT + 10, P.XS.base + (long long)p * P.XS.stride + p, P.XS.stride, slo, shi, XT,
                           P.SS, p, ss_tag);
            const int e1 = sh.epoch;
            sh.epoch = e0;  // both analyses run side by side, meeting the same barriers
            replay_analyse(sh, P, P.stg + P.stg_floats, DYT + 10, P.X.base + (long long)p * P.X.stride + p, P.X.stride,
                           xlo, xhi, DYT, P.S, p, s_tag);
            if (sh.epoch != e1) sh.fail("the two analyses meet different barriers", e1);
        }
        if (plane_i > 0 && L >= 1) {
            sh.phase = "A: synthesis of the previous dx";
            synthesis();
        }
        if (plane_i == 2) break;
        sh.barrier();
        sh.phase = "B: staging";
        if (plane_i == 0) {
            replay_stage(sh, P, P.stg, XT + 10, 0);
            replay_stage(sh, P, P.stg + P.stg_floats, DYT + 10, 0);
        }
        sh.phase = "B: dx conv tiles";
        for (int cl = 1; cl < ncls; ++cl) {
            const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
            const int n = H >> (l + 1), m = W >> (l + 1);
            for (int local = 0; local < P.sub_begin[cl] - P.sub_begin[cl - 1]; ++local) {
                const int tr = (int)fastdiv_host(local, P.div_ntc[l]), tc = local - tr * P.ntc[l];
                for (int t = 0; t < KK; ++t) sh.read(P.wbase + (long long)cl * P.wcls + t, 0, all, WTS, "weights");
                const Buf& S = P.S[l];
                replay_window(sh, P, S.base + (long long)s * S.sub, S.stride, S.base + (long long)s * S.sub,
                              S.base + (long long)(s + 1) * S.sub, n, m, tr, tc, s_tag(l, s), "dy subband window", 0);
                const Buf& Q = P.Q[l];
                const long long out = Q.base + (long long)s * Q.sub + (long long)tr * TR * Q.stride + (long long)tc * TC;
                for (int o = 0; o < TR; ++o)
                    for (int j = 0; j < TC; ++j)
                        sh.write(out + (long long)o * Q.stride + j, Q.base + (long long)s * Q.sub,
                                 Q.base + (long long)(s + 1) * Q.sub, q_tag(l, s), "Q tile");
            }
        }
        for (int t = 0; t < P.n_base_tiles; ++t) {
            const int tr = (int)fastdiv_host(t, P.div_ntc[kMaxL]), tc = t - tr * P.ntc[kMaxL];
            for (int q = 0; q < KK; ++q) sh.read(P.wbase + q, 0, all, WTS, "base weights");
            replay_window(sh, P, P.X.base, P.X.stride, xlo, xhi, H, W, tr, tc, DYT, "dy window", 0);
            if (L >= 1) {
                const long long yo = P.Y.base + (long long)tr * TR * P.Y.stride + (long long)tc * TC;
                for (int o = 0; o < TR; ++o)
                    for (int e = 0; e < TC; ++e) sh.write(yo + (long long)o * P.Y.stride + e, ylo, yhi, YT, "Y tile");
            } else {
                for (int o = 0; o < TR; ++o)
                    if (tr * TR + o < P.Hr)
                        for (int e = 0; e < TC; ++e)
                            check_global((long long)(tr * TR + o) * P.Wr + tc * TC + e, plane, "dx store");
            }
        }
        sh.phase = "B: correlation tiles";
        int covered = 0;
        for (int ct = 0; ct < ncorr; ++ct)
            for (int k = 0; k < P.tpt; ++k) {
                int cl = 0;
                while (ct >= P.cls_thr[cl + 1]) ++cl;
                const int lvl = (cl == 0) ? kMaxL : ((cl - 1) >> 2);
                const int first = (ct - P.cls_thr[cl]) * P.tpt;
                const int cnt = std::min(P.tpt, P.cls_tiles[cl] - first);
                if (cnt < 1) sh.fail("thread without tiles", ct);
                if (k >= cnt) continue;
                const int local = first + k;
                ++covered;
                const int tr = (int)fastdiv_host(local, P.div_ntc[lvl]), tc = local - tr * P.ntc[lvl];
                if (cl == 0) {
                    replay_window(sh, P, P.XS.base, P.XS.stride, slo, shi, H, W, tr, tc, XT, "x window", 0);
                    replay_dtile(sh, P, P.X.base + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi, H, W, tr, tc, DYT,
                                 align);
                } else {
                    const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
                    const int n = H >> (l + 1), m = W >> (l + 1);
                    const Buf& SS = P.SS[l];
                    const Buf& S = P.S[l];
                    replay_window(sh, P, SS.base + (long long)s * SS.sub, SS.stride, SS.base + (long long)s * SS.sub,
                                  SS.base + (long long)(s + 1) * SS.sub, n, m, tr, tc, ss_tag(l, s), "x subband window", 0);
                    replay_dtile(sh, P, S.base + (long long)s * S.sub + (long long)p * S.stride + p, S.stride,
                                 S.base + (long long)s * S.sub, S.base + (long long)(s + 1) * S.sub, n, m, tr, tc,
                                 s_tag(l, s), align);
                }
            }
        if (covered != P.n_all_tiles) sh.fail("correlation tiles covered", covered);
    }
    // Reduction scratch after the walk.
    sh.barrier();
    sh.phase = "reduction";
    const long long red_end = (long long)P.red + (long long)ncorr * KK + P.nthreads / 32;
    if (red_end > P.smem_floats) sh.fail("reduction scratch", red_end);
    for (int ct = 0; ct < ncorr; ++ct)
        for (int t = 0; t < KK; ++t) sh.write(P.red + (long long)ct * KK + t, P.red, red_end, RED, "class sums");
    for (int w = 0; w < P.nthreads / 32; ++w) sh.write(P.red + (long long)ncorr * KK + w, P.red, red_end, RED, "dy sums");
    sh.barrier();
    for (int k2 = 0; k2 < ncls; ++k2)
        for (int th = P.cls_thr[k2]; th < P.cls_thr[k2 + 1]; ++th)
            for (int t = 0; t < KK; ++t) sh.read(P.red + (long long)th * KK + t, P.red, red_end, RED, "class reduction");
    if ((long long)P.nv + ncls * KK + 1 > P.smem_floats) sh.fail("final-step scratch", P.nv);
    Plan Pin, Pw;
    const bool one = make_plan(&d, kBackwardInput, kB200SMs, &Pin) == WTCONV_OK &&
                     make_plan(&d, kBackwardWeight, kB200SMs, &Pw) == WTCONV_OK && prefer_one_pass(P, Pin, Pw);
    std::printf("bwd: smem %d B, threads %d (%d conv + %d correlation), TR %d, groups %d, library picks %s%s\n",
                P.smem_floats * 4, P.nthreads, P.corr0, ncorr, TR, P.groups, one ? "one pass" : "two passes",
                P.oct ? ", channel octets" : "");
}

// NHWC: the kernels address element e (plane-relative, row-major over the
// real Hr x Wr plane) of plane (b, c), strip `rank`, at
//   b*Hr*Wr*C + c  +  rank*H*Wr*C  +  e*C     (e < real rows of the strip x Wr).
// Every (b, c, rank, e) must land on a distinct element of the B*C*Hr*Wr
// tensor, and every element must be reached.
void check_nhwc_map(const wtconv_desc_t& d) {
    Plan P;
    if (make_plan(&d, kForward, kB200SMs, &P) != WTCONV_OK) return;
    const long long hw = (long long)P.Hr * P.Wr, n = (long long)P.B * P.C * hw;
    if (n > (1LL << 26)) return;
    std::vector<unsigned char> seen(n, 0);
    for (int b = 0; b < P.B; ++b)
        for (int c = 0; c < P.C; ++c)
            for (int rank = 0; rank < P.nstrips; ++rank) {
                const int rows = std::max(0, std::min(P.H, P.Hr - rank * P.H));
                const long long base = (long long)b * hw * P.C + c + (long long)rank * P.H * P.Wr * P.C;
                for (long long e = 0; e < (long long)rows * P.Wr; ++e) {
                    const long long off = base + e * P.C;
                    if (off < 0 || off >= n || seen[off]) {
                        std::printf("FAIL nhwc element map b %d c %d strip %d e %lld -> %lld\n", b, c, rank, e, off);
                        std::exit(1);
                    }
                    seen[off] = 1;
                }
            }
    for (long long i = 0; i < n; ++i)
        if (!seen[i]) {
            std::printf("FAIL nhwc element %lld never addressed\n", i);
            std::exit(1);
        }
    std::printf("nhwc: %lld elements, each addressed once\n", n);
}

}  // namespace

int main(int argc, char** argv) {
    if (argc != 8 && argc != 9) {
        std::printf("usage: plan_access_check B C H W k L dtype [layout]\n");
        return 2;
    }
    wtconv_desc_t d{};
    d.B = std::atoi(argv[1]); d.C = std::atoi(argv[2]); d.H = std::atoi(argv[3]); d.W = std::atoi(argv[4]);
    d.k = std::atoi(argv[5]); d.L = std::atoi(argv[6]); d.dtype = std::atoi(argv[7]);
    d.layout = argc == 9 ? std::atoi(argv[8]) : WTCONV_NCHW;
    if (validate(&d) != WTCONV_OK) {
        std::printf("invalid (status %d)\n", (int)validate(&d));
        return 3;
    }
    check_fused(d, kForward);
    check_fused(d, kBackwardInput);
    check_bwdw(d);
    check_bwd(d);
    if (d.layout == WTCONV_NHWC) check_nhwc_map(d);
    std::printf("OK\n");
    return 0;
}
