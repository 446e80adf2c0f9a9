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

// Warp-specialised kernels: the analysis of a plane is shared by the
// producer warps; the replay of one warp's share visits only the work items
// of that warp (item t belongs to producer thread t mod np).
int g_share = -1, g_share_np = 1;
bool mine(long long idx) { return g_share < 0 || (int)((idx % g_share_np) / 32) == g_share; }

// Replays stage_plane: 16-byte chunk ch of this CTA's rows (strip `rank`) of
// the stored plane -> staging floats [stg + 4ch, stg + 4ch + 4).
// False while replaying an analysis whose plane copy the kernel skips (the
// weight gradient's dy when its tiles read the staging; COPY = false).
bool g_copy_plane = true;

int real_rows_host(const Plan& P, int rank) { return std::max(0, std::min(P.H, P.Hr - rank * P.H)); }

void replay_stage(Shadow& sh, const Plan& P, long long stg, int tag, int rank) {
    const long long strip_bytes = (long long)P.H * P.W * P.esize;
    const long long plane_bytes = (long long)P.Hr * P.Wr * P.esize;
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
            if (!mine((long long)i * (W / 4) + q)) continue;
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
        if (!mine(item)) continue;
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
            if (!mine((long long)i * m + j)) continue;
            const long long s0 = src + 2LL * i * ss + 2LL * j;
            sh.read(s0, slo, shi, stag, "haar src");
            sh.read(s0 + 1, slo, shi, stag, "haar src");
            sh.read(s0 + ss, slo, shi, stag, "haar src");
            sh.read(s0 + ss + 1, slo, shi, stag, "haar src");
        }
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < m; ++j)
            for (int s = 0; s < 4; ++s) {
                if (!mine((long long)i * m + j)) continue;
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

// Replays copy_halos for strip `rank`: every halo row of X and of every
// level's subbands is read from the CTA that owns the row (its own tag) and
// written into this CTA's padding rows.
void replay_halos(std::vector<Shadow>& shs, const Plan& P, int rank) {
    Shadow& me = shs[rank];
    auto one = [&](const Buf& b, int nsub_lg, int rows, int cols, FastDiv dcols, int tagbase, bool per_sub_tag) {
        const int pad = P.p;
        const int n = (2 * pad << nsub_lg) * cols;
        const long long span = (long long)(1 << nsub_lg) * (b.sub ? b.sub : 0);
        const long long lo = b.base, hi = nsub_lg ? b.base + span : b.base + (long long)(rows + 2 * pad) * b.stride;
        for (int t = 0; t < n; ++t) {
            const int rest = (int)fastdiv_host(t, dcols), c = t - rest * cols;
            if (rest != t / cols) me.fail("halo column division", t);
            const int hr = rest >> nsub_lg, s = rest - (hr << nsub_lg);
            const int i = hr < pad ? hr - pad : rows + hr - pad;
            const int g = rank * rows + i;
            if (g < 0 || g >= P.nstrips * rows) continue;
            const int owner = g / rows, lr = g - owner * rows;
            if (owner == rank) me.fail("halo row owned by the copying strip", g);
            const long long col = b.base + (long long)s * b.sub + c + pad;
            const int tag = per_sub_tag ? tagbase + s : tagbase;
            const long long slo = nsub_lg ? b.base + (long long)s * b.sub : lo;
            const long long shi = nsub_lg ? b.base + (long long)(s + 1) * b.sub : hi;
            shs[owner].read(col + (long long)(lr + pad) * b.stride, slo, shi, tag, "halo source");
            me.write(col + (long long)(i + pad) * b.stride, slo, shi, tag, "halo row");
        }
    };
    one(P.X, 0, P.H, P.W, P.div_w, XT, false);
    for (int l = 0; l < P.L; ++l) one(P.S[l], 2, P.H >> (l + 1), P.W >> (l + 1), P.div_m[l], s_tag(l, 0), true);
}

void barrier_all(std::vector<Shadow>& shs) {
    for (auto& sh : shs) sh.barrier();
}

void check_ws_all(const Plan& P, Kind kind);
void check_duo_all(const Plan& P, Kind kind);

void check_fused(const wtconv_desc_t& d, Kind kind) {
    Plan P;
    const wtconv_status_t st = make_plan(&d, kind, &P);
    if (st == WTCONV_OK && P.duo) {
        check_duo_all(P, kind);
        return;
    }
    if (st == WTCONV_OK && P.ws) {
        check_ws_all(P, kind);
        return;
    }
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
    std::vector<Shadow> shs(NS, Shadow(P.smem_floats));
    const long long all = P.smem_floats;
    if (P.grid < 1 || P.grid > (long long)P.B * P.C) shs[0].fail("grid", P.grid);
    const int xrows = P.ntr[kMaxL] * TR + 2 * p;
    const long long xlo = P.X.base, xhi = P.X.base + (long long)xrows * P.X.stride;
    const long long ylo = P.Y.base, yhi = P.Y.base + (long long)P.ntr[kMaxL] * TR * P.Y.stride;
    for (int cl = 0; cl < ncls; ++cl)
        if ((P.wbase + cl * P.wcls) % 4) shs[0].fail("weight class not 16-byte aligned", P.wbase + cl * P.wcls);
    const int ntc = P.ntc[kMaxL];
    const long long plane = (long long)P.Hr * P.Wr;

    // Phase A's synthesis of the previous plane: rows 2i, 2i+1 x columns 4q..4q+3.
    auto synthesis = [&](Shadow& sh, int rank) {
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
                    if (store) check_global((long long)(rank * H + 2 * i + rr) * P.Wr + 4 * q + e, plane, "y store");
                }
            }
        }
    };

    // The persistent walk over two planes and the final synthesis, with the
    // kernel's barriers (cluster-wide with strips) as phase boundaries:
    //   stage(0) | A(0) | B(0): stage(1), halos(0), | tiles(0) | A(1) | B(1) ... | A(end)
    for (int r = 0; r < NS; ++r) {
        shs[r].phase = "initial staging";
        replay_stage(shs[r], P, P.stg, XT + 10, r);
    }
    for (int unit = 0; unit <= 2; ++unit) {
        barrier_all(shs);
        for (int r = 0; r < NS; ++r) {
            Shadow& sh = shs[r];
            if (unit < 2) {
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
            for (int r = 0; r < NS; ++r) {
                shs[r].phase = "A: analysis";
                g_rank = r;
                const int e0 = shs[r].epoch;
                replay_analyse(shs[r], P, P.stg, XT + 10, P.X.base + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi,
                               XT, P.S, p, s_tag);
                if (r + 1 < NS) shs[r].epoch = e0;  // replay the next strip from the same phase
                else for (int q = 0; q + 1 < NS; ++q) shs[q].epoch = shs[r].epoch;
            }
        }
        if (unit > 0 && L >= 1)
            for (int r = 0; r < NS; ++r) {
                shs[r].phase = "A: synthesis";
                synthesis(shs[r], r);
            }
        if (unit == 2) break;
        barrier_all(shs);
        for (int r = 0; r < NS; ++r) {
            shs[r].phase = "B: staging";
            if (unit + 1 < 2) replay_stage(shs[r], P, P.stg, XT + 10, r);
        }
        if (NS > 1) {
            for (int r = 0; r < NS; ++r) {
                shs[r].phase = "B: halo copy";
                replay_halos(shs, P, r);
            }
            // Local barrier after the copy: a new phase for each CTA (the other
            // CTAs' phase is unchanged, so remote reads still conflict with
            // their later writes only through this CTA's epoch -- the replay
            // keeps the cluster in lockstep, which is the stricter check).
            barrier_all(shs);
        }
        for (int r = 0; r < NS; ++r) {
            Shadow& sh = shs[r];
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
    std::printf("fused(kind %d): smem %d B, threads %d, TR %d, tiles %d+%d, merged %d, strips %d\n", (int)kind,
                P.smem_floats * 4, P.nthreads, TR, P.n_sub_tiles, P.n_base_tiles, P.merged, NS);
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
    const int ncls = 1 + 4 * L, NS = P.nstrips;
    check_divs(P);
    check_div(P.div_w, W, (long long)(2 * p * 4) * W + 1, "W");
    std::vector<Shadow> shs(NS, Shadow(P.smem_floats));
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
    //   stage(0) | analysis(0) | stage(1), halos(0) | correlation(0) | analysis(1) | ... | reduction
    for (int r = 0; r < NS; ++r) {
        shs[r].phase = "initial staging";
        replay_stage(shs[r], P, P.stg, XT + 10, r);
        replay_stage(shs[r], P, P.stg + P.stg_floats, DYT + 10, r);
    }
    for (int plane = 0; plane < 2; ++plane) {
        barrier_all(shs);
        for (int r = 0; r < NS; ++r) {
            Shadow& sh = shs[r];
            sh.phase = "analysis";
            g_rank = r;
            const int e0 = sh.epoch;
            replay_analyse(sh, P, P.stg, XT + 10, P.X.base + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi, XT, P.S,
                           p, s_tag);
            g_copy_plane = !dys;
            replay_analyse(sh, P, P.stg + P.stg_floats, DYT + 10, P.DY.base, P.DY.stride, dlo, dhi, DYT, P.Q, 0, q_tag);
            g_copy_plane = true;
            if (r + 1 < NS) sh.epoch = e0;
            else for (int q = 0; q + 1 < NS; ++q) shs[q].epoch = sh.epoch;
        }
        barrier_all(shs);
        for (int r = 0; r < NS; ++r) {
            shs[r].phase = "staging";
            if (plane == 0) {
                replay_stage(shs[r], P, P.stg, XT + 10, r);
                if (!dys) replay_stage(shs[r], P, P.stg + P.stg_floats, DYT + 10, r);
            }
        }
        if (NS > 1) {
            for (int r = 0; r < NS; ++r) {
                shs[r].phase = "halo copy";
                replay_halos(shs, P, r);
            }
            barrier_all(shs);
        }
        for (int r = 0; r < NS; ++r) {
            Shadow& sh = shs[r];
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
    }
    const long long red_end = (long long)P.red + (long long)P.nthreads * KK + P.nthreads;
    barrier_all(shs);
    for (int r = 0; r < NS; ++r) {
        Shadow& sh = shs[r];
        sh.phase = "reduction";
        if (red_end > P.smem_floats) sh.fail("reduction scratch", red_end);
        for (int tid = 0; tid < P.nthreads; ++tid)
            for (int t = 0; t < KK; ++t) sh.write(P.red + (long long)tid * KK + t, P.red, red_end, RED, "class sums");
        for (int w = 0; w < P.nthreads / 32; ++w)
            sh.write(P.red + (long long)P.nthreads * KK + w, P.red, red_end, RED, "warp dy sums");
    }
    barrier_all(shs);
    for (int r = 0; r < NS; ++r)
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
    std::printf("bwdw: smem %d B, threads %d, TR %d, tiles %d (<= %d per thread), groups %d, strips %d%s\n",
                P.smem_floats * 4, P.nthreads, TR, P.n_all_tiles, P.tpt, P.groups, NS, dys ? ", dy read from staging" : "");
}

// Fused backward: dx conv tiles (the input-gradient pass: dy in X / S, dx
// in Q / Y) and correlation tiles (x windows in XS / SS against dy tiles at
// the interior of X / S) in one walk.
void check_bwd(const wtconv_desc_t& d) {
    Plan P;
    const wtconv_status_t st = make_plan(&d, kBackward, &P);
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
    std::printf("bwd: smem %d B, threads %d (%d conv + %d correlation), TR %d, groups %d\n", P.smem_floats * 4,
                P.nthreads, P.corr0, ncorr, TR, P.groups);
}



// ---------------------------------------------------------------------------
// Warp-specialised forward / input gradient (wtconv_ws.cuh).  Every role's
// sequence of mbarrier waits and arrivals is written out below exactly as
// the kernel executes it; a scheduler then runs the roles (and the landing
// of every bulk copy) in random orders, one action at a time, and
//   - fails if no role can move (deadlock) or a wait would see its barrier
//     two phases ahead (the parity test would then be wrong),
//   - replays every shared-memory access of each action with tags that carry
//     the plane (and, for the weights, the channel) they belong to, so a
//     buffer overwritten before its last reader, or read before its writer,
//     fails the tag check; and checks every output is stored exactly once.
// ---------------------------------------------------------------------------
int g_tag_off = 0;
int s_tag_ws(int l, int s) { return s_tag(l, s) + g_tag_off; }
int plane_off(int j) { return 1000 * (j + 1); }
int chan_off(int c) { return 1000 * (c + 1); }

struct MBar {
    int expected = 0, pending = 0, phase = 0;
    long long tx = 0;
    void init(int n) { expected = pending = n; phase = 0; tx = 0; }
    void maybe_complete() {
        if (pending == 0 && tx == 0) {
            ++phase;
            pending = expected;
        }
    }
    void arrive(int for_phase = -1) {
        if (pending <= 0) { std::printf("FAIL mbarrier arrival beyond its count\n"); std::exit(1); }
        if (for_phase >= 0 && for_phase != phase) {
            std::printf("FAIL ws: arrival meant for phase %d lands in phase %d\n", for_phase, phase);
            std::exit(1);
        }
        --pending;
        maybe_complete();
    }
};

enum WsOp { OP_WAIT, OP_ARRIVE, OP_ISSUE, OP_ANALYSE, OP_TILES };
struct Op {
    WsOp k;
    int bar, a, b;  // WAIT: bar, phase a | ARRIVE: bar, phase a | ISSUE: plane a | ANALYSE: plane a, warp b | TILES: step a, warp-tile b
};

// Host copy of ws_describe.
void ws_desc_host(const Plan& P, int t, int& win, int& out, int& wcl, int& level, int& r0, int& c0, bool& base) {
    const int TR = 8, TC = 4;
    if (t < P.n_sub_tiles) {
        int cl = 1;
        while (t >= P.sub_begin[cl]) ++cl;
        const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
        const int local = t - P.sub_begin[cl - 1];
        const int tr = local / P.ntc[l], tc = local - tr * P.ntc[l];
        win = P.S[l].base + s * P.S[l].sub + tr * TR * P.S[l].stride + tc * TC;
        out = P.Q[l].base + s * P.Q[l].sub + tr * TR * P.Q[l].stride + tc * TC;
        wcl = cl;
        level = l;
        r0 = tr;  // tile row / column of the subband
        c0 = tc;
        base = false;
    } else {
        const int bt = t - P.sub_pad;
        const int tr = bt / P.ntc[kMaxL], tc = bt - tr * P.ntc[kMaxL];
        win = P.X.base + tr * TR * P.X.stride + tc * TC;
        out = 0;
        wcl = 0;
        level = kMaxL;
        r0 = tr * TR;
        c0 = tc * TC;
        base = true;
    }
}

void check_ws(const Plan& P, int u0, int n, unsigned seed, bool verbose) {
    const int K = P.k, KK = K * K, p = P.p, L = P.L, H = P.H, W = P.W, ncls = 1 + 4 * L;
    const int NSTG = P.nstg, np = P.npw * 32, nsub = P.n_sub_tiles, ntiles = P.n_step_tiles, nwt = P.nwt;
    const int ncw = P.ncw, npw = P.npw;
    Shadow sh(P.smem_floats);
    sh.phase = "ws layout";
    if (P.TR != 8 || P.TC != 4 || P.padded || P.nstrips != 1) sh.fail("ws plan shape", P.TR);
    if (!(L == 0 || (P.pyr && L <= P.pyr_levels) || (!P.pyr && L == 1))) sh.fail("ws analysis is not one pass", L);
    if (P.nthreads != (ncw + npw + 1) * 32 || P.nthreads > kWsMaxThreads || NSTG < 2 || NSTG > kWsMaxStg || npw < 1 ||
        P.s_slots < 2 || P.s_slots > kWsMaxSSlots || P.x_slots != kWsQSlots)
        sh.fail("ws threads / staging slots", P.nthreads);
    if (nwt != (ntiles + 31) / 32 || P.sub_pad != (nsub + 31) / 32 * 32 || ntiles != P.sub_pad + P.n_base_tiles)
        sh.fail("ws tile counts", ntiles);
    if (P.smem_floats % 4 || P.smem_floats * 4LL > 227 * 1024) sh.fail("ws smem size", P.smem_floats);
    // Regions: disjoint, in bounds, aligned.
    struct R { long long lo, hi; const char* what; };
    std::vector<R> regs;
    regs.push_back({P.mbar, P.mbar + 2LL * kNumBars, "mbarriers"});
    regs.push_back({P.desc, P.desc + 4LL * ntiles, "tile descriptors"});
    for (int i = 0; i < P.x_slots; ++i)
        regs.push_back({P.wbase + (long long)i * P.w_slot, P.wbase + (long long)i * P.w_slot + ncls * P.wcls + 1, "weights"});
    for (int i = 0; i < NSTG; ++i)
        regs.push_back({P.stg + (long long)i * P.stg_floats, P.stg + (long long)(i + 1) * P.stg_floats, "staging"});
    const long long xsize = (long long)(P.ntr[kMaxL] * 8 + 2 * p) * P.X.stride;
    if (xsize > P.x_slot) sh.fail("X slot too small", P.x_slot);
    for (int i = 0; i < P.x_slots; ++i) regs.push_back({P.X.base + (long long)i * P.x_slot, P.X.base + (long long)i * P.x_slot + xsize, "X"});
    for (int l = 0; l < L; ++l) {
        for (int i = 0; i < P.s_slots; ++i)
            regs.push_back({P.S[l].base + (long long)i * P.s_slot, P.S[l].base + (long long)i * P.s_slot + 4LL * P.S[l].sub, "S"});
        for (int i = 0; i < kWsQSlots; ++i)
            regs.push_back({P.Q[l].base + (long long)i * P.q_slot, P.Q[l].base + (long long)i * P.q_slot + 4LL * P.Q[l].sub, "Q"});
    }
    for (size_t a = 0; a < regs.size(); ++a) {
        if (regs[a].lo < 0 || regs[a].hi > P.smem_floats) sh.fail(std::string(regs[a].what) + " outside shared memory", regs[a].lo);
        for (size_t b = a + 1; b < regs.size(); ++b)
            if (regs[a].lo < regs[b].hi && regs[b].lo < regs[a].hi)
                sh.fail(std::string(regs[a].what) + " overlaps " + regs[b].what, regs[a].lo);
    }
    if (P.mbar % 2 || P.desc % 4 || P.stg % 4 || P.stg_floats % 4 || P.wbase % 4 || P.w_slot % 4 || P.x_slot % 4 ||
        P.s_slot % 4 || P.q_slot % 4)
        sh.fail("ws alignment", 0);
    const long long plane_bytes = (long long)H * W * P.esize;
    if (plane_bytes % 16 || plane_bytes != 4LL * P.stg_floats || plane_bytes >= (1LL << 20))
        sh.fail("bulk copy size", plane_bytes);
    if (P.X.stride >= 4096) sh.fail("window stride field", P.X.stride);
    for (int l = 0; l < L; ++l)
        if (P.S[l].stride >= 4096 || P.Q[l].stride >= 4096) sh.fail("stride field", l);

    // Role programs.
    // Roles: producer warps [0, npw), the copy warp npw, conv warps after it.
    const int NS = P.s_slots, NX = P.x_slots, R = kWsBarRing;
    std::vector<std::vector<Op>> prog(npw + 1 + ncw);
    for (int pw = 0; pw < npw; ++pw) {
        auto& g = prog[pw];
        for (int j = 0; j < n; ++j) {
            g.push_back({OP_WAIT, kBarStgFull + j % NSTG, j / NSTG, 0});
            if (j >= NS && P.sub_pad > 0) g.push_back({OP_WAIT, kBarSub + (j - NS) % R, (j - NS) / R, 0});
            if (j >= NX) g.push_back({OP_WAIT, kBarBase + (j - NX) % 3, (j - NX) / 3, 0});
            g.push_back({OP_ANALYSE, 0, j, pw});
            g.push_back({OP_ARRIVE, kBarStgEmpty + j % NSTG, j / NSTG, 0});
            g.push_back({OP_ARRIVE, kBarAna + j % R, j / R, 0});
        }
    }
    {
        auto& g = prog[npw];
        for (int q = 0; q < n; ++q) {
            if (q >= NSTG) g.push_back({OP_WAIT, kBarStgEmpty + q % NSTG, (q - NSTG) / NSTG, 0});
            g.push_back({OP_ISSUE, 0, q, 0});
        }
        for (int q = std::max(0, n - NSTG); q < n; ++q) g.push_back({OP_WAIT, kBarStgFull + q % NSTG, q / NSTG, 0});
    }
    // Conv warps take tasks from a shared counter (see the kernel): their
    // programs are appended one task at a time when the role asks for work.
    const int nsub_pad = P.sub_pad, nsub_wt = nsub_pad / 32, nbase_wt = nwt - nsub_wt, per_step = nsub_wt + nbase_wt;
    const int ntasks = n * per_step;
    int next_task = 0;
    auto grab = [&](std::vector<Op>& g) {
        const int t = next_task++;
        int j, wt;
        if (t < nsub_wt) {
            j = 0;
            wt = t;
        } else {
            const int h = t - nsub_wt;
            j = 1 + h / per_step;
            wt = h - (j - 1) * per_step;
            if (j == n) wt += nsub_wt;
        }
        const bool is_sub = wt < nsub_wt;
        const int jj = is_sub ? j : j - 1;
        if (is_sub) {
            g.push_back({OP_WAIT, kBarAna + jj % R, jj / R, 0});
        } else if (nsub_wt > 0) {
            g.push_back({OP_WAIT, kBarSub + jj % R, jj / R, 0});
        } else {
            g.push_back({OP_WAIT, kBarAna + jj % R, jj / R, 0});
        }
        g.push_back({OP_TILES, 0, j, wt});
        g.push_back({OP_ARRIVE, is_sub ? kBarSub + jj % R : kBarBase + jj % 3, is_sub ? jj / R : jj / 3, 0});
    };

    MBar bars[kNumBars];
    for (int i = 0; i < NSTG; ++i) {
        bars[kBarStgFull + i].init(1);
        bars[kBarStgEmpty + i].init(npw);
    }
    for (int i = 0; i < kWsBarRing; ++i) {
        bars[kBarAna + i].init(npw);
        bars[kBarSub + i].init(nsub_wt > 0 ? nsub_wt : 1);
    }
    for (int i = 0; i < 3; ++i) bars[kBarBase + i].init(nbase_wt);

    std::vector<size_t> pc(prog.size(), 0);
    std::vector<int> landing;  // planes whose bulk copy is in flight
    const long long plane_elems = (long long)H * W;
    std::vector<std::vector<int>> stored(n, std::vector<int>(plane_elems, 0));
    const long long units = (long long)P.B * P.C;
    auto chan = [&](int j) { return (u0 + j) / P.B; };
    unsigned rng = seed * 2654435761u + 12345u;
    auto rnd = [&]() { rng = rng * 1664525u + 1013904223u; return rng >> 8; };

    // The hardware tests parity only: try_wait.parity(k & 1) passes whenever
    // the current phase's parity differs from k's.  So a wait is only
    // meaningful while the barrier is in phase k (blocks) or k + 1 (passes);
    // two phases ahead it would block for good, and one phase behind (the
    // phase before k still open) it would pass at once with k not complete.
    auto wait_ok = [&](const Op& o, int role) {
        const MBar& m = bars[o.bar];
        if (m.phase < o.a) {
            std::printf("FAIL ws: role %d (%s) waits on barrier %d for phase %d while phase %d is still open "
                        "(parity would pass it at once; seed %u)\n", role,
                        role < npw ? "producer" : role == npw ? "copy" : "conv", o.bar, o.a, m.phase, seed);
            std::exit(1);
        }
        if (m.phase > o.a + 1) {
            std::printf("FAIL ws: role %d (%s) wait on barrier %d for phase %d sees phase %d (two ahead; seed %u)\n", role,
                        role < npw ? "producer" : role == npw ? "copy" : "conv", o.bar, o.a, m.phase, seed);
            std::exit(1);
        }
        return ((m.phase ^ o.a) & 1) != 0;  // the hardware's test; equals m.phase == o.a + 1 here
    };
    auto land = [&](int j) {
        sh.barrier();
        sh.phase = "ws: bulk copy lands";
        const long long stg = P.stg + (long long)(j % NSTG) * P.stg_floats;
        const long long u = u0 + j;
        const long long b = u % P.B, c = u / P.B;
        check_global(((b * P.C + c) * plane_elems * P.esize + plane_bytes) - 1, units * plane_elems * P.esize,
                     "bulk copy source");
        for (long long f = 0; f < P.stg_floats; ++f) sh.write(stg + f, stg, stg + P.stg_floats, XT + 10 + plane_off(j), "staging");
        MBar& m = bars[kBarStgFull + j % NSTG];
        m.tx -= plane_bytes;
        if (m.tx < 0) sh.fail("bulk copy transaction count", m.tx);
        m.maybe_complete();
    };
    auto analyse = [&](int j, int pw, int seg) {
        sh.barrier();
        sh.phase = "ws: analysis share";
        g_share = pw;
        g_share_np = np;
        g_tag_off = plane_off(j);
        g_rank = 0;
        const long long stg = P.stg + (long long)(j % NSTG) * P.stg_floats;
        const long long xs = P.X.base + (long long)(j % P.x_slots) * P.x_slot;
        Buf sb[kMaxL];
        for (int l = 0; l < kMaxL; ++l) {
            sb[l] = P.S[l];
            sb[l].base += (j % P.s_slots) * P.s_slot;
        }
        const int stag = XT + 10 + plane_off(j), xt = XT + plane_off(j);
        const long long xlo = xs, xhi = xs + xsize;
        if (seg == 0) {
            const int c = chan(j);
            if (j < P.x_slots || c != chan(j - P.x_slots)) {
                const long long ws = P.wbase + (long long)(j % P.x_slots) * P.w_slot;
                for (int t = 0; t < ncls * KK; ++t) {
                    if (!mine(t)) continue;
                    const int cl = t / KK, tap = t - cl * KK;
                    sh.write(ws + (long long)cl * P.wcls + tap, ws, ws + ncls * P.wcls, WTS + chan_off(c), "ws weights");
                }
                if (pw == 0) sh.write(ws + P.bias, ws + P.bias, ws + P.bias + 1, BIAS + chan_off(c), "ws bias");
            }
            if (P.pyr) {
                replay_pyramid(sh, P, stg, stag, xs + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi, xt, sb, p, s_tag_ws);
            } else {
                const Buf& b0 = sb[0];
                replay_unpack(sh, P, stg, stag, xs + (long long)p * P.X.stride + p, P.X.stride, xlo, xhi, xt,
                              L >= 1 ? b0.base + (long long)p * b0.stride + p : 0, b0.stride, b0.sub, b0.base, s_tag_ws, L >= 1);
            }
        } else {
            const int done = P.pyr ? P.pyr_levels : (L >= 1 ? 1 : 0);
            const int l = done + seg - 1;
            const int nn = H >> (l + 1), m = W >> (l + 1);
            const Buf& s0 = sb[l - 1];
            const Buf& s1 = sb[l];
            replay_haar(sh, s0.base + (long long)p * s0.stride + p, s0.stride, s0.base, s0.base + s0.sub, s_tag_ws(l - 1, 0), nn,
                        m, s1.base + (long long)p * s1.stride + p, s1.stride, s1.sub, s1.base, s1.base + 4LL * s1.sub, s_tag_ws,
                        l);
        }
        g_share = -1;
    };
    auto tiles = [&](int j, int wt) {
        sh.barrier();
        for (int lane = 0; lane < 32; ++lane) {
            const int t = 32 * wt + lane;
            if (t >= ntiles) continue;
            if (t >= nsub && t < P.sub_pad) continue;  // padding
            int win, out, wcl, level, r0, c0;
            bool base;
            ws_desc_host(P, t, win, out, wcl, level, r0, c0, base);
            if (base ? j < 1 : j >= n) continue;
            const int jj = base ? j - 1 : j;
            const int c = chan(jj);
            const long long ws = P.wbase + (long long)(jj % P.x_slots) * P.w_slot;
            sh.phase = base ? "ws: base tile" : "ws: sub tile";
            if ((ws + (long long)wcl * P.wcls) % 4) sh.fail("weight class alignment", ws);
            for (int q = 0; q < KK; ++q)
                sh.read(ws + (long long)wcl * P.wcls + q, ws, ws + ncls * P.wcls, WTS + chan_off(c), "ws weights read");
            if (base) {
                sh.read(ws + P.bias, ws + P.bias, ws + P.bias + 1, BIAS + chan_off(c), "ws bias read");
                const long long xs = P.X.base + (long long)(jj % P.x_slots) * P.x_slot;
                if (win != P.X.base + (r0 / 8) * 8 * P.X.stride + c0) sh.fail("base descriptor", t);
                replay_window(sh, P, xs, P.X.stride, xs, xs + xsize, H, W, r0 / 8, c0 / 4, XT + plane_off(jj), "ws base window", 0);
                // Synthesis epilogue reads (synth_tile).
                const long long qs = (long long)(jj % kWsQSlots) * P.q_slot;
                auto qread = [&](int l, int s2, int pr, int pc, bool need) {
                    const Buf& Q = P.Q[l];
                    const long long lo = qs + Q.base + (long long)s2 * Q.sub, hi = lo + Q.sub;
                    const long long a = lo + (long long)pr * Q.stride + pc;
                    if (need) {
                        if (pr >= (H >> (l + 1)) || pc >= (W >> (l + 1))) sh.fail("synthesis position outside the subband", l);
                        sh.read(a, lo, hi, q_tag(l, s2) + plane_off(jj), "ws synthesis Q read");
                    } else {
                        sh.touch(a, lo, hi, "ws synthesis Q read (unused)");
                    }
                };
                // A level-l position (pr, pc) feeds outputs of rows
                // [pr << (l+1), (pr+1) << (l+1)); it is needed when one of them
                // lies in this tile and in the plane.
                auto need = [&](int l, int pr) {
                    const int lo = std::max(pr << (l + 1), r0), hi = std::min((pr + 1) << (l + 1), std::min(r0 + 8, H));
                    return lo < hi;
                };
                for (int l = kMaxL - 1; l >= 3; --l) {
                    if (l >= L) continue;
                    const int pr = r0 >> (l + 1), pcc = c0 >> (l + 1);
                    for (int s2 = 0; s2 < 4; ++s2) qread(l, s2, pr, pcc, need(l, pr));
                }
                if (L >= 3)
                    for (int s2 = 0; s2 < 4; ++s2) qread(2, s2, r0 >> 3, c0 >> 3, need(2, r0 >> 3));
                if (L >= 2)
                    for (int ah = 0; ah < 2; ++ah)
                        for (int s2 = 0; s2 < 4; ++s2) qread(1, s2, (r0 >> 2) + ah, c0 >> 2, need(1, (r0 >> 2) + ah));
                if (L >= 1)
                    for (int a = 0; a < 4; ++a)
                        for (int s2 = 0; s2 < 4; ++s2) {
                            const long long addr = qs + P.Q[0].base + (long long)s2 * P.Q[0].sub +
                                                   (long long)((r0 >> 1) + a) * P.Q[0].stride + (c0 >> 1);
                            if (addr % 2) sh.fail("level-0 pair load not 8-byte aligned", addr);
                            for (int e = 0; e < 2; ++e) qread(0, s2, (r0 >> 1) + a, (c0 >> 1) + e, need(0, (r0 >> 1) + a));
                        }
                for (int o = 0; o < 8; ++o) {
                    if (r0 + o >= H) continue;
                    if (c0 + 4 > W) sh.fail("base tile column", c0);
                    for (int e = 0; e < 4; ++e) ++stored[jj][(long long)(r0 + o) * W + c0 + e];
                }
            } else {
                const int s2 = (wcl - 1) & 3;
                const Buf& S = P.S[level];
                const Buf& Q = P.Q[level];
                const long long ss = (long long)(jj % P.s_slots) * P.s_slot, qq = (long long)(jj % kWsQSlots) * P.q_slot;
                const long long slo = ss + S.base + (long long)s2 * S.sub;
                replay_window(sh, P, slo, S.stride, slo, slo + S.sub, H >> (level + 1), W >> (level + 1), r0, c0,
                              s_tag(level, s2) + plane_off(jj), "ws subband window", 0);
                const long long o0 = qq + out;
                if (o0 % 4) sh.fail("Q tile not 16-byte aligned", o0);
                const long long qlo = qq + Q.base + (long long)s2 * Q.sub;
                for (int o = 0; o < 8; ++o)
                    for (int e = 0; e < 4; ++e)
                        sh.write(o0 + (long long)o * Q.stride + e, qlo, qlo + Q.sub, q_tag(level, s2) + plane_off(jj), "ws Q tile");
            }
        }
    };

    const int nroles = (int)prog.size();
    long long steps = 0;
    // seed 0: producers first where possible; 1: conv warps first; others random.
    auto runnable = [&](int r) -> bool {
        if (pc[r] >= prog[r].size()) return r > npw && next_task < ntasks;  // a conv warp can take a task
        const Op& o = prog[r][pc[r]];
        if (o.k == OP_WAIT) return wait_ok(o, r);
        return true;
    };
    for (;;) {
        std::vector<int> ready;
        for (int r = 0; r < nroles; ++r)
            if (runnable(r)) ready.push_back(r);
        const bool all_done = [&] {
            for (int r = 0; r < nroles; ++r)
                if (pc[r] < prog[r].size()) return false;
            return next_task >= ntasks;
        }();
        if (all_done && landing.empty()) break;
        if (ready.empty() && landing.empty()) {
            std::printf("FAIL ws: deadlock after %lld actions (seed %u); next ops:", steps, seed);
            for (int r = 0; r < nroles; ++r)
                if (pc[r] < prog[r].size())
                    std::printf(" [role %d op %d bar %d a %d]", r, (int)prog[r][pc[r]].k, prog[r][pc[r]].bar, prog[r][pc[r]].a);
            std::printf("\n");
            std::exit(1);
        }
        ++steps;
        // Choose: a landing or a role.
        const size_t nchoice = ready.size() + landing.size();
        size_t pick;
        if (seed == 0) pick = !ready.empty() ? 0 : ready.size();          // lowest role first (producers)
        else if (seed == 1) pick = !ready.empty() ? ready.size() - 1 : ready.size();  // conv warps first
        else pick = rnd() % nchoice;
        if (pick >= ready.size()) {
            const size_t li = pick - ready.size();
            const int j = landing[li];
            landing.erase(landing.begin() + li);
            land(j);
            continue;
        }
        const int r = ready[pick];
        if (pc[r] >= prog[r].size()) {  // a conv warp takes the next task
            grab(prog[r]);
            continue;
        }
        const Op o = prog[r][pc[r]];
        switch (o.k) {
            case OP_WAIT: ++pc[r]; break;
            case OP_ARRIVE: bars[o.bar].arrive(o.a); ++pc[r]; break;
            case OP_ISSUE: {
                MBar& m = bars[kBarStgFull + o.a % NSTG];
                m.tx += plane_bytes;  // arrive.expect_tx: expect, then arrive
                m.arrive();
                landing.push_back(o.a);
                ++pc[r];
                break;
            }
            case OP_ANALYSE: analyse(o.a, o.b, 0); ++pc[r]; break;
            case OP_TILES: tiles(o.a, o.b); ++pc[r]; break;
        }
    }
    for (int j = 0; j < n; ++j)
        for (long long e = 0; e < plane_elems; ++e)
            if (stored[j][e] != 1) {
                std::printf("FAIL ws: plane %d output %lld stored %d times\n", j, e, stored[j][e]);
                std::exit(1);
            }
    for (int i = 0; i < kNumBars; ++i)
        if (bars[i].expected && bars[i].pending != bars[i].expected) {
            std::printf("FAIL ws: barrier %d left with %d of %d arrivals pending\n", i, bars[i].pending, bars[i].expected);
            std::exit(1);
        }
    if (verbose)
        std::printf("ws: smem %d B, threads %d (%d conv + %d producer warps + 1 copy warp), rings stg %d X %d S %d, tiles %d+%d, planes %d from %d\n",
                    P.smem_floats * 4, P.nthreads, ncw, npw, NSTG, P.x_slots, P.s_slots, nsub, P.n_base_tiles, n, u0);
}

void check_ws_all(const Plan& P, Kind kind) {
    const long long units = (long long)P.B * P.C;
    const int n = (int)std::min<long long>(units, 9);
    // From the first unit, and across a channel boundary.
    const int u_alt = (int)std::min<long long>(std::max(0, P.B - 4), units - n);
    for (unsigned seed = 0; seed < 40; ++seed) check_ws(P, seed % 2 ? u_alt : 0, n, seed, seed == 0);
    // A short run (fewer planes than staging slots) and a single plane.
    check_ws(P, 0, std::min(n, 2), 3, false);
    check_ws(P, 0, 1, 4, false);
    std::printf("fused(kind %d): warp-specialised\n", (int)kind);
}

// ---------------------------------------------------------------------------
// Two alternating warp groups (wtconv_duo.cuh): the kernel's half-cycle
// schedule replayed with its barriers as phase boundaries (a CTA barrier
// ends every half-cycle; inside A the group barrier splits the analysis from
// the staging of the next plane), every access checked against tags that
// carry the plane (and, for the weights, the channel).
// ---------------------------------------------------------------------------
void check_duo(const Plan& P, int u0, int n) {
    const int K = P.k, KK = K * K, p = P.p, L = P.L, H = P.H, W = P.W, ncls = 1 + 4 * L;
    const int nsub = P.n_sub_tiles, ntiles = P.n_step_tiles;
    Shadow sh(P.smem_floats);
    sh.phase = "duo layout";
    if (P.TR != 8 || P.TC != 4 || P.padded || P.nstrips != 1 || P.nthreads != kDuoThreads || P.sub_pad != nsub ||
        ntiles != nsub + P.n_base_tiles)
        sh.fail("duo plan", P.nthreads);
    if (P.smem_floats % 4 || P.smem_floats * 4LL > 227 * 1024 || P.gbase % 4 || P.gsize % 4) sh.fail("duo smem", 0);
    if (P.gbase < 4LL * ntiles || P.gbase + 2LL * P.gsize > P.smem_floats) sh.fail("duo groups", P.gbase);
    const long long xsize = (long long)(P.ntr[kMaxL] * 8 + 2 * p) * P.X.stride;
    struct R { long long lo, hi; const char* what; };
    std::vector<R> regs;
    for (int i = 0; i < 2; ++i) {
        regs.push_back({P.wbase + (long long)i * P.w_slot, P.wbase + (long long)i * P.w_slot + ncls * P.wcls + 1, "weights"});
        regs.push_back({P.X.base + (long long)i * P.x_slot, P.X.base + (long long)i * P.x_slot + xsize, "X"});
        for (int l = 0; l < L; ++l)
            regs.push_back({P.Q[l].base + (long long)i * P.q_slot, P.Q[l].base + (long long)i * P.q_slot + 4LL * P.Q[l].sub, "Q"});
    }
    regs.push_back({P.stg, P.stg + (long long)P.stg_floats, "staging"});
    for (int l = 0; l < L; ++l) regs.push_back({P.S[l].base, P.S[l].base + 4LL * P.S[l].sub, "S"});
    for (size_t a = 0; a < regs.size(); ++a) {
        if (regs[a].lo < 0 || regs[a].hi > P.gsize) sh.fail(std::string(regs[a].what) + " outside its group", regs[a].lo);
        for (size_t b = a + 1; b < regs.size(); ++b)
            if (regs[a].lo < regs[b].hi && regs[b].lo < regs[a].hi)
                sh.fail(std::string(regs[a].what) + " overlaps " + regs[b].what, regs[a].lo);
    }
    if (P.stg % 4 || P.w_slot % 4 || P.x_slot % 4 || P.q_slot % 4 || (P.gbase + P.stg) % 4 || (P.gbase + P.gsize) % 4)
        sh.fail("duo alignment", 0);
    const long long plane_elems = (long long)H * W, units = (long long)P.B * P.C;
    std::vector<std::vector<int>> stored(n, std::vector<int>(plane_elems, 0));
    auto chan = [&](int j) { return (u0 + j) / P.B; };
    // Local plane j of group g = g + 2k.
    auto stage = [&](int g, int k) {
        const long long gb = P.gbase + (long long)g * P.gsize;
        const int j = g + 2 * k;
        const long long u = u0 + j;
        check_global(((u % P.B) * P.C + u / P.B) * plane_elems * P.esize + (long long)P.plane_chunks * 16 - 1,
                     units * plane_elems * P.esize, "staging source");
        for (long long f = 0; f < P.stg_floats; ++f)
            sh.write(gb + P.stg + f, gb + P.stg, gb + P.stg + P.stg_floats, XT + 10 + plane_off(j), "duo staging");
    };
    auto analyse = [&](int g, int k) {
        const long long gb = P.gbase + (long long)g * P.gsize;
        const int j = g + 2 * k;
        g_share = -1;
        g_tag_off = plane_off(j);
        g_rank = 0;
        const int c = chan(j);
        const long long ws = gb + P.wbase + (long long)(k & 1) * P.w_slot;
        if (k < 2 || c != chan(j - 4)) {
            for (int t = 0; t < ncls * KK; ++t) {
                const int cl = t / KK, tap = t - cl * KK;
                sh.write(ws + (long long)cl * P.wcls + tap, ws, ws + ncls * P.wcls, WTS + chan_off(c), "duo weights");
            }
            sh.write(ws + P.bias, ws + P.bias, ws + P.bias + 1, BIAS + chan_off(c), "duo bias");
        }
        Buf sb[kMaxL];
        for (int l = 0; l < kMaxL; ++l) {
            sb[l] = P.S[l];
            sb[l].base += gb;
        }
        const long long xs = gb + P.X.base + (long long)(k & 1) * P.x_slot;
        replay_analyse(sh, P, gb + P.stg, XT + 10 + plane_off(j), xs + (long long)p * P.X.stride + p, P.X.stride, xs,
                       xs + xsize, XT + plane_off(j), sb, p, s_tag_ws);
    };
    auto tiles = [&](int g, int k, int m) {
        const long long gb = P.gbase + (long long)g * P.gsize;
        for (int t = 0; t < ntiles; ++t) {
            const bool base = t >= nsub;
            if (base ? k < 1 : k >= m) continue;
            const int kk = base ? k - 1 : k, j = g + 2 * kk;
            int win, out, wcl, level, r0, c0;
            bool b2;
            ws_desc_host(P, t, win, out, wcl, level, r0, c0, b2);
            const long long ws = gb + P.wbase + (long long)(kk & 1) * P.w_slot;
            sh.phase = base ? "duo: base tile" : "duo: sub tile";
            for (int q = 0; q < KK; ++q)
                sh.read(ws + (long long)wcl * P.wcls + q, ws, ws + ncls * P.wcls, WTS + chan_off(chan(j)), "duo weights read");
            if (base) {
                sh.read(ws + P.bias, ws + P.bias, ws + P.bias + 1, BIAS + chan_off(chan(j)), "duo bias read");
                const long long xs = gb + P.X.base + (long long)(kk & 1) * P.x_slot;
                replay_window(sh, P, xs, P.X.stride, xs, xs + xsize, H, W, r0 / 8, c0 / 4, XT + plane_off(j), "duo base window", 0);
                const long long qs = gb + (long long)(kk & 1) * P.q_slot;
                auto need = [&](int l, int pr) {
                    const int lo = std::max(pr << (l + 1), r0), hi = std::min((pr + 1) << (l + 1), std::min(r0 + 8, H));
                    return lo < hi;
                };
                auto qread = [&](int l, int s2, int pr, int pc, bool nd) {
                    const Buf& Q = P.Q[l];
                    const long long lo = qs + Q.base + (long long)s2 * Q.sub, hi = lo + Q.sub;
                    const long long a = lo + (long long)pr * Q.stride + pc;
                    if (nd) sh.read(a, lo, hi, q_tag(l, s2) + plane_off(j), "duo synthesis Q read");
                    else sh.touch(a, lo, hi, "duo synthesis Q read (unused)");
                };
                for (int l = kMaxL - 1; l >= 3; --l) {
                    if (l >= L) continue;
                    for (int s2 = 0; s2 < 4; ++s2) qread(l, s2, r0 >> (l + 1), c0 >> (l + 1), need(l, r0 >> (l + 1)));
                }
                if (L >= 3)
                    for (int s2 = 0; s2 < 4; ++s2) qread(2, s2, r0 >> 3, c0 >> 3, need(2, r0 >> 3));
                if (L >= 2)
                    for (int ah = 0; ah < 2; ++ah)
                        for (int s2 = 0; s2 < 4; ++s2) qread(1, s2, (r0 >> 2) + ah, c0 >> 2, need(1, (r0 >> 2) + ah));
                if (L >= 1)
                    for (int a = 0; a < 4; ++a)
                        for (int s2 = 0; s2 < 4; ++s2)
                            for (int e = 0; e < 2; ++e) qread(0, s2, (r0 >> 1) + a, (c0 >> 1) + e, need(0, (r0 >> 1) + a));
                for (int o = 0; o < 8; ++o) {
                    if (r0 + o >= H) continue;
                    for (int e = 0; e < 4; ++e) ++stored[j][(long long)(r0 + o) * W + c0 + e];
                }
            } else {
                const int s2 = (wcl - 1) & 3;
                const Buf& S = P.S[level];
                const Buf& Q = P.Q[level];
                const long long slo = gb + S.base + (long long)s2 * S.sub;
                replay_window(sh, P, slo, S.stride, slo, slo + S.sub, H >> (level + 1), W >> (level + 1), r0, c0,
                              s_tag(level, s2) + plane_off(j), "duo subband window", 0);
                const long long qq = gb + (long long)(kk & 1) * P.q_slot;
                const long long qlo = qq + Q.base + (long long)s2 * Q.sub;
                for (int o = 0; o < 8; ++o)
                    for (int e = 0; e < 4; ++e)
                        sh.write(qq + out + (long long)o * Q.stride + e, qlo, qlo + Q.sub, q_tag(level, s2) + plane_off(j), "duo Q tile");
            }
        }
    };
    const int mg[2] = {(n + 1) / 2, n / 2};
    for (int g = 0; g < 2; ++g)
        if (mg[g] > 0) stage(g, 0);
    const int Hh = std::max(2 * mg[0] + 2, 2 * mg[1] + 3);
    for (int h = 0; h < Hh; ++h) {
        sh.barrier();
        int a_grp = -1, a_k = -1;
        for (int g = 0; g < 2; ++g) {
            const bool runs_a = ((h + g) & 1) == 0;
            if (runs_a) {
                const int k = (h - g) >> 1;
                if (k >= 0 && k < mg[g]) {
                    sh.phase = "duo: analysis";
                    analyse(g, k);
                    a_grp = g;
                    a_k = k;
                }
            } else {
                const int k = (h - 1 - g) >> 1;
                if (k >= 0 && k <= mg[g]) tiles(g, k, mg[g]);
            }
        }
        if (a_grp >= 0 && a_k + 1 < mg[a_grp]) {
            sh.barrier();  // the group barrier after the analysis
            sh.phase = "duo: staging";
            stage(a_grp, a_k + 1);
        }
    }
    for (int j = 0; j < n; ++j)
        for (long long e = 0; e < plane_elems; ++e)
            if (stored[j][e] != 1) {
                std::printf("FAIL duo: plane %d output %lld stored %d times\n", j, e, stored[j][e]);
                std::exit(1);
            }
}

void check_duo_all(const Plan& P, Kind kind) {
    const long long units = (long long)P.B * P.C;
    const int n = (int)std::min<long long>(units, 9);
    const int u_alt = (int)std::min<long long>(std::max(0, P.B - 4), units - n);
    check_duo(P, 0, n);
    check_duo(P, u_alt, n);
    check_duo(P, 0, std::min(n, 2));
    check_duo(P, 0, 1);
    std::printf("fused(kind %d): two alternating warp groups, smem %d B\n", (int)kind, P.smem_floats * 4);
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
    check_bwd(d);
    std::printf("OK\n");
    return 0;
}
