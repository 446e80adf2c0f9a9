// Host-side argument validation and on-chip planning for the WTConv kernels.
// Plain C++ (no CUDA types), so that the planner can also be compiled by a
// host compiler to check every shared-memory access the kernels make.
#pragma once

#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "../../include/wtconv.h"
#include "wtconv_plan.h"

namespace wtc {

constexpr int kSmemLimitFloats = 227 * 1024 / 4;
constexpr int kSmemPerSM = 228 * 1024;
// SMs of a B200: the SM count planned for when no CUDA device can be
// queried (host-only planning; nothing can launch then).
constexpr int kB200SMs = 148;

// kBackward: the fused backward (dx and the weight-gradient partials in one
// pass over x and dy).
enum Kind { kForward = 0, kBackwardInput = 1, kBackwardWeight = 2, kBackward = 3 };

inline int round4(int v) { return (v + 3) & ~3; }
inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Row stride (floats, multiple of 4) of a buffer read by tiles laid out
// ntc per tile row.  Consecutive lanes walk the tile columns and wrap to the
// next tile row (TR rows down), so TR * stride/4 == ntc (mod 8) puts each
// quarter-warp's 16-byte accesses on 8 distinct bank groups.
inline int pick_stride(int min_floats, int TR, int ntc) {
    const int s = round4(min_floats);
    for (int t = 0; t < 8; ++t) {
        const int c = s + 4 * t;
        if ((((TR * (c / 4) - ntc) % 8) + 8) % 8 == 0) return c;
    }
    return s;
}

// Conv tiles of height TR (4 columns wide) over the base plane and every subband.
inline int count_tiles(const wtconv_desc_t* d, int TR) {
    int n = ceil_div(d->H, TR) * ceil_div(d->W, 4);
    for (int l = 0; l < d->L; ++l) n += 4 * ceil_div(d->H >> (l + 1), TR) * ceil_div(d->W >> (l + 1), 4);
    return n;
}

// Threads of a CTA for `tiles` conv tiles: a multiple of 4 warps (one warp
// per SM sub-partition each) once there are more than 128 tiles, so no
// sub-partition carries an extra warp of tiles; at most max_threads.
inline int tile_threads(int tiles, int max_threads) {
    const int t = tiles <= 128 ? std::max(64, ceil_div(tiles, 32) * 32) : ceil_div(tiles, 128) * 128;
    return std::min(t, max_threads);
}

// CTAs per SM that the shared memory of one CTA allows (the register
// budget of the launch bounds allows two).
inline int ctas_per_sm(int smem_floats) {
    return std::max(1, std::min(2, kSmemPerSM / (smem_floats * 4 + 1024)));
}

// CTAs of `nthreads` threads one SM holds: the least of what its shared
// memory, its 64K registers at the kernels' register cap (every launch bound
// allows at most 128 registers a thread) and its 64 warps allow.
inline int resident_ctas(int nthreads, int smem_floats) {
    const int by_smem = kSmemPerSM / (smem_floats * 4 + 1024);
    const int by_regs = 65536 / (std::max(nthreads, 32) * 128);
    const int by_warps = 64 / std::max(ceil_div(nthreads, 32), 1);
    return std::max(1, std::min(std::min(by_smem, by_regs), std::min(by_warps, 32)));
}

// Weight-gradient batch groups (grid.y): the CTA of group g walks planes
// b = g, g + groups, ...  Chosen to minimise waves x planes-per-CTA over the
// resident CTA slots, with at most 64 planes per CTA so every per-thread
// running sum stays short.
inline int pick_groups(int B, int C, long long slots) {
    int best = 1;
    long long best_cost = -1;
    for (int g = 1; g <= B; ++g) {
        const int planes = ceil_div(B, g);
        if (planes > 64 && g != B) continue;
        const long long waves = (C * (long long)g + slots - 1) / slots;
        const long long cost = waves * (planes + 1);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = g;
        }
    }
    return best;
}

inline bool is_supported_k(int k) { return k == 1 || k == 3 || k == 5 || k == 7; }

inline wtconv_status_t validate(const wtconv_desc_t* d) {
    if (!d) return WTCONV_ERR_NULLPTR;
    if (d->dtype != WTCONV_F32 && d->dtype != WTCONV_BF16) return WTCONV_ERR_DTYPE;
    if (d->B <= 0 || d->C <= 0 || d->H <= 0 || d->W <= 0) return WTCONV_ERR_BAD_SHAPE;
    if (!is_supported_k(d->k)) return WTCONV_ERR_BAD_K;
    if (d->L < 0 || d->L > kMaxL) return WTCONV_ERR_BAD_L;
    if (d->layout != WTCONV_NCHW && d->layout != WTCONV_NHWC) return WTCONV_ERR_LAYOUT;
    if ((d->W % 4) != 0) return WTCONV_ERR_BAD_SHAPE;
    // NCHW planes are staged in 16-byte chunks: whole planes if H and W are
    // multiples of 2^L, else (zero-padded on chip) row by row.  NHWC planes
    // are gathered element by element.
    const long long esize = d->dtype == WTCONV_BF16 ? 2 : 4;
    const bool padded = (d->H % (1 << d->L)) != 0 || (d->W % (1 << d->L)) != 0;
    if (d->layout == WTCONV_NCHW &&
        (padded ? ((long long)d->W * esize) % 16 != 0 : ((long long)d->H * d->W * esize) % 16 != 0))
        return WTCONV_ERR_BAD_SHAPE;
    // Index arithmetic in the kernels is 32-bit within a plane and 64-bit across planes.
    if ((long long)d->H * d->W > (1LL << 30)) return WTCONV_ERR_BAD_SHAPE;
    if ((long long)d->B * d->C > (1LL << 31) - 1) return WTCONV_ERR_BAD_SHAPE;
    return WTCONV_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The plan for tile height TR with every plane split into `nstrips`
// horizontal strips of H / nstrips rows (one CTA of a thread-block cluster
// per strip; 1 = whole planes, no cluster).  Every field that describes
// on-chip rows (H, ntr, buffers, tiles) describes one strip.
// dy_stg (weight gradient on strips of fp32 planes whose height is whole
// tiles): no DY buffer; the correlation tiles read dy from its staging.
// num_sms (the device's SM count) sizes the persistent forward grid and the
// weight gradient's batch groups.
inline wtconv_status_t make_plan_for(const wtconv_desc_t* d, Kind kind, int TR, int nstrips, int num_sms, Plan* P,
                                     bool dy_stg = false, bool octets = true) {
    memset(P, 0, sizeof(*P));
    if (num_sms < 1) return WTCONV_ERR_UNSUPPORTED;
    // The plane the CTAs hold: H and W rounded up to multiples of 2^L.
    const int m = 1 << d->L;
    const int Hv = (d->H + m - 1) / m * m, Wv = (d->W + m - 1) / m * m;
    if (nstrips < 1 || nstrips > kMaxStrips || Hv % nstrips) return WTCONV_ERR_UNSUPPORTED;
    if (kind == kBackward && nstrips != 1) return WTCONV_ERR_UNSUPPORTED;  // whole planes only
    if (dy_stg && (kind != kBackwardWeight || nstrips == 1 || d->dtype != WTCONV_F32 || Hv != d->H || Wv != d->W))
        return WTCONV_ERR_UNSUPPORTED;
    const int Hs = Hv / nstrips;
    if (nstrips > 1 && (Hs % m != 0 || Hs % 4 != 0)) return WTCONV_ERR_UNSUPPORTED;
    P->B = d->B; P->C = d->C; P->H = Hs; P->W = Wv; P->k = d->k; P->L = d->L;
    P->Hp = Hv;
    P->Hr = d->H;
    P->Wr = d->W;
    P->padded = (Hv != d->H || Wv != d->W) ? 1 : 0;
    P->nstrips = nstrips;
    P->nhwc = d->layout == WTCONV_NHWC ? 1 : 0;
    P->div_wr = make_fastdiv(P->Wr);
    const int p = d->k / 2, k = d->k, L = d->L, H = Hs, W = Wv, KK = k * k;
    P->p = p;
    P->esize = d->dtype == WTCONV_BF16 ? 2 : 4;
    P->TC = 4;
    P->TR = TR;
    const int TC = P->TC;
    const int WV4 = 4 * ((TC + k - 1 + 3) / 4);  // floats read per window row

    P->ntr[kMaxL] = ceil_div(H, TR);
    P->ntc[kMaxL] = ceil_div(W, TC);
    for (int l = 0; l < L; ++l) {
        P->ntr[l] = ceil_div(H >> (l + 1), TR);
        P->ntc[l] = ceil_div(W >> (l + 1), TC);
    }

    long long off = 0;
    const int ncls = 1 + 4 * L;
    if (kind != kBackwardWeight) {
        P->wcls = round4(KK);  // each class 16-byte aligned
        P->wbase = (int)off;
        off += (long long)ncls * P->wcls;
        P->bias = (int)off;
        off += 4;
    }
    // Padded input plane and padded subbands of every level (the fused
    // backward holds two sets: dy in X / S, x in XS / SS).
    auto padded = [&](Buf& X, Buf* S) {
        {
            const int ntc = P->ntc[kMaxL];
            const int rows = P->ntr[kMaxL] * TR + 2 * p;
            const int need = std::max(W + 2 * p, (ntc - 1) * TC + WV4);
            X.stride = pick_stride(need, TR, ntc);
            X.base = (int)off;
            off += round4(rows * X.stride);
        }
        for (int l = 0; l < L; ++l) {
            const int m = W >> (l + 1);
            const int ntc = P->ntc[l];
            const int rows = P->ntr[l] * TR + 2 * p;
            const int need = std::max(m + 2 * p, (ntc - 1) * TC + WV4);
            S[l].stride = pick_stride(need, TR, ntc);
            S[l].sub = round4(rows * S[l].stride);
            S[l].base = (int)off;
            off += 4LL * S[l].sub;
        }
    };
    padded(P->X, P->S);
    if (kind == kBackward) padded(P->XS, P->SS);
    // Tile-rounded, unpadded planes: conv outputs (forward) or dy subbands.
    for (int l = 0; l < L; ++l) {
        const int rows = P->ntr[l] * TR;
        P->Q[l].stride = round4(P->ntc[l] * TC);
        P->Q[l].sub = round4(rows * P->Q[l].stride);
        P->Q[l].base = (int)off;
        off += 4LL * P->Q[l].sub;
    }
    if (kind != kBackwardWeight && L >= 1) {
        // Written by base tiles (lanes walk tile columns, like the windows).
        const int ntc = P->ntc[kMaxL];
        P->Y.stride = pick_stride(ntc * TC, TR, ntc);
        P->Y.base = (int)off;
        off += round4(P->ntr[kMaxL] * TR * P->Y.stride);
    }
    if (kind == kBackwardWeight && !dy_stg) {
        const int rows = P->ntr[kMaxL] * TR;
        P->DY.stride = round4(P->ntc[kMaxL] * TC);
        P->DY.base = (int)off;
        off += round4(rows * P->DY.stride);
    }
    // Staging of the next plane(s), stored format (W elements per row).
    {
        const long long bytes = (long long)H * W * P->esize;
        P->plane_chunks = (int)(bytes / 16);
        P->stg_floats = (int)(bytes / 4);
        P->row_chunks = (int)((long long)P->Wr * P->esize / 16);
        P->div_rowc = make_fastdiv(std::max(P->row_chunks, 1));
        P->stg = (int)off;
        off += (kind == kBackwardWeight || kind == kBackward ? 2LL : 1LL) * P->stg_floats;
    }
    // NHWC channel octets: a pixel's 8 channels are one 16- or 32-byte run,
    // loaded once for the cluster's 8 planes instead of element by element
    // per plane.  Whole, unpadded planes whose pixels split into 8 runs of an
    // even number of pixels (moved 4 at a time, or 2 where the run is not a
    // multiple of 4: 28 x 28 planes, 98 pixels a run).
    // The weight gradient's x and dy runs take the octet buffer in turn; the
    // fused backward holds both (x run at tbuf, dy run after it).
    // The fused backward only with 4 pixels a step (28 x 28 planes, 2 a
    // step, measured 149.5 -> 191.5 us against its gather).
    long long oct_floats = 0;  // shared memory of the octet buffers
    if (octets && P->nhwc && nstrips == 1 && !P->padded && !dy_stg && d->C % 8 == 0 &&
        ((long long)H * W) % (kind == kBackward ? 32 : 16) == 0) {
        P->oct = 1;
        P->opix = H * W / 8;
        P->og = P->opix % 4 == 0 ? 4 : 2;
        P->div_opix = make_fastdiv(P->opix);
        P->tbuf = (int)off;
        oct_floats = (kind == kBackward ? 2LL : 1LL) * P->stg_floats;
        if (L >= 1 && kind != kBackwardWeight) {  // outputs of the synthesis (L = 0: the base tiles store them)
            P->obuf = (int)(off + oct_floats);
            oct_floats += P->stg_floats;
        }
        off += oct_floats;
    }
    if (dy_stg) {
        // The dy staging holds the strip as H rows of W floats: the DY layout
        // exactly when H is whole tiles and W is whole tile columns.
        if (H % TR != 0 || W % TC != 0) return WTCONV_ERR_UNSUPPORTED;
        P->DY.base = P->stg + P->stg_floats;
        P->DY.stride = W;
        P->DY.sub = 0;
        P->dy_stg = 1;
    }

    // Tiles and threads.
    int nsub = 0;
    P->sub_begin[0] = 0;
    for (int l = 0; l < L; ++l)
        for (int s = 0; s < 4; ++s) {
            nsub += P->ntr[l] * P->ntc[l];
            P->sub_begin[1 + 4 * l + s] = nsub;
        }
    P->n_sub_tiles = nsub;
    P->n_base_tiles = P->ntr[kMaxL] * P->ntc[kMaxL];
    P->n_all_tiles = 0;
    for (int cl = 0; cl < ncls; ++cl) {
        const int lv = cl == 0 ? kMaxL : (cl - 1) >> 2;
        P->cls_tiles[cl] = P->ntr[lv] * P->ntc[lv];
        P->n_all_tiles += P->cls_tiles[cl];
    }
    P->nv = ncls * KK + 1;

    P->pyr = (L >= 1 && H % 4 == 0) ? 1 : 0;
    P->pyr_levels = std::min(L, 4);
    P->pyr_lg = std::max(P->pyr_levels - 2, 0);
    P->div_rw = make_fastdiv(std::max(W >> (P->pyr_lg + 2), 1));
    P->div_q4 = make_fastdiv(W / 4);
    P->div_w = make_fastdiv(W);
    for (int l = 0; l < L; ++l) P->div_m[l] = make_fastdiv(W >> (l + 1));
    for (int l = 0; l <= kMaxL; ++l) P->div_ntc[l] = make_fastdiv(std::max(P->ntc[l], 1));

    if (kind == kBackward) {
        // dx conv tiles one per thread (warps [0, corr0/32)); the correlation
        // tiles in class runs on the remaining threads.
        P->base_tid0 = P->n_sub_tiles;
        P->tile_end = P->base_tid0 + P->n_base_tiles;
        P->corr0 = ceil_div(P->tile_end, 32) * 32;
        const int budget = kBwdMaxThreads - P->corr0;
        if (budget < 32 * ncls / 32 || budget < 32) return WTCONV_ERR_UNSUPPORTED;
        int tpt = 1, used = 0;
        for (;; ++tpt) {
            used = 0;
            for (int cl = 0; cl < ncls; ++cl) used += ceil_div(P->cls_tiles[cl], tpt);
            if (used <= budget) break;
        }
        P->tpt = tpt;
        P->cls_thr[0] = 0;
        for (int cl = 0; cl < ncls; ++cl) P->cls_thr[cl + 1] = P->cls_thr[cl] + ceil_div(P->cls_tiles[cl], tpt);
        P->nthreads = std::max(64, ceil_div(P->corr0 + used, 32) * 32);
        P->merged = 1;
        P->an_split = ceil_div(P->nthreads / 2, 32) * 32;
        P->n_fin = L >= 1 ? (H / 2) * (W / 4) : 0;
        P->fin_off = 0;
        // Reduction scratch (correlation threads' sums, then one sum of dy
        // per warp) aliases the buffers from offset 0 after the walk.
        P->red = 0;
        off = std::max(off, (long long)used * KK + P->nthreads / 32);
    } else if (kind == kBackwardWeight) {
        // The fewest tiles per thread whose class-pure thread ranges fit.
        int tpt = 1, used = 0;
        for (;; ++tpt) {
            used = 0;
            for (int cl = 0; cl < ncls; ++cl) used += ceil_div(P->cls_tiles[cl], tpt);
            if (used <= (nstrips > 1 ? kStripMaxThreads : kBwdwMaxThreads)) break;
        }
        P->tpt = tpt;
        P->cls_thr[0] = 0;
        for (int cl = 0; cl < ncls; ++cl) P->cls_thr[cl + 1] = P->cls_thr[cl] + ceil_div(P->cls_tiles[cl], tpt);
        P->nthreads = std::max(tile_threads(used, nstrips > 1 ? kStripMaxThreads : kBwdwMaxThreads),
                               ceil_div(used, 32) * 32);
        // Reduction scratch aliases the (then dead) buffers from offset 0.
        P->red = 0;
        off = std::max(off, (long long)P->nthreads * (KK + 1));
    } else {
        // Subband and base tiles run the same code, so they share warps.
        P->base_tid0 = P->n_sub_tiles;
        P->tile_end = P->base_tid0 + P->n_base_tiles;
        P->nthreads = tile_threads(P->tile_end, nstrips > 1 ? kStripMaxThreads : kFusedMaxThreads);
        P->merged = P->tile_end <= P->nthreads ? 1 : 0;
        P->n_fin = L >= 1 ? (H / 2) * (W / 4) : 0;
        // Threads the analysis keeps busy (whole warps); the synthesis items
        // start on the others.
        long long an_items;
        if (P->pyr) {
            const int G = 1 << P->pyr_lg;
            an_items = (long long)(H >> (P->pyr_lg + 2)) * (W >> (P->pyr_lg + 2)) * G * G;
        } else {
            an_items = (long long)(L >= 1 ? H / 2 : H) * (W / 4);
        }
        const long long busy = ceil_div((int)std::min<long long>(an_items, 1 << 30), 32) * 32LL;
        P->fin_off = busy >= P->nthreads ? 0 : (int)busy;
    }
    // Halo push constants (strips; see wtconv_plan.h): per buffer the row
    // chunks, the reach and the warp-0 offset of its row groups.
    if (nstrips > 1) {
        const int nw = P->nthreads / 32;
        int gbase = 0;
        for (int bi = 0; bi <= L; ++bi) {
            const int rows = bi == 0 ? H : H >> bi, cols = bi == 0 ? W : W >> bi, nsub_lg = bi == 0 ? 0 : 2;
            P->hal_nq[bi] = (cols + 2 * p + 3) >> 2;
            P->hal_reach[bi] = (p + rows - 1) / rows;
            P->hal_g0[bi] = gbase % nw;
            gbase += (2 * P->hal_reach[bi]) << nsub_lg;
        }
    }
    // Weight gradients: the final step's scratch (summed partials, weights, a flag).
    if (kind == kBackwardWeight || kind == kBackward) off = std::max(off, (long long)P->nv + ncls * KK + 4);
    off = round4((int)std::min<long long>(off, 1LL << 30));
    if (off > kSmemLimitFloats) return WTCONV_ERR_UNSUPPORTED;
    // The weight gradient's octets add two CTA barriers and a staging step
    // after the tiles: measured slower than the gather at one CTA per SM
    // (64 x 64, L = 4: 483 -> 534 us), faster at two (stage1: 178 -> 164 us).
    if (P->oct && kind == kBackwardWeight && ctas_per_sm((int)off) < 2) return WTCONV_ERR_UNSUPPORTED;
    P->smem_floats = (int)off;
    if (kind == kBackwardWeight || kind == kBackward) {
        // The groups (and so the workspace) are chosen without the octet
        // buffer, so that both layouts of a shape get the same workspace size
        // (the choice is not monotone in the slots).
        const int smem_groups = P->smem_floats - (int)oct_floats;
        const long long slots = (long long)num_sms * resident_ctas(P->nthreads, smem_groups);
        P->groups = pick_groups(P->B, P->C * nstrips, slots);
        P->parts = P->groups * nstrips;
    } else {
        const long long units = (long long)P->B * P->C;
        P->grid = (int)std::min<long long>(units, (long long)num_sms * ctas_per_sm(P->smem_floats));
        P->groups = 1;
    }
    return WTCONV_OK;
}

// Tile rows on the busiest SM sub-partition per plane and SM: the tile-phase
// length of one CTA (its warp-tiles spread over 4 sub-partitions, times the
// tile height), times the CTAs of a plane, over the CTAs an SM holds.
// Cluster strips carry a halo exchange on top (weighted 15%).
inline int plan_ctas_per_sm(const Plan& P) {
    return P.nthreads > 256 ? 1 : ctas_per_sm(P.smem_floats);
}

inline double plan_cost(const Plan& P, Kind kind) {
    int per_smsp;
    if (kind == kBackward)
        per_smsp = ceil_div(ceil_div(P.tile_end, 32) + P.tpt * ceil_div(P.cls_thr[1 + 4 * P.L], 32), 4);
    else if (kind == kBackwardWeight)
        per_smsp = P.tpt * ceil_div(ceil_div(P.cls_thr[1 + 4 * P.L], 32), 4);
    else
        per_smsp = ceil_div(ceil_div(P.tile_end, 32), 4);
    const double c = (double)per_smsp * P.TR * P.nstrips / plan_ctas_per_sm(P);
    if (P.nstrips > kMaxPortableStrips) return 1.3 * c;  // a 16-CTA cluster needs 16 SMs of one GPC
    return P.nstrips > 1 ? 1.15 * c : c;
}

// The whole backward: the one-pass plan P against the input- and
// weight-gradient plans Pin and Pw.  The one pass when its tile-row cost is
// lower; on equal costs, when one of the two passes also runs one CTA per SM
// (then neither path hides an analysis phase behind a second CTA's tiles, and
// the one pass saves a pass over dy and one analysis of it).  Measured on the
// 64 whole-plane points of the shape sweep: the one pass is faster exactly at
// 32x32, L = 1 (cost 4 vs 7) and at 64x64, L = 3 and 4 (cost 40 vs 12 + 28, the
// weight pass at one CTA per SM), by 5-20%, and slower by 8-30% everywhere else
// (32x32 at L = 4, k = 3 is within 1% either way).  NHWC planes that both
// passes gather element by element (no channel octets): the one pass, which
// gathers x and dy once where the two passes gather dy twice; measured 1.2-1.45x
// faster at six shapes (16x16 to 64x64, L = 1 to 4, C = 6 to 100).  NHWC planes
// that the one pass holds on channel octets: the one pass (below).
inline bool prefer_one_pass(const Plan& P, const Plan& Pin, const Plan& Pw) {
    if (P.nhwc && !Pin.oct && !Pw.oct) return true;
    // NHWC with the one pass on channel octets: measured 0.51-1.01x the two
    // passes at eleven shapes (32x32 to 64x64, L = 1 to 4, stage1 fp32 and
    // bf16), the one pass moving one run of x and one of dy a plane where the
    // two passes move dy twice.
    if (P.nhwc && P.oct) return true;
    const double c1 = plan_cost(P, kBackward);
    const double c2 = plan_cost(Pin, kBackwardInput) + plan_cost(Pw, kBackwardWeight);
    if (c1 < c2 * (1.0 - 1e-9)) return true;
    if (c1 > c2 * (1.0 + 1e-9)) return false;
    return plan_ctas_per_sm(Pin) == 1 || plan_ctas_per_sm(Pw) == 1;
}

// Chooses the fewest strips that fit (whole planes, else clusters of 2, 4,
// 8, 16 strips), and for that count the tile height (7 or 8 rows) with the
// lowest plan_cost.  Every cluster strip adds barriers and halo exchanges
// per plane that the tile count does not show: at 128 x 128 (L = 2..4) two
// strips measured 1.7-1.9x faster than eight, and at every shape measured
// fewer strips were faster (also where twice the strips would fit two CTAs
// per SM: 4 strips at 128 x 128 and 16 at 256 x 256, L = 1, measured within
// 3% of 2 and 8).
inline wtconv_status_t make_plan(const wtconv_desc_t* d, Kind kind, int num_sms, Plan* P) {
    bool have = false;
    double best = 0.0;
    Plan cand;
    for (int n = 1; n <= kMaxStrips && !have; n *= 2) {
        // The weight gradient on strips may read dy from its staging (no DY
        // buffer) when that is what lets this strip count fit.
        for (int alias = 0; alias < 2 && !have; ++alias) {
            if (alias && (kind != kBackwardWeight || n == 1)) break;
            for (int TR = 7; TR <= 8; ++TR) {
                wtconv_status_t st = make_plan_for(d, kind, TR, n, num_sms, &cand, alias == 1);
                // NHWC planes whose octet buffer does not fit: the element-by-element gather.
                if (st != WTCONV_OK && n == 1 && d->layout == WTCONV_NHWC)
                    st = make_plan_for(d, kind, TR, n, num_sms, &cand, alias == 1, false);
                if (st != WTCONV_OK) continue;
                const double c = plan_cost(cand, kind);
                if (!have || c < best) {
                    best = c;
                    *P = cand;
                    have = true;
                }
            }
        }
    }
    if (!have) {
        memset(P, 0, sizeof(*P));
        return WTCONV_ERR_UNSUPPORTED;
    }
    return WTCONV_OK;
}

}  // namespace wtc
