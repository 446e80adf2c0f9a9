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
constexpr int kNumSMs = 148;  // B200; sizes the persistent grids

enum Kind { kForward = 0, kBackwardInput = 1, kBackwardWeight = 2 };

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

// Tile height: the one with the shorter tile phase, i.e. fewer tile rows on
// the busiest SM sub-partition (warp-tiles per sub-partition x TR).
inline int pick_tile_rows(const wtconv_desc_t* d, int max_threads) {
    int best = 7;
    long long best_cost = -1;
    for (int TR = 7; TR <= 8; ++TR) {
        const int tiles = count_tiles(d, TR);
        const int threads = tile_threads(tiles, max_threads);
        const long long warp_tiles = ceil_div(tiles, 32);
        const long long per_smsp = ceil_div((int)std::min<long long>(warp_tiles, 1 << 30), 4);
        const long long iters = ceil_div(tiles, threads);
        const long long cost = std::max(per_smsp, iters) * TR;
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = TR;
        }
    }
    return best;
}

// CTAs per SM that the shared memory of one CTA allows (the register
// budget of the launch bounds allows two).
inline int ctas_per_sm(int smem_floats) {
    return std::max(1, std::min(2, kSmemPerSM / (smem_floats * 4 + 1024)));
}

// Weight-gradient batch groups (grid.y): the CTA of group g walks planes
// b = g, g + groups, ...  Chosen to minimise waves x planes-per-CTA over the
// resident CTA slots, with at most 64 planes per CTA so every per-thread
// running sum stays short.
inline int pick_groups(int B, int C, int smem_floats) {
    const long long slots = (long long)kNumSMs * ctas_per_sm(smem_floats);
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
    if ((d->H % (1 << d->L)) != 0 || (d->W % (1 << d->L)) != 0) return WTCONV_ERR_BAD_SHAPE;
    if ((d->W % 4) != 0) return WTCONV_ERR_BAD_SHAPE;
    // Planes are staged in 16-byte chunks.
    const long long esize = d->dtype == WTCONV_BF16 ? 2 : 4;
    if (((long long)d->H * d->W * esize) % 16 != 0) return WTCONV_ERR_BAD_SHAPE;
    // Index arithmetic in the kernels is 32-bit within a plane and 64-bit across planes.
    if ((long long)d->H * d->W > (1LL << 30)) return WTCONV_ERR_BAD_SHAPE;
    if ((long long)d->B * d->C > (1LL << 31) - 1) return WTCONV_ERR_BAD_SHAPE;
    return WTCONV_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline wtconv_status_t make_plan(const wtconv_desc_t* d, Kind kind, Plan* P) {
    memset(P, 0, sizeof(*P));
    P->B = d->B; P->C = d->C; P->H = d->H; P->W = d->W; P->k = d->k; P->L = d->L;
    const int p = d->k / 2, k = d->k, L = d->L, H = d->H, W = d->W, KK = k * k;
    P->p = p;
    P->esize = d->dtype == WTCONV_BF16 ? 2 : 4;
    P->TC = 4;
    P->TR = pick_tile_rows(d, kind == kBackwardWeight ? kBwdwMaxThreads : kFusedMaxThreads);
    const int TR = P->TR, TC = P->TC;
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
    // Padded input plane.
    {
        const int ntc = P->ntc[kMaxL];
        const int rows = P->ntr[kMaxL] * TR + 2 * p;
        const int need = std::max(W + 2 * p, (ntc - 1) * TC + WV4);
        P->X.stride = pick_stride(need, TR, ntc);
        P->X.base = (int)off;
        off += round4(rows * P->X.stride);
    }
    // Padded subbands of every level.
    for (int l = 0; l < L; ++l) {
        const int m = W >> (l + 1);
        const int ntc = P->ntc[l];
        const int rows = P->ntr[l] * TR + 2 * p;
        const int need = std::max(m + 2 * p, (ntc - 1) * TC + WV4);
        P->S[l].stride = pick_stride(need, TR, ntc);
        P->S[l].sub = round4(rows * P->S[l].stride);
        P->S[l].base = (int)off;
        off += 4LL * P->S[l].sub;
    }
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
    if (kind == kBackwardWeight) {
        const int rows = P->ntr[kMaxL] * TR;
        P->DY.stride = round4(P->ntc[kMaxL] * TC);
        P->DY.base = (int)off;
        off += round4(rows * P->DY.stride);
    }
    // Staging of the next plane(s), stored format.
    {
        const long long bytes = (long long)H * W * P->esize;
        P->plane_chunks = (int)(bytes / 16);
        P->stg_floats = (int)(bytes / 4);
        P->stg = (int)off;
        off += (kind == kBackwardWeight ? 2LL : 1LL) * P->stg_floats;
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
    P->cls_begin[0] = 0;
    P->cls_begin[1] = P->n_base_tiles;
    for (int cl = 1; cl < ncls; ++cl) {
        const int l = (cl - 1) >> 2;
        P->cls_begin[cl + 1] = P->cls_begin[cl] + P->ntr[l] * P->ntc[l];
    }
    P->n_all_tiles = P->cls_begin[ncls];
    P->nv = ncls * KK + 1;

    P->pyr = (L >= 1 && H % 4 == 0) ? 1 : 0;
    P->pyr_levels = std::min(L, 4);
    P->pyr_lg = std::max(P->pyr_levels - 2, 0);
    P->div_rw = make_fastdiv(std::max(W >> (P->pyr_lg + 2), 1));
    P->div_q4 = make_fastdiv(W / 4);
    for (int l = 0; l < L; ++l) P->div_m[l] = make_fastdiv(W >> (l + 1));
    for (int l = 0; l <= kMaxL; ++l) P->div_ntc[l] = make_fastdiv(std::max(P->ntc[l], 1));

    if (kind == kBackwardWeight) {
        // One tile per thread for the whole walk.
        if (P->n_all_tiles > kBwdwMaxThreads) return WTCONV_ERR_UNSUPPORTED;
        P->nthreads = tile_threads(P->n_all_tiles, kBwdwMaxThreads);
        if (P->nthreads < P->n_all_tiles) P->nthreads = ceil_div(P->n_all_tiles, 32) * 32;
        // Reduction scratch aliases the (then dead) buffers from offset 0.
        P->red = 0;
        off = std::max(off, (long long)P->nthreads * (KK + 1));
    } else {
        // Subband and base tiles run the same code, so they share warps.
        P->base_tid0 = P->n_sub_tiles;
        P->tile_end = P->base_tid0 + P->n_base_tiles;
        P->nthreads = tile_threads(P->tile_end, kFusedMaxThreads);
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
    off = round4((int)std::min<long long>(off, 1LL << 30));
    if (off > kSmemLimitFloats) return WTCONV_ERR_UNSUPPORTED;
    P->smem_floats = (int)off;
    if (kind == kBackwardWeight) {
        P->groups = pick_groups(P->B, P->C, P->smem_floats);
    } else {
        const long long units = (long long)P->B * P->C;
        P->grid = (int)std::min<long long>(units, (long long)kNumSMs * ctas_per_sm(P->smem_floats));
        P->groups = 1;
    }
    return WTCONV_OK;
}

}  // namespace wtc
