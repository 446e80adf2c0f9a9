// Shared-memory and tile plan for the fused WTConv kernels.
//
// A CTA stages whole (b, c) planes on chip, one after another (persistent):
// while it computes one plane, cp.async copies the next plane into a staging
// buffer.  Every buffer below lives in dynamic shared memory; offsets and
// strides are in floats.  The plan is built on the host (wtconv_planner.h)
// and passed to the kernels by value.
//
// Buffers:
//   STG    raw staging of the next plane(s), as stored in HBM (float or bf16):
//          x (forward), dy (input gradient), x then dy (weight gradient).
//   X      padded input plane, p = k/2 zero rows/cols around it.
//   S[l]   padded un-normalised Haar subbands of level l (4 planes) of X.
//   Q[l]   forward: subband conv outputs of level l (4 planes, tile-rounded);
//          weight gradient: Haar subbands of dy (4 planes, tile-rounded).
//   Y      forward (L >= 1): base-branch outputs (tile-rounded), kept until
//          the synthesis adds the wavelet terms and stores the plane.
//   DY     weight gradient: dy plane (tile-rounded).
//   XS, SS[l]  fused backward: padded x plane and padded x subbands (the
//          correlation windows); there X and S hold the padded dy plane and
//          dy subbands (the dx conv windows, and the correlation's dy tiles
//          at their interior), Q and Y the dx conv outputs.
//   W      forward: folded weights, one class (K*K floats) per subband and the base.
//
// Padded buffers: `base` is the offset of padded element (-p, -p), so a
// conv window for the output tile whose top-left output is (r0, c0) starts
// at base + r0 * stride + c0, which is 16-byte aligned (stride and c0 are
// multiples of 4).  Unpadded buffers: element (i, j) is at base + i*stride + j.
#pragma once

#include <stdint.h>

namespace wtc {

constexpr int kMaxL = 6;
constexpr int kMaxStrips = 16;          // CTAs of a cluster sharing one plane
constexpr int kMaxPortableStrips = 8;   // larger clusters need the non-portable opt-in
constexpr int kMaxCls = 1 + 4 * kMaxL;

// Division by a runtime constant d as a multiply-high and a shift:
//   n / d == (umulhi(n, mul) + n) >> shift   for 0 <= n < 2^31,
// with shift = ceil(log2 d) and mul = floor(2^32 (2^shift - d) / d) + 1.
struct FastDiv {
    uint32_t mul;
    uint32_t shift;
};

inline uint32_t fastdiv_host(uint32_t n, FastDiv f) {
    return (uint32_t)(((((uint64_t)n * f.mul) >> 32) + n) >> f.shift);
}

inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    FastDiv f;
    f.shift = l;
    f.mul = (uint32_t)(((((uint64_t)1 << l) - d) << 32) / d + 1);
    return f;
}

// Thread budgets (also the kernels' __launch_bounds__, two CTAs per SM).
constexpr int kFusedMaxThreads = 256;
constexpr int kBwdwMaxThreads = 256;
// Planes split into cluster strips: one CTA per SM at most (their strips'
// buffers are large), so those instantiations take 512 threads at one CTA
// per SM (the same 128-register budget).
constexpr int kStripMaxThreads = 512;
constexpr int kBwdMaxThreads = 512;  // fused backward: one CTA per SM

struct Buf {
    int base;    // float offset (see above)
    int stride;  // floats per row, multiple of 4
    int sub;     // floats between the 4 subband planes (0 for single planes)
};

struct Plan {
    // H is the height of the rows a CTA holds: the plane, or one of its
    // nstrips strips (a thread-block cluster of nstrips CTAs per plane, CTA
    // rank r holding plane rows [r*H, (r+1)*H) and, in its padding rows, the
    // neighbouring strips' halo rows).  Hp is the plane height.
    int B, C, H, W, k, L, p;
    int Hp, nstrips;
    // The plane in global memory is Hr x Wr.  When Hr or Wr is not a multiple
    // of 2^L the CTAs hold it zero-padded to Hp x W (multiples of 2^L; padded
    // = 1): the real rows are staged row by row (row_chunks 16-byte chunks
    // each) into staging rows of W elements, and only real outputs are
    // stored.
    int Hr, Wr, padded, row_chunks;
    // Activation layout in global memory: 0 = NCHW, 1 = NHWC (planes
    // gathered element by element, C elements apart; the general
    // instantiations and the one-pass backward only).
    int nhwc;
    // NHWC channel octets (whole planes, C a multiple of 8): clusters of 8
    // CTAs, CTA r of a cluster holding channel 8o + r of the planes (b, octet
    // o) the cluster walks.  Each CTA loads its run of opix pixels of the
    // plane's 8 channels (8 * esize contiguous bytes a pixel) into its octet
    // buffer at tbuf (stg_floats floats, pixel j at 8 * esize * j bytes) and
    // scatters channel q to CTA q's staging (the weight gradient: the x run,
    // then the dy run, through the same buffer; the fused backward: the x
    // run at tbuf and the dy run at tbuf + stg_floats).
    // The synthesis (forward, input gradient, fused backward) stores each
    // output into the output octet buffer at obuf (stg_floats floats) of the
    // CTA that owns its pixel, as row r of
    // [8 channels][opix pixels] (stored format); the owner writes the 8
    // channels of its pixels as whole runs.
    // og: pixels a scatter / write-out step moves (4, or 2 where opix is not
    // a multiple of 4).
    int oct, opix, tbuf, obuf, og;
    FastDiv div_opix;
    int parts;           // weight gradient: partial vectors per channel (groups * nstrips)
    int TR, TC;          // output tile: TR rows x TC cols per thread (TC = 4: two column pairs)
    int esize;           // bytes per stored activation (4 or 2)
    int nthreads;        // CTA size
    int smem_floats;     // dynamic shared memory, in floats (multiple of 4)
    int grid;            // forward: number of persistent CTAs
    int groups;          // weight gradient: batch groups (grid.y)
    int wbase, wcls;     // forward: folded weights of class cl (0 = base, 1 + 4l + s) at wbase + cl*wcls
    int bias;            // forward: folded bias
    int red;             // weight gradient: reduction scratch (aliases the plane buffers)
    int stg;             // staging buffer offset; one stored plane occupies stg_floats floats
    int stg_floats;
    int dy_stg;          // weight gradient (strips): DY aliases the dy staging (see the kernel)
    int plane_chunks;    // 16-byte chunks per stored plane
    Buf X, Y, DY, XS;
    Buf S[kMaxL], Q[kMaxL], SS[kMaxL];
    int ntr[kMaxL + 1], ntc[kMaxL + 1];  // tile grid per level; index kMaxL = full resolution
    // Tile enumeration.  Forward: subband tiles in class order (l, s) first,
    // counted by sub_begin; base tiles separately.  Weight gradient: class cl
    // (0 = base, 1 + 4l + s) has cls_tiles[cl] tiles and the contiguous
    // thread range [cls_thr[cl], cls_thr[cl+1]); its j-th thread owns the
    // class's tiles [j*tpt, min((j+1)*tpt, cls_tiles[cl])) for the whole walk,
    // so every thread accumulates one class only.
    int sub_begin[kMaxCls + 1];
    int n_sub_tiles, n_base_tiles;
    int cls_tiles[kMaxCls];
    int cls_thr[kMaxCls + 1];
    int tpt;             // weight gradient: tiles per thread (at most)
    int n_all_tiles;
    int nv;              // weight gradient: floats per partial vector = ncls*k*k + 1
    // Forward tile index space: subband tiles [0, n_sub_tiles), base tiles
    // [base_tid0, tile_end); thread t takes the indices t, t + nthreads, ...
    int base_tid0, tile_end;
    int merged;          // forward: tile_end <= nthreads (one tile per thread)
    // Forward synthesis work items (L >= 1): rows 2i, 2i+1 x columns 4q..4q+3;
    // thread t takes items (t - fin_off) mod nthreads + k * nthreads, so the
    // threads that the analysis leaves idle start first.
    int n_fin, fin_off;
    // Fused backward: threads [0, corr0) run the dx conv tiles (one each),
    // threads [corr0, corr0 + cls_thr[ncls]) the correlation tiles (class
    // runs as in the weight gradient); in the analysis threads [0, an_split)
    // take x and the rest take dy.
    int corr0, an_split;
    // Strips: halo push constants of buffer b (0 = X, 1 + l = S[l]): 16-byte
    // chunks of a padded row, strips reached, and the first of its row groups
    // that warp 0 takes (the groups of buffers < b, modulo the warps).
    int hal_nq[kMaxL + 1], hal_reach[kMaxL + 1], hal_g0[kMaxL + 1];
    int pyr;             // analysis by the one-pass pyramid (H % 4 == 0 and L >= 1)
    int pyr_levels;      // levels the pyramid computes (min(L, 4)); the rest run level by level
    int pyr_lg;          // pyramid lane groups cover (4 * 2^pyr_lg)^2 pixel regions
    FastDiv div_rw;      // (W >> (pyr_lg + 2)): pyramid regions per row
    FastDiv div_q4;                 // W / 4: 4-column groups per row
    FastDiv div_w;                  // W
    FastDiv div_rowc;               // row_chunks
    FastDiv div_wr;                 // Wr (NHWC staging)
    FastDiv div_m[kMaxL];           // W >> (l+1)
    FastDiv div_ntc[kMaxL + 1];     // tile columns per tile row
};

// CTAs per cluster: the strips of a plane, or the 8 CTAs of a channel octet
// (also compiled by host-only tools, without the CUDA qualifiers).
#ifdef __CUDACC__
#define WTC_HD __host__ __device__
#else
#define WTC_HD
#endif
inline WTC_HD int cluster_ctas(const Plan& P) { return P.oct ? 8 : P.nstrips; }
#undef WTC_HD

}  // namespace wtc
