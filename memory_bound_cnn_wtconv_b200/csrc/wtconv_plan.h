// Shared-memory and tile plan for the fused WTConv kernels.
//
// One CTA stages one whole (b, c) plane on chip.  Every buffer below lives in
// dynamic shared memory; offsets and strides are in floats.  The plan is built
// on the host (wtconv_plan.cpp) and passed to the kernels by value.
//
// Buffers:
//   X      padded input plane (x in the forward, dy in the input gradient,
//          x in the weight gradient), p = k/2 zero rows/cols around it.
//   S[l]   padded un-normalised Haar subbands of level l (4 planes).
//   Q[l]   forward: subband conv outputs of level l (4 planes, tile-rounded);
//          weight gradient: Haar subbands of dy (4 planes, tile-rounded).
//   Z      forward: coarse-level synthesis at half resolution (aliases S[0]).
//   DY     weight gradient: dy plane (tile-rounded).
//
// Padded buffers: `base` is the offset of padded element (-p, -p), so a
// conv window for the output tile whose top-left output is (r0, c0) starts
// at base + r0 * stride + c0, which is 16-byte aligned (stride and c0 are
// multiples of 4).  Unpadded buffers: element (i, j) is at base + i*stride + j.
#pragma once

namespace wtc {

constexpr int kMaxL = 6;
constexpr int kMaxCls = 1 + 4 * kMaxL;

struct Buf {
    int base;    // float offset (see above)
    int stride;  // floats per row, multiple of 4
    int sub;     // floats between the 4 subband planes (0 for single planes)
};

struct Plan {
    int B, C, H, W, k, L, p;
    int TR, TC;          // output tile: TR rows x TC cols per thread
    int nthreads;        // CTA size
    int smem_floats;     // dynamic shared memory, in floats (multiple of 4)
    int groups;          // weight gradient: batch groups (grid.y)
    int wbase, wcls;     // folded weights: class cl (0 = base, 1 + 4l + s) at wbase + cl*wcls
    int bias;            // folded bias (forward)
    int red;             // weight gradient: reduction scratch (aliases S / Q)
    Buf X, DY, Z;
    Buf S[kMaxL], Q[kMaxL];
    int ntr[kMaxL + 1], ntc[kMaxL + 1];  // tile grid per level; index kMaxL = full resolution
    // Tile enumeration.  Forward: subband tiles in class order (l, s) first,
    // counted by sub_begin; base tiles separately.  Weight gradient: every
    // class (base first) gets a contiguous thread range cls_begin[cl].
    int sub_begin[kMaxCls + 1];
    int n_sub_tiles, n_base_tiles;
    int cls_begin[kMaxCls + 1];
    int n_all_tiles;
    int nv;              // weight gradient: floats per partial vector = ncls*k*k + 1
};

}  // namespace wtc
