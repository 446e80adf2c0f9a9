// Fused WTConv kernels for sm_100a (B200).
//
// Method: "Fast and Memory-Efficient Wavelet Convolutions via I/O-Aware
// Reformulation" (arXiv 2608.10805), Abstract -- the three reformulations:
//   (1) the Haar analysis butterflies are recomputed on chip for every level
//       from the staged input plane; no subband ever reaches HBM;
//   (2) the synthesis is one pass over the output: output (h, w) receives,
//       for every level l, the signed sum of that level's four conv outputs
//       at (h >> (l+1), w >> (l+1)), the signs given by bit l of h and w;
//   (3) per-channel and per-subband scales (and the orthonormal 2^-(l+1)
//       factors of analysis and synthesis) are folded into the conv weights,
//       so the butterflies are pure add/sub.
//
// Un-normalised butterflies: U_{l,s} = 2^(l+1) S_{l,s} (S orthonormal), so a
// level-l conv with weights  wt_scale * wt_w * 4^-(l+1)  yields exactly the
// term  2^-(l+1) * Shat_{l,s}  that the closed-form synthesis adds.
//
// Depthwise convolution is not a dense contraction, so the convs run on the
// FP32 pipes, with the packed f32x2 FMA (64 multiply-adds per warp
// instruction, half the issue slots of scalar FMAs): a thread owns a TR x 4
// output tile as TR x 2 column pairs, streams its window's TR+K-1 input rows
// from shared memory once with 128-bit loads, and keeps the K*K folded
// weights in registers.
//
// CTAs are persistent: each walks a run of planes; while it computes one
// plane, cp.async copies the next one from HBM into a staging buffer.  Per
// plane, a phase of on-chip analysis (and of the previous plane's synthesis)
// and a phase of conv tiles, separated by CTA barriers (cluster barriers when
// a plane is split into strips across a thread-block cluster).
//
// Kernels: wtconv_fused_kernel (forward; input gradient with BWD),
// wtconv_bwdw_partial_kernel (weight gradient, with its final step in the
// tail) and wtconv_backward_kernel (input and weight gradients in one pass).
#pragma once

#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <type_traits>
#include <cuda_bf16.h>
#include <stdint.h>

#include "wtconv_plan.h"

namespace wtc {

namespace cg = cooperative_groups;

__device__ __forceinline__ int fdiv(int n, FastDiv f) {
    return (int)((__umulhi((uint32_t)n, f.mul) + (uint32_t)n) >> f.shift);
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// ---------------------------------------------------------------------------
// Asynchronous plane staging (cp.async, 16-byte chunks, no register round trip).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

__device__ __forceinline__ void stage_plane(float* stg, const void* src, int chunks, int tid, int nt) {
    const char* g = static_cast<const char*>(src);
    char* d = reinterpret_cast<char*>(stg);
    for (int ch = tid; ch < chunks; ch += nt) cp_async16(d + 16 * ch, g + 16 * ch);
}

// Activations in global memory.  NCHW: plane (b, c) is Hr x Wr contiguous
// elements.  NHWC: the C channels of a pixel are adjacent, so plane (b, c)
// starts at element b*Hr*Wr*C + c and its elements are C apart.  `act_es`
// is that element stride; an offset within a plane is (h*Wr + w) * act_es.
// NHWC is a runtime layout of the general instantiations and the one-pass
// backward only (NHW = false compiles the plain NCHW walk).
template <bool NHW>
__device__ __forceinline__ size_t act_es(const Plan& P) {
    return (NHW && P.nhwc) ? (size_t)P.C : (size_t)1;
}
template <bool NHW>
__device__ __forceinline__ size_t plane_origin(const Plan& P, int b, int c) {
    const size_t hw = (size_t)P.Hr * P.Wr;
    return (NHW && P.nhwc) ? (size_t)b * hw * P.C + c : ((size_t)b * P.C + c) * hw;
}

// NHWC staging: this CTA's `rows` real rows of Wr elements, each element C
// elements from the next, into staging rows of W elements.  fp32 elements
// go by 4-byte cp.async; bf16 elements (2 bytes, below the smallest
// cp.async) by plain loads and shared stores.
__device__ __forceinline__ void stage_nhwc(float* stg, const void* src, const Plan& P, int rows, int tid, int nt) {
    const int n = rows * P.Wr;
    const size_t es = (size_t)P.C;
    if (P.esize == 4) {
        const float* g = static_cast<const float*>(src);
        for (int e = tid; e < n; e += nt) {
            const int r = fdiv(e, P.div_wr), col = e - r * P.Wr;
            cp_async4(stg + r * P.W + col, g + (size_t)e * es);
        }
    } else {
        const unsigned short* g = static_cast<const unsigned short*>(src);
        unsigned short* d = reinterpret_cast<unsigned short*>(stg);
#pragma unroll 4
        for (int e = tid; e < n; e += nt) {
            const int r = fdiv(e, P.div_wr), col = e - r * P.Wr;
            d[r * P.W + col] = __ldg(g + (size_t)e * es);
        }
    }
}

// This CTA's rows of a plane into staging: one contiguous copy, or (planes
// zero-padded on chip) its `rows` real rows, each Wr elements, into staging
// rows of W elements (the padding was zeroed once and is never written), or
// the NHWC gather above.
__device__ __forceinline__ void stage_rows(float* stg, const void* src, const Plan& P, int rows, int tid, int nt) {
    if (P.nhwc) {
        stage_nhwc(stg, src, P, rows, tid, nt);
        return;
    }
    if (!P.padded) {
        stage_plane(stg, src, P.plane_chunks, tid, nt);
        return;
    }
    const char* g = static_cast<const char*>(src);
    char* d = reinterpret_cast<char*>(stg);
    const int rc = P.row_chunks;
    const size_t sbytes = (size_t)P.Wr * P.esize, dbytes = (size_t)P.W * P.esize;
    for (int ch = tid; ch < rows * rc; ch += nt) {
        const int r = fdiv(ch, P.div_rowc), c = ch - r * rc;
        cp_async16(d + r * dbytes + 16 * c, g + r * sbytes + 16 * c);
    }
}

// Real rows of strip `rank` (all H of them unless the plane was padded).
__device__ __forceinline__ int real_rows(const Plan& P, int rank) {
    return max(0, min(P.H, P.Hr - rank * P.H));
}

// 4 consecutive staged elements (element index e, a multiple of 4), as floats.
template <typename T>
__device__ __forceinline__ float4 stg_load4(const float* stg, int e);

template <>
__device__ __forceinline__ float4 stg_load4<float>(const float* stg, int e) {
    return *reinterpret_cast<const float4*>(stg + e);
}

template <>
__device__ __forceinline__ float4 stg_load4<__nv_bfloat16>(const float* stg, int e) {
    const uint2 r = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(stg) + e);
    const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// Store 4 activations to global memory (16 bytes as float, 8 as bf16).
template <typename T>
__device__ __forceinline__ void gst4(T* p, float4 v);

template <>
__device__ __forceinline__ void gst4<float>(float* p, float4 v) {
    *reinterpret_cast<float4*>(p) = v;
}

template <>
__device__ __forceinline__ void gst4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 r;
    r.x = *reinterpret_cast<uint32_t*>(&a);
    r.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = r;
}

// Store 4 activations that are `es` elements apart (es = 1: gst4).
template <typename T>
__device__ __forceinline__ void gst1(T* p, float v);
template <>
__device__ __forceinline__ void gst1<float>(float* p, float v) {
    *p = v;
}
template <>
__device__ __forceinline__ void gst1<__nv_bfloat16>(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
}
template <typename T>
__device__ __forceinline__ void gst4s(T* p, float4 v, size_t es) {
    if (es == 1) {
        gst4<T>(p, v);
    } else {
        gst1<T>(p, v.x);
        gst1<T>(p + es, v.y);
        gst1<T>(p + 2 * es, v.z);
        gst1<T>(p + 3 * es, v.w);
    }
}

// Store 4 / 2 floats to a shared address congruent to P (mod 4) floats.
template <int P>
__device__ __forceinline__ void sts4(float* dst, float4 v) {
    if constexpr (P % 4 == 0) {
        *reinterpret_cast<float4*>(dst) = v;
    } else if constexpr (P % 2 == 0) {
        reinterpret_cast<float2*>(dst)[0] = make_float2(v.x, v.y);
        reinterpret_cast<float2*>(dst)[1] = make_float2(v.z, v.w);
    } else {
        dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
    }
}

template <int P>
__device__ __forceinline__ void sts2(float* dst, float a, float b) {
    if constexpr (P % 2 == 0) {
        *reinterpret_cast<float2*>(dst) = make_float2(a, b);
    } else {
        dst[0] = a; dst[1] = b;
    }
}

__device__ __forceinline__ void zero_smem(float* sm, int nfloats, int tid, int nt) {
    float4* s4 = reinterpret_cast<float4*>(sm);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = tid; i < (nfloats >> 2); i += nt) s4[i] = z;
}

// ---------------------------------------------------------------------------
// Unpack the staged H x W plane into the plane buffer (element (0,0) at
// `dst`, congruent to PD mod 4 floats) and, if `level0`, run the level-0
// un-normalised butterflies into the 4 subband planes at `sb` (element (0,0),
// congruent to PD mod 2).  One work item = rows 2i, 2i+1 x columns 4q..4q+3,
// i.e. two 2x2 blocks.  Returns the thread's sum of the unpacked values if SUM.
// COPY = false: the plane buffer is not written (its reader uses the staging).
// ---------------------------------------------------------------------------
template <typename T, int PD, bool SUM, bool COPY = true>
__device__ __forceinline__ float unpack_level0(const float* stg, int H, int W, FastDiv dq4, float* dst, int ds,
                                               float* sb, int sbs, int sbsub, bool level0, int tid, int nt) {
    const int W4 = W >> 2;
    float sum = 0.f;
    if (level0) {
        const int n = (H >> 1) * W4;
        for (int t = tid; t < n; t += nt) {
            const int i = fdiv(t, dq4), q = t - i * W4;
            const int r0 = 2 * i, c0 = 4 * q;
            const float4 a = stg_load4<T>(stg, r0 * W + c0);
            const float4 b = stg_load4<T>(stg, (r0 + 1) * W + c0);
            if (COPY) {
                sts4<PD>(dst + r0 * ds + c0, a);
                sts4<PD>(dst + (r0 + 1) * ds + c0, b);
            }
            if (SUM) sum += ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w));
            const float apb0 = a.x + a.y, amb0 = a.x - a.y, cpd0 = b.x + b.y, cmd0 = b.x - b.y;
            const float apb1 = a.z + a.w, amb1 = a.z - a.w, cpd1 = b.z + b.w, cmd1 = b.z - b.w;
            float* d = sb + i * sbs + 2 * q;
            sts2<PD>(d, apb0 + cpd0, apb1 + cpd1);              // LL
            sts2<PD>(d + sbsub, apb0 - cpd0, apb1 - cpd1);      // LH: difference between rows
            sts2<PD>(d + 2 * sbsub, amb0 + cmd0, amb1 + cmd1);  // HL: difference between columns
            sts2<PD>(d + 3 * sbsub, amb0 - cmd0, amb1 - cmd1);  // HH
        }
    } else {
        const int n = H * W4;
        for (int t = tid; t < n; t += nt) {
            const int i = fdiv(t, dq4), q = t - i * W4;
            const float4 a = stg_load4<T>(stg, i * W + 4 * q);
            if (COPY) sts4<PD>(dst + i * ds + 4 * q, a);
            if (SUM) sum += (a.x + a.y) + (a.z + a.w);
        }
    }
    return sum;
}

// One un-normalised 2-D Haar analysis step on chip: the (2n) x (2m) plane at
// `src` (element (0,0), row stride `ss`) becomes 4 planes n x m at `dst`
// (element (0,0), row stride `ds`, plane step `dsub`), order LL, LH, HL, HH.
__device__ __forceinline__ void haar_level(const float* src, int ss, int n, int m, FastDiv dm, float* dst,
                                           int ds, int dsub, int tid, int nt) {
    for (int t = tid; t < n * m; t += nt) {
        const int i = fdiv(t, dm), j = t - i * m;
        const float* s0 = src + 2 * i * ss + 2 * j;
        const float a = s0[0], b = s0[1], c = s0[ss], d = s0[ss + 1];
        const float apb = a + b, amb = a - b, cpd = c + d, cmd = c - d;
        float* d0 = dst + i * ds + j;
        d0[0] = apb + cpd;
        d0[dsub] = apb - cpd;
        d0[2 * dsub] = amb + cmd;
        d0[3 * dsub] = amb - cmd;
    }
}

// Where one analysis level writes: element (i, j) of subband s at
// base + s*sub + i*stride + j (`base` already includes any padding offset).
struct LevelDst {
    float* base;
    int stride;
    int sub;
};
struct Levels {
    LevelDst d[4];  // indexed by compile-time constants only (kept in registers)
};

__device__ __forceinline__ void butterfly(float a, float b, float c, float d, float& ll, float& lh, float& hl,
                                          float& hh) {
    const float apb = a + b, amb = a - b, cpd = c + d, cmd = c - d;
    ll = apb + cpd;  // LL
    lh = apb - cpd;  // LH: difference between rows
    hl = amb + cmd;  // HL: difference between columns
    hh = amb - cmd;  // HH
}

// Analysis pyramid of one staged plane in a single pass (no CTA barrier):
// the `np` threads [0, np) each own 4x4 pixel blocks; they unpack the block
// into the plane buffer `dst` (element (0,0), row stride ds, congruent to PD
// mod 4 floats), run levels 0 and 1 in registers, and levels 2 ..
// `levels`-1 (levels <= 4) by xor-shuffles inside groups of 4^(l-1) lanes
// that cover one 2^(l+1) x 2^(l+1) region.  Lane groups: a region of
// (4G)^2 pixels, G = 2^lg, occupies G*G consecutive lanes (block (by, bx) of
// the region at lane offset by*G + bx).  Returns the thread's sum of the
// unpacked values if SUM; COPY = false leaves the plane buffer unwritten.
template <typename T, int PD, bool SUM, bool COPY = true>
__device__ __forceinline__ float analysis_pyramid(const float* stg, int H, int W, int levels, int lg, FastDiv drw,
                                                  float* dst, int ds, const Levels& levs, int np, int ptid) {
    const LevelDst* lev = levs.d;
    const int G = 1 << lg, G2 = G * G;
    const int nreg_w = W >> (lg + 2);
    const int items = (H >> (lg + 2)) * nreg_w * G2;
    const int lane = ptid & 31;
    float sum = 0.f;
    for (int base = ptid & ~31; base < items; base += np) {
        const int item = base + lane;
        const bool valid = item < items;  // whole lane groups are valid or not
        const int it = valid ? item : 0;
        const int r = it >> (2 * lg), o = it & (G2 - 1);
        const int by = o >> lg, bx = o & (G - 1);
        const int rrow = fdiv(r, drw), rcol = r - rrow * nreg_w;
        const int brow = rrow * G + by, bcol = rcol * G + bx;  // 4x4 block coordinates
        const int r0 = 4 * brow, c0 = 4 * bcol;
        float4 v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = stg_load4<T>(stg, (r0 + q) * W + c0);
        if (valid) {
            if (COPY) {
#pragma unroll
                for (int q = 0; q < 4; ++q) sts4<PD>(dst + (r0 + q) * ds + c0, v[q]);
            }
            if (SUM) {
#pragma unroll
                for (int q = 0; q < 4; ++q) sum += (v[q].x + v[q].y) + (v[q].z + v[q].w);
            }
        }
        // Level 0: the block's 2x2 positions.
        float ll[2][2];
#pragma unroll
        for (int pi = 0; pi < 2; ++pi) {
            const float4 A = v[2 * pi], B = v[2 * pi + 1];
            float l0, h0, g0, d0, l1, h1, g1, d1;
            butterfly(A.x, A.y, B.x, B.y, l0, h0, g0, d0);
            butterfly(A.z, A.w, B.z, B.w, l1, h1, g1, d1);
            if (valid) {
                float* q = lev[0].base + (2 * brow + pi) * lev[0].stride + 2 * bcol;
                sts2<PD>(q, l0, l1);
                sts2<PD>(q + lev[0].sub, h0, h1);
                sts2<PD>(q + 2 * lev[0].sub, g0, g1);
                sts2<PD>(q + 3 * lev[0].sub, d0, d1);
            }
            ll[pi][0] = l0;
            ll[pi][1] = l1;
        }
        if (levels < 2) continue;
        // Level 1: the block itself.
        float mine, lh, hl, hh;
        butterfly(ll[0][0], ll[0][1], ll[1][0], ll[1][1], mine, lh, hl, hh);
        if (valid) {
            float* q = lev[1].base + brow * lev[1].stride + bcol;
            q[0] = mine; q[lev[1].sub] = lh; q[2 * lev[1].sub] = hl; q[3 * lev[1].sub] = hh;
        }
        // Levels 2..: the 2x2 group of lanes that differ in bit (l-2) of by / bx.
#pragma unroll
        for (int l = 2; l < 4; ++l) {
            if (l >= levels) break;
            const int sh = l - 2;
            const float vh = __shfl_xor_sync(0xffffffffu, mine, 1 << sh);
            const float vv = __shfl_xor_sync(0xffffffffu, mine, G << sh);
            const float vd = __shfl_xor_sync(0xffffffffu, vh, G << sh);
            const int py = (by >> sh) & 1, px = (bx >> sh) & 1;
            const float a = py ? (px ? vd : vv) : (px ? vh : mine);
            const float b = py ? (px ? vv : vd) : (px ? mine : vh);
            const float c = py ? (px ? vh : mine) : (px ? vd : vv);
            const float d = py ? (px ? mine : vh) : (px ? vv : vd);
            float nll;
            butterfly(a, b, c, d, nll, lh, hl, hh);
            const int m = (2 << sh) - 1;
            if (valid && (by & m) == 0 && (bx & m) == 0) {
                float* q = lev[l].base + (brow >> (l - 1)) * lev[l].stride + (bcol >> (l - 1));
                q[0] = nll; q[lev[l].sub] = lh; q[2 * lev[l].sub] = hl; q[3 * lev[l].sub] = hh;
            }
            mine = nll;
        }
    }
    return sum;
}

// ---------------------------------------------------------------------------
// A window row as NW2 aligned pairs e[k] = (r[2k], r[2k+1]), loaded straight
// into register pairs with 128-bit shared loads (a trailing odd pair with a
// 64-bit load).  Lanes walk 16-byte-apart windows, so every quarter-warp's
// 128-bit loads hit 8 distinct bank groups.  For output column pair jp
// (columns 2jp, 2jp+1) and tap v the inputs are columns 2jp+v and 2jp+v+1:
//   v even: the pair e[jp + v/2]              -> one packed FMA;
//   v odd:  e[jp + v/2].y and e[jp + v/2 + 1].x -> two scalar FMAs.
// No register moves are needed to build shifted pairs.
// ---------------------------------------------------------------------------
template <int NW2>
struct WinRow {
    float2 e[NW2];
    __device__ __forceinline__ void load(const float* rp) {
#pragma unroll
        for (int k = 0; k < NW2 / 2; ++k) {
            const float4 v = *reinterpret_cast<const float4*>(rp + 4 * k);
            e[2 * k] = make_float2(v.x, v.y);
            e[2 * k + 1] = make_float2(v.z, v.w);
        }
        if constexpr (NW2 % 2 == 1) e[NW2 - 1] = *reinterpret_cast<const float2*>(rp + 2 * (NW2 - 1));
    }
};

// acc (output columns 2jp, 2jp+1) += w * input columns (2jp+v, 2jp+v+1).
template <int NW2>
__device__ __forceinline__ float2 tap(float2 acc, float w, const WinRow<NW2>& row, int jp, int v) {
    if ((v & 1) == 0) return ffma2(make_float2(w, w), row.e[jp + (v >> 1)], acc);
    acc.x = fmaf(w, row.e[jp + (v >> 1)].y, acc.x);
    acc.y = fmaf(w, row.e[jp + (v >> 1) + 1].x, acc.y);
    return acc;
}

// acc (split by column parity) += d (columns 2jp, 2jp+1) * input columns (2jp+v, 2jp+v+1).
template <int NW2>
__device__ __forceinline__ float2 ctap(float2 acc, float2 d, const WinRow<NW2>& row, int jp, int v) {
    if ((v & 1) == 0) return ffma2(d, row.e[jp + (v >> 1)], acc);
    acc.x = fmaf(d.x, row.e[jp + (v >> 1)].y, acc.x);
    acc.y = fmaf(d.y, row.e[jp + (v >> 1) + 1].x, acc.y);
    return acc;
}

// Register-tiled depthwise conv of one TR x TC output tile (TC/2 column pairs):
//   out[o][j] = init + sum_{u<K, v<K} w[u*K+v] * win[(o+u)*stride + j+v]
// `win` is the 16-byte aligned window origin (input element (r0-p, c0-p)).
// Output row o is handed to emit(o, acc[o]) once its last input row is in.
template <int K, int TR, int TC, class Emit>
__device__ __forceinline__ void conv_tile(const float* __restrict__ win, int stride, const float (&w)[K * K],
                                          float2 init, Emit&& emit) {
    constexpr int NP = TC / 2;
    constexpr int NW2 = (TC + K - 1) / 2;
    float2 acc[TR][NP];
#pragma unroll
    for (int r = 0; r < TR + K - 1; ++r) {
        WinRow<NW2> row;
        row.load(win + r * stride);
#pragma unroll
        for (int u = 0; u < K; ++u) {
            const int o = r - u;
            if (o >= 0 && o < TR) {
#pragma unroll
                for (int jp = 0; jp < NP; ++jp) {
                    float2 a = (u == 0) ? init : acc[o][jp];
#pragma unroll
                    for (int v = 0; v < K; ++v) a = tap<NW2>(a, w[u * K + v], row, jp, v);
                    acc[o][jp] = a;
                }
            }
        }
        const int oc = r - (K - 1);
        if (oc >= 0 && oc < TR) emit(oc, acc[oc]);
    }
}

// Correlation sums of one thread: split by column parity (float2, the even
// taps as packed FMAs) for K <= 5; one float per tap for K = 7, whose 49
// float2 sums would not fit the register budget beside the D tile.
template <int K>
struct CorrAcc {
    using type = float2;
};
template <>
struct CorrAcc<7> {
    using type = float;
};
__device__ __forceinline__ float acc_total(float2 a) { return a.x + a.y; }
__device__ __forceinline__ float acc_total(float a) { return a; }
template <class A>
__device__ __forceinline__ A acc_zero() {
    if constexpr (std::is_same_v<A, float2>) return make_float2(0.f, 0.f); else return 0.f;
}

// Correlation of one TR x TC tile of D with the K x K shifts of S (float2
// sums split by column parity: sum the two halves at the end):
//   acc[u*K+v] += sum_{o<TR, j<TC} D[o][j] * S[o+u][j+v]
// `swin` is the S window origin (element (r0-p, c0-p)), `dt` the D tile origin.
// D rows load as 128-bit (DLD = 4) or 64-bit pairs (2; the faster of the two
// was measured per activation type), or as single floats (1) where the tile
// sits at an odd float offset (the interior of a padded buffer, p odd).
template <int K, int TR, int TC, int DLD>
__device__ __forceinline__ void corr_tile(const float* __restrict__ swin, int sstride,
                                          const float* __restrict__ dt, int dstride,
                                          typename CorrAcc<K>::type (&acc)[K * K]) {
    constexpr int NP = TC / 2;
    constexpr int NW2 = (TC + K - 1) / 2;
    float2 d[TR][NP];
#pragma unroll
    for (int r = 0; r < TR + K - 1; ++r) {
        if (r < TR) {
            if constexpr (DLD == 1) {
#pragma unroll
                for (int q = 0; q < NP; ++q)
                    d[r][q] = make_float2(dt[r * dstride + 2 * q], dt[r * dstride + 2 * q + 1]);
            } else if constexpr (DLD == 4) {
#pragma unroll
                for (int q = 0; q < NP / 2; ++q) {
                    const float4 v = *reinterpret_cast<const float4*>(dt + r * dstride + 4 * q);
                    d[r][2 * q] = make_float2(v.x, v.y);
                    d[r][2 * q + 1] = make_float2(v.z, v.w);
                }
            } else {
#pragma unroll
                for (int q = 0; q < NP; ++q) d[r][q] = *reinterpret_cast<const float2*>(dt + r * dstride + 2 * q);
            }
        }
        WinRow<NW2> row;
        row.load(swin + r * sstride);
#pragma unroll
        for (int u = 0; u < K; ++u) {
            const int o = r - u;
            if (o >= 0 && o < TR) {
#pragma unroll
                for (int v = 0; v < K; ++v) {
                    if constexpr (std::is_same_v<typename CorrAcc<K>::type, float2>) {
                        float2 a = acc[u * K + v];
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) a = ctap<NW2>(a, d[o][jp], row, jp, v);
                        acc[u * K + v] = a;
                    } else {
                        float a = acc[u * K + v];
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            // input columns 2jp+v and 2jp+v+1 of the window row
                            const int c = 2 * jp + v;
                            const float s0 = (c & 1) ? row.e[c >> 1].y : row.e[c >> 1].x;
                            const float s1 = (c & 1) ? row.e[(c + 1) >> 1].x : row.e[(c + 1) >> 1].y;
                            a = fmaf(d[o][jp].x, s0, a);
                            a = fmaf(d[o][jp].y, s1, a);
                        }
                        acc[u * K + v] = a;
                    }
                }
            }
        }
    }
}

template <int K>
__device__ __forceinline__ void load_weights(const float* wsm, float (&w)[K * K]) {
    constexpr int KK = K * K;
#pragma unroll
    for (int q = 0; q < KK / 4; ++q) {
        const float4 v = reinterpret_cast<const float4*>(wsm)[q];
        w[4 * q + 0] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int t = (KK / 4) * 4; t < KK; ++t) w[t] = wsm[t];
}

// 4^-(l+1), exact.
__device__ __forceinline__ float quarter_pow(int l) {
    float s = 0.25f;
    for (int i = 0; i < l; ++i) s *= 0.25f;
    return s;
}

// ---------------------------------------------------------------------------
// Staging and analysis of one plane by the threads [0, np) (ptid = thread
// index among them): the staged plane becomes the plane buffer (element
// (0,0) at `dst`, row stride ds, congruent to PD mod 4 floats) and the Haar
// subbands of every level (level l in bufs[l]; `pad` is the zero border of
// those buffers).  `sync()` synchronises the np threads between the levels
// that run one at a time (levels >= 4, or every level without the pyramid).
// ---------------------------------------------------------------------------
enum : int { kToS = 0, kToQ = 1, kToSS = 2 };

template <typename T, int PD, bool SUM, int DST, bool COPY = true, class Sync>
__device__ __forceinline__ float analyse_plane(float* sm, const Plan& P, const float* stg, float* dst, int ds, int pad,
                                               int np, int ptid, Sync&& sync) {
    const int H = P.H, W = P.W, L = P.L;
    // Level l's subbands go to P.S[l], P.Q[l] or P.SS[l] (DST); every index
    // below is a compile-time constant or goes through the parameter
    // directly, so no copy of the kernel parameter is made.
    auto buf = [&](int l) -> const Buf& { return DST == kToQ ? P.Q[l] : (DST == kToSS ? P.SS[l] : P.S[l]); };
    float sum;
    int done;  // levels complete
    if (P.pyr) {
        Levels lev;
#pragma unroll
        for (int l = 0; l < 4; ++l) {
            const Buf& b = buf(l < L ? l : 0);
            lev.d[l] = LevelDst{sm + b.base + pad * b.stride + pad, b.stride, b.sub};
        }
        sum = analysis_pyramid<T, PD, SUM, COPY>(stg, H, W, P.pyr_levels, P.pyr_lg, P.div_rw, dst, ds, lev, np, ptid);
        done = P.pyr_levels;
    } else {
        const Buf& b = buf(0);
        sum = unpack_level0<T, PD, SUM, COPY>(stg, H, W, P.div_q4, dst, ds, sm + b.base + pad * b.stride + pad, b.stride,
                                        b.sub, L >= 1, ptid, np);
        done = L >= 1 ? 1 : 0;
    }
    for (int l = done; l < L; ++l) {
        sync();
        const Buf& s0 = buf(l - 1);
        const Buf& s1 = buf(l);
        haar_level(sm + s0.base + pad * s0.stride + pad, s0.stride, H >> (l + 1), W >> (l + 1), P.div_m[l],
                   sm + s1.base + pad * s1.stride + pad, s1.stride, s1.sub, ptid, np);
    }
    return sum;
}

// ---------------------------------------------------------------------------
// Planes split into strips across a thread-block cluster.
// ---------------------------------------------------------------------------
// Barrier of everything that shares a plane: the CTA, or the whole cluster
// when the plane is split into strips or the cluster holds a channel octet
// (then it also orders the shared-memory accesses of the cluster's CTAs to
// each other's buffers).
template <bool GENERAL, bool OCT = false>
__device__ __forceinline__ void plane_sync(const Plan& P) {
    if constexpr (OCT) {
        cg::this_cluster().sync();
        return;
    }
    if constexpr (GENERAL) {
        if (P.nstrips > 1) {
            cg::this_cluster().sync();
            return;
        }
    }
    __syncthreads();
}

// The two halves of a cluster barrier, for work that can run between this
// CTA's arrival and the others': arrive (release: this CTA's earlier shared
// and distributed-shared stores become visible to the cluster) and wait
// (acquire).  Every thread of every CTA of the cluster executes them in the
// same order, alternating.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory"); }

// Send this CTA's rows that other strips hold as halo rows, for one padded
// buffer: nsub planes (1 or 4) of `rows` x `cols` interior elements behind
// `pad` border rows and columns.  Halo row i (i in [-pad, 0) or
// [rows, rows + pad)) of strip t = rank + d is plane row t*rows + i, i.e. row
// d*rows + i of this strip; the CTA that owns the row stores it straight into
// strip t's shared memory (same offsets: every CTA of the cluster runs the
// same plan).  Strip t below (d > 0) takes rows into its top halo, strip t
// above (d < 0) into its bottom halo, each a contiguous run of rows; only
// strips within ceil(pad / rows) can need this strip's rows (coarse levels may
// have fewer rows than pad).  Halo rows outside the plane are never written
// and stay zero.  A row goes whole, padding columns included (zero on both
// sides), as 16-byte stores from its 16-byte aligned start (the row stride
// covers the rounding).  The stores need no reply; the cluster barrier after
// them (release / acquire) makes them visible.
__device__ __forceinline__ void st_cluster4(unsigned addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_cluster2(unsigned addr, unsigned a, unsigned b) {
    asm volatile("st.shared::cluster.v2.b32 [%0], {%1, %2};\n" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void st_cluster1(unsigned addr, unsigned a) {
    asm volatile("st.shared::cluster.b32 [%0], %1;\n" ::"r"(addr), "r"(a) : "memory");
}

// NHWC channel octets: 4 outputs of pixels px .. px + 3 (one row; px a
// multiple of 4) of this CTA's channel into the output octet buffer of the
// CTA that owns them (og = 2: each pixel pair to its own owner, since a
// run boundary may fall between them).  oaddr: this CTA's output octet
// buffer (shared window address); ocol: byte offset of this CTA's channel
// row in it.
template <typename T>
__device__ __forceinline__ void st_octet_out(const Plan& P, unsigned oaddr, unsigned ocol, int px, float4 v) {
    auto dst_of = [&](int x) {
        const int owner = fdiv(x, P.div_opix), j = x - owner * P.opix;
        unsigned d;
        asm("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(d) : "r"(oaddr), "r"(owner));
        return d + ocol + (unsigned)j * (unsigned)sizeof(T);
    };
    if constexpr (sizeof(T) == 4) {
        if (P.og == 4) {
            st_cluster4(dst_of(px), v);
        } else {
            st_cluster2(dst_of(px), __float_as_uint(v.x), __float_as_uint(v.y));
            st_cluster2(dst_of(px + 2), __float_as_uint(v.z), __float_as_uint(v.w));
        }
    } else {
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
        __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
        const unsigned ua = *reinterpret_cast<uint32_t*>(&a), ub = *reinterpret_cast<uint32_t*>(&b);
        if (P.og == 4) {
            st_cluster2(dst_of(px), ua, ub);
        } else {
            st_cluster1(dst_of(px), ua);
            st_cluster1(dst_of(px + 2), ub);
        }
    }
}

// One buffer's halo rows (see above), as row groups: for every direction d
// and subband s, the run of halo rows i0 .. i0 + n - 1 of strip t = rank + d.
// The groups of all buffers are numbered in order; warp w takes every nw-th
// from w (the planner gives the buffer's chunks per row nq, its reach and g0,
// the offset of this buffer's first group that warp 0 takes, so no index is
// divided here).  A warp's lanes copy a row's 16-byte chunks, loading up to
// two per lane before storing them.
__device__ __forceinline__ void push_halo_rows(float* sm, unsigned local, const Buf& b, int nsub_lg, int rows, int nq,
                                               int reach, int g0, int pad, int rank, int nstrips, int warp, int lane,
                                               int nw) {
    const int ngroups = (2 * reach) << nsub_lg;
    int g = warp - g0;
    if (g < 0) g += nw;
    for (; g < ngroups; g += nw) {
        const int di = g >> nsub_lg, s = g - (di << nsub_lg);
        const int d = di < reach ? di - reach : di - reach + 1;
        const int t = rank + d;
        if (t < 0 || t >= nstrips) continue;
        int i0, n;
        if (d > 0) {
            i0 = max(-pad, -d * rows);
            n = min(0, (1 - d) * rows) - i0;
        } else {
            i0 = max(rows, -d * rows);
            n = min(rows + pad, (1 - d) * rows) - i0;
        }
        if (n <= 0) continue;
        unsigned tsm;  // strip t's copy of this shared memory in the cluster window
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(tsm) : "r"(local), "r"(t));
        for (int j = 0; j < n; ++j) {
            const int i = i0 + j;
            const int row = b.base + s * b.sub;
            const float* src = sm + row + (d * rows + i + pad) * b.stride;
            const unsigned dst = tsm + 4u * (unsigned)(row + (i + pad) * b.stride);
            for (int q0 = 0; q0 < nq; q0 += 64) {
                float4 v[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int q = q0 + lane + 32 * k;
                    if (q < nq) v[k] = *reinterpret_cast<const float4*>(src + 4 * q);
                }
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int q = q0 + lane + 32 * k;
                    if (q < nq) st_cluster4(dst + 16u * (unsigned)q, v[k]);
                }
            }
        }
    }
}

// Halo rows of the padded input strip (X) and, for the subband convs, of
// every level's padded subbands (S), sent to the strips that hold them.
__device__ __forceinline__ void push_halos(float* sm, const Plan& P, int rank, int tid, int nt) {
    const int p = P.p, warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
    const unsigned local = static_cast<unsigned>(__cvta_generic_to_shared(sm));
    push_halo_rows(sm, local, P.X, 0, P.H, P.hal_nq[0], P.hal_reach[0], P.hal_g0[0], p, rank, P.nstrips, warp, lane, nw);
#pragma unroll
    for (int l = 0; l < kMaxL; ++l)
        if (l < P.L)
            push_halo_rows(sm, local, P.S[l], 2, P.H >> (l + 1), P.hal_nq[l + 1], P.hal_reach[l + 1], P.hal_g0[l + 1], p,
                           rank, P.nstrips, warp, lane, nw);
}

// ---------------------------------------------------------------------------
// Forward (BWD = false) and input gradient (BWD = true).
// The input gradient is the same pass applied to dy with every kernel
// rotated by 180 degrees and no bias: the transpose of the forward map.
// ---------------------------------------------------------------------------
// One conv tile, its addressing decoded: window origin (padded S or X),
// output origin (Q or Y), folded weights, and the initial value (the folded
// bias for base tiles, 0 for subband tiles).
struct TileJob {
    int win, out, wts;  // float offsets into shared memory (out: into y when L = 0)
    int wstride, ostride;
    int row0;           // base tiles: first output row
    bool base, valid;
};

// Tile t of the forward index space (subband tiles, then base tiles from
// base_tid0).
__device__ __forceinline__ TileJob decode_tile(const Plan& P, int t, int TR, int TC) {
    TileJob j;
    j.valid = true;
    if (t < P.n_sub_tiles) {
        int cl = 1;
        while (t >= P.sub_begin[cl]) ++cl;  // sub_begin[cl] = end of class cl's tiles
        const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
        const int local = t - P.sub_begin[cl - 1];
        const int tr = fdiv(local, P.div_ntc[l]), tc = local - tr * P.ntc[l];
        const Buf& S = P.S[l];
        const Buf& Q = P.Q[l];
        j.win = S.base + s * S.sub + tr * TR * S.stride + tc * TC;
        j.out = Q.base + s * Q.sub + tr * TR * Q.stride + tc * TC;
        j.wts = P.wbase + cl * P.wcls;
        j.wstride = S.stride;
        j.ostride = Q.stride;
        j.row0 = 0;
        j.base = false;
    } else if (t >= P.base_tid0 && t < P.tile_end) {
        const int bt = t - P.base_tid0;
        const int tr = fdiv(bt, P.div_ntc[kMaxL]), tc = bt - tr * P.ntc[kMaxL];
        j.win = P.X.base + tr * TR * P.X.stride + tc * TC;
        j.row0 = tr * TR;
        // L >= 1: Y in shared memory.  L = 0: the output plane itself.
        j.out = P.L >= 1 ? P.Y.base + tr * TR * P.Y.stride + tc * TC : (tr * TR) * P.Wr + tc * TC;
        j.ostride = P.L >= 1 ? P.Y.stride : P.W;
        j.wts = P.wbase;
        j.wstride = P.X.stride;
        j.base = true;
    } else {
        j = TileJob{0, 0, 0, 0, 0, 0, false, false};
    }
    return j;
}

// Reformulation (2): the synthesis of one work item, output rows 2i, 2i+1 x
// columns 4q..4q+3 (the level-0 positions (i, 2q) and (i, 2q+1)), added to
// the base-branch outputs in Y and stored (the only HBM write; of the
// planes zero-padded on chip, only the first `rows` rows and Wr columns).
// Output (h, w) receives, for every level l, the signed sum of the four
// level-l conv outputs at (h >> (l+1), w >> (l+1)), with LH negated when
// bit l of h is set, HL when bit l of w is set and HH when exactly one is.
// The levels >= 1 are gathered Horner-style along the item's path: level l's
// signed sum for the level-(l-1) position on the path is added to that
// position's LL term, so the level-0 butterfly carries every coarser level.
// LL: the level count when the caller has dispatched on it (the Horner walk
// then has no per-level tests), or 0 for any L (P.L).
template <typename T, bool GUARD, int LL = 0>
__device__ __forceinline__ void synth_item(const float* sm, const Plan& P, T* yp, int t, int rows, unsigned oaddr = 0u,
                                           unsigned ocol = 0u) {
    const int i = fdiv(t, P.div_q4), q = t - i * (P.W >> 2);
    const int j0 = 2 * q;
    const int L = LL > 0 ? LL : P.L;
    float c0 = 0.f, c1 = 0.f;  // coarse terms for LL at (i, j0) and (i, j0 + 1)
    if (L >= 2) {
        float v = 0.f;
#pragma unroll
        for (int l = (LL > 0 ? LL : kMaxL) - 1; l >= 1; --l) {
            if (LL == 0 && l >= P.L) continue;
            const Buf& Q = P.Q[l];
            const float* r = sm + Q.base + (i >> l) * Q.stride + (j0 >> l);
            const float q0 = r[0] + v, q1 = r[Q.sub], q2 = r[2 * Q.sub], q3 = r[3 * Q.sub];
            const bool bi = (i >> (l - 1)) & 1;
            const float t0 = bi ? q0 - q1 : q0 + q1;
            const float t1 = bi ? q2 - q3 : q2 + q3;
            if (l > 1) {
                v = ((j0 >> (l - 1)) & 1) ? t0 - t1 : t0 + t1;
            } else {
                c0 = t0 + t1;
                c1 = t0 - t1;
            }
        }
    }
    const Buf& Q = P.Q[0];
    const float* r = sm + Q.base + i * Q.stride + j0;
    float2 ll = *reinterpret_cast<const float2*>(r);
    const float2 lh = *reinterpret_cast<const float2*>(r + Q.sub);
    const float2 hl = *reinterpret_cast<const float2*>(r + 2 * Q.sub);
    const float2 hh = *reinterpret_cast<const float2*>(r + 3 * Q.sub);
    ll.x += c0;
    ll.y += c1;
    const float* yr = sm + P.Y.base + (2 * i) * P.Y.stride + 4 * q;
    float4 top = *reinterpret_cast<const float4*>(yr);
    float4 bot = *reinterpret_cast<const float4*>(yr + P.Y.stride);
    {
        const float a0 = ll.x + lh.x, b0 = hl.x + hh.x, a1 = ll.y + lh.y, b1 = hl.y + hh.y;
        top.x += a0 + b0; top.y += a0 - b0; top.z += a1 + b1; top.w += a1 - b1;
    }
    {
        const float a0 = ll.x - lh.x, b0 = hl.x - hh.x, a1 = ll.y - lh.y, b1 = hl.y - hh.y;
        bot.x += a0 + b0; bot.y += a0 - b0; bot.z += a1 + b1; bot.w += a1 - b1;
    }
    // yp: this CTA's rows in y (row stride Wr elements, each act_es apart);
    // only real outputs are stored.
    if (!GUARD) {
        T* yo = yp + (size_t)(2 * i) * P.Wr + 4 * q;
        gst4<T>(yo, top);
        gst4<T>(yo + P.Wr, bot);
    } else if (oaddr != 0u) {
        // Channel octets (whole planes): to the owners' output octet buffers.
        const int px = (2 * i) * P.W + 4 * q;
        st_octet_out<T>(P, oaddr, ocol, px, top);
        st_octet_out<T>(P, oaddr, ocol, px + P.W, bot);
    } else if (4 * q < P.Wr) {
        const size_t es = act_es<true>(P);
        T* yo = yp + ((size_t)(2 * i) * P.Wr + 4 * q) * es;
        if (2 * i < rows) gst4s<T>(yo, top, es);
        if (2 * i + 1 < rows) gst4s<T>(yo + (size_t)P.Wr * es, bot, es);
    }
}

// NHWC channel octets.  load_octet: this CTA's run of opix pixels (from
// pixel crank * opix) of the 8 channels starting at `src` (channel 8o of
// pixel 0 of the plane pair's batch element), 8 * esize contiguous bytes a
// pixel, into the octet buffer by 16-byte cp.async (pixel j at byte
// 8 * esize * j).
__device__ __forceinline__ void load_octet(float* tb, const void* src, const Plan& P, int crank, int tid, int nt) {
    const int cpp = P.esize / 2;  // 16-byte chunks a pixel: 2 (fp32) or 1 (bf16)
    const size_t pstride = (size_t)P.C * P.esize;
    const char* g = static_cast<const char*>(src) + (size_t)crank * P.opix * pstride;
    char* t = reinterpret_cast<char*>(tb);
    const int n = P.opix * cpp;
    for (int ch = tid; ch < n; ch += nt) {
        const int j = cpp == 2 ? ch >> 1 : ch, h = ch - j * cpp;
        cp_async16(t + 16 * ch, g + (size_t)j * pstride + 16 * h);
    }
}

// scatter_octet: channel q of the octet buffer's pixels (the buffer at
// tbuf, P.tbuf if negative) into CTA q's
// staging at `stg` (pixel crank * opix + j of the plane, stored format), og
// pixels a step as one distributed shared store per channel (og = 4: 16
// bytes in fp32, 8 in bf16; og = 2: 8 or 4).  The cluster barrier after it
// makes the stores visible.
__device__ __forceinline__ void scatter_octet(float* sm, int stg, const Plan& P, int crank, int tid, int nt,
                                              int tbuf = -1) {
    const unsigned local = static_cast<unsigned>(__cvta_generic_to_shared(sm + stg));
    // CTA q's copy of the staging (mapped per store: few registers live, the
    // weight gradient's correlation sums stay in registers meanwhile).
    auto remote = [&](int q) {
        unsigned a;
        asm("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(a) : "r"(local), "r"(q));
        return a;
    };
    const float* tb = sm + (tbuf >= 0 ? tbuf : P.tbuf);
    if (P.og == 2) {
        // Two pixels a step: 8-byte (fp32) or 4-byte (bf16) stores.
        for (int gq = tid; gq < (P.opix >> 1); gq += nt) {
            const int j = 2 * gq;
            const unsigned off = (unsigned)(crank * P.opix + j) * (unsigned)P.esize;
            if (P.esize == 4) {
                const float4* t = reinterpret_cast<const float4*>(tb) + 2 * j;
                const float4 a0 = t[0], b0 = t[1], a1 = t[2], b1 = t[3];
                st_cluster2(remote(0) + off, __float_as_uint(a0.x), __float_as_uint(a1.x));
                st_cluster2(remote(1) + off, __float_as_uint(a0.y), __float_as_uint(a1.y));
                st_cluster2(remote(2) + off, __float_as_uint(a0.z), __float_as_uint(a1.z));
                st_cluster2(remote(3) + off, __float_as_uint(a0.w), __float_as_uint(a1.w));
                st_cluster2(remote(4) + off, __float_as_uint(b0.x), __float_as_uint(b1.x));
                st_cluster2(remote(5) + off, __float_as_uint(b0.y), __float_as_uint(b1.y));
                st_cluster2(remote(6) + off, __float_as_uint(b0.z), __float_as_uint(b1.z));
                st_cluster2(remote(7) + off, __float_as_uint(b0.w), __float_as_uint(b1.w));
            } else {
                const uint4* t = reinterpret_cast<const uint4*>(tb) + j;
                const uint4 r0 = t[0], r1 = t[1];
                const unsigned w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    st_cluster1(remote(q) + off, __byte_perm(w0[q >> 1], w1[q >> 1], (q & 1) ? 0x7632u : 0x5410u));
            }
        }
        return;
    }
    const int ng = P.opix >> 2;
    for (int gq = tid; gq < ng; gq += nt) {
        const int j = 4 * gq;
        const unsigned off = (unsigned)(crank * P.opix + j) * (unsigned)P.esize;
        if (P.esize == 4) {
            // Pixel i's channels 0-3 at float4 2i, channels 4-7 at 2i + 1.
            const float4* t = reinterpret_cast<const float4*>(tb) + 2 * j;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float4 v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) v[i] = t[2 * i + h];
                st_cluster4(remote(4 * h) + off, make_float4(v[0].x, v[1].x, v[2].x, v[3].x));
                st_cluster4(remote(4 * h + 1) + off, make_float4(v[0].y, v[1].y, v[2].y, v[3].y));
                st_cluster4(remote(4 * h + 2) + off, make_float4(v[0].z, v[1].z, v[2].z, v[3].z));
                st_cluster4(remote(4 * h + 3) + off, make_float4(v[0].w, v[1].w, v[2].w, v[3].w));
            }
        } else {
            // bf16: word w of a pixel holds channels 2w (low half) and 2w + 1.
            const uint4* t = reinterpret_cast<const uint4*>(tb) + j;
            const uint4 r0 = t[0], r1 = t[1], r2 = t[2], r3 = t[3];
            const unsigned w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
            const unsigned w2[4] = {r2.x, r2.y, r2.z, r2.w}, w3[4] = {r3.x, r3.y, r3.z, r3.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const unsigned sel = (q & 1) ? 0x7632u : 0x5410u;
                st_cluster2(remote(q) + off, __byte_perm(w0[q >> 1], w1[q >> 1], sel),
                            __byte_perm(w2[q >> 1], w3[q >> 1], sel));
            }
        }
    }
}

// stream_octet_out: this CTA's pixels (crank * opix + j) of the output
// octet buffer ([8 channels][opix pixels], stored format) to y, og pixels a
// step, the 8 channels of a pixel as one 32-byte (fp32) or 16-byte (bf16)
// run; `dst` is channel 8o of pixel 0 of the plane's batch element.
template <typename T>
__device__ __forceinline__ void stream_octet_out(const float* sm, const Plan& P, T* dst, int crank, int tid, int nt) {
    const size_t pstride = (size_t)P.C;
    T* g = dst + (size_t)crank * P.opix * pstride;
    const T* ob = reinterpret_cast<const T*>(sm + P.obuf);
    if (P.og == 2) {
        // Two pixels a step.
        for (int gq = tid; gq < (P.opix >> 1); gq += nt) {
            const int j = 2 * gq;
            if constexpr (sizeof(T) == 4) {
                float2 c[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) c[q] = *reinterpret_cast<const float2*>(ob + (size_t)q * P.opix + j);
                float* o = reinterpret_cast<float*>(g + (size_t)j * pstride);
                *reinterpret_cast<float4*>(o) = make_float4(c[0].x, c[1].x, c[2].x, c[3].x);
                *reinterpret_cast<float4*>(o + 4) = make_float4(c[4].x, c[5].x, c[6].x, c[7].x);
                *reinterpret_cast<float4*>(o + pstride) = make_float4(c[0].y, c[1].y, c[2].y, c[3].y);
                *reinterpret_cast<float4*>(o + pstride + 4) = make_float4(c[4].y, c[5].y, c[6].y, c[7].y);
            } else {
                unsigned c[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) c[q] = *reinterpret_cast<const unsigned*>(ob + (size_t)q * P.opix + j);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const unsigned sel = i ? 0x7632u : 0x5410u;
                    uint4 v;
                    v.x = __byte_perm(c[0], c[1], sel);
                    v.y = __byte_perm(c[2], c[3], sel);
                    v.z = __byte_perm(c[4], c[5], sel);
                    v.w = __byte_perm(c[6], c[7], sel);
                    *reinterpret_cast<uint4*>(g + (size_t)(j + i) * pstride) = v;
                }
            }
        }
        return;
    }
    const int ng = P.opix >> 2;
    for (int gq = tid; gq < ng; gq += nt) {
        const int j = 4 * gq;
        if constexpr (sizeof(T) == 4) {
            float4 c[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) c[q] = *reinterpret_cast<const float4*>(ob + (size_t)q * P.opix + j);
            float* o = reinterpret_cast<float*>(g + (size_t)j * pstride);
            const size_t ps = pstride;
            *reinterpret_cast<float4*>(o) = make_float4(c[0].x, c[1].x, c[2].x, c[3].x);
            *reinterpret_cast<float4*>(o + 4) = make_float4(c[4].x, c[5].x, c[6].x, c[7].x);
            *reinterpret_cast<float4*>(o + ps) = make_float4(c[0].y, c[1].y, c[2].y, c[3].y);
            *reinterpret_cast<float4*>(o + ps + 4) = make_float4(c[4].y, c[5].y, c[6].y, c[7].y);
            *reinterpret_cast<float4*>(o + 2 * ps) = make_float4(c[0].z, c[1].z, c[2].z, c[3].z);
            *reinterpret_cast<float4*>(o + 2 * ps + 4) = make_float4(c[4].z, c[5].z, c[6].z, c[7].z);
            *reinterpret_cast<float4*>(o + 3 * ps) = make_float4(c[0].w, c[1].w, c[2].w, c[3].w);
            *reinterpret_cast<float4*>(o + 3 * ps + 4) = make_float4(c[4].w, c[5].w, c[6].w, c[7].w);
        } else {
            // bf16: channel q's 4 pixels are one 8-byte word pair (pixel i in
            // half i & 1 of word i >> 1).
            uint2 c[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) c[q] = *reinterpret_cast<const uint2*>(ob + (size_t)q * P.opix + j);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const unsigned sel = (i & 1) ? 0x7632u : 0x5410u;
                auto w = [&](int q) { return (i >> 1) ? c[q].y : c[q].x; };
                uint4 v;
                v.x = __byte_perm(w(0), w(1), sel);
                v.y = __byte_perm(w(2), w(3), sel);
                v.z = __byte_perm(w(4), w(5), sel);
                v.w = __byte_perm(w(6), w(7), sel);
                *reinterpret_cast<uint4*>(g + (size_t)(j + i) * pstride) = v;
            }
        }
    }
}

// Shared pieces of the two forward schedules (NHW: the NHWC layout may occur).
template <int K, typename T, bool BWD, bool NHW>
struct FusedCtx {
    float* sm;
    const Plan& P;
    const T* x;
    const float *base_w, *base_b, *base_scale, *wt_w, *wt_scale;
    long long units;
    int u0, u1;
    size_t plane_elems;  // Hr * Wr
    size_t strip_off;    // first element of this CTA's strip within a plane (plane-relative index)

    // Units run channel-major: unit u is plane (b, c) = (u mod B, u / B).
    // Offset of this CTA's rows of plane (b, c).
    __device__ __forceinline__ size_t rows_of(int b, int c) const {
        return plane_origin<NHW>(P, b, c) + strip_off * act_es<NHW>(P);
    }
    __device__ __forceinline__ const T* src(int b, int c) const { return x + rows_of(b, c); }
    // Reformulation (3): fold the scales (and the Haar factors) into the
    // weights of channel c (threads [0, np)).
    __device__ __forceinline__ void fold(int c, int np, int ptid) const {
        constexpr int KK = K * K;
        const int ncls = 1 + 4 * P.L;
        for (int t = ptid; t < ncls * KK; t += np) {
            const int cl = t / KK, tap = t - cl * KK;
            const int src_tap = BWD ? (KK - 1 - tap) : tap;
            float v;
            if (cl == 0) {
                v = base_scale[c] * base_w[c * KK + src_tap];
            } else {
                const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
                const int pi = (l * P.C + c) * 4 + s;
                v = (wt_scale[pi] * wt_w[pi * KK + src_tap]) * quarter_pow(l);
            }
            sm[P.wbase + cl * P.wcls + tap] = v;
        }
        if (ptid == 0) sm[P.bias] = BWD ? 0.f : base_scale[c] * base_b[c];
    }
};

// Forward / input gradient.  Persistent CTAs walk a run of planes with two
// CTA barriers per plane:
//   phase A(u): fold the weights when the channel changes and analyse the
//               staged plane u (writes X, S); the threads the analysis leaves
//               idle start on the synthesis of plane u-1 (reads Q, Y; writes y);
//   phase B(u): start staging plane u+1, then run every conv tile of plane u:
//               subband tiles write Q, base tiles write Y (y itself if L = 0).
// Within a phase the buffers written (A: X, S, weights; B: staging, Q, Y) and
// the buffers read (A: staging, Q, Y; B: S, X, weights) are disjoint.
// GENERAL: planes split into strips across a cluster and / or zero-padded on
// chip, or NHWC activations (a separate instantiation, so the common walk of
// whole planes that are multiples of 2^L carries none of that code).  OCT
// (with GENERAL): NHWC channel octets, the barriers cluster-wide, staging
// by octet runs and scatters, outputs through the owners' output octet
// buffers, written out in phase B of the next plane.
template <int K, int TR, int TC, typename T, bool BWD, bool GENERAL, bool OCT = false>
__global__ void __launch_bounds__(GENERAL ? kStripMaxThreads : kFusedMaxThreads, GENERAL ? 1 : 2) wtconv_fused_kernel(
    const T* __restrict__ x, const float* __restrict__ base_w, const float* __restrict__ base_b,
    const float* __restrict__ base_scale, const float* __restrict__ wt_w,
    const float* __restrict__ wt_scale, T* __restrict__ y, const Plan P) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    constexpr int p = K / 2, KK = K * K, NP = TC / 2;
    static_assert(TC == 4, "4-column tiles");
    const int tid = threadIdx.x, nt = blockDim.x;
    static_assert(!OCT || GENERAL, "channel octets run in the general walk");
    const long long units = (long long)P.B * (OCT ? P.C / 8 : P.C);
    // With strips, the nstrips CTAs of a cluster walk the same planes; with
    // channel octets (NHWC), the 8 CTAs of a cluster walk the same (b, octet)
    // units, CTA r taking channel 8 * octet + r.
    const bool strips = GENERAL && P.nstrips > 1;
    constexpr bool oct = OCT;
    const int cs = OCT ? 8 : (GENERAL ? P.nstrips : 1);
    const int crank = cs > 1 ? (int)cg::this_cluster().block_rank() : 0;
    const int rank = strips ? crank : 0;  // strip of the plane
    const long long team = cs > 1 ? blockIdx.x / cs : blockIdx.x;
    const long long teams = cs > 1 ? gridDim.x / cs : gridDim.x;
    FusedCtx<K, T, BWD, GENERAL> cx{sm, P, x, base_w, base_b, base_scale, wt_w, wt_scale, units,
                           (int)((team * units) / teams), (int)(((team + 1) * units) / teams),
                           (size_t)P.Hr * P.Wr, (size_t)rank * P.H * P.Wr};
    const int myrows = real_rows(P, rank);
    const int u0 = cx.u0, u1 = cx.u1;
    auto csync = [&]() { __syncthreads(); };
    float* X0 = sm + P.X.base + p * P.X.stride + p;
    int ft = tid - P.fin_off;
    if (ft < 0) ft += nt;
    // In the one-tile-per-thread schedule each thread's tile is fixed.
    const TileJob fixed = P.merged ? decode_tile(P, tid, TR, TC) : TileJob{0, 0, 0, 0, 0, 0, false, false};

    zero_smem(sm, P.smem_floats, tid, nt);
    __syncthreads();
    // (b, c) of the plane being analysed / tiled, of the previous plane, and of the next
    // (with octets, c is the octet and chan(c) this CTA's channel).
    int cur_b = u0 % P.B, cur_c = u0 / P.B;
    int prev_b = 0, prev_c = 0;
    auto chan = [&](int c) { return oct ? 8 * c + crank : c; };
    auto stage = [&](const T* src) {
        if constexpr (GENERAL) {
            stage_rows(sm + P.stg, src, P, myrows, tid, nt);
        } else {
            stage_plane(sm + P.stg, src, P.plane_chunks, tid, nt);
        }
    };
    auto octet_src = [&](int b, int c) { return x + plane_origin<GENERAL>(P, b, 8 * c); };
    // Octets with a synthesis (L >= 1): outputs go through the owners' output
    // octet buffers (oaddr != 0), written out in phase B of the next plane.
    const bool oct_out = oct && P.L >= 1;
    const unsigned oaddr = oct_out ? static_cast<unsigned>(__cvta_generic_to_shared(sm + P.obuf)) : 0u;
    const unsigned ocol = (unsigned)crank * (unsigned)P.opix * (unsigned)sizeof(T);
    if (oct) {
        // Octets: the first plane's octet run, then its scatter once every
        // CTA of the cluster runs and has zeroed its shared memory.
        if (u0 < u1) load_octet(sm + P.tbuf, octet_src(cur_b, cur_c), P, crank, tid, nt);
        cp_async_commit();
        cp_async_wait_all();
        plane_sync<GENERAL, OCT>(P);
        if (u0 < u1) scatter_octet(sm, P.stg, P, crank, tid, nt);
    } else {
        if (u0 < u1) stage(cx.src(cur_b, cur_c));
        cp_async_commit();
    }
    int folded_c = -1;
    for (int u = u0; u <= u1; ++u) {
        cp_async_wait_all();
        plane_sync<GENERAL, OCT>(P);  // plane u staged; every tile of plane u-1 done (its halo rows are free)
        int nb = cur_b + 1, nc = cur_c;
        if (nb == P.B) {
            nb = 0;
            ++nc;
        }
        // Phase A.
        if (u < u1) {
            if (oct) {
                // The next plane's octet run (the buffer's last reader, the
                // scatter of phase B(u-1), is behind the barrier above).
                if (u + 1 < u1) load_octet(sm + P.tbuf, octet_src(nb, nc), P, crank, tid, nt);
                cp_async_commit();
            }
            if (cur_c != folded_c) {
                cx.fold(chan(cur_c), nt, tid);
                folded_c = cur_c;
            }
            analyse_plane<T, p, false, kToS>(sm, P, sm + P.stg, X0, P.X.stride, p, nt, tid, csync);
        }
        if (u > u0 && P.L >= 1) {
            T* yp = y + cx.rows_of(prev_b, chan(prev_c));
            // One synthesis loop per level count (uniform dispatch), so that
            // the items' level walk is unrolled with no per-level tests.
            switch (P.L) {
                case 1: for (int t = ft; t < P.n_fin; t += nt) synth_item<T, GENERAL, 1>(sm, P, yp, t, myrows, oaddr, ocol); break;
                case 2: for (int t = ft; t < P.n_fin; t += nt) synth_item<T, GENERAL, 2>(sm, P, yp, t, myrows, oaddr, ocol); break;
                case 3: for (int t = ft; t < P.n_fin; t += nt) synth_item<T, GENERAL, 3>(sm, P, yp, t, myrows, oaddr, ocol); break;
                case 4: for (int t = ft; t < P.n_fin; t += nt) synth_item<T, GENERAL, 4>(sm, P, yp, t, myrows, oaddr, ocol); break;
                default: for (int t = ft; t < P.n_fin; t += nt) synth_item<T, GENERAL>(sm, P, yp, t, myrows, oaddr, ocol); break;
            }
        }
        if (u == u1) break;
        if (strips) {
            __syncthreads();  // this strip's X and S of plane u complete
            push_halos(sm, P, rank, tid, nt);
        }
        if (oct) cp_async_wait_all();  // this thread's chunks of the next octet run
        plane_sync<GENERAL, OCT>(P);  // X, S and halo rows of plane u ready (every strip); Q and Y of plane u-1 consumed
        // Phase B.
        if (oct) {
            // Every CTA of the cluster is past its analysis of plane u: the
            // next plane goes into all eight stagings; and past its synthesis
            // of plane u-1: this CTA's pixels of it are complete.
            if (u + 1 < u1) scatter_octet(sm, P.stg, P, crank, tid, nt);
            if (oct_out && u > u0) stream_octet_out<T>(sm, P, y + plane_origin<GENERAL>(P, prev_b, 8 * prev_c), crank, tid, nt);
        } else {
            if (u + 1 < u1) stage(cx.src(nb, nc));
            cp_async_commit();
        }
        // One tile loop per output kind (a uniform branch), each with a
        // single conv-tile call site.
        if (P.L >= 1) {
            // Subband tiles write Q, base tiles Y (both on chip).
            for (int t = tid; t < P.tile_end; t += nt) {
                const TileJob j = P.merged ? fixed : decode_tile(P, t, TR, TC);
                if (!j.valid) continue;
                float w[KK];
                load_weights<K>(sm + j.wts, w);
                const float b0 = j.base ? sm[P.bias] : 0.f;
                float* out = sm + j.out;
                const int os = j.ostride;
                conv_tile<K, TR, TC>(sm + j.win, j.wstride, w, make_float2(b0, b0), [&](int o, float2(&a)[NP]) {
                    *reinterpret_cast<float4*>(out + o * os) = make_float4(a[0].x, a[0].y, a[1].x, a[1].y);
                });
            }
        } else {
            // L = 0: every tile is a base tile, and the base branch is the
            // whole output.
            const size_t es = act_es<GENERAL>(P);
            for (int t = tid; t < P.tile_end; t += nt) {
                const TileJob j = P.merged ? fixed : decode_tile(P, t, TR, TC);
                if (!j.valid) continue;
                float w[KK];
                load_weights<K>(sm + j.wts, w);
                const float b0 = sm[P.bias];
                T* yo = y + cx.rows_of(cur_b, chan(cur_c)) + (size_t)j.out * es;
                const int h0 = j.row0;
                conv_tile<K, TR, TC>(sm + j.win, j.wstride, w, make_float2(b0, b0), [&](int o, float2(&a)[NP]) {
                    if (h0 + o < myrows)
                        gst4s<T>(yo + (size_t)o * P.Wr * es, make_float4(a[0].x, a[0].y, a[1].x, a[1].y), es);
                });
            }
        }
        prev_b = cur_b;
        prev_c = cur_c;
        cur_b = nb;
        cur_c = nc;
    }
    cp_async_wait_all();
    if (oct_out && u1 > u0) {
        plane_sync<GENERAL, OCT>(P);  // the last plane's outputs are in every owner's buffer
        stream_octet_out<T>(sm, P, y + plane_origin<GENERAL>(P, prev_b, 8 * prev_c), crank, tid, nt);
    }
}

// ---------------------------------------------------------------------------
// Weight gradient, final step (in the tail of the kernels that write the
// partial vectors): the last CTA of channel c to publish its partial vector
// sums the channel's `parts` vectors in a fixed order (so the result does not
// depend on which CTA is last), scales the level sums by 4^-(l+1) (they were
// accumulated on un-normalised subbands), and writes the five gradients; each
// dot product is one warp's fixed xor-tree.  Arrival counters (one per
// channel) are zero before the launch and reset by the last CTA.
// ---------------------------------------------------------------------------
struct GradArgs {
    const float *base_w, *base_b, *base_scale, *wt_w, *wt_scale;
    float *d_base_w, *d_base_b, *d_base_scale, *d_wt_w, *d_wt_scale;
    unsigned* counters;
};

__device__ __forceinline__ void finish_channel_if_last(float* sm, const Plan& P, const float* part, int c,
                                                       const GradArgs& ga, int tid, int nt) {
    const int KK = P.k * P.k, L = P.L, C = P.C, nv = P.nv, ncls = 1 + 4 * L;
    // Shared scratch from offset 0 (every buffer is dead by now): gsum, wts,
    // then the "last" flag.
    int* last = reinterpret_cast<int*>(sm + nv + ncls * KK);
    __syncthreads();  // this CTA's partial vector is written; the reduction scratch is read
    if (tid == 0) {
        __threadfence();  // publish it before counting in
        *last = atomicAdd(&ga.counters[c], 1u) == (unsigned)(P.parts - 1);
    }
    __syncthreads();
    if (!*last) return;
    __threadfence();  // every partial vector of the channel is visible
    float* gsum = sm;       // nv: summed partials
    float* wts = sm + nv;   // ncls*KK: the channel's base_w then wt_w[l][c][s]
    const float* pc = part + (size_t)c * P.parts * nv;
    for (int t = tid; t < nv; t += nt) {
        float s = 0.f;
        for (int g = 0; g < P.parts; ++g) s += __ldcg(pc + (size_t)g * nv + t);
        gsum[t] = s;
    }
    for (int t = tid; t < ncls * KK; t += nt) {
        const int cl = t / KK, tap = t - cl * KK;
        if (cl == 0) {
            wts[t] = ga.base_w[c * KK + tap];
        } else {
            const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
            wts[t] = ga.wt_w[((l * C + c) * 4 + s) * KK + tap];
        }
    }
    __syncthreads();
    for (int t = tid; t < 4 * L * KK; t += nt) {
        const int l = t / (4 * KK);
        gsum[KK + t] *= quarter_pow(l);
    }
    __syncthreads();
    const float sdy = gsum[ncls * KK];
    const float bs = ga.base_scale[c];
    for (int t = tid; t < KK; t += nt) ga.d_base_w[c * KK + t] = bs * gsum[t];
    for (int t = tid; t < 4 * L * KK; t += nt) {
        const int k2 = t / KK, tap = t - k2 * KK;
        const int l = k2 >> 2, s = k2 & 3;
        const int pi = (l * C + c) * 4 + s;
        ga.d_wt_w[pi * KK + tap] = ga.wt_scale[pi] * gsum[KK + t];
    }
    const int warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
    for (int cl = warp; cl < ncls; cl += nw) {
        float a = 0.f;
        for (int tap = lane; tap < KK; tap += 32) a = fmaf(wts[cl * KK + tap], gsum[cl * KK + tap], a);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) {
            if (cl == 0) {
                ga.d_base_b[c] = bs * sdy;
                ga.d_base_scale[c] = fmaf(ga.base_b[c], sdy, a);
            } else {
                const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
                ga.d_wt_scale[(l * C + c) * 4 + s] = a;
            }
        }
    }
    if (tid == 0) ga.counters[c] = 0u;
}

// ---------------------------------------------------------------------------
// Weight gradient, stage 1: grid (C, groups).  The CTA of (c, g) walks the
// planes b = g, g + groups, ... of channel c, staging the next (x, dy) pair
// while it computes the current one.  Thread t owns a run of tiles of one
// class (base, or level l subband s) for the whole walk and accumulates their
// K*K correlation sums in registers; the CTA then reduces each class over its
// threads in a fixed order and writes one partial vector (plus sum dy).
// ---------------------------------------------------------------------------
// GENERAL: the plane is split into strips across a cluster and / or
// zero-padded on chip, or NHWC activations (a separate instantiation, so
// whole-plane walks keep every register for the sums).  OCT (with GENERAL):
// NHWC channel octets, clusters of the 8 channels of an octet; the x run and
// then the dy run of the next plane go through the octet buffer (the dy run
// loaded during the correlation tiles and scattered after them).
template <int K, int TR, int TC, typename T, bool GENERAL, bool OCT = false>
__global__ void __launch_bounds__(GENERAL ? kStripMaxThreads : kBwdwMaxThreads, GENERAL ? 1 : 2) wtconv_bwdw_partial_kernel(
    const T* __restrict__ x, const T* __restrict__ dy, float* __restrict__ part, const GradArgs ga, const Plan P) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    constexpr int p = K / 2, KK = K * K;
    constexpr int DLD = sizeof(T) == 2 ? 4 : 2;
    const int tid = threadIdx.x, nt = blockDim.x;
    // blockIdx.x = c * nstrips + (strip rank within the cluster); with NHWC
    // channel octets, clusters of the 8 channels of an octet (rank c mod 8).
    static_assert(!OCT || GENERAL, "channel octets run in the general walk");
    const bool strips = GENERAL && P.nstrips > 1;
    constexpr bool oct = OCT;
    const int rank = strips ? (int)cg::this_cluster().block_rank() : 0;
    const int crank = oct ? (int)cg::this_cluster().block_rank() : 0;
    const int c = strips ? blockIdx.x / P.nstrips : blockIdx.x, g = blockIdx.y, G = P.groups;
    const size_t strip_off = (size_t)rank * P.H * P.Wr * act_es<GENERAL>(P);
    const int myrows = real_rows(P, rank);
    auto csync = [&]() { __syncthreads(); };

    // dys: the correlation tiles read dy straight from its staging buffer
    // (P.DY aliases it; strips of fp32 planes whose height is whole tiles),
    // so the next dy strip is staged only after them.
    const bool dys = GENERAL && P.dy_stg;
    zero_smem(sm, P.smem_floats, tid, nt);
    __syncthreads();
    auto stage = [&](size_t off, bool with_dy) {
        if constexpr (GENERAL) {
            stage_rows(sm + P.stg, x + off, P, myrows, tid, nt);
            if (with_dy) stage_rows(sm + P.stg + P.stg_floats, dy + off, P, myrows, tid, nt);
        } else {
            stage_plane(sm + P.stg, x + off, P.plane_chunks, tid, nt);
            stage_plane(sm + P.stg + P.stg_floats, dy + off, P.plane_chunks, tid, nt);
        }
    };
    // Octets: the x and dy runs of the octet's planes go through one octet
    // buffer in turn, each scattered into the cluster's stagings.
    const size_t oct_off = (size_t)(c - crank);  // channel 8o: NHWC element offset of the octet
    auto octet_run = [&](const T* src, int b) {
        load_octet(sm + P.tbuf, src + plane_origin<GENERAL>(P, b, 0) + oct_off, P, crank, tid, nt);
    };
    if (oct) {
        if (g < P.B) octet_run(x, g);
        cp_async_commit();
        cp_async_wait_all();
        plane_sync<GENERAL, OCT>(P);  // every CTA of the cluster running, its shared memory zeroed; x run complete
        if (g < P.B) scatter_octet(sm, P.stg, P, crank, tid, nt);
        __syncthreads();  // the octet buffer consumed
        if (g < P.B) octet_run(dy, g);
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        if (g < P.B) scatter_octet(sm, P.stg + P.stg_floats, P, crank, tid, nt);
    } else {
        if (g < P.B) stage(plane_origin<GENERAL>(P, g, c) + strip_off, true);
        cp_async_commit();
    }

    // This thread's class and its run of that class's tiles.
    int cl = -1, first = 0, cnt = 0;
    if (tid < P.cls_thr[1 + 4 * P.L]) {
        cl = 0;
        while (tid >= P.cls_thr[cl + 1]) ++cl;
        first = (tid - P.cls_thr[cl]) * P.tpt;
        cnt = min(P.tpt, P.cls_tiles[cl] - first);
    }
    const int lvl = cl <= 0 ? kMaxL : ((cl - 1) >> 2);
    // The class's window buffer (padded X or subband S) and dy buffer (DY or
    // its subband Q), the same for every plane: one tile call site, no
    // per-plane buffer selection.
    int wb = 0, ws = 0, db = 0, dsd = 0;
    if (cl == 0) {
        wb = P.X.base; ws = P.X.stride; db = P.DY.base; dsd = P.DY.stride;
    } else if (cl > 0) {
        const int l = (cl - 1) >> 2, s2 = (cl - 1) & 3;
        wb = P.S[l].base + s2 * P.S[l].sub; ws = P.S[l].stride;
        db = P.Q[l].base + s2 * P.Q[l].sub; dsd = P.Q[l].stride;
    }
    using Acc = typename CorrAcc<K>::type;
    Acc acc[KK];
#pragma unroll
    for (int t = 0; t < KK; ++t) acc[t] = acc_zero<Acc>();
    float sdy = 0.f, sdy_c = 0.f;  // compensated running sum of dy over the walk

    float* X0 = sm + P.X.base + p * P.X.stride + p;
    for (int b = g; b < P.B; b += G) {
        cp_async_wait_all();
        plane_sync<GENERAL, OCT>(P);  // staged pair complete; previous correlations done (halo rows free)
        if (oct) {
            if (b + G < P.B) octet_run(x, b + G);  // the buffer's last reader is behind the barrier above
            cp_async_commit();
        }
        analyse_plane<T, p, false, kToS>(sm, P, sm + P.stg, X0, P.X.stride, p, nt, tid, csync);
        const float s = dys ? analyse_plane<T, 0, true, kToQ, false>(sm, P, sm + P.stg + P.stg_floats, sm + P.DY.base,
                                                                     P.DY.stride, 0, nt, tid, csync)
                            : analyse_plane<T, 0, true, kToQ>(sm, P, sm + P.stg + P.stg_floats, sm + P.DY.base,
                                                              P.DY.stride, 0, nt, tid, csync);
        {
            const float yv = s - sdy_c;
            const float tv = sdy + yv;
            sdy_c = (tv - sdy) - yv;
            sdy = tv;
        }
        if (strips) {
            __syncthreads();  // this strip's analyses complete (staging consumed)
            push_halos(sm, P, rank, tid, nt);
            cluster_arrive();  // this strip's halo stores released
            if (b + G < P.B) stage(plane_origin<GENERAL>(P, b + G, c) + strip_off, !dys);
            cp_async_commit();
            cluster_wait();  // every strip's X, S and halo rows ready
        } else if (oct) {
            cp_async_wait_all();     // this thread's chunks of the next x run
            plane_sync<GENERAL, OCT>(P);  // both analyses complete in every CTA of the cluster
            if (b + G < P.B) scatter_octet(sm, P.stg, P, crank, tid, nt);
            __syncthreads();  // the octet buffer consumed
            if (b + G < P.B) octet_run(dy, b + G);
            cp_async_commit();
        } else {
            plane_sync<GENERAL, OCT>(P);  // both analyses complete
            if (b + G < P.B) stage(plane_origin<GENERAL>(P, b + G, c) + strip_off, !dys);
            cp_async_commit();
        }
        for (int k = 0; k < cnt; ++k) {
            const int local = first + k;
            const int tr = fdiv(local, P.div_ntc[lvl]), tc = local - tr * P.ntc[lvl];
            corr_tile<K, TR, TC, DLD>(sm + wb + tr * TR * ws + tc * TC, ws, sm + db + tr * TR * dsd + tc * TC, dsd, acc);
        }
        if (oct) {
            cp_async_wait_all();
            __syncthreads();  // the next dy run complete
            if (b + G < P.B) scatter_octet(sm, P.stg + P.stg_floats, P, crank, tid, nt);
        }
        if (dys) {
            __syncthreads();  // every dy tile read (dy is this CTA's own; no other CTA reads it)
            if (b + G < P.B)
                stage_rows(sm + P.stg + P.stg_floats, dy + plane_origin<GENERAL>(P, b + G, c) + strip_off, P,
                           myrows, tid, nt);
            cp_async_commit();
        }
    }
    cp_async_wait_all();
    plane_sync<GENERAL, OCT>(P);  // the cluster leaves together

    // Fixed-order reduction of every class over its threads.
    float* red = sm + P.red;
#pragma unroll
    for (int t = 0; t < KK; ++t) red[tid * KK + t] = acc_total(acc[t]);
    // sum dy: a fixed xor-tree inside each warp, then the warps in order.
    float sw = sdy;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sw += __shfl_xor_sync(0xffffffffu, sw, o);
    if ((tid & 31) == 0) red[nt * KK + (tid >> 5)] = sw;
    __syncthreads();
    float* out = part + ((size_t)c * P.parts + (size_t)g * P.nstrips + rank) * P.nv;
    const int ncls = 1 + 4 * P.L;
    for (int t = tid; t < ncls * KK; t += nt) {
        const int k2 = t / KK, tap = t - k2 * KK;
        float s = 0.f;
        for (int th = P.cls_thr[k2]; th < P.cls_thr[k2 + 1]; ++th) s += red[th * KK + tap];
        out[t] = s;
    }
    if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < (nt >> 5); ++w) s += red[nt * KK + w];
        out[ncls * KK] = s;
    }
    finish_channel_if_last(sm, P, part, c, ga, tid, nt);
}

// ---------------------------------------------------------------------------
// Fused backward: dx and the weight-gradient partials in one pass over x and
// dy (each read once; dx written once).  Grid (C, groups) of one CTA per SM;
// the CTA of (c, g) walks the planes b = g, g + groups, ... of channel c.
// Per plane, phase A: threads [0, an_split) analyse x into XS / SS, the rest
// analyse dy into X / S (and sum it), then every thread takes synthesis items
// of the previous plane's dx; phase B: stage the next (x, dy) pair, threads
// [0, corr0) run one dx conv tile each (the input-gradient pass: dy with
// every kernel rotated by 180 degrees, no bias) and threads [corr0, ...) run
// their runs of correlation tiles (x windows against dy tiles) into
// registers.  After the walk: the last plane's synthesis, then the
// fixed-order reduction of the correlation sums into one partial vector.
// ---------------------------------------------------------------------------
template <int K, int TR, int TC, typename T, bool OCT = false>
__global__ void __launch_bounds__(kBwdMaxThreads, 1) wtconv_backward_kernel(
    const T* __restrict__ x, const T* __restrict__ dy, const float* __restrict__ base_w,
    const float* __restrict__ base_b, const float* __restrict__ base_scale, const float* __restrict__ wt_w,
    const float* __restrict__ wt_scale, T* __restrict__ dx, float* __restrict__ part, const GradArgs ga,
    const Plan P) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    constexpr int p = K / 2, KK = K * K, NP = TC / 2;
    constexpr int DLD = (p % 2 == 0) ? 2 : 1;  // dy tiles sit at the interior of padded buffers
    static_assert(TC == 4, "4-column tiles");
    const int tid = threadIdx.x, nt = blockDim.x;
    const int c = blockIdx.x, g = blockIdx.y, G = P.groups;
    const size_t plane_elems = (size_t)P.Hr * P.Wr;
    const int myrows = real_rows(P, 0);
    auto csync = [&]() { __syncthreads(); };
    FusedCtx<K, T, true, true> cx{sm, P, dy, base_w, base_b, base_scale, wt_w, wt_scale, 0, 0, 0, plane_elems, 0};
    const size_t es = act_es<true>(P);

    zero_smem(sm, P.smem_floats, tid, nt);
    __syncthreads();
    cx.fold(c, nt, tid);  // the channel is fixed: dx weights folded once
    // NHWC channel octets: clusters of the 8 channels of an octet (rank c mod
    // 8).  The x run and the dy run of the next plane are loaded into the two
    // octet buffers during phase A and scattered in phase B by the dx-tile
    // threads, which also write out the previous plane's dx from the output
    // octet buffer; the plane barriers are cluster-wide.
    const int crank = OCT ? (int)cg::this_cluster().block_rank() : 0;
    const size_t oct_off = (size_t)(c - crank);  // channel 8o: NHWC element offset of the octet
    auto octet_runs = [&](int b) {
        load_octet(sm + P.tbuf, x + plane_origin<true>(P, b, 0) + oct_off, P, crank, tid, nt);
        load_octet(sm + P.tbuf + P.stg_floats, dy + plane_origin<true>(P, b, 0) + oct_off, P, crank, tid, nt);
    };
    auto octet_scatter = [&](int ptid, int np) {
        scatter_octet(sm, P.stg, P, crank, ptid, np, P.tbuf);
        scatter_octet(sm, P.stg + P.stg_floats, P, crank, ptid, np, P.tbuf + P.stg_floats);
    };
    const unsigned oaddr = (OCT && P.L >= 1) ? static_cast<unsigned>(__cvta_generic_to_shared(sm + P.obuf)) : 0u;
    const unsigned ocol = (unsigned)crank * (unsigned)P.opix * (unsigned)sizeof(T);
    if constexpr (OCT) {
        if (g < P.B) octet_runs(g);
        cp_async_commit();
        cp_async_wait_all();
        cg::this_cluster().sync();  // every CTA of the cluster running, its shared memory zeroed; the runs complete
        if (g < P.B) octet_scatter(tid, nt);
    } else {
        if (g < P.B) {
            const size_t off = plane_origin<true>(P, g, c);
            stage_rows(sm + P.stg, x + off, P, myrows, tid, nt);
            stage_rows(sm + P.stg + P.stg_floats, dy + off, P, myrows, tid, nt);
        }
        cp_async_commit();
    }

    const bool x_side = tid < P.an_split;
    float* XS0 = sm + P.XS.base + p * P.XS.stride + p;
    float* X0 = sm + P.X.base + p * P.X.stride + p;
    const int ct = tid - P.corr0;
    const int ncorr = P.cls_thr[1 + 4 * P.L];
    float sdy = 0.f, sdy_c = 0.f;  // compensated running sum of dy over the walk (dy-side threads)
    float* red = sm + P.red;

    // The plane walk, instantiated once per role (whole warps): CORR = false
    // runs this thread's dx conv tile, CORR = true its correlation tiles.
    // Both instantiations meet the same CTA barriers in the same order, and
    // only the correlation one keeps the K*K accumulators.
    auto walk = [&](auto corr_tag) {
        constexpr bool CORR = decltype(corr_tag)::value;
        TileJob job = TileJob{0, 0, 0, 0, 0, 0, false, false};
        int cl = -1, first = 0, cnt = 0;
        if constexpr (!CORR) {
            job = decode_tile(P, tid, TR, TC);
        } else if (ct < ncorr) {
            cl = 0;
            while (ct >= P.cls_thr[cl + 1]) ++cl;
            first = (ct - P.cls_thr[cl]) * P.tpt;
            cnt = min(P.tpt, P.cls_tiles[cl] - first);
        }
        const int lvl = cl <= 0 ? kMaxL : ((cl - 1) >> 2);
        // The correlation class's x-window buffer (XS or SS) and dy-tile
        // buffer (the interior of X or S), selected once: one tile call site.
        int wb = 0, ws = 0, db = 0, dsd = 0;
        if constexpr (CORR) {
            if (cl == 0) {
                wb = P.XS.base; ws = P.XS.stride; db = P.X.base + p * P.X.stride + p; dsd = P.X.stride;
            } else if (cl > 0) {
                const int l = (cl - 1) >> 2, s2 = (cl - 1) & 3;
                wb = P.SS[l].base + s2 * P.SS[l].sub; ws = P.SS[l].stride;
                db = P.S[l].base + s2 * P.S[l].sub + p * P.S[l].stride + p; dsd = P.S[l].stride;
            }
        }
        using Acc = typename CorrAcc<K>::type;
        Acc acc[CORR ? KK : 1];
#pragma unroll
        for (int t = 0; t < (CORR ? KK : 1); ++t) acc[t] = acc_zero<Acc>();

        int prev_b = -1;
        for (int b = g;; b += G) {
            const bool have = b < P.B;
            cp_async_wait_all();
            // Staged pair complete (octets: scattered by every CTA of the
            // cluster, and the previous output write-outs done); every tile
            // of the previous plane done.
            if constexpr (OCT) cg::this_cluster().sync(); else __syncthreads();
            // Phase A.
            if constexpr (OCT) {
                if (have && b + G < P.B) octet_runs(b + G);  // the buffers' last readers are behind the barrier above
                cp_async_commit();
            }
            if (have) {
                if (x_side) {
                    analyse_plane<T, p, false, kToSS>(sm, P, sm + P.stg, XS0, P.XS.stride, p, P.an_split, tid, csync);
                } else {
                    const float sv = analyse_plane<T, p, true, kToS>(sm, P, sm + P.stg + P.stg_floats, X0, P.X.stride,
                                                                     p, nt - P.an_split, tid - P.an_split, csync);
                    const float yv = sv - sdy_c;
                    const float tv = sdy + yv;
                    sdy_c = (tv - sdy) - yv;
                    sdy = tv;
                }
            }
            if (prev_b >= 0 && P.L >= 1) {
                T* yp = dx + plane_origin<true>(P, prev_b, c);
                for (int t = tid; t < P.n_fin; t += nt) synth_item<T, true>(sm, P, yp, t, myrows, oaddr, ocol);
            }
            if (!have) break;
            // Both analyses complete (octets: in every CTA of the cluster, and
            // their dx outputs of the previous plane stored); the previous
            // plane's Q and Y consumed.
            if constexpr (OCT) {
                cp_async_wait_all();
                cg::this_cluster().sync();
            } else {
                __syncthreads();
            }
            // Phase B.
            if constexpr (OCT) {
                if constexpr (!CORR) {
                    if (b + G < P.B) octet_scatter(tid, P.corr0);
                    if (P.L >= 1 && prev_b >= 0)
                        stream_octet_out<T>(sm, P, dx + plane_origin<true>(P, prev_b, 0) + oct_off, crank, tid, P.corr0);
                }
            } else {
                if (b + G < P.B) {
                    const size_t off = plane_origin<true>(P, b + G, c);
                    stage_rows(sm + P.stg, x + off, P, myrows, tid, nt);
                    stage_rows(sm + P.stg + P.stg_floats, dy + off, P, myrows, tid, nt);
                }
                cp_async_commit();
            }
            if constexpr (!CORR) {
                if (job.valid) {
                    float w[KK];
                    load_weights<K>(sm + job.wts, w);
                    if (P.L >= 1 || !job.base) {
                        float* out = sm + job.out;
                        const int os = job.ostride;
                        conv_tile<K, TR, TC>(sm + job.win, job.wstride, w, make_float2(0.f, 0.f),
                                             [&](int o, float2(&a)[NP]) {
                                                 *reinterpret_cast<float4*>(out + o * os) =
                                                     make_float4(a[0].x, a[0].y, a[1].x, a[1].y);
                                             });
                    } else {
                        T* yo = dx + plane_origin<true>(P, b, c) + (size_t)job.out * es;
                        const int h0 = job.row0;
                        conv_tile<K, TR, TC>(sm + job.win, job.wstride, w, make_float2(0.f, 0.f),
                                             [&](int o, float2(&a)[NP]) {
                                                 if (h0 + o < myrows)
                                                     gst4s<T>(yo + (size_t)o * P.Wr * es,
                                                              make_float4(a[0].x, a[0].y, a[1].x, a[1].y), es);
                                             });
                    }
                }
            } else {
                for (int k = 0; k < cnt; ++k) {
                    const int local = first + k;
                    const int tr = fdiv(local, P.div_ntc[lvl]), tc = local - tr * P.ntc[lvl];
                    corr_tile<K, TR, TC, DLD>(sm + wb + tr * TR * ws + tc * TC, ws, sm + db + tr * TR * dsd + tc * TC,
                                              dsd, acc);
                }
            }
            prev_b = b;
        }
        cp_async_wait_all();
        if constexpr (OCT) {
            cg::this_cluster().sync();  // the last plane's dx outputs in every owner's buffer
            if constexpr (!CORR) {
                if (P.L >= 1 && prev_b >= 0)
                    stream_octet_out<T>(sm, P, dx + plane_origin<true>(P, prev_b, 0) + oct_off, crank, tid, P.corr0);
            }
        }
        __syncthreads();  // the last synthesis (and write-out) done: the buffers are free
        if constexpr (CORR) {
            if (ct < ncorr) {
#pragma unroll
                for (int t = 0; t < KK; ++t) red[ct * KK + t] = acc_total(acc[t]);
            }
        }
    };
    if (tid < P.corr0) {
        walk(std::false_type{});
    } else {
        walk(std::true_type{});
    }

    // Fixed-order reduction of every class over its correlation threads.
    float sw = sdy;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sw += __shfl_xor_sync(0xffffffffu, sw, o);
    if ((tid & 31) == 0) red[ncorr * KK + (tid >> 5)] = sw;
    __syncthreads();
    float* out = part + ((size_t)c * P.parts + g) * P.nv;
    const int ncls = 1 + 4 * P.L;
    for (int t = tid; t < ncls * KK; t += nt) {
        const int k2 = t / KK, tap = t - k2 * KK;
        float s = 0.f;
        for (int th = P.cls_thr[k2]; th < P.cls_thr[k2 + 1]; ++th) s += red[th * KK + tap];
        out[t] = s;
    }
    if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < (nt >> 5); ++w) s += red[ncorr * KK + w];
        out[ncls * KK] = s;
    }
    finish_channel_if_last(sm, P, part, c, ga, tid, nt);
}

}  // namespace wtc
