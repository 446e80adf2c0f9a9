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
//       factors of analysis and synthesis) are folded into the conv weights
//       once per CTA, so the butterflies are pure add/sub.
//
// Un-normalised butterflies: U_{l,s} = 2^(l+1) S_{l,s} (S orthonormal), so a
// level-l conv with weights  wt_scale * wt_w * 4^-(l+1)  yields exactly the
// term  2^-(l+1) * Shat_{l,s}  that the closed-form synthesis adds.
//
// Depthwise convolution is not a dense contraction, so every conv here runs
// on the FP32 FMA pipes: each thread owns a TR x TC output tile, streams the
// (TR+K-1) input rows of its window from shared memory once with 128-bit
// loads, and keeps the K*K folded weights in registers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "wtconv_plan.h"

namespace wtc {

// ---------------------------------------------------------------------------
// Activation storage: 4 consecutive elements at a time (W % 4 == 0).
// ---------------------------------------------------------------------------
template <typename T>
struct Act;

template <>
struct Act<float> {
    static __device__ __forceinline__ float4 load4(const float* p) {
        return __ldg(reinterpret_cast<const float4*>(p));
    }
    static __device__ __forceinline__ void store4(float* p, float4 v) {
        *reinterpret_cast<float4*>(p) = v;
    }
};

template <>
struct Act<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
        uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&r.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&r.y);
        float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        return make_float4(fa.x, fa.y, fb.x, fb.y);
    }
    static __device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
        __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
        uint2 r;
        r.x = *reinterpret_cast<uint32_t*>(&a);
        r.y = *reinterpret_cast<uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = r;
    }
};

// Store 4 floats to a shared address that is congruent to P (mod 4) floats.
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

__device__ __forceinline__ void zero_smem(float* sm, int nfloats, int tid, int nt) {
    float4* s4 = reinterpret_cast<float4*>(sm);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = tid; i < (nfloats >> 2); i += nt) s4[i] = z;
}

// Copy an H x W plane from global memory into a shared buffer whose element
// (0, 0) sits at `dst` (congruent to P mod 4 floats); optionally returns the
// thread's running sum of the loaded values (weight gradient's sum of dy).
template <typename T, int P, bool SUM>
__device__ __forceinline__ float load_plane(const T* __restrict__ src, int H, int W, float* dst,
                                            int stride, int tid, int nt) {
    constexpr int U = 4;
    const int W4 = W >> 2;
    const int n = H * W4;
    float s = 0.f;
    for (int t0 = tid; t0 < n; t0 += U * nt) {
        float4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = t0 + u * nt;
            if (t < n) {
                const int i = t / W4, j = (t - i * W4) * 4;
                v[u] = Act<T>::load4(src + (size_t)i * W + j);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = t0 + u * nt;
            if (t < n) {
                const int i = t / W4, j = (t - i * W4) * 4;
                sts4<P>(dst + i * stride + j, v[u]);
                if (SUM) s += (v[u].x + v[u].y) + (v[u].z + v[u].w);
            }
        }
    }
    return s;
}

// One un-normalised 2-D Haar analysis step on chip: the (2n) x (2m) plane at
// `src` (element (0,0), row stride `ss`) becomes 4 planes n x m at `dst`
// (element (0,0), row stride `ds`, plane step `dsub`), order LL, LH, HL, HH.
__device__ __forceinline__ void haar_level(const float* src, int ss, int n, int m, float* dst, int ds,
                                           int dsub, int tid, int nt) {
    for (int t = tid; t < n * m; t += nt) {
        const int i = t / m, j = t - i * m;
        const float* s0 = src + 2 * i * ss + 2 * j;
        const float a = s0[0], b = s0[1], c = s0[ss], d = s0[ss + 1];
        const float apb = a + b, amb = a - b, cpd = c + d, cmd = c - d;
        float* d0 = dst + i * ds + j;
        d0[0] = apb + cpd;          // LL
        d0[dsub] = apb - cpd;       // LH: difference between rows
        d0[2 * dsub] = amb + cmd;   // HL: difference between columns
        d0[3 * dsub] = amb - cmd;   // HH
    }
}

// ---------------------------------------------------------------------------
// Register-tiled depthwise conv of one TR x TC output tile.
//   out[o][j] = init + sum_{u<K, v<K} w[u*K+v] * win[(o+u)*stride + j+v]
// `win` is the 16-byte aligned window origin (input element (r0-p, c0-p)).
// Each input row is loaded once; output row o is handed to emit(o, acc[o])
// as soon as its last input row has been consumed.
// ---------------------------------------------------------------------------
template <int K, int TR, int TC, class Emit>
__device__ __forceinline__ void conv_tile(const float* __restrict__ win, int stride, const float (&w)[K * K],
                                          float init, Emit&& emit) {
    constexpr int WV = (TC + K - 1 + 3) / 4;
    float acc[TR][TC];
#pragma unroll
    for (int r = 0; r < TR + K - 1; ++r) {
        float row[4 * WV];
        const float* rp = win + r * stride;
#pragma unroll
        for (int q = 0; q < WV; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(rp + 4 * q);
            row[4 * q + 0] = v.x; row[4 * q + 1] = v.y; row[4 * q + 2] = v.z; row[4 * q + 3] = v.w;
        }
#pragma unroll
        for (int u = 0; u < K; ++u) {
            const int o = r - u;
            if (o >= 0 && o < TR) {
#pragma unroll
                for (int j = 0; j < TC; ++j) {
                    float a = (u == 0) ? init : acc[o][j];
#pragma unroll
                    for (int v = 0; v < K; ++v) a = fmaf(w[u * K + v], row[j + v], a);
                    acc[o][j] = a;
                }
            }
        }
        const int oc = r - (K - 1);
        if (oc >= 0 && oc < TR) emit(oc, acc[oc]);
    }
}

// Correlation of one TR x TC tile of D with the K x K shifts of S:
//   acc[u*K+v] += sum_{o<TR, j<TC} D[o][j] * S[o+u][j+v]
// `swin` is the S window origin (element (r0-p, c0-p)), `dt` the D tile origin.
template <int K, int TR, int TC>
__device__ __forceinline__ void corr_tile(const float* __restrict__ swin, int sstride,
                                          const float* __restrict__ dt, int dstride, float (&acc)[K * K]) {
    constexpr int WV = (TC + K - 1 + 3) / 4;
    float d[TR][TC];
#pragma unroll
    for (int r = 0; r < TR + K - 1; ++r) {
        if (r < TR) {
#pragma unroll
            for (int q = 0; q < TC / 4; ++q) {
                const float4 v = *reinterpret_cast<const float4*>(dt + r * dstride + 4 * q);
                d[r][4 * q + 0] = v.x; d[r][4 * q + 1] = v.y; d[r][4 * q + 2] = v.z; d[r][4 * q + 3] = v.w;
            }
        }
        float row[4 * WV];
        const float* rp = swin + r * sstride;
#pragma unroll
        for (int q = 0; q < WV; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(rp + 4 * q);
            row[4 * q + 0] = v.x; row[4 * q + 1] = v.y; row[4 * q + 2] = v.z; row[4 * q + 3] = v.w;
        }
#pragma unroll
        for (int u = 0; u < K; ++u) {
            const int o = r - u;
            if (o >= 0 && o < TR) {
#pragma unroll
                for (int v = 0; v < K; ++v) {
                    float a = acc[u * K + v];
#pragma unroll
                    for (int j = 0; j < TC; ++j) a = fmaf(d[o][j], row[j + v], a);
                    acc[u * K + v] = a;
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
// Forward (BWD = false) and input gradient (BWD = true).  One CTA per plane.
// The input gradient is the same pass applied to dy with every kernel
// rotated by 180 degrees and no bias: the transpose of the forward map.
// ---------------------------------------------------------------------------
template <int K, int TR, int TC, typename T, bool BWD>
__global__ void __launch_bounds__(512) wtconv_fused_kernel(
    const T* __restrict__ x, const float* __restrict__ base_w, const float* __restrict__ base_b,
    const float* __restrict__ base_scale, const float* __restrict__ wt_w,
    const float* __restrict__ wt_scale, T* __restrict__ y, const Plan P) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    constexpr int p = K / 2, KK = K * K;
    static_assert(TC % 4 == 0, "tile width must be a multiple of 4");
    const int tid = threadIdx.x, nt = blockDim.x;
    const int plane = blockIdx.x;
    const int c = plane % P.C;
    const int H = P.H, W = P.W, L = P.L;

    zero_smem(sm, P.smem_floats, tid, nt);
    __syncthreads();

    // Reformulation (3): fold the scales (and the Haar factors) into the weights.
    const int ncls = 1 + 4 * L;
    for (int t = tid; t < ncls * KK; t += nt) {
        const int cl = t / KK, tap = t - cl * KK;
        const int src = BWD ? (KK - 1 - tap) : tap;
        float v;
        if (cl == 0) {
            v = base_scale[c] * base_w[c * KK + src];
        } else {
            const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
            const int pi = (l * P.C + c) * 4 + s;
            v = (wt_scale[pi] * wt_w[pi * KK + src]) * quarter_pow(l);
        }
        sm[P.wbase + cl * P.wcls + tap] = v;
    }
    if (tid == 0) sm[P.bias] = BWD ? 0.f : base_scale[c] * base_b[c];

    // Stage the plane (the only HBM read).
    const size_t poff = (size_t)plane * H * W;
    load_plane<T, p, false>(x + poff, H, W, sm + P.X.base + p * P.X.stride + p, P.X.stride, tid, nt);
    __syncthreads();

    // Reformulation (1): analysis butterflies for every level, on chip.
    for (int l = 0; l < L; ++l) {
        const float* src = (l == 0) ? sm + P.X.base + p * P.X.stride + p
                                    : sm + P.S[l - 1].base + p * P.S[l - 1].stride + p;
        const int ss = (l == 0) ? P.X.stride : P.S[l - 1].stride;
        haar_level(src, ss, H >> (l + 1), W >> (l + 1), sm + P.S[l].base + p * P.S[l].stride + p,
                   P.S[l].stride, P.S[l].sub, tid, nt);
        __syncthreads();
    }

    // Per-subband depthwise convs, folded weights -> Q[l].
    for (int t = tid; t < P.n_sub_tiles; t += nt) {
        int cl = 1;
        while (t >= P.sub_begin[cl]) ++cl;  // sub_begin[cl] = end of class cl's tiles
        const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
        const int local = t - P.sub_begin[cl - 1];
        const int tr = local / P.ntc[l], tc = local - tr * P.ntc[l];
        float w[KK];
        load_weights<K>(sm + P.wbase + cl * P.wcls, w);
        const Buf& S = P.S[l];
        const Buf& Q = P.Q[l];
        const float* win = sm + S.base + s * S.sub + tr * TR * S.stride + tc * TC;
        float* out = sm + Q.base + s * Q.sub + tr * TR * Q.stride + tc * TC;
        conv_tile<K, TR, TC>(win, S.stride, w, 0.f, [&](int o, float(&a)[TC]) {
#pragma unroll
            for (int q = 0; q < TC / 4; ++q)
                *reinterpret_cast<float4*>(out + o * Q.stride + 4 * q) =
                    make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
        });
    }
    __syncthreads();

    // Reformulation (2), levels >= 1: their signed sum at half resolution
    // (constant over each 2x2 output block), indexed by the bits of (i, j).
    const int n0 = H >> 1, m0 = W >> 1;
    if (L >= 2) {
        for (int t = tid; t < n0 * m0; t += nt) {
            const int i = t / m0, j = t - i * m0;
            float z = 0.f;
            for (int l = 1; l < L; ++l) {
                const Buf& Q = P.Q[l];
                const float* q = sm + Q.base + (i >> l) * Q.stride + (j >> l);
                const float q0 = q[0], q1 = q[Q.sub], q2 = q[2 * Q.sub], q3 = q[3 * Q.sub];
                const int a = (i >> (l - 1)) & 1, b = (j >> (l - 1)) & 1;
                const float t0 = a ? q0 - q1 : q0 + q1;
                const float t1 = a ? q2 - q3 : q2 + q3;
                z += b ? t0 - t1 : t0 + t1;
            }
            sm[P.Z.base + i * P.Z.stride + j] = z;
        }
        __syncthreads();
    }

    // Base conv + level-0 signed sum + coarse sum -> y (the only HBM write).
    {
        float w[KK];
        load_weights<K>(sm + P.wbase, w);
        const float bias = sm[P.bias];
        const int ntc = P.ntc[kMaxL];
        T* yp = y + poff;
        for (int t = tid; t < P.n_base_tiles; t += nt) {
            const int tr = t / ntc, tc = t - tr * ntc;
            const float* win = sm + P.X.base + tr * TR * P.X.stride + tc * TC;
            conv_tile<K, TR, TC>(win, P.X.stride, w, bias, [&](int o, float(&a)[TC]) {
                const int h = tr * TR + o;
                if (h >= H) return;
                const int w0 = tc * TC;
                if (L >= 1) {
                    const Buf& Q = P.Q[0];
                    const int i = h >> 1;
                    const float sg = (h & 1) ? -1.f : 1.f;
#pragma unroll
                    for (int pos = 0; pos < TC / 2; ++pos) {
                        const int j = (w0 >> 1) + pos;
                        const float* q = sm + Q.base + i * Q.stride + j;
                        float q0 = q[0];
                        if (L >= 2) q0 += sm[P.Z.base + i * P.Z.stride + j];
                        const float t0 = fmaf(sg, q[Q.sub], q0);
                        const float t1 = fmaf(sg, q[3 * Q.sub], q[2 * Q.sub]);
                        a[2 * pos] += t0 + t1;
                        a[2 * pos + 1] += t0 - t1;
                    }
                }
#pragma unroll
                for (int q = 0; q < TC / 4; ++q)
                    Act<T>::store4(yp + (size_t)h * W + w0 + 4 * q,
                                   make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]));
            });
        }
    }
}

// ---------------------------------------------------------------------------
// Weight gradient, stage 1: grid (C, groups).  The CTA of (c, g) walks the
// planes b = g, g + groups, ... of channel c.  Thread t owns one tile of one
// class (base, or level l subband s) for the whole walk and accumulates its
// K*K correlation sums in registers; the CTA then reduces each class over its
// threads in a fixed order and writes one partial vector (plus sum dy).
// ---------------------------------------------------------------------------
template <int K, int TR, int TC, typename T>
__global__ void __launch_bounds__(512) wtconv_bwdw_partial_kernel(const T* __restrict__ x,
                                                                  const T* __restrict__ dy,
                                                                  float* __restrict__ part, const Plan P) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    constexpr int p = K / 2, KK = K * K;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int c = blockIdx.x, g = blockIdx.y, G = P.groups;
    const int H = P.H, W = P.W, L = P.L;

    zero_smem(sm, P.smem_floats, tid, nt);

    int cl = -1, tr = 0, tc = 0;
    if (tid < P.n_all_tiles) {
        cl = 0;
        while (tid >= P.cls_begin[cl + 1]) ++cl;
        const int lvl = (cl == 0) ? kMaxL : ((cl - 1) >> 2);
        const int local = tid - P.cls_begin[cl];
        tr = local / P.ntc[lvl];
        tc = local - tr * P.ntc[lvl];
    }
    float acc[KK];
#pragma unroll
    for (int t = 0; t < KK; ++t) acc[t] = 0.f;
    float sdy = 0.f;
    __syncthreads();

    for (int b = g; b < P.B; b += G) {
        const size_t poff = ((size_t)b * P.C + c) * H * W;
        load_plane<T, p, false>(x + poff, H, W, sm + P.X.base + p * P.X.stride + p, P.X.stride, tid, nt);
        sdy += load_plane<T, 0, true>(dy + poff, H, W, sm + P.DY.base, P.DY.stride, tid, nt);
        __syncthreads();
        for (int l = 0; l < L; ++l) {
            const float* xs = (l == 0) ? sm + P.X.base + p * P.X.stride + p
                                       : sm + P.S[l - 1].base + p * P.S[l - 1].stride + p;
            const int xss = (l == 0) ? P.X.stride : P.S[l - 1].stride;
            haar_level(xs, xss, H >> (l + 1), W >> (l + 1), sm + P.S[l].base + p * P.S[l].stride + p,
                       P.S[l].stride, P.S[l].sub, tid, nt);
            const float* ds = (l == 0) ? sm + P.DY.base : sm + P.Q[l - 1].base;
            const int dss = (l == 0) ? P.DY.stride : P.Q[l - 1].stride;
            haar_level(ds, dss, H >> (l + 1), W >> (l + 1), sm + P.Q[l].base, P.Q[l].stride, P.Q[l].sub,
                       tid, nt);
            __syncthreads();
        }
        if (cl == 0) {
            corr_tile<K, TR, TC>(sm + P.X.base + tr * TR * P.X.stride + tc * TC, P.X.stride,
                                 sm + P.DY.base + tr * TR * P.DY.stride + tc * TC, P.DY.stride, acc);
        } else if (cl > 0) {
            const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
            const Buf& S = P.S[l];
            const Buf& Q = P.Q[l];
            corr_tile<K, TR, TC>(sm + S.base + s * S.sub + tr * TR * S.stride + tc * TC, S.stride,
                                 sm + Q.base + s * Q.sub + tr * TR * Q.stride + tc * TC, Q.stride, acc);
        }
        __syncthreads();
    }

    // Fixed-order reduction of every class over its threads.
    float* red = sm + P.red;
#pragma unroll
    for (int t = 0; t < KK; ++t) red[tid * KK + t] = acc[t];
    red[nt * KK + tid] = sdy;
    __syncthreads();
    float* out = part + ((size_t)c * G + g) * P.nv;
    const int ncls = 1 + 4 * L;
    for (int t = tid; t < ncls * KK; t += nt) {
        const int k2 = t / KK, tap = t - k2 * KK;
        float s = 0.f;
        for (int th = P.cls_begin[k2]; th < P.cls_begin[k2 + 1]; ++th) s += red[th * KK + tap];
        out[t] = s;
    }
    if (tid == 0) {
        float s = 0.f;
        for (int th = 0; th < nt; ++th) s += red[nt * KK + th];
        out[ncls * KK] = s;
    }
}

}  // namespace wtc
