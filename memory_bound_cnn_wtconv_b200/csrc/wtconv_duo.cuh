// Forward / input gradient of the fused WTConv layer with two alternating
// warp groups (sm_100a).
//
// Method: "Fast and Memory-Efficient Wavelet Convolutions via I/O-Aware
// Reformulation" (arXiv 2608.10805), Abstract -- the analysis recomputed on
// chip, the synthesis as one closed-form pass over the output, the scales
// folded into the conv weights (wtconv_kernels.cuh states the arithmetic).
//
// Schedule.  One persistent CTA per SM of two groups of 8 warps.  The CTA's
// run of (b, c) planes is dealt to the groups alternately (group g takes the
// planes g, g + 2, ... of the run); each group owns a full set of buffers.
// A group alternates two kinds of half-cycle:
//   A(k)  wait for its staged plane p_k, fold the channel's weights (when the
//         channel changed) into the weight slot k%2, analyse p_k into the X
//         slot k%2 and S, then stage p_{k+1} (cp.async);
//   B(k)  every conv tile of the step: the subband tiles of p_k (S -> Q slot
//         k%2) and the base tiles of p_{k-1} (X slot (k-1)%2), whose
//         epilogue adds the closed-form synthesis of every level (Q slot
//         (k-1)%2) and stores y.
// The groups run in opposite phases, with one CTA barrier per half-cycle:
// while group 0 runs B its partner runs A and vice versa, so the FMA pipes
// always hold one group's tiles (two warps per SM sub-partition, enough to
// keep them busy) while the other group's analysis -- latency-bound, light
// on the FMA pipes -- proceeds beside them.  Within a half-cycle the buffers
// a group writes and reads are disjoint, and the two groups touch only their
// own buffers (and the shared, read-only tile descriptors).
#pragma once

#include "wtconv_ws.cuh"

namespace wtc {

template <int K, typename T, bool BWD>
__global__ void __launch_bounds__(kDuoThreads, 1) wtconv_duo_kernel(
    const T* __restrict__ x, const float* __restrict__ base_w, const float* __restrict__ base_b,
    const float* __restrict__ base_scale, const float* __restrict__ wt_w, const float* __restrict__ wt_scale,
    T* __restrict__ y, const Plan P) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    int4* desc = reinterpret_cast<int4*>(sm + P.desc);
    constexpr int p = K / 2, KK = K * K;
    constexpr int GT = kDuoThreads / 2;  // threads of a group
    const int tid = threadIdx.x, grp = tid / GT, gt = tid - grp * GT;
    float* gsm = sm + P.gbase + grp * P.gsize;  // this group's buffers
    const long long units = (long long)P.B * P.C;
    const int u0 = (int)(((long long)blockIdx.x * units) / gridDim.x);
    const int u1 = (int)(((long long)(blockIdx.x + 1) * units) / gridDim.x);
    const int n = u1 - u0;
    const int m = (n - grp + 1) / 2;  // planes of this group: local planes grp, grp + 2, ...
    const size_t plane_elems = (size_t)P.H * P.W;
    const int nsub = P.n_sub_tiles, ntiles = P.n_step_tiles;

    zero_smem(sm, P.smem_floats, tid, kDuoThreads);
    __syncthreads();
    for (int t = tid; t < ntiles; t += kDuoThreads) desc[t] = ws_describe(P, t);
    __syncthreads();
    if (n <= 0) return;

    // Barrier of this group's 256 threads (ids 1 and 2; 0 is the CTA's).
    auto gsync = [&]() { asm volatile("bar.sync %0, %1;\n" ::"r"(1 + grp), "r"(GT) : "memory"); };
    // Plane p_k of this group: unit u0 + grp + 2k.
    auto unit_of = [&](int k) { return u0 + grp + 2 * k; };
    auto stage = [&](int k) {
        const int u = unit_of(k);
        const T* src = x + ((size_t)(u % P.B) * P.C + u / P.B) * plane_elems;
        stage_plane(gsm + P.stg, src, P.plane_chunks, gt, GT);
        cp_async_commit();
    };
    if (m > 0) stage(0);

    // Half-cycle h: group 0 runs A(h/2) on even h and B((h-1)/2) on odd h;
    // group 1 runs B((h-2)/2) on even h and A((h-1)/2) on odd h.
    const int m0 = (n + 1) / 2, m1 = n / 2;
    const int H = 2 * m0 + 2 > 2 * m1 + 3 ? 2 * m0 + 2 : 2 * m1 + 3;
    for (int h = 0; h < H; ++h) {
        const bool runs_a = ((h + grp) & 1) == 0;
        if (runs_a) {
            const int k = (h - grp) >> 1;
            if (k >= 0 && k < m) {
                cp_async_wait_all();
                gsync();  // p_k staged (every thread's copies)
                const int u = unit_of(k), c = u / P.B;
                float* wslot = gsm + P.wbase + (k & 1) * P.w_slot;
                // The slot last held p_{k-2}: two planes back in the run.
                if (k < 2 || c != (u - 4) / P.B)
                    ws_fold<K, BWD>(wslot, P, c, base_w, base_b, base_scale, wt_w, wt_scale, GT, gt);
                float* X0 = gsm + (k & 1) * P.x_slot + P.X.base + p * P.X.stride + p;
                analyse_plane<T, p, false, kToS>(gsm, P, gsm + P.stg, X0, P.X.stride, p, GT, gt, gsync);
                gsync();  // staging read by every thread of the group
                if (k + 1 < m) stage(k + 1);
            }
        } else {
            const int k = (h - 1 - grp) >> 1;
            if (k >= 0 && k <= m) {
                const bool sub_on = k < m, base_on = k >= 1;
                const float* s_buf = gsm;
                const float* w_sub = gsm + P.wbase + (k & 1) * P.w_slot;
                float* q_sub = gsm + (k & 1) * P.q_slot;
                const float* x_buf = gsm + ((k - 1) & 1) * P.x_slot;
                const float* w_base = gsm + P.wbase + ((k - 1) & 1) * P.w_slot;
                const float* q_base = gsm + ((k - 1) & 1) * P.q_slot;
                const int ub = base_on ? unit_of(k - 1) : u0;
                T* yp = y + ((size_t)(ub % P.B) * P.C + ub / P.B) * plane_elems;
                for (int t = gt; t < ntiles; t += GT) {
                    const bool base = t >= nsub;
                    if (base ? !base_on : !sub_on) continue;
                    const int4 d = desc[t];
                    const float* win = (base ? x_buf : s_buf) + d.x;
                    const float* wsl = base ? w_base : w_sub;
                    float w[KK];
                    load_weights<K>(wsl + d.z, w);
                    const float b0 = base ? wsl[P.bias] : 0.f;
                    float2 acc[8][2];
                    conv_tile_regs<K, 8>(win, d.w & 0xfff, w, make_float2(b0, b0), acc);
                    if (!base) {
                        float* out = q_sub + d.y;
                        const int os = (d.w >> 12) & 0xfff;
#pragma unroll
                        for (int o = 0; o < 8; ++o)
                            *reinterpret_cast<float4*>(out + o * os) =
                                make_float4(acc[o][0].x, acc[o][0].y, acc[o][1].x, acc[o][1].y);
                    } else {
                        const int r0 = d.y >> 16, c0 = d.y & 0xffff;
                        synth_tile(q_base, P, r0, c0, acc);
                        T* yo = yp + (size_t)r0 * P.W + c0;
#pragma unroll
                        for (int o = 0; o < 8; ++o)
                            if (r0 + o < P.H)
                                gst4<T>(yo + (size_t)o * P.W,
                                        make_float4(acc[o][0].x, acc[o][0].y, acc[o][1].x, acc[o][1].y));
                    }
                }
            }
        }
        __syncthreads();  // end of the half-cycle
    }
    cp_async_wait_all();
}

}  // namespace wtc
