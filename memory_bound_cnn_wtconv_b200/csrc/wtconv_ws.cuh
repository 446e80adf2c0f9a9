// Warp-specialised forward / input gradient of the fused WTConv layer (sm_100a).
//
// Method: "Fast and Memory-Efficient Wavelet Convolutions via I/O-Aware
// Reformulation" (arXiv 2608.10805), Abstract -- the analysis recomputed on
// chip, the synthesis as one closed-form pass over the output, the scales
// folded into the conv weights (wtconv_kernels.cuh states the arithmetic).
//
// Schedule.  One persistent CTA per SM walks a run of (b, c) planes.  Its
// warps have three roles that run concurrently, handing buffers to each
// other through mbarriers (no CTA-wide barrier in the walk):
//   copy warp       one lane issues one bulk copy of each whole plane into a
//                   ring of NSTG staging slots, as soon as the slot is free;
//   producer warps  plane j: fold the channel's weights if the weight slot
//                   holds another channel, and run the Haar analysis from
//                   staging into the X slot j%NX (padded plane) and the S
//                   slot j%NS (padded subbands of every level), up to NS
//                   planes ahead of the sub tiles;
//   conv warps      the subband conv tiles of each plane (S slot j%NS ->
//                   Q slot j%3) and its base conv tiles (X slot j%NX), whose
//                   epilogue adds the closed-form synthesis of every level
//                   (read from Q slot j%3) and stores y.  Sub tiles are padded
//                   to whole warp-tiles, so no warp-tile holds both kinds.
// So the FMA pipes are fed by the conv warps while the analysis of the next
// planes and the loads from HBM proceed beside them; x is read once and y
// written once.
//
// Buffer hand-offs (mbarrier phases; the k-th use of a barrier slot waits
// for parity k & 1):
//   stg_full[j%NSTG]   bulk copy of plane j landed         (1 arrival + tx bytes)
//   stg_empty[j%NSTG]  every producer warp read plane j   (npw arrivals)
//   ana[j%16]          X, S and weights of plane j ready  (npw arrivals)
//   sub[j%16]          sub tiles of plane j done          (one per sub warp-tile)
//   base[j%3]          base tiles of plane j done         (one per base warp-tile)
// Conv warps take warp-tile tasks from a shared counter in the order
// S_0, S_1, B_0, S_2, B_1, ... (S_j: a sub warp-tile of plane j, B_j: a base
// warp-tile of plane j).  A parity wait is only meaningful while the phase
// before the awaited one has completed: the producer and copy warps wait in
// order, and a conv warp takes a task of plane j only after every task
// before it was taken, with at most ncw <= 8 of them unfinished, which (16
// ring slots) leaves the phase of plane j - 16 complete.  Copy, plane q:
// waits stg_empty(q-NSTG).  Producer,
// plane j: waits stg_full(j), sub(j-NS) [S slot], base(j-3) [X, weight and Q
// slots; NX = 3].  S_j waits ana(j) and arrives on sub(j);
// B_j waits sub(j) [its Q; with L = 0, ana(j)] and arrives on base(j).  No
// wait can see its barrier two phases ahead: the next phase of the barrier
// it waits for needs the waiting task's own arrival, directly or through
// the analysis the producer can only finish after it.  No arrival lands in
// an earlier phase than its own: ana(j) implies sub(j-16) complete (the
// analysis of plane j-16+NS waited for it), and B_j's wait for sub(j) implies
// base(j-3) complete (the analysis of plane j waited for it).
// The bulk copies are issued by the copy warp alone.  Every wait gives up
// after kWaitLimitNs, counts the time-out in g_wait_timeouts (read by the
// host through wtconv_wait_timeouts) and ends the role; the copy lane then
// waits (again with a limit) for the copies it has in flight before the CTA
// exits.
#pragma once

#include "wtconv_kernels.cuh"

namespace wtc {

// Time-outs of mbarrier waits in this translation unit (see the header).
static __device__ unsigned int g_wait_timeouts;

constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* b, unsigned count) {
    asm volatile("mbarrier.init.shared.b64 [%0], %1;\n" ::"r"(smem_addr(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared.b64 st, [%0];\n}\n" ::"r"(smem_addr(b)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* b, unsigned bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared.b64 st, [%0], %1;\n}\n" ::"r"(smem_addr(b)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(b)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the completion of the phase of parity `parity`; false after
// kWaitLimitNs (counted in g_wait_timeouts).
__device__ __forceinline__ bool mbar_wait(uint64_t* b, unsigned parity) {
    if (mbar_try_wait(b, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(b, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicAdd(&g_wait_timeouts, 1u);
            return false;
        }
    }
}

// One bulk copy global -> shared (16-byte aligned addresses, size a multiple
// of 16), completing `bytes` of transaction count on the mbarrier.  No
// multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// Conv tile descriptor (one per tile of a conv step, built once per CTA; sub
// tiles [0, n_sub_tiles), padding up to sub_pad, base tiles after it):
//   x  window origin (float offset into slot 0 of S, or of X for base tiles)
//   y  sub tiles: output origin in slot 0 of Q;  base tiles: (r0 << 16) | c0
//   z  weight class offset within a weight slot
//   w  bit 31: base tile;  bits 0..11: window row stride;  bits 12..23: Q row stride
__device__ __forceinline__ int4 ws_describe(const Plan& P, int t) {
    constexpr int TR = 8, TC = 4;
    int4 d;
    if (t < P.n_sub_tiles) {
        int cl = 1;
        while (t >= P.sub_begin[cl]) ++cl;
        const int l = (cl - 1) >> 2, s = (cl - 1) & 3;
        const int local = t - P.sub_begin[cl - 1];
        const int tr = local / P.ntc[l], tc = local - tr * P.ntc[l];
        int sb = 0, ss = 0, sst = 0, qb = 0, qs = 0, qst = 0;
#pragma unroll
        for (int q = 0; q < kMaxL; ++q)
            if (q == l) {
                sb = P.S[q].base; ss = P.S[q].sub; sst = P.S[q].stride;
                qb = P.Q[q].base; qs = P.Q[q].sub; qst = P.Q[q].stride;
            }
        d.x = sb + s * ss + tr * TR * sst + tc * TC;
        d.y = qb + s * qs + tr * TR * qst + tc * TC;
        d.z = cl * P.wcls;
        d.w = sst | (qst << 12);
    } else if (t < P.sub_pad) {
        d = make_int4(0, 0, 0, 0);  // padding of the sub tiles to whole warp-tiles (never run)
    } else {
        const int bt = t - P.sub_pad;
        const int tr = bt / P.ntc[kMaxL], tc = bt - tr * P.ntc[kMaxL];
        d.x = P.X.base + tr * TR * P.X.stride + tc * TC;
        d.y = ((tr * TR) << 16) | (tc * TC);
        d.z = 0;
        d.w = (int)(0x80000000u | (unsigned)P.X.stride);
    }
    return d;
}

// Register-tiled depthwise conv of one 8 x 4 output tile into acc
// (conv_tile's arithmetic, with every output row kept for the epilogue).
template <int K, int TR>
__device__ __forceinline__ void conv_tile_regs(const float* __restrict__ win, int stride, const float (&w)[K * K],
                                               float2 init, float2 (&acc)[TR][2]) {
    constexpr int NW2 = (4 + K - 1) / 2;
#pragma unroll
    for (int r = 0; r < TR + K - 1; ++r) {
        WinRow<NW2> row;
        row.load(win + r * stride);
#pragma unroll
        for (int u = 0; u < K; ++u) {
            const int o = r - u;
            if (o >= 0 && o < TR) {
#pragma unroll
                for (int jp = 0; jp < 2; ++jp) {
                    float2 a = (u == 0) ? init : acc[o][jp];
#pragma unroll
                    for (int v = 0; v < K; ++v) a = tap<NW2>(a, w[u * K + v], row, jp, v);
                    acc[o][jp] = a;
                }
            }
        }
    }
}

// Reformulation (2) in the epilogue of a base tile: the 8 x 4 outputs at
// (r0 + o, c0 + j) (r0 a multiple of 8, c0 of 4) receive, for every level
// l, the signed sum of the four level-l conv outputs at
// (h >> (l+1), w >> (l+1)): LH negated where bit l of h is set, HL where bit
// l of w is, HH where exactly one is.  Evaluated Horner-style from the
// coarsest level down (each level's signed sum added to the next finer LL
// term): levels >= 3 touch one position of the tile, level 2 one position
// with two row signs, level 1 two positions, level 0 eight.  `qs` is the Q
// slot of the plane.
__device__ __forceinline__ void synth_tile(const float* qs, const Plan& P, int r0, int c0, float2 (&acc)[8][2]) {
    const int L = P.L;
    float t = 0.f;  // coarse term at the tile's unique level-2 position
#pragma unroll
    for (int l = kMaxL - 1; l >= 3; --l) {
        if (l >= L) continue;
        const Buf& Q = P.Q[l];
        const float* q = qs + Q.base + (r0 >> (l + 1)) * Q.stride + (c0 >> (l + 1));
        const float q0 = q[0] + t, q1 = q[Q.sub], q2 = q[2 * Q.sub], q3 = q[3 * Q.sub];
        const bool bi = (r0 >> l) & 1, bj = (c0 >> l) & 1;
        const float a = bi ? q0 - q1 : q0 + q1;
        const float b = bi ? q2 - q3 : q2 + q3;
        t = bj ? a - b : a + b;
    }
    float t2[2] = {0.f, 0.f};  // coarse term at the level-1 rows (r0 >> 2) + ah
    if (L >= 3) {
        const Buf& Q = P.Q[2];
        const float* q = qs + Q.base + (r0 >> 3) * Q.stride + (c0 >> 3);
        const float q0 = q[0] + t, q1 = q[Q.sub], q2 = q[2 * Q.sub], q3 = q[3 * Q.sub];
        const bool bj = (c0 >> 2) & 1;
#pragma unroll
        for (int ah = 0; ah < 2; ++ah) {
            const float a = ah ? q0 - q1 : q0 + q1;
            const float b = ah ? q2 - q3 : q2 + q3;
            t2[ah] = bj ? a - b : a + b;
        }
    }
    float t1[4][2] = {};  // coarse term at the level-0 positions ((r0 >> 1) + a, (c0 >> 1) + b)
    if (L >= 2) {
        const Buf& Q = P.Q[1];
#pragma unroll
        for (int ah = 0; ah < 2; ++ah) {
            const float* q = qs + Q.base + ((r0 >> 2) + ah) * Q.stride + (c0 >> 2);
            const float q0 = q[0] + t2[ah], q1 = q[Q.sub], q2 = q[2 * Q.sub], q3 = q[3 * Q.sub];
#pragma unroll
            for (int al = 0; al < 2; ++al) {
                const float a = al ? q0 - q1 : q0 + q1;
                const float b = al ? q2 - q3 : q2 + q3;
                t1[2 * ah + al][0] = a + b;
                t1[2 * ah + al][1] = a - b;
            }
        }
    }
    if (L >= 1) {
        const Buf& Q = P.Q[0];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const float* q = qs + Q.base + ((r0 >> 1) + a) * Q.stride + (c0 >> 1);
            const float2 ll = *reinterpret_cast<const float2*>(q);
            const float2 lh = *reinterpret_cast<const float2*>(q + Q.sub);
            const float2 hl = *reinterpret_cast<const float2*>(q + 2 * Q.sub);
            const float2 hh = *reinterpret_cast<const float2*>(q + 3 * Q.sub);
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const float vll = (b ? ll.y : ll.x) + t1[a][b];
                const float vlh = b ? lh.y : lh.x, vhl = b ? hl.y : hl.x, vhh = b ? hh.y : hh.x;
                const float at = vll + vlh, bt = vhl + vhh;  // output row 2a
                const float ab = vll - vlh, bb = vhl - vhh;  // output row 2a + 1
                acc[2 * a][b].x += at + bt;
                acc[2 * a][b].y += at - bt;
                acc[2 * a + 1][b].x += ab + bb;
                acc[2 * a + 1][b].y += ab - bb;
            }
        }
    }
}

// Reformulation (3): the folded weights of channel c into one weight slot
// (threads [0, np)); the input gradient takes every kernel rotated by 180
// degrees and no bias.
template <int K, bool BWD>
__device__ __forceinline__ void ws_fold(float* wdst, const Plan& P, int c, const float* base_w, const float* base_b,
                                        const float* base_scale, const float* wt_w, const float* wt_scale, int np,
                                        int ptid) {
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
        wdst[cl * P.wcls + tap] = v;
    }
    if (ptid == 0) wdst[ncls * P.wcls] = BWD ? 0.f : base_scale[c] * base_b[c];
}

// Ring position of plane j for a ring of `depth` slots: slot = j % depth and
// use = j / depth, advanced one plane at a time (no division in the loops).
struct RingPos {
    int slot = 0, use = 0;
    __device__ __forceinline__ void next(int depth) {
        if (++slot == depth) {
            slot = 0;
            ++use;
        }
    }
};

template <int K, typename T, bool BWD>
__global__ void __launch_bounds__(kWsMaxThreads, 1) wtconv_ws_kernel(
    const T* __restrict__ x, const float* __restrict__ base_w, const float* __restrict__ base_b,
    const float* __restrict__ base_scale, const float* __restrict__ wt_w, const float* __restrict__ wt_scale,
    T* __restrict__ y, const Plan P) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P.mbar);
    int4* desc = reinterpret_cast<int4*>(sm + P.desc);
    constexpr int p = K / 2, KK = K * K;
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const long long units = (long long)P.B * P.C;
    const int u0 = (int)(((long long)blockIdx.x * units) / gridDim.x);
    const int u1 = (int)(((long long)(blockIdx.x + 1) * units) / gridDim.x);
    const int n = u1 - u0;
    const size_t plane_elems = (size_t)P.H * P.W;
    const int NSTG = P.nstg, NX = P.x_slots, NS = P.s_slots;

    zero_smem(sm, P.smem_floats, tid, nt);
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // the zeroed staging, before any bulk copy
    __syncthreads();
    for (int t = tid; t < P.n_step_tiles; t += nt) desc[t] = ws_describe(P, t);
    if (tid == 0) {
        for (int i = 0; i < NSTG; ++i) {
            mbar_init(&bars[kBarStgFull + i], 1);
            mbar_init(&bars[kBarStgEmpty + i], P.npw);
        }
        for (int i = 0; i < kWsBarRing; ++i) {
            mbar_init(&bars[kBarAna + i], P.npw);
            mbar_init(&bars[kBarSub + i], P.sub_pad > 0 ? P.sub_pad / 32 : 1);  // unused when L = 0
        }
        for (int i = 0; i < 3; ++i) mbar_init(&bars[kBarBase + i], P.nwt - P.sub_pad / 32);
        *reinterpret_cast<int*>(bars + kNumBars) = 0;  // task counter
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (n <= 0) return;

    if (warp == P.ncw + P.npw) {
        // ------------------------------------------------------------------
        // Copy warp (one lane): one bulk copy per plane into the staging
        // ring, as soon as every producer warp has read the slot's previous
        // plane.
        // ------------------------------------------------------------------
        if (lane != 0) return;
        const unsigned plane_bytes = (unsigned)(plane_elems * sizeof(T));
        int b = u0 % P.B, c = u0 / P.B;
        RingPos st;
        int issued = 0;
        for (int q = 0; q < n; ++q) {
            if (q >= NSTG && !mbar_wait(&bars[kBarStgEmpty + st.slot], (unsigned)((st.use - 1) & 1))) break;
            mbar_arrive_expect_tx(&bars[kBarStgFull + st.slot], plane_bytes);
            bulk_load(sm + P.stg + st.slot * P.stg_floats, x + ((size_t)b * P.C + c) * plane_elems, plane_bytes,
                      &bars[kBarStgFull + st.slot]);
            ++issued;
            st.next(NSTG);
            if (++b == P.B) {
                b = 0;
                ++c;
            }
        }
        // The last copies have landed in a normal run (the producer warps
        // waited for them); after a time-out elsewhere, do not leave the CTA
        // with a copy in flight.
        for (int q = issued > NSTG ? issued - NSTG : 0; q < issued; ++q)
            if (!mbar_wait(&bars[kBarStgFull + q % NSTG], (unsigned)((q / NSTG) & 1))) break;
        return;
    }

    if (warp >= P.ncw) {
        // ------------------------------------------------------------------
        // Producer warps: fold and analyse plane after plane, up to NS planes
        // ahead of the sub tiles.
        // ------------------------------------------------------------------
        const int np = P.npw * 32, ptid = tid - P.ncw * 32;
        int b = u0 % P.B, c = u0 / P.B;
        RingPos st, xr, sr, br, sbr;  // staging, X / weights, S; base(j - NX); sub(j - NS)
        for (int j = 0; j < n; ++j) {
            bool ok = mbar_wait(&bars[kBarStgFull + st.slot], (unsigned)(st.use & 1));
            if (ok && j >= NS && P.sub_pad > 0) ok = mbar_wait(&bars[kBarSub + sbr.slot], (unsigned)(sbr.use & 1));
            if (ok && j >= NX) ok = mbar_wait(&bars[kBarBase + br.slot], (unsigned)(br.use & 1));
            if (!ok) return;
            // Plane j - NX (the last in this weight slot) is of the same
            // channel exactly when b >= NX.
            float* wslot = sm + P.wbase + xr.slot * P.w_slot;
            if (j < NX || b < NX) ws_fold<K, BWD>(wslot, P, c, base_w, base_b, base_scale, wt_w, wt_scale, np, ptid);
            float* X0 = sm + xr.slot * P.x_slot + P.X.base + p * P.X.stride + p;
            analyse_plane<T, p, false, kToS>(sm + sr.slot * P.s_slot, P, sm + P.stg + st.slot * P.stg_floats, X0,
                                             P.X.stride, p, np, ptid, [] {});
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[kBarStgEmpty + st.slot]);
                mbar_arrive(&bars[kBarAna + (j & (kWsBarRing - 1))]);
            }
            st.next(NSTG);
            xr.next(NX);
            sr.next(NS);
            if (j >= NX) br.next(3);
            if (j >= NS) sbr.next(kWsBarRing);
            if (++b == P.B) {
                b = 0;
                ++c;
            }
        }
        return;
    }

    // ----------------------------------------------------------------------
    // Conv warps.
    // ----------------------------------------------------------------------
    const int nsub = P.n_sub_tiles, ntiles = P.n_step_tiles, nwt = P.nwt, ncw = P.ncw;
    const int nsub_pad = P.sub_pad, nsub_wt = nsub_pad / 32;  // warp-tiles [0, nsub_wt) hold sub tiles
    // Slot bases of the planes of step j: sub tiles of plane j (S, Q,
    // weights), base tiles of plane j-1 (X, Q, weights, y).
    struct StepBufs {
        const float *s, *w_sub, *x, *w_base, *q_base;
        float* q_sub;
        T* y;
    };
    // One tile of step j (lane's tile t), if it exists.
    auto run_tile = [&](int t, bool sub_on, bool base_on, const StepBufs& sb) {
        if (t >= ntiles || (t >= nsub && t < nsub_pad)) return;  // past the end, or sub-tile padding
        const bool base = t >= nsub_pad;
        if (base ? !base_on : !sub_on) return;
        const int4 d = desc[t];
        const float* win = (base ? sb.x : sb.s) + d.x;
        const float* wsl = base ? sb.w_base : sb.w_sub;
        float w[KK];
        load_weights<K>(wsl + d.z, w);
        const float b0 = base ? wsl[P.bias] : 0.f;
        float2 acc[8][2];
        conv_tile_regs<K, 8>(win, d.w & 0xfff, w, make_float2(b0, b0), acc);
        if (!base) {
            float* out = sb.q_sub + d.y;
            const int os = (d.w >> 12) & 0xfff;
#pragma unroll
            for (int o = 0; o < 8; ++o)
                *reinterpret_cast<float4*>(out + o * os) = make_float4(acc[o][0].x, acc[o][0].y, acc[o][1].x, acc[o][1].y);
        } else {
            const int r0 = d.y >> 16, c0 = d.y & 0xffff;
            synth_tile(sb.q_base, P, r0, c0, acc);
            T* yo = sb.y + (size_t)r0 * P.W + c0;
#pragma unroll
            for (int o = 0; o < 8; ++o)
                if (r0 + o < P.H)
                    gst4<T>(yo + (size_t)o * P.W, make_float4(acc[o][0].x, acc[o][0].y, acc[o][1].x, acc[o][1].y));
        }
    };
    // Tasks (one warp-tile each), taken from a shared counter in this
    // order: step j = the sub warp-tiles of plane j (j < n), then the base
    // warp-tiles of plane j-1 (j >= 1).  Each task waits for its own inputs
    // only and arrives once on its plane's barrier, so a warp never holds
    // back work that is ready.
    const int nbase_wt = nwt - nsub_wt, per_step = nsub_wt + nbase_wt;
    const int ntasks = n * per_step;  // n sub steps, n base steps
    int* task_ctr = reinterpret_cast<int*>(bars + kNumBars);
    for (;;) {
        int g = 0;
        if (lane == 0) g = atomicAdd(task_ctr, 1);
        g = __shfl_sync(0xffffffffu, g, 0);
        if (g >= ntasks) break;
        // Step j and warp-tile wt of this task.
        int j, wt;
        if (g < nsub_wt) {
            j = 0;
            wt = g;
        } else {
            const int h = g - nsub_wt;
            j = 1 + h / per_step;
            wt = h - (j - 1) * per_step;  // sub warp-tiles of plane j first, then base ones
            if (j == n) wt += nsub_wt;    // the last step holds base warp-tiles only
        }
        const bool is_sub = wt < nsub_wt;
        const int jj = is_sub ? j : j - 1;  // plane of the task
        const int u = u0 + jj;
        if (is_sub) {
            // ana(j) also means base(j-3) is complete: the Q slot is free.
            if (!mbar_wait(&bars[kBarAna + (jj & (kWsBarRing - 1))], (unsigned)((jj / kWsBarRing) & 1))) return;
        } else if (nsub_wt > 0) {
            if (!mbar_wait(&bars[kBarSub + (jj & (kWsBarRing - 1))], (unsigned)((jj / kWsBarRing) & 1))) return;
        } else if (!mbar_wait(&bars[kBarAna + (jj & (kWsBarRing - 1))], (unsigned)((jj / kWsBarRing) & 1))) {
            return;  // L = 0: no sub tiles; the base tiles take the analysis directly
        }
        StepBufs sb;
        const int xsl = jj % NX, qsl = jj % kWsQSlots;
        sb.s = sm + (jj % NS) * P.s_slot;
        sb.w_sub = sb.w_base = sm + P.wbase + xsl * P.w_slot;
        sb.q_sub = sm + qsl * P.q_slot;
        sb.q_base = sb.q_sub;
        sb.x = sm + xsl * P.x_slot;
        sb.y = y + ((size_t)(u % P.B) * P.C + u / P.B) * plane_elems;
        run_tile(32 * wt + lane, is_sub, !is_sub, sb);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(is_sub ? &bars[kBarSub + (jj & (kWsBarRing - 1))] : &bars[kBarBase + jj % 3]);
    }
}

}  // namespace wtc
