// Kernel instantiations and launchers for one kernel size; included by
// wtconv_k<K>.cu with WTC_K defined.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "wtconv_kernels.cuh"
#include "wtconv_launch.h"

#ifndef WTC_K
#error "define WTC_K before including wtconv_kinst.cuh"
#endif

#define WTC_CAT2(a, b) a##b
#define WTC_CAT(a, b) WTC_CAT2(a, b)

namespace wtc {

namespace {

constexpr int kMaxDevices = 64;

// cudaFuncSetAttribute for the dynamic shared-memory opt-in (and the
// non-portable cluster-size opt-in for 16-CTA clusters), once per kernel and
// device.  The attributes are idempotent, so host threads racing on the first
// call both set them; the flags are atomic so that the race is benign.
template <class F>
cudaError_t opt_in_smem(F* fn, std::atomic<bool> (&done)[kMaxDevices]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(true, std::memory_order_release);
    return e;
}

// Launch configuration; planes split into strips (and NHWC channel octets)
// run as clusters of cluster_ctas(P) CTAs along x.
struct Launch {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    Launch(const Plan& P, dim3 grid, cudaStream_t s) {
        cfg = cudaLaunchConfig_t{};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(P.nthreads);
        cfg.dynamicSmemBytes = (size_t)P.smem_floats * 4;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 0;
        if (cluster_ctas(P) > 1) {
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = cluster_ctas(P);
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.numAttrs = 1;
        }
    }
};

template <int TR, typename T, bool BWD, bool GENERAL, bool OCT = false>
cudaError_t fused_typed(const Plan& P, const FusedArgs& a, cudaStream_t s) {
    static std::atomic<bool> done[kMaxDevices] = {};
    auto* fn = wtconv_fused_kernel<WTC_K, TR, 4, T, BWD, GENERAL, OCT>;
    cudaError_t e = opt_in_smem(fn, done);
    if (e != cudaSuccess) return e;
    // Persistent grid: every resident CTA slot (cluster slot, for strips and
    // octets) of the device, at most one CTA (cluster) per plane (octet).
    const int cs = cluster_ctas(P);
    const long long units = (long long)P.B * (P.oct ? P.C / 8 : P.C);
    long long teams = 0;
    Launch L(P, dim3(1), s);
    if (cs > 1) {
        L.cfg.gridDim = dim3(cs * 64);  // any multiple of the cluster size, for the query
        int clusters = 0;
        if ((e = cudaOccupancyMaxActiveClusters(&clusters, fn, &L.cfg)) != cudaSuccess) return e;
        if (clusters < 1) return cudaErrorInvalidConfiguration;
        teams = clusters;
    } else {
        int dev = 0, sms = 0, per_sm = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, P.nthreads, (size_t)P.smem_floats * 4)) !=
            cudaSuccess)
            return e;
        teams = (long long)sms * std::max(per_sm, 1);
    }
    L.cfg.gridDim = dim3((unsigned)(std::min<long long>(units, teams) * cs));
    e = cudaLaunchKernelEx(&L.cfg, fn, static_cast<const T*>(a.x), a.base_w, a.base_b, a.base_scale, a.wt_w,
                           a.wt_scale, static_cast<T*>(a.y), P);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int TR, typename T, bool GENERAL, bool OCT = false>
cudaError_t bwdw_typed(const Plan& P, const BwdwArgs& a, cudaStream_t s) {
    static std::atomic<bool> done[kMaxDevices] = {};
    auto* fn = wtconv_bwdw_partial_kernel<WTC_K, TR, 4, T, GENERAL, OCT>;
    cudaError_t e = opt_in_smem(fn, done);
    if (e != cudaSuccess) return e;
    Launch L(P, dim3(P.C * P.nstrips, P.groups), s);
    if (cluster_ctas(P) > 1) {
        // A cluster that can never be resident is an error, not a hang.
        int clusters = 0;
        if ((e = cudaOccupancyMaxActiveClusters(&clusters, fn, &L.cfg)) != cudaSuccess) return e;
        if (clusters < 1) return cudaErrorInvalidConfiguration;
    }
    e = cudaLaunchKernelEx(&L.cfg, fn, static_cast<const T*>(a.x), static_cast<const T*>(a.dy), a.part, a.ga, P);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int TR, typename T>
cudaError_t fused_t(const Plan& P, bool bwd, const FusedArgs& a, cudaStream_t s) {
    // NHWC channel octets, and the general instantiation for cluster
    // strips, planes padded on chip and / or the NHWC gather.
    if (P.oct)
        return bwd ? fused_typed<TR, T, true, true, true>(P, a, s) : fused_typed<TR, T, false, true, true>(P, a, s);
    if (P.nstrips > 1 || P.padded || P.nhwc)
        return bwd ? fused_typed<TR, T, true, true>(P, a, s) : fused_typed<TR, T, false, true>(P, a, s);
    return bwd ? fused_typed<TR, T, true, false>(P, a, s) : fused_typed<TR, T, false, false>(P, a, s);
}

template <int TR, typename T, bool OCT = false>
cudaError_t bwd_typed(const Plan& P, const BwdArgs& a, cudaStream_t s) {
    static std::atomic<bool> done[kMaxDevices] = {};
    auto* fn = wtconv_backward_kernel<WTC_K, TR, 4, T, OCT>;
    cudaError_t e = opt_in_smem(fn, done);
    if (e != cudaSuccess) return e;
    const GradArgs& g = a.ga;
    if constexpr (OCT) {
        // Clusters of the 8 channels of an octet (grid.x = C, a multiple of 8).
        Launch L(P, dim3(P.C, P.groups), s);
        int clusters = 0;
        if ((e = cudaOccupancyMaxActiveClusters(&clusters, fn, &L.cfg)) != cudaSuccess) return e;
        if (clusters < 1) return cudaErrorInvalidConfiguration;
        e = cudaLaunchKernelEx(&L.cfg, fn, static_cast<const T*>(a.x), static_cast<const T*>(a.dy), g.base_w,
                               g.base_b, g.base_scale, g.wt_w, g.wt_scale, static_cast<T*>(a.dx), a.part, g, P);
        if (e != cudaSuccess) return e;
    } else {
        fn<<<dim3(P.C, P.groups), P.nthreads, (size_t)P.smem_floats * 4, s>>>(
            static_cast<const T*>(a.x), static_cast<const T*>(a.dy), g.base_w, g.base_b, g.base_scale, g.wt_w,
            g.wt_scale, static_cast<T*>(a.dx), a.part, g, P);
    }
    return cudaGetLastError();
}

template <int TR>
cudaError_t fused_tr(const Plan& P, int dtype, bool bwd, const FusedArgs& a, cudaStream_t s) {
    if (dtype == 0) return fused_t<TR, float>(P, bwd, a, s);
    return fused_t<TR, __nv_bfloat16>(P, bwd, a, s);
}

template <int TR>
cudaError_t bwdw_tr(const Plan& P, int dtype, const BwdwArgs& a, cudaStream_t s) {
    const bool strips = P.nstrips > 1 || P.padded || P.nhwc;  // the general instantiation
    if (P.oct)
        return dtype == 0 ? bwdw_typed<TR, float, true, true>(P, a, s) : bwdw_typed<TR, __nv_bfloat16, true, true>(P, a, s);
    if (dtype == 0) return strips ? bwdw_typed<TR, float, true>(P, a, s) : bwdw_typed<TR, float, false>(P, a, s);
    return strips ? bwdw_typed<TR, __nv_bfloat16, true>(P, a, s) : bwdw_typed<TR, __nv_bfloat16, false>(P, a, s);
}

}  // namespace

cudaError_t WTC_CAT(launch_fused_k, WTC_K)(const Plan& P, int dtype, bool bwd, const FusedArgs& a,
                                           cudaStream_t s) {
    switch (P.TR) {
        case 7: return fused_tr<7>(P, dtype, bwd, a, s);
        case 8: return fused_tr<8>(P, dtype, bwd, a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t WTC_CAT(launch_bwd_k, WTC_K)(const Plan& P, int dtype, const BwdArgs& a, cudaStream_t s) {
    switch (P.TR) {
        case 7:
            if (P.oct) return dtype == 0 ? bwd_typed<7, float, true>(P, a, s) : bwd_typed<7, __nv_bfloat16, true>(P, a, s);
            return dtype == 0 ? bwd_typed<7, float>(P, a, s) : bwd_typed<7, __nv_bfloat16>(P, a, s);
        case 8:
            if (P.oct) return dtype == 0 ? bwd_typed<8, float, true>(P, a, s) : bwd_typed<8, __nv_bfloat16, true>(P, a, s);
            return dtype == 0 ? bwd_typed<8, float>(P, a, s) : bwd_typed<8, __nv_bfloat16>(P, a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t WTC_CAT(launch_bwdw_k, WTC_K)(const Plan& P, int dtype, const BwdwArgs& a, cudaStream_t s) {
    switch (P.TR) {
        case 7: return bwdw_tr<7>(P, dtype, a, s);
        case 8: return bwdw_tr<8>(P, dtype, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace wtc
