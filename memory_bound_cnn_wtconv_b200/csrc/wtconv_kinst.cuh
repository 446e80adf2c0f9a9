// Kernel instantiations and launchers for one kernel size; included by
// wtconv_k<K>.cu with WTC_K defined.
#include <cuda_bf16.h>

#include <algorithm>

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

// cudaFuncSetAttribute for the dynamic shared-memory opt-in, once per kernel
// and device (idempotent; a repeated call is harmless).
template <class F>
cudaError_t opt_in_smem(F* fn, bool (&done)[kMaxDevices]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev] = true;
    return e;
}

template <int TR, typename T, bool BWD>
cudaError_t fused_typed(const Plan& P, const FusedArgs& a, cudaStream_t s) {
    static bool done[kMaxDevices] = {};
    auto* fn = wtconv_fused_kernel<WTC_K, TR, 4, T, BWD>;
    cudaError_t e = opt_in_smem(fn, done);
    if (e != cudaSuccess) return e;
    // Persistent grid: every resident CTA slot of the device, at most one CTA per plane.
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, P.nthreads, (size_t)P.smem_floats * 4)) !=
        cudaSuccess)
        return e;
    const long long units = (long long)P.B * P.C;
    const int grid = (int)std::min<long long>(units, (long long)sms * std::max(per_sm, 1));
    fn<<<grid, P.nthreads, (size_t)P.smem_floats * 4, s>>>(
        static_cast<const T*>(a.x), a.base_w, a.base_b, a.base_scale, a.wt_w, a.wt_scale, static_cast<T*>(a.y),
        P);
    return cudaGetLastError();
}

template <int TR, typename T>
cudaError_t bwdw_typed(const Plan& P, const BwdwArgs& a, cudaStream_t s) {
    static bool done[kMaxDevices] = {};
    auto* fn = wtconv_bwdw_partial_kernel<WTC_K, TR, 4, T>;
    cudaError_t e = opt_in_smem(fn, done);
    if (e != cudaSuccess) return e;
    fn<<<dim3(P.C, P.groups), P.nthreads, (size_t)P.smem_floats * 4, s>>>(
        static_cast<const T*>(a.x), static_cast<const T*>(a.dy), a.part, P);
    return cudaGetLastError();
}

template <int TR>
cudaError_t fused_tr(const Plan& P, int dtype, bool bwd, const FusedArgs& a, cudaStream_t s) {
    if (dtype == 0) return bwd ? fused_typed<TR, float, true>(P, a, s) : fused_typed<TR, float, false>(P, a, s);
    return bwd ? fused_typed<TR, __nv_bfloat16, true>(P, a, s) : fused_typed<TR, __nv_bfloat16, false>(P, a, s);
}

template <int TR>
cudaError_t bwdw_tr(const Plan& P, int dtype, const BwdwArgs& a, cudaStream_t s) {
    if (dtype == 0) return bwdw_typed<TR, float>(P, a, s);
    return bwdw_typed<TR, __nv_bfloat16>(P, a, s);
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

cudaError_t WTC_CAT(launch_bwdw_k, WTC_K)(const Plan& P, int dtype, const BwdwArgs& a, cudaStream_t s) {
    switch (P.TR) {
        case 7: return bwdw_tr<7>(P, dtype, a, s);
        case 8: return bwdw_tr<8>(P, dtype, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace wtc
