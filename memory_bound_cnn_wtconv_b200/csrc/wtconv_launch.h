// Launchers for one kernel size K, defined in wtconv_k<K>.cu and called by the
// C ABI in wtconv_api.cu after validation and planning.
#pragma once

#include <cuda_runtime.h>

#include "wtconv_kernels.cuh"
#include "wtconv_plan.h"
#include "wtconv_planner.h"

namespace wtc {

struct FusedArgs {
    const void* x;
    const float *base_w, *base_b, *base_scale, *wt_w, *wt_scale;
    void* y;
};

struct BwdwArgs {
    const void* x;
    const void* dy;
    float* part;
    GradArgs ga;
};

struct BwdArgs {
    const void* x;
    const void* dy;
    void* dx;
    float* part;
    GradArgs ga;
};

#define WTC_DECLARE_LAUNCHERS(KV)                                                                     \
    cudaError_t launch_fused_k##KV(const Plan& P, int dtype, bool bwd, const FusedArgs& a, cudaStream_t s); \
    cudaError_t launch_bwdw_k##KV(const Plan& P, int dtype, const BwdwArgs& a, cudaStream_t s);           \
    cudaError_t launch_bwd_k##KV(const Plan& P, int dtype, const BwdArgs& a, cudaStream_t s);

WTC_DECLARE_LAUNCHERS(1)
WTC_DECLARE_LAUNCHERS(3)
WTC_DECLARE_LAUNCHERS(5)
WTC_DECLARE_LAUNCHERS(7)

#undef WTC_DECLARE_LAUNCHERS

// Dispatch on the kernel size (every entry point launches through these).
inline cudaError_t launch_fused(const Plan& P, int dtype, bool bwd, const FusedArgs& a, cudaStream_t s) {
    switch (P.k) {
        case 1: return launch_fused_k1(P, dtype, bwd, a, s);
        case 3: return launch_fused_k3(P, dtype, bwd, a, s);
        case 5: return launch_fused_k5(P, dtype, bwd, a, s);
        case 7: return launch_fused_k7(P, dtype, bwd, a, s);
        default: return cudaErrorInvalidValue;
    }
}

inline cudaError_t launch_bwdw(const Plan& P, int dtype, const BwdwArgs& a, cudaStream_t s) {
    switch (P.k) {
        case 1: return launch_bwdw_k1(P, dtype, a, s);
        case 3: return launch_bwdw_k3(P, dtype, a, s);
        case 5: return launch_bwdw_k5(P, dtype, a, s);
        case 7: return launch_bwdw_k7(P, dtype, a, s);
        default: return cudaErrorInvalidValue;
    }
}

inline cudaError_t launch_bwd(const Plan& P, int dtype, const BwdArgs& a, cudaStream_t s) {
    switch (P.k) {
        case 1: return launch_bwd_k1(P, dtype, a, s);
        case 3: return launch_bwd_k3(P, dtype, a, s);
        case 5: return launch_bwd_k5(P, dtype, a, s);
        case 7: return launch_bwd_k7(P, dtype, a, s);
        default: return cudaErrorInvalidValue;
    }
}

inline GradArgs grad_args(const float* base_w, const float* base_b, const float* base_scale, const float* wt_w,
                          const float* wt_scale, float* d_base_w, float* d_base_b, float* d_base_scale,
                          float* d_wt_w, float* d_wt_scale, unsigned* counters) {
    return GradArgs{base_w, base_b, base_scale, wt_w, wt_scale, d_base_w, d_base_b, d_base_scale,
                    d_wt_w, d_wt_scale, counters};
}

// SM count of the current device, which the plans size their grids for; a
// B200's 148 when no device can be queried (then nothing can launch, and
// only host-side planning, such as a workspace size, is asked for).
inline int planning_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();  // clear the (non-sticky) query error
        return kB200SMs;
    }
    return n;
}

// Weight-gradient workspace: the partial vectors, then one arrival counter
// per channel (16-byte aligned).
inline size_t partial_floats(const Plan& P) { return (size_t)P.C * P.parts * P.nv; }
inline size_t counters_offset_floats(const Plan& P) { return (partial_floats(P) + 3) & ~(size_t)3; }
inline size_t workspace_bytes_of(const Plan& P) { return (counters_offset_floats(P) + (size_t)P.C) * 4; }

}  // namespace wtc
