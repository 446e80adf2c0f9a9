// Launchers for one kernel size K, defined in wtconv_k<K>.cu and called by the
// C ABI in wtconv_api.cu after validation and planning.
#pragma once

#include <cuda_runtime.h>

#include "wtconv_kernels.cuh"
#include "wtconv_plan.h"

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

// Weight-gradient workspace: the partial vectors, then one arrival counter
// per channel (16-byte aligned).
inline size_t partial_floats(const Plan& P) { return (size_t)P.C * P.parts * P.nv; }
inline size_t counters_offset_floats(const Plan& P) { return (partial_floats(P) + 3) & ~(size_t)3; }
inline size_t workspace_bytes_of(const Plan& P) { return (counters_offset_floats(P) + (size_t)P.C) * 4; }

}  // namespace wtc
