// Launchers for one kernel size K, defined in wtconv_k<K>.cu and called by the
// C ABI in wtconv_api.cu after validation and planning.
#pragma once

#include <cuda_runtime.h>

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
};

struct BwdArgs {
    const void* x;
    const void* dy;
    const float *base_w, *base_b, *base_scale, *wt_w, *wt_scale;
    void* dx;
    float* part;
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

cudaError_t launch_bwdw_finish(const Plan& P, const float* part, const float* base_w, const float* base_b,
                               const float* base_scale, const float* wt_w, const float* wt_scale,
                               float* d_base_w, float* d_base_b, float* d_base_scale, float* d_wt_w,
                               float* d_wt_scale, cudaStream_t s);

}  // namespace wtc
