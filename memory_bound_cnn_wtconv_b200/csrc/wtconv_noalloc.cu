// wtconv_backward_weight_noalloc: the weight gradient without a caller-provided
// workspace, for callers that cannot allocate device memory (see
// include/wtconv.h).  The per-block partial sums live in a fixed-size
// device array owned by this library instead of in a cudaMalloc'd buffer.
#include <cuda_runtime.h>

#include "../../include/wtconv.h"
#include "wtconv_launch.h"
#include "wtconv_plan.h"
#include "wtconv_planner.h"

namespace wtc {
namespace {

// Partial sums of the weight gradient: at most this many floats (4 MiB).
// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocScratchFloats = (size_t)1 << 20;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Device address of g_noalloc_scratch in the current context.  Looked up on
// every call (a host-side lookup, no device work), so that a new context on
// the device (after cudaDeviceReset, or a context other than the primary one)
// gets its own module's address.  The host-side name is only a stand-in for
// the device array and must never be passed to a kernel.
float* scratch_address(cudaError_t* err) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    return *err == cudaSuccess ? static_cast<float*>(p) : nullptr;
}

}  // namespace
}  // namespace wtc

using namespace wtc;

extern "C" wtconv_status_t wtconv_backward_weight_noalloc(
    const wtconv_desc_t* d, const void* x, const void* dy, const float* base_w, const float* base_b,
    const float* base_scale, const float* wt_w, const float* wt_scale, float* d_base_w, float* d_base_b,
    float* d_base_scale, float* d_wt_w, float* d_wt_scale, wtconv_stream_t stream) {
    wtconv_status_t st = validate(d);
    if (st != WTCONV_OK) return st;
    if (!x || !dy || !base_w || !base_b || !base_scale || !d_base_w || !d_base_b || !d_base_scale)
        return WTCONV_ERR_NULLPTR;
    if (d->L > 0 && (!wt_w || !wt_scale || !d_wt_w || !d_wt_scale)) return WTCONV_ERR_NULLPTR;
    if (!aligned16(x) || !aligned16(dy)) return WTCONV_ERR_MISALIGNED;
    Plan P;
    st = make_plan(d, kBackwardWeight, planning_sm_count(), &P);
    if (st != WTCONV_OK) return st;
    // The partials and the per-channel arrival counters of this plan
    // (workspace_bytes_of); beyond the fixed array the call is rejected (use
    // wtconv_backward_weight with a workspace instead).
    if (workspace_bytes_of(P) > kNoAllocScratchFloats * sizeof(float)) return WTCONV_ERR_WORKSPACE;
    cudaError_t err = cudaSuccess;
    float* part = scratch_address(&err);
    if (part == nullptr) return WTCONV_ERR_CUDA;
    // Every partial slot the final step reads is written by the same launch;
    // only the counters are cleared.
    unsigned* counters = reinterpret_cast<unsigned*>(part + counters_offset_floats(P));
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(counters, 0, (size_t)P.C * sizeof(unsigned), s) != cudaSuccess) return WTCONV_ERR_CUDA;
    BwdwArgs a{x, dy, part,
               grad_args(base_w, base_b, base_scale, wt_w, wt_scale, d_base_w, d_base_b, d_base_scale, d_wt_w,
                         d_wt_scale, counters)};
    if (launch_bwdw(P, d->dtype, a, s) != cudaSuccess) return WTCONV_ERR_CUDA;
    return WTCONV_OK;
}
