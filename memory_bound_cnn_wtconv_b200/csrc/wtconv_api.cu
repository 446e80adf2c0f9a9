// C ABI of the WTConv library: argument validation, on-chip planning and
// kernel dispatch.  Declarations and contracts: include/wtconv.h.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "../../include/wtconv.h"
#include "wtconv_kernels.cuh"
#include "wtconv_launch.h"
#include "wtconv_plan.h"
#include "wtconv_planner.h"

namespace wtc {

namespace {

// Workspace both weight-gradient paths accept: the larger of the two plans'.
size_t workspace_bytes_any(const wtconv_desc_t* d, int sms) {
    Plan P;
    size_t n = 0;
    if (make_plan(d, kBackwardWeight, sms, &P) == WTCONV_OK) n = workspace_bytes_of(P);
    if (make_plan(d, kBackward, sms, &P) == WTCONV_OK) n = std::max(n, workspace_bytes_of(P));
    return n;
}

// Shared checks of the calls that write parameter gradients.
wtconv_status_t check_grad_args(const wtconv_desc_t* d, const void* x, const void* dy, const float* base_w,
                                const float* base_b, const float* base_scale, const float* wt_w,
                                const float* wt_scale, const float* d_base_w, const float* d_base_b,
                                const float* d_base_scale, const float* d_wt_w, const float* d_wt_scale) {
    if (!x || !dy || !base_w || !base_b || !base_scale || !d_base_w || !d_base_b || !d_base_scale)
        return WTCONV_ERR_NULLPTR;
    if (d->L > 0 && (!wt_w || !wt_scale || !d_wt_w || !d_wt_scale)) return WTCONV_ERR_NULLPTR;
    if (!aligned16(x) || !aligned16(dy)) return WTCONV_ERR_MISALIGNED;
    return WTCONV_OK;
}

// The one-pass kernel on plan P (validated arguments).
wtconv_status_t run_one_pass(const wtconv_desc_t* d, const Plan& P, int sms, const void* x, const void* dy,
                             const float* base_w, const float* base_b, const float* base_scale, const float* wt_w,
                             const float* wt_scale, void* dx, float* d_base_w, float* d_base_b,
                             float* d_base_scale, float* d_wt_w, float* d_wt_scale, void* workspace,
                             size_t workspace_bytes, cudaStream_t s) {
    if (!workspace || workspace_bytes < workspace_bytes_any(d, sms)) return WTCONV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return WTCONV_ERR_MISALIGNED;
    float* part = static_cast<float*>(workspace);
    unsigned* counters = reinterpret_cast<unsigned*>(part + counters_offset_floats(P));
    if (cudaMemsetAsync(counters, 0, (size_t)P.C * sizeof(unsigned), s) != cudaSuccess) return WTCONV_ERR_CUDA;
    BwdArgs a{x, dy, dx, part,
              grad_args(base_w, base_b, base_scale, wt_w, wt_scale, d_base_w, d_base_b, d_base_scale, d_wt_w,
                        d_wt_scale, counters)};
    if (launch_bwd(P, d->dtype, a, s) != cudaSuccess) return WTCONV_ERR_CUDA;
    return WTCONV_OK;
}

}  // namespace

}  // namespace wtc

using namespace wtc;

extern "C" {

const char* wtconv_status_string(wtconv_status_t s) {
    switch (s) {
        case WTCONV_OK: return "ok";
        case WTCONV_ERR_NULLPTR: return "a required pointer is NULL";
        case WTCONV_ERR_BAD_SHAPE: return "bad shape (B, C, H, W > 0; W % 4 == 0; rows of whole 16-byte chunks)";
        case WTCONV_ERR_BAD_K: return "unsupported kernel size (k must be 1, 3, 5 or 7)";
        case WTCONV_ERR_BAD_L: return "unsupported level count (0 <= L <= 6)";
        case WTCONV_ERR_MISALIGNED: return "activation pointer not 16-byte aligned";
        case WTCONV_ERR_DTYPE: return "unknown activation dtype";
        case WTCONV_ERR_WORKSPACE: return "workspace missing or too small";
        case WTCONV_ERR_UNSUPPORTED: return "plane too large to stage on chip";
        case WTCONV_ERR_CUDA: return "CUDA runtime error";
        case WTCONV_ERR_LAYOUT: return "unknown activation layout (0 = NCHW, 1 = NHWC)";
    }
    return "unknown status";
}

size_t wtconv_workspace_bytes(const wtconv_desc_t* d) {
    if (validate(d) != WTCONV_OK) return 0;
    return workspace_bytes_any(d, planning_sm_count());
}

wtconv_status_t wtconv_forward(const wtconv_desc_t* d, const void* x, const float* base_w, const float* base_b,
                               const float* base_scale, const float* wt_w, const float* wt_scale, void* y,
                               wtconv_stream_t stream) {
    wtconv_status_t st = validate(d);
    if (st != WTCONV_OK) return st;
    if (!x || !y || !base_w || !base_b || !base_scale) return WTCONV_ERR_NULLPTR;
    if (d->L > 0 && (!wt_w || !wt_scale)) return WTCONV_ERR_NULLPTR;
    if (!aligned16(x) || !aligned16(y)) return WTCONV_ERR_MISALIGNED;
    Plan P;
    st = make_plan(d, kForward, planning_sm_count(), &P);
    if (st != WTCONV_OK) return st;
    FusedArgs a{x, base_w, base_b, base_scale, wt_w, wt_scale, y};
    return launch_fused(P, d->dtype, false, a, (cudaStream_t)stream) == cudaSuccess ? WTCONV_OK
                                                                                   : WTCONV_ERR_CUDA;
}

wtconv_status_t wtconv_backward_input(const wtconv_desc_t* d, const void* dy, const float* base_w,
                                      const float* base_scale, const float* wt_w, const float* wt_scale,
                                      void* dx, wtconv_stream_t stream) {
    wtconv_status_t st = validate(d);
    if (st != WTCONV_OK) return st;
    if (!dy || !dx || !base_w || !base_scale) return WTCONV_ERR_NULLPTR;
    if (d->L > 0 && (!wt_w || !wt_scale)) return WTCONV_ERR_NULLPTR;
    if (!aligned16(dy) || !aligned16(dx)) return WTCONV_ERR_MISALIGNED;
    Plan P;
    st = make_plan(d, kBackwardInput, planning_sm_count(), &P);
    if (st != WTCONV_OK) return st;
    // base_b is unused by the transpose; pass base_scale as a valid pointer.
    FusedArgs a{dy, base_w, base_scale, base_scale, wt_w, wt_scale, dx};
    return launch_fused(P, d->dtype, true, a, (cudaStream_t)stream) == cudaSuccess ? WTCONV_OK
                                                                                  : WTCONV_ERR_CUDA;
}

wtconv_status_t wtconv_backward_weight(const wtconv_desc_t* d, const void* x, const void* dy,
                                       const float* base_w, const float* base_b, const float* base_scale,
                                       const float* wt_w, const float* wt_scale, float* d_base_w,
                                       float* d_base_b, float* d_base_scale, float* d_wt_w,
                                       float* d_wt_scale, void* workspace, size_t workspace_bytes,
                                       wtconv_stream_t stream) {
    wtconv_status_t st = validate(d);
    if (st != WTCONV_OK) return st;
    st = check_grad_args(d, x, dy, base_w, base_b, base_scale, wt_w, wt_scale, d_base_w, d_base_b, d_base_scale,
                         d_wt_w, d_wt_scale);
    if (st != WTCONV_OK) return st;
    const int sms = planning_sm_count();
    Plan P;
    st = make_plan(d, kBackwardWeight, sms, &P);
    if (st != WTCONV_OK) return st;
    if (!workspace || workspace_bytes < workspace_bytes_any(d, sms)) return WTCONV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return WTCONV_ERR_MISALIGNED;
    float* part = static_cast<float*>(workspace);
    unsigned* counters = reinterpret_cast<unsigned*>(part + counters_offset_floats(P));
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(counters, 0, (size_t)P.C * sizeof(unsigned), s) != cudaSuccess) return WTCONV_ERR_CUDA;
    BwdwArgs a{x, dy, part,
               grad_args(base_w, base_b, base_scale, wt_w, wt_scale, d_base_w, d_base_b, d_base_scale, d_wt_w,
                         d_wt_scale, counters)};
    if (launch_bwdw(P, d->dtype, a, s) != cudaSuccess) return WTCONV_ERR_CUDA;
    return WTCONV_OK;
}

wtconv_status_t wtconv_backward(const wtconv_desc_t* d, const void* x, const void* dy, const float* base_w,
                                const float* base_b, const float* base_scale, const float* wt_w,
                                const float* wt_scale, void* dx, float* d_base_w, float* d_base_b,
                                float* d_base_scale, float* d_wt_w, float* d_wt_scale, void* workspace,
                                size_t workspace_bytes, wtconv_stream_t stream) {
    wtconv_status_t st = validate(d);
    if (st != WTCONV_OK) return st;
    if (!dx) return WTCONV_ERR_NULLPTR;
    st = check_grad_args(d, x, dy, base_w, base_b, base_scale, wt_w, wt_scale, d_base_w, d_base_b, d_base_scale,
                         d_wt_w, d_wt_scale);
    if (st != WTCONV_OK) return st;
    if (!aligned16(dx)) return WTCONV_ERR_MISALIGNED;
    const int sms = planning_sm_count();
    // The one pass where its plan exists and the planner prefers it to the
    // two passes' plans (prefer_one_pass: tile rows on the busiest SM
    // sub-partition, then CTAs per SM); else the input- and weight-gradient
    // passes, with the same results.
    Plan P, Pin, Pw;
    st = make_plan(d, kBackward, sms, &P);
    if (st != WTCONV_OK && st != WTCONV_ERR_UNSUPPORTED) return st;
    bool one_pass = st == WTCONV_OK;
    if (one_pass && make_plan(d, kBackwardInput, sms, &Pin) == WTCONV_OK &&
        make_plan(d, kBackwardWeight, sms, &Pw) == WTCONV_OK)
        one_pass = prefer_one_pass(P, Pin, Pw);
    if (one_pass)
        return run_one_pass(d, P, sms, x, dy, base_w, base_b, base_scale, wt_w, wt_scale, dx, d_base_w, d_base_b,
                            d_base_scale, d_wt_w, d_wt_scale, workspace, workspace_bytes, (cudaStream_t)stream);
    // Check everything the weight pass checks before the input pass writes dx.
    st = make_plan(d, kBackwardWeight, sms, &Pw);
    if (st != WTCONV_OK) return st;
    if (!workspace || workspace_bytes < workspace_bytes_any(d, sms)) return WTCONV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return WTCONV_ERR_MISALIGNED;
    st = wtconv_backward_input(d, dy, base_w, base_scale, wt_w, wt_scale, dx, stream);
    if (st != WTCONV_OK) return st;
    return wtconv_backward_weight(d, x, dy, base_w, base_b, base_scale, wt_w, wt_scale, d_base_w, d_base_b,
                                  d_base_scale, d_wt_w, d_wt_scale, workspace, workspace_bytes, stream);
}

wtconv_status_t wtconv_backward_one_pass(const wtconv_desc_t* d, const void* x, const void* dy,
                                         const float* base_w, const float* base_b, const float* base_scale,
                                         const float* wt_w, const float* wt_scale, void* dx, float* d_base_w,
                                         float* d_base_b, float* d_base_scale, float* d_wt_w, float* d_wt_scale,
                                         void* workspace, size_t workspace_bytes, wtconv_stream_t stream) {
    wtconv_status_t st = validate(d);
    if (st != WTCONV_OK) return st;
    if (!dx) return WTCONV_ERR_NULLPTR;
    st = check_grad_args(d, x, dy, base_w, base_b, base_scale, wt_w, wt_scale, d_base_w, d_base_b, d_base_scale,
                         d_wt_w, d_wt_scale);
    if (st != WTCONV_OK) return st;
    if (!aligned16(dx)) return WTCONV_ERR_MISALIGNED;
    const int sms = planning_sm_count();
    Plan P;
    st = make_plan(d, kBackward, sms, &P);
    if (st != WTCONV_OK) return st;
    return run_one_pass(d, P, sms, x, dy, base_w, base_b, base_scale, wt_w, wt_scale, dx, d_base_w, d_base_b,
                        d_base_scale, d_wt_w, d_wt_scale, workspace, workspace_bytes, (cudaStream_t)stream);
}

}  // extern "C"
