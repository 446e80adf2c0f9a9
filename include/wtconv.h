/*
 * wtconv.h -- C ABI of the B200 (sm_100a) wavelet-convolution (WTConv) library.
 *
 * The layer (arXiv 2608.10805, "Fast and Memory-Efficient Wavelet
 * Convolutions via I/O-Aware Reformulation", Abstract) is, per sample b and
 * channel c, the sum of two branches on an H x W plane:
 *
 *   base branch:     yb = base_scale[c] * (dwconv(x, base_w[c]) + base_b[c])
 *   wavelet branch:  an L-level orthonormal 2-D Haar analysis that splits the
 *                    plane into LL/LH/HL/HH subbands and recurses on the raw
 *                    LL subband; every subband s of level l gets its own
 *                    depthwise k x k conv scaled by wt_scale[l][c][s]; the
 *                    inverse Haar synthesis adds each coarser level's
 *                    reconstruction into the next finer LL.
 *   y = yb + (wavelet branch)
 *
 * dwconv is cross-correlation with "same" zero padding (p = k/2) at each
 * subband's own resolution.  Subband order: 0 = LL, 1 = LH (high-pass along
 * H, i.e. between rows), 2 = HL (high-pass along W), 3 = HH.  One Haar step
 * maps the 2x2 block (a b / c d) to ((a+b+c+d), (a+b-c-d), (a-b+c-d),
 * (a-b-c+d)) / 2.
 *
 * The kernels apply the abstract's three reformulations: the Haar analysis
 * is recomputed on chip for every level (nothing but x is read from HBM), the
 * synthesis is one pass over the output indexed by the bits of the output
 * coordinates (nothing but y is written), and the per-channel and
 * per-subband scales are folded into the conv weights before the convs run.
 *
 * Conventions for every entry point:
 *   - Layouts.  Activations are NCHW or NHWC (desc->layout), contiguous,
 *     stored as float32 or bf16 (desc->dtype); arithmetic is float32; x, dy,
 *     y and dx of one call share the layout.  Parameters and gradients are
 *     float32, contiguous:  base_w [C][k][k], base_b [C], base_scale [C],
 *     wt_w [L][C][4][k][k], wt_scale [L][C][4].
 *   - Pointers are DEVICE pointers on the current device; activation pointers
 *     must be 16-byte aligned and W must be a multiple of 4.
 *   - Ownership.  The caller owns every buffer.  The library allocates
 *     nothing, keeps no pointer after returning, and never synchronises: all
 *     work is enqueued on `stream` (0 = the legacy default stream).
 *   - Gradients are overwritten, not accumulated.
 *   - Errors.  Arguments are validated on the host before any launch; a
 *     non-OK status means nothing was enqueued and no output was touched.
 *     A launch failure returns WTCONV_ERR_CUDA.  Faults of an enqueued kernel
 *     surface at the caller's next synchronisation, as for any CUDA call.
 *   - Limits: k in {1, 3, 5, 7}; 0 <= L <= 6.  H and W need not be
 *     multiples of 2^L: such planes are zero-padded at the bottom and right to
 *     the next multiples on chip, the layer applied, and only the H x W outputs
 *     written (the input gradient is the transpose of that cropped map; the
 *     weight gradients sum over the padded plane, where dy is zero); their rows
 *     must be whole 16-byte chunks (W a multiple of 4 for fp32, 8 for bf16).
 *     A plane that does not fit on one SM is split into 2, 4, 8 or 16 row
 *     strips held by the CTAs of a thread-block cluster (strip height a
 *     multiple of 2^L and of 4; 16-CTA clusters use the non-portable cluster
 *     size); planes that still do not fit return WTCONV_ERR_UNSUPPORTED.
 *   - Plans (grid sizes, the weight gradient's batch groups and so its
 *     workspace size) are made for the SM count of the device current at the
 *     call and for the descriptor's layout; make the wtconv_workspace_bytes
 *     call and the call that uses the workspace with the same device current.
 *     Both layouts of a shape need the same workspace size.
 *   - L = 0 is the base branch only; wt_w and wt_scale may then be NULL.
 *   - Calls are reentrant; apart from the fixed scratch array of
 *     wtconv_backward_weight_noalloc (see there), the library holds no
 *     global state.
 */
#ifndef WTCONV_H
#define WTCONV_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *wtconv_stream_t; /* same type as cudaStream_t */

typedef enum {
    WTCONV_OK = 0,
    WTCONV_ERR_NULLPTR = 1,     /* a required pointer is NULL */
    WTCONV_ERR_BAD_SHAPE = 2,   /* B, C, H or W <= 0, W % 4 != 0, or rows not whole 16-byte chunks where needed */
    WTCONV_ERR_BAD_K = 3,       /* k not in {1, 3, 5, 7} */
    WTCONV_ERR_BAD_L = 4,       /* L < 0 or L > 6 */
    WTCONV_ERR_MISALIGNED = 5,  /* an activation pointer is not 16-byte aligned */
    WTCONV_ERR_DTYPE = 6,       /* unknown activation dtype */
    WTCONV_ERR_WORKSPACE = 7,   /* workspace missing or smaller than wtconv_workspace_bytes() */
    WTCONV_ERR_UNSUPPORTED = 8, /* valid shape whose plane (or strip) does not fit on chip */
    WTCONV_ERR_CUDA = 9,        /* a CUDA runtime call or kernel launch failed */
    WTCONV_ERR_LAYOUT = 10      /* unknown activation layout */
} wtconv_status_t;

typedef enum { WTCONV_F32 = 0, WTCONV_BF16 = 1 } wtconv_dtype_t; /* activation storage */

/* Activation layout: NCHW, or NHWC (channels last: element (b, c, h, w) at
 * ((b*H + h)*W + w)*C + c).  With NHWC, where C is a multiple of 8 and a
 * plane is held whole (H*W a multiple of 16, no zero padding), clusters of
 * 8 CTAs move the 8 channels of a pixel as one 16- or 32-byte run; other
 * NHWC planes are gathered and scattered element by element (C elements
 * apart).  The on-chip pass, and so every result bit, is the NCHW one; the
 * parameters' layouts do not change. */
typedef enum { WTCONV_NCHW = 0, WTCONV_NHWC = 1 } wtconv_layout_t;

typedef struct {
    int B, C, H, W; /* batch, channels, height, width */
    int k;          /* odd depthwise kernel size, shared by the base and subband convs */
    int L;          /* number of wavelet decomposition levels */
    int dtype;      /* a wtconv_dtype_t value */
    int layout;     /* a wtconv_layout_t value (0 = NCHW) */
} wtconv_desc_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *wtconv_status_string(wtconv_status_t s);

/* Bytes of device workspace wtconv_backward_weight, wtconv_backward and
 * wtconv_backward_one_pass need for `d` on the current device (0 if `d` is
 * invalid); one size serves all three.  Planned for 148 SMs (a B200) when no
 * CUDA device can be queried.  The forward and input-gradient calls need
 * none: every intermediate stays on chip. */
size_t wtconv_workspace_bytes(const wtconv_desc_t *d);

/* Forward pass: y = WTConv(x), the fused layer of the Abstract with its three
 * reformulations (on-chip Haar analysis, closed-form synthesis, scales folded
 * into the weights).  x, y: [B][C][H][W] in desc->dtype; x and y must not
 * overlap.  Reads x once and writes y once. */
wtconv_status_t wtconv_forward(const wtconv_desc_t *d, const void *x,
                               const float *base_w, const float *base_b, const float *base_scale,
                               const float *wt_w, const float *wt_scale,
                               void *y, wtconv_stream_t stream);

/* Gradient with respect to the input: dx = J^T dy, the transpose of the
 * forward map (the same pass run on dy with every kernel rotated by 180
 * degrees and no bias), one of the backward passes of the training step
 * whose speedup the Abstract reports; the same three reformulations apply
 * to the transposed map.  dy, dx: [B][C][H][W] in desc->dtype; must not
 * overlap. */
wtconv_status_t wtconv_backward_input(const wtconv_desc_t *d, const void *dy,
                                      const float *base_w, const float *base_scale,
                                      const float *wt_w, const float *wt_scale,
                                      void *dx, wtconv_stream_t stream);

/* Gradients with respect to every parameter, summed over the batch and all
 * positions (overwritten); the other backward pass of the Abstract's
 * training step, with the subbands of x and dy recomputed on chip
 * (reformulation (1)) and the folded scales' gradients recovered from the
 * unscaled correlations (reformulation (3)):
 *   d_base_w[c][u][v]   = base_scale[c] * sum dy[h][w] x[h+u-p][w+v-p]
 *   d_base_b[c]         = base_scale[c] * sum dy
 *   d_base_scale[c]     = sum dy * (dwconv(x, base_w[c]) + base_b[c])
 *   d_wt_w[l][c][s]     = wt_scale[l][c][s] * sum D_{l,s}[i][j] S_{l,s}[i+u-p][j+v-p]
 *   d_wt_scale[l][c][s] = sum D_{l,s} * dwconv(S_{l,s}, wt_w[l][c][s])
 * with S / D the Haar subbands of x / dy.  The reduction order is fixed, so
 * repeated calls return bitwise-identical results.  `workspace` (device,
 * at least wtconv_workspace_bytes(d) bytes) holds per-block partial sums. */
wtconv_status_t wtconv_backward_weight(const wtconv_desc_t *d, const void *x, const void *dy,
                                       const float *base_w, const float *base_b, const float *base_scale,
                                       const float *wt_w, const float *wt_scale,
                                       float *d_base_w, float *d_base_b, float *d_base_scale,
                                       float *d_wt_w, float *d_wt_scale,
                                       void *workspace, size_t workspace_bytes,
                                       wtconv_stream_t stream);

/* Whole backward of the layer (the backward half of the Abstract's training
 * step): dx (as wtconv_backward_input) and every parameter gradient (as
 * wtconv_backward_weight, bitwise-repeatable).  The library picks the path
 * from the plans, not by timing: the one-pass kernel of
 * wtconv_backward_one_pass where its plan exists and the planner's cost
 * (conv-tile rows on the busiest SM sub-partition) is below that of the two
 * passes together, or equal to it while one of the two passes runs one CTA
 * per SM, or the activations are NHWC and either both passes would gather
 * them element by element or the one pass holds them on channel octets;
 * else wtconv_backward_input then wtconv_backward_weight.  Both paths give the same results.  dx:
 * [B][C][H][W] in desc->dtype, not overlapping x or dy.  Workspace as for
 * wtconv_backward_weight.  Every argument is checked before either pass is
 * enqueued. */
wtconv_status_t wtconv_backward(const wtconv_desc_t *d, const void *x, const void *dy,
                                const float *base_w, const float *base_b, const float *base_scale,
                                const float *wt_w, const float *wt_scale, void *dx,
                                float *d_base_w, float *d_base_b, float *d_base_scale,
                                float *d_wt_w, float *d_wt_scale,
                                void *workspace, size_t workspace_bytes, wtconv_stream_t stream);

/* The one-pass backward: the results of wtconv_backward from one kernel that
 * reads x and dy once and writes dx once (the fewest HBM bytes of any
 * backward, per the Abstract's I/O model), at the cost of an on-chip
 * footprint that holds one CTA per SM.  Only whole planes: a plane split
 * into cluster strips returns WTCONV_ERR_UNSUPPORTED.  Arguments as for
 * wtconv_backward. */
wtconv_status_t wtconv_backward_one_pass(const wtconv_desc_t *d, const void *x, const void *dy,
                                         const float *base_w, const float *base_b, const float *base_scale,
                                         const float *wt_w, const float *wt_scale, void *dx,
                                         float *d_base_w, float *d_base_b, float *d_base_scale,
                                         float *d_wt_w, float *d_wt_scale,
                                         void *workspace, size_t workspace_bytes, wtconv_stream_t stream);

/* The paper has no counterpart to this entry point.
 *
 * Same result as wtconv_backward_weight, for callers that cannot allocate
 * device memory -- for example code running inside a fixed memory budget, an
 * allocator hook, or a runtime that forbids cudaMalloc while a stream is being
 * captured.  Instead of a workspace argument it uses a fixed array inside this
 * library (4 MiB of device memory per GPU that loads the library, held until
 * the process exits) for the per-block partial sums; it calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *   - Size limit: its partial sums (at most wtconv_workspace_bytes(d) bytes)
 *     must fit in 2^20 floats; larger problems return WTCONV_ERR_WORKSPACE (use
 *     wtconv_backward_weight).
 *   - Every call looks up the array's address in the current context (a
 *     host-side lookup), so a context created after cudaDeviceReset, or a
 *     non-primary context, gets its own copy of the array.  Under lazy module
 *     loading the first call in a context may load the library's device code;
 *     make one call before any stream capture.
 *   - Every call shares the one array: calls whose kernels overlap on the GPU
 *     (different streams, no ordering between them) race and corrupt each
 *     other's results.  Calls ordered on one stream are safe.  Each call
 *     enqueues, on `stream`, one memset of its per-channel arrival counters
 *     (C unsigned ints) and then the kernel; the partial sums are never
 *     cleared, since each call overwrites every partial it later reads.
 * Arguments, layouts and gradients as for wtconv_backward_weight. */
wtconv_status_t wtconv_backward_weight_noalloc(const wtconv_desc_t *d, const void *x, const void *dy,
                                               const float *base_w, const float *base_b, const float *base_scale,
                                               const float *wt_w, const float *wt_scale,
                                               float *d_base_w, float *d_base_b, float *d_base_scale,
                                               float *d_wt_w, float *d_wt_scale, wtconv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WTCONV_H */
