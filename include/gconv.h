/*
 * gconv.h -- C ABI of libgconv.so: FP32 contiguous-NCHW 2D convolution forward
 * (grouped, depthwise, dense, asymmetric kernels) and the fused
 * conv -> +bias -> *scale -> sigmoid -> GroupNorm chain, on NVIDIA B200
 * (sm_100a).
 *
 * Sources for the operations (web pages on the subject):
 *  - "GroupConv Atlas" (xiangguozhang.com/projects/groupconv-atlas), section
 *    "Fix the experiment": FP32, contiguous NCHW grouped convolution with
 *    general geometry (the direct-mapping kernel "supports general convolution
 *    geometry").
 *  - POPCORNBENCH "Kimi-K2.6__l2_p21" transcript: the Model
 *    Conv2d(8->32, 3x3) -> x + bias[K,1,1] -> x * scale[K,1,1] -> sigmoid ->
 *    GroupNorm(8 groups, eps 1e-5, affine weight/bias), and the final design's
 *    folding of the conv bias and the extra bias into one per-channel vector.
 *  - POPCORNBENCH "Kimi-K2.6__l1_p62" transcript: the asymmetric Conv2d with a
 *    (5, 9) kernel, the output size (H + 2p - d(R-1) - 1)/s + 1 and the index
 *    map in_y = out_y*stride - pad + kh*dilation.
 *
 * Conventions shared by every entry point:
 *  - Tensors are FP32, contiguous, row-major: x[N][C][H][W], w[K][C/groups][R][S],
 *    y[N][K][P][Q].  Offsets are computed in 64-bit.  Pointers need only
 *    4-byte alignment; 16-byte alignment enables the vector paths.
 *  - x, w, bias, scale, gamma, beta and y are DEVICE pointers owned by the
 *    caller.  The library never frees or retains them.
 *  - The operation is a cross-correlation (no kernel flip): output channel k
 *    belongs to group k / (K/groups) and reads input channels
 *    [gi*C/groups, (gi+1)*C/groups); taps outside the image read zero.
 *  - Stride, padding and dilation are the same along H and W, except in
 *    gconv2d_fwd_ex, which takes them per axis; the kernel may be non-square
 *    (R != S).
 *  - Every call is asynchronous on `stream` (0 = legacy default stream).  It
 *    performs no host synchronisation and no device allocation, except the
 *    one-time workspace allocation described at gconv_reserve_workspace.
 *  - Errors: arguments are validated on the host first; on any error nothing
 *    is launched and y is untouched.  A launch failure reported by the CUDA
 *    runtime returns GCONV_ERR_CUDA.  Shapes that are valid but outside what
 *    the kernels implement return GCONV_ERR_UNSUPPORTED (never a fallback).
 *  - y must not overlap x, w or any parameter vector.
 */
#ifndef GCONV_H_
#define GCONV_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define GCONV_API __attribute__((visibility("default")))
#else
#define GCONV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gconv_status {
    GCONV_OK = 0,
    GCONV_ERR_INVALID_ARG = 1,   /* a size, pointer or parameter is invalid */
    GCONV_ERR_UNSUPPORTED = 2,   /* valid shape that no kernel implements */
    GCONV_ERR_CUDA = 3,          /* the CUDA runtime reported an error */
    GCONV_ERR_WORKSPACE = 4,     /* workspace too small and cannot grow now */
    GCONV_ERR_TIMEOUT = 5        /* a bounded device wait gave up (see gconv_get_last_device_error) */
} gconv_status_t;

/* Human-readable name of a status code (static string, never NULL). */
GCONV_API const char *gconv_status_string(gconv_status_t status);

/* Output extents P, Q of a convolution: P = floor((H + 2*pad - dilation*(R-1) - 1)/stride) + 1
 * and likewise Q from W and S ("Kimi-K2.6__l1_p62", output-size formula).
 * Returns GCONV_ERR_INVALID_ARG when an argument is out of range or the
 * kernel does not fit (P or Q < 1).  P and Q are host pointers. */
GCONV_API gconv_status_t gconv2d_output_size(int H, int W, int R, int S, int stride, int pad,
                                   int dilation, int *P, int *Q);

/* Grouped / depthwise / dense convolution forward:
 *   y[n,k,p,q] = bias[k] + sum_{c<C/g, r<R, s<S} w[k,c,r,s] * x[n, gi*C/g + c,
 *                                    p*stride - pad + r*dilation, q*stride - pad + s*dilation]
 * ("GroupConv Atlas", "Fix the experiment"; "Kimi-K2.6__l1_p62", index map).
 * bias: [K] device pointer or NULL for none.
 * Requires N >= 1, C, K, R, S, stride, dilation >= 1, pad >= 0,
 * groups >= 1 dividing C and K, P, Q >= 1, and every tensor smaller than
 * 2^31 elements per sample plane product (N*C*H*W, N*K*P*Q < 2^62).
 * Workspace: shapes that run on the tensor-core implicit GEMM keep their
 * split weights in the library-owned workspace of the current device (see
 * gconv_reserve_workspace); when the GEMM cannot stage x itself (rows not a
 * multiple of 16 bytes, more than 32 output channels per group, ...) the
 * workspace also holds two padded copies of x, about 2 * N*C*(H+pad)*(W+pad)
 * floats (about 540 MB for x[8,32,512,512]).  gconv2d_chain_workspace_size
 * and gconv2d_plan_name report what a shape needs.  Calls on different
 * streams that can overlap on the GPU share that workspace and must be
 * ordered by the caller; calls on one stream are always safe. */
GCONV_API gconv_status_t gconv2d_fwd(const float *x, const float *w, const float *bias,
                           int N, int C, int H, int W, int K, int R, int S,
                           int stride, int pad, int dilation, int groups,
                           float *y, cudaStream_t stream);

/* Convolution forward with stride, padding and dilation given per axis
 * ("Kimi-K2.6__l1_p62", ModelNew.forward: the layer's padding, stride and
 * dilation may each be an (h, w) tuple, which a single int cannot carry; the
 * transcript's fix is a signature taking padding_h, padding_w, dilation_h,
 * dilation_w, stride_h and stride_w):
 *   y[n,k,p,q] = bias[k] + sum_{c,r,s} w[k,c,r,s] * x[n, gi*C/g + c,
 *                       p*stride_h - pad_h + r*dil_h, q*stride_w - pad_w + s*dil_w]
 *   P = floor((H + 2*pad_h - dil_h*(R-1) - 1)/stride_h) + 1,
 *   Q = floor((W + 2*pad_w - dil_w*(S-1) - 1)/stride_w) + 1.
 * Equal values on both axes give exactly gconv2d_fwd (same kernels, same
 * bits).  Unequal ones run on the general-geometry direct kernel, or on the
 * implicit GEMM when both strides are 1 and the groups are wide enough.
 * Arguments, layout, alignment, streams, workspace and errors as
 * gconv2d_fwd (each stride and dilation >= 1, each padding >= 0). */
GCONV_API gconv_status_t gconv2d_fwd_ex(const float *x, const float *w, const float *bias,
                           int N, int C, int H, int W, int K, int R, int S,
                           int stride_h, int stride_w, int pad_h, int pad_w, int dil_h, int dil_w,
                           int groups, float *y, cudaStream_t stream);

/* Convolution with a per-output-channel affine epilogue and a clamp:
 *   y[n,k,p,q] = min(max(conv(x, w)[n,k,p,q] * scale[k] + shift[k], lo), hi)
 * This is the depthwise convolution of a MobileNetV2 inverted-residual block
 * ("GroupConv Atlas", "Fix the experiment": the block the page substitutes
 * one convolution in) fused with the BatchNorm in inference form that
 * follows it, folded into scale = gamma / sqrt(running_var + eps) and
 * shift = beta - running_mean * scale (+ conv bias * scale), and the ReLU6
 * (lo = 0, hi = 6).
 * scale, shift: [K] device pointers, or NULL for 1 and 0.  lo <= hi (either
 * may be infinite; -INFINITY, +INFINITY gives no clamp).  Shapes, layout,
 * alignment, streams and errors as gconv2d_fwd; lo > hi or a NaN bound is
 * GCONV_ERR_INVALID_ARG. */
GCONV_API gconv_status_t gconv2d_affine_clamp_fwd(const float *x, const float *w,
                           int N, int C, int H, int W, int K, int R, int S,
                           int stride, int pad, int dilation, int groups,
                           const float *scale, const float *shift, float lo, float hi,
                           float *y, cudaStream_t stream);

/* Fused chain ("Kimi-K2.6__l2_p21", Model forward):
 *   z = conv(x, w) + bias[k]          (bias [K] or NULL; the caller folds the
 *                                       conv bias and the extra [K,1,1] bias)
 *   a = 1 / (1 + exp(-(z * scale[k])))
 *   per (n, G) with G < gn_groups, over channels [G*K/gn_groups, (G+1)*K/gn_groups)
 *   and all P*Q positions: mu = mean(a), var = mean((a - mu)^2)
 *   y = (a - mu) / sqrt(var + eps) * gamma[k] + beta[k]
 * scale, gamma, beta: [K] device pointers (required).  gn_groups must divide K;
 * eps >= 0.  y receives the result (it also holds a between the two passes).
 * GroupNorm statistics are merged deterministically (fixed order), so equal
 * inputs give bit-identical outputs.
 * Scratch: per-tile partial statistics live in a library-owned workspace on
 * the current device (see gconv_reserve_workspace).  Calls on different
 * streams that overlap on the GPU share that workspace and must not run
 * concurrently. */
GCONV_API gconv_status_t gconv2d_bias_scale_sigmoid_groupnorm_fwd(
    const float *x, const float *w, const float *bias,
    int N, int C, int H, int W, int K, int R, int S,
    int stride, int pad, int dilation, int groups,
    const float *scale, int gn_groups, const float *gamma, const float *beta,
    float eps, float *y, cudaStream_t stream);

/* Allocation-free variant of gconv2d_bias_scale_sigmoid_groupnorm_fwd (the
 * pages have no counterpart: this is an addition for callers of this
 * library).  Same arguments, same result, same kernels; the only difference
 * is where the GroupNorm partial statistics live.  The regular entry point
 * keeps them in a workspace it grows with cudaMalloc; this one uses a
 * fixed-size scratch array in device memory that every GPU loading the
 * library reserves until process exit (gconv_noalloc_scratch_capacity()
 * bytes, 4 MiB), so it never calls cudaMalloc, cudaFree or any other
 * allocator.  It is meant for callers that cannot allocate device memory at
 * call time: code recording a CUDA graph (allocation is not allowed while a
 * stream is being captured), engines that must not stall on an implicit
 * device synchronisation or must keep a fixed memory budget after start-up,
 * and hosts whose allocator is owned by another framework.
 * - It always runs the direct (CUDA-core) convolution kernels, whose only
 *   scratch is the partial statistics; shapes whose partials need more than
 *   the capacity return GCONV_ERR_WORKSPACE and launch nothing; use the
 *   regular entry point for them.
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - Every call on a device shares the one array and leaves its contents
 *   behind; each call writes every entry it later reads, so nothing needs to
 *   start at zero.  Calls whose kernels overlap on the GPU (for example on two
 *   streams without ordering between them) race on the array and must be
 *   serialised by the caller. */
GCONV_API gconv_status_t gconv2d_bias_scale_sigmoid_groupnorm_fwd_noalloc(
    const float *x, const float *w, const float *bias,
    int N, int C, int H, int W, int K, int R, int S,
    int stride, int pad, int dilation, int groups,
    const float *scale, int gn_groups, const float *gamma, const float *beta,
    float eps, float *y, cudaStream_t stream);

/* Bytes of the fixed scratch array the allocation-free chain may use. */
GCONV_API size_t gconv_noalloc_scratch_capacity(void);

/* Bytes of workspace the fused chain needs for this shape (0 on invalid input
 * or when the chain's conv stage runs on the direct kernels, whose only scratch
 * is the partial statistics: then the size of those). */
GCONV_API size_t gconv2d_chain_workspace_size(int N, int C, int H, int W, int K, int R, int S,
                                    int stride, int pad, int dilation, int groups,
                                    int gn_groups);

/* Make sure the current device's workspace holds at least `bytes`.  The chain
 * grows the workspace on demand (cudaMalloc) the first time a shape needs more;
 * growing is impossible while `stream` capture is active, in which case the
 * chain returns GCONV_ERR_WORKSPACE.  Call this (or one un-captured chain call)
 * before capturing a CUDA graph.  The workspace lives until process exit. */
GCONV_API gconv_status_t gconv_reserve_workspace(size_t bytes);

/* Name of the kernel variant the dispatcher selects for a convolution shape
 * (for records and A/B measurements); "unsupported" / "invalid" otherwise.
 * `chain` != 0 asks about the fused chain's conv stage. */
GCONV_API const char *gconv2d_plan_name(int N, int C, int H, int W, int K, int R, int S,
                              int stride, int pad, int dilation, int groups, int chain);

/* gconv2d_plan_name for the per-axis geometry of gconv2d_fwd_ex. */
GCONV_API const char *gconv2d_plan_name_ex(int N, int C, int H, int W, int K, int R, int S,
                              int stride_h, int stride_w, int pad_h, int pad_w, int dil_h, int dil_w,
                              int groups);

/* Force a kernel family for subsequent calls on this process, by name:
 * "direct_stream", "direct_blocked", "direct" (streaming when possible, else
 * blocked), "direct_cpasync" (blocked, cp.async staging), "generic",
 * "igemm"; a ":kt1" / ":kt2" / ":kt4" / ":kt8" suffix also fixes the direct
 * kernels' output channels per thread.  "auto" restores per-shape dispatch
 * (the measured table compiled into the library, then the planner's rules).
 * A forced family that cannot run a shape makes that call return
 * GCONV_ERR_UNSUPPORTED.  Returns GCONV_ERR_INVALID_ARG for an unknown name.
 * Intended for measurement (A/B runs, regenerating the table). */
GCONV_API gconv_status_t gconv_force_kernel(const char *name);

/* Status of the bounded waits inside the kernels since the last query:
 * GCONV_ERR_TIMEOUT when a kernel gave up waiting for its own asynchronous
 * copies, GCONV_OK otherwise.  After a timeout every output of the calls
 * made since the last query is invalid, not only the tile that gave up: an
 * aborted CTA skips its remaining tiles, and in the fused chain a missing or
 * partial GroupNorm partial spoils the statistics of its whole (image,
 * group).  Reading clears the flag.  Synchronises with the current device. */
GCONV_API gconv_status_t gconv_device_error_status(void);

/* The same status after the work queued on `stream` so far has finished:
 * synchronises `stream` (NULL: the legacy default stream) first, then reads
 * and clears the flags as gconv_device_error_status.  GCONV_ERR_CUDA when
 * the synchronisation itself reports an error (for example a launch that
 * failed). */
GCONV_API gconv_status_t gconv_get_last_device_error(cudaStream_t stream);

/* Self-test of the device-side failure path.  Every wait inside the kernels
 * (on TMA and cp.async completion, on pipeline stages, on tensor-core
 * commits) is bounded: a wait that runs out raises a device error flag,
 * stops the kernel's pipeline and returns, instead of hanging the GPU.  This
 * call launches one CTA (one warp) on `stream` that waits on an mbarrier no
 * thread ever arrives on, with that same bounded wait limited to `spins`
 * polls (1 .. 2^24); the wait runs out, the flag is raised and the kernel
 * returns.  The next gconv_get_last_device_error(stream) then reports
 * GCONV_ERR_TIMEOUT (and clears the flag) while the CUDA context stays
 * usable.  The pages have no counterpart: this exists so the failure path
 * can be tested without faulting a GPU.  Returns GCONV_ERR_INVALID_ARG for
 * `spins` out of range, GCONV_ERR_CUDA when the launch fails. */
GCONV_API gconv_status_t gconv_selftest_wait_timeout(unsigned int spins, cudaStream_t stream);

/* Library version string. */
GCONV_API const char *gconv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GCONV_H_ */
