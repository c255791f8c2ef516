/*
 * dwconv2d.h - depthwise 2-D convolution on NVIDIA B200 (sm_100a): C ABI.
 *
 * The operation (page "LeanMlir Proofs/Architectures/Depthwise",
 * lean.brettkoonce.com, section "Depthwise conv2d forward"), generalised to a
 * batch axis, stride s, dilation d and per-side padding:
 *
 *   y[n,ho,wo,c] = sum_{kh<kH, kw<kW} X(n, ho*sh + kh*dh - pt,
 *                                         wo*sw + kw*dw - pl, c) * W[c,kh,kw]
 *                  + b[c]
 *
 * where X is x inside [0,H) x [0,W) and 0 outside (zero padding).  It is a
 * cross-correlation (the kernel is not flipped) and has no cross-channel
 * mixing: channel c of y reads only channel c of x and filter c.  The input
 * gradient (sections "Closed-form input gradient ... direct formula" and
 * "Depthwise conv input-VJP") is the transpose of the linear part:
 *
 *   dx[n,hi,wi,c] = sum over (kh,kw) with hi + pt - kh*dh = ho*sh,
 *                   wi + pl - kw*dw = wo*sw, 0 <= ho < Ho, 0 <= wo < Wo
 *                   of W[c,kh,kw] * dy[n,ho,wo,c]
 *
 * which at stride 1 is the reversed-kernel correlation of dy with the
 * complementary pads d(k-1) - p_lo, and at stride 2 is the zero-upsample of
 * dy onto the forward's sampled positions followed by that correlation
 * (sections "Stride-2 SAME depthwise input-VJP" and "Stride-2 XLA-SAME
 * depthwise input-VJP"); both are computed without materialising anything.
 * The weight and bias gradients are the sums of the sections "Depthwise
 * weight-VJP" and "Depthwise bias gradient - closed-form formula".  With a
 * channel multiplier M (desc->multiplier) output channel o = c*M + j reads
 * input channel c through filter o; M = 1 is the formula above.
 *
 * Conventions for every entry point:
 *   - Activations (x, y, dy, dx) are dense, of the element type desc->atype
 *     (float32 by default, or float16 / bfloat16), in the layout of
 *     desc->layout: DW_NHWC = [N][H][W][C] (C innermost), DW_NCHW =
 *     [N][C][H][W] (W innermost).  y and dy have C*M channels.
 *   - Weights are [C*M][kH][kW] row-major (the PyTorch [C*M,1,kH,kW] grouped
 *     weight, contiguous), float32 or float16 per desc->wtype.  float16 weights
 *     are widened exactly to float32; accumulation is always float32, taps in
 *     kh-major / kw-minor order, then the bias is added.  With weights that are
 *     exactly representable in float16, the float16 and float32 weight paths
 *     return bit-identical results.
 *   - Bias is float32 [C*M] or NULL (NULL means zero).
 *   - All data pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates, frees or retains them (the weight gradient takes a
 *     caller workspace; its no-allocation variant uses a fixed array inside
 *     the library).  Unaligned pointers are accepted (a slower kernel is
 *     chosen).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous: they enqueue kernels and return without synchronising.
 *     They make no device allocation and may be captured in a CUDA graph once
 *     the same descriptor shape has been run once outside capture on that
 *     device.
 *   - Errors: invalid descriptors (sizes <= 0, stride or dilation < 1,
 *     negative pads, an empty output, unknown enum values, NULL required
 *     pointers) return DW_ERR_INVALID_ARG and launch nothing; an output buffer
 *     that overlaps an input returns DW_ERR_ALIAS and launches nothing;
 *     DW_ALGO_TILED on a shape the tiled kernels do not cover returns
 *     DW_ERR_UNSUPPORTED; a failed launch returns DW_ERR_CUDA.
 */
#ifndef DWCONV2D_H_
#define DWCONV2D_H_

#include <stdint.h>

/* Exported entry points keep default visibility when the library is built
 * with -fvisibility=hidden. */
#if defined(__GNUC__)
#define DW_API __attribute__((visibility("default")))
#else
#define DW_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t dw_status_t;
enum {
    DW_OK = 0,
    DW_ERR_INVALID_ARG = 1,
    DW_ERR_UNSUPPORTED = 2,
    DW_ERR_ALIAS = 3,
    DW_ERR_CUDA = 4,
    DW_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up waiting on a copy */
    DW_ERR_TOO_LARGE = 6       /* needs more scratch than the fixed device array holds */
};

enum { DW_NHWC = 0, DW_NCHW = 1 };                 /* dw_desc_t.layout   */
enum { DW_F32 = 0, DW_F16 = 1, DW_BF16 = 2 };      /* .wtype (F32/F16), .atype */
enum { DW_PAD_EXPLICIT = 0, DW_PAD_SAME = 1 };     /* dw_desc_t.pad_mode */
enum { DW_ALGO_AUTO = 0, DW_ALGO_DIRECT = 1, DW_ALGO_TILED = 2 }; /* .algo */
/* activation of dwconv2d_fwd_bn_act: identity, max(u,0), min(max(u,0),6),
 * u / (1 + exp(-u)) */
enum { DW_ACT_NONE = 0, DW_ACT_RELU = 1, DW_ACT_RELU6 = 2, DW_ACT_SILU = 3 };

/*
 * Problem descriptor.  N,H,W,C are the INPUT (x / dx) extents.  pad_mode
 * DW_PAD_SAME ignores the pad_* fields and uses the XLA rule per axis:
 * Ho = ceil(H/sh), total = max((Ho-1)*sh + dh*(kH-1) + 1 - H, 0),
 * pt = floor(total/2), pb = total - pt (the odd pad at the bottom/right, the
 * page's "XLA-SAME" odd-position decimation at stride 2).  DW_PAD_EXPLICIT
 * uses pad_top/bottom/left/right as given (>= 0); Ho = floor((H + pt + pb -
 * dh*(kH-1) - 1)/sh) + 1, same for Wo.
 * algo: DW_ALGO_AUTO picks the fastest kernel that covers the shape;
 * DW_ALGO_DIRECT forces the one-thread-per-output kernel (any shape);
 * DW_ALGO_TILED forces the TMA-tiled kernels (DW_ERR_UNSUPPORTED if they do
 * not cover the shape).
 * multiplier: M output channels per input channel (0 and 1 both mean the
 * plain depthwise convolution, M = 1; at most 4096).  With M > 1 the
 * forward maps C input channels to C*M output channels: output channel
 * o = c*M + j reads only input channel c = o / M, through filter w[o] and
 * bias b[o] (a grouped convolution with groups = C, as in the page
 * "Incorrect stableHLO for grouped convolution gradient", a conv from 4 to
 * 8 channels with groups = 4).  Then w is [C*M,kH,kW], b [C*M], y and dy
 * have C*M channels, x and dx have C; every entry point applies it.
 * atype: element type of the activations x, y, dy and dx: DW_F32 (0, the
 * default), DW_F16 or DW_BF16.  16-bit activations are widened to float32
 * exactly, every sum is formed in float32 exactly as for DW_F32, and each
 * result is rounded once (to nearest even) to atype; the weight gradient's
 * dW and db, bias and batch-norm statistics stay float32.  Extends the
 * pages' f16 weights to the activations.
 */
typedef struct dw_desc {
    int64_t N, H, W, C;
    int32_t kH, kW;
    int32_t stride_h, stride_w;
    int32_t dil_h, dil_w;
    int32_t pad_mode;
    int32_t pad_top, pad_bottom, pad_left, pad_right;
    int32_t layout;
    int32_t wtype;
    int32_t algo;
    int32_t multiplier;
    int32_t atype;
} dw_desc_t;

/* Output extents Ho, Wo of the forward for `desc` (host only, no CUDA call).
 * Returns DW_ERR_INVALID_ARG for an invalid descriptor. */
DW_API dw_status_t dwconv2d_out_shape(const dw_desc_t* desc, int64_t* Ho, int64_t* Wo);

/* Resolved pads {top, bottom, left, right} for `desc` (host only). */
DW_API dw_status_t dwconv2d_resolved_pads(const dw_desc_t* desc, int32_t pads[4]);

/*
 * Forward: y = depthwise(x; w) + b (Co = C*M output channels; Co = C at M = 1).
 *   x: [N,H,W,C] or [N,C,H,W] of desc->atype (float32 by default), read only.
 *   w: [Co,kH,kW] float32 or float16 (desc->wtype), read only.
 *   b: [Co] float32 or NULL, read only.
 *   y: [N,Ho,Wo,Co] or [N,Co,Ho,Wo] of desc->atype, every element written.
 * y must not overlap x, w or b (DW_ERR_ALIAS).
 * Page: LeanMlir Depthwise, "Depthwise conv2d forward"; strided forms
 * "Stride-2 SAME" / "Stride-2 XLA-SAME depthwise conv" (computed directly at
 * the sampled positions, never as a decimated stride-1 pass).
 */
DW_API dw_status_t dwconv2d_fwd(const dw_desc_t* desc, const void* x, const void* w,
                                const float* b, void* y, void* stream);

/*
 * Forward with a fused epilogue: y = act(BN(depthwise(x; w) + b)), where BN
 * is inference-mode batch normalisation with per-channel running statistics,
 *   BN(z)[c] = gamma[c] * (z - mean[c]) / sqrt(var[c] + eps) + beta[c],
 * and act one of DW_ACT_*.  The normalisation and the activation are applied
 * to each output in registers before its single store, so y is written once
 * and never re-read.
 *   x, w, b, y: as for dwconv2d_fwd.
 *   gamma, beta, mean, var: [Co] float32 each, read only; either all four are
 *       given or all four are NULL (then BN is the identity and only the
 *       activation is applied).
 *   eps: finite, >= 0.
 *   act: DW_ACT_NONE .. DW_ACT_SILU.
 * Each channel's scale gamma/sqrt(var+eps) and shift beta - mean*scale are
 * formed in float32 (IEEE division and square root) and applied as one fused
 * multiply-add (the tiled kernels fold them into the filter and bias they
 * hold: scale*w and scale*b + shift); silu is u / (1 + expf(-u)) with a fast
 * division (a few ulp).  y must not overlap any input (DW_ERR_ALIAS);
 * a mixed set of NULL statistics, a negative or non-finite eps or an unknown
 * act is DW_ERR_INVALID_ARG.
 * Page: LeanMlir Depthwise, the section on the MLIR lowering, which names a
 * depthwise conv + batch-norm emitter; the pages do not spell the
 * normalisation out, and the inference-mode form above is the reading taken.
 */
DW_API dw_status_t dwconv2d_fwd_bn_act(const dw_desc_t* desc, const void* x, const void* w,
                                       const float* b, const float* gamma, const float* beta,
                                       const float* mean, const float* var, float eps,
                                       int32_t act, void* y, void* stream);

/*
 * Input gradient: dx = J^T dy for the forward of `desc` (bias plays no part;
 * with a multiplier, dx channel c sums its M output channels c*M ..).
 *   dy: [N,Ho,Wo,Co] or [N,Co,Ho,Wo] of desc->atype, read only.
 *   w:  [Co,kH,kW] float32 or float16, read only.
 *   dx: [N,H,W,C] or [N,C,H,W] of desc->atype, every element written (positions no
 *       output reads get 0; nothing is accumulated into previous contents).
 * dx must not overlap dy or w (DW_ERR_ALIAS).
 * Page: LeanMlir Depthwise, "Closed-form input gradient ... direct formula",
 * its reversed-kernel form, and the stride-2 / XLA-SAME input-VJP sections
 * (the forward's actual low pad is used, never a symmetric one).
 */
DW_API dw_status_t dwconv2d_bwd_input(const dw_desc_t* desc, const void* dy, const void* w,
                                      void* dx, void* stream);

/*
 * Weight and bias gradients of the forward of `desc` (o < Co = C*M):
 *   dW[o,kh,kw] = sum_{n,ho,wo} dy[n,ho,wo,o] * X(n, ho*sh + kh*dh - pt,
 *                                                 wo*sw + kw*dw - pl, o/M)
 *   db[o]       = sum_{n,ho,wo} dy[n,ho,wo,o]
 *   x:  [N,H,W,C] or [N,C,H,W] of desc->atype, read only.
 *   dy: [N,Ho,Wo,Co] or [N,Co,Ho,Wo] of desc->atype, read only.
 *   dw: [Co,kH,kW] float32, every element written (also when desc->wtype is
 *       DW_F16 or the activations are 16-bit: gradients are produced in
 *       float32).
 *   db: [Co] float32 or NULL (then the bias gradient is not produced).
 *   workspace: device memory of at least dwconv2d_bwd_weight_workspace_size()
 *       bytes, caller-owned; its contents on entry do not matter and are
 *       overwritten.
 * The sums are reduced in a fixed order (float32 products over a few
 * outputs folded into float64, then float64 partials summed in order), so
 * repeated calls give bit-identical results on the same device.
 * dw, db and workspace must not overlap x, dy or each other (DW_ERR_ALIAS);
 * a workspace smaller than required returns DW_ERR_INVALID_ARG.
 * Page: LeanMlir Depthwise, "Depthwise weight-VJP", "Depthwise bias gradient
 * - closed-form formula" and the stride-2 / XLA-SAME weight and bias VJP
 * sections.
 */
DW_API dw_status_t dwconv2d_bwd_weight(const dw_desc_t* desc, const void* x, const void* dy,
                                       float* dw, float* db, void* workspace,
                                       uint64_t workspace_bytes, void* stream);

/* Workspace bytes dwconv2d_bwd_weight needs for `desc` (host only; depends
 * on the problem, not on the device or the pointers). */
DW_API dw_status_t dwconv2d_bwd_weight_workspace_size(const dw_desc_t* desc, uint64_t* bytes);

/*
 * Weight and bias gradients for callers that cannot allocate device memory.
 * The source pages have no counterpart to this entry point: it is the same
 * computation as dwconv2d_bwd_weight, but its scratch is a fixed array inside
 * the library instead of a caller workspace.  It is meant for code that
 * cannot allocate at the call site: programs whose device memory is an arena
 * reserved up front and that may not allocate more, and latency-critical
 * paths where cudaMalloc / cudaFree are not acceptable because they can
 * synchronise the device.
 *   - Arguments and results as dwconv2d_bwd_weight (x, dy, dw, db are the
 *     caller's device buffers; db may be NULL).
 *   - The scratch is one array of DW_NOALLOC_SCRATCH_BYTES bytes per device;
 *     every GPU that loads the library holds it until the process exits.
 *     A problem whose dwconv2d_bwd_weight_workspace_size() exceeds it returns
 *     DW_ERR_TOO_LARGE and launches nothing.
 *   - The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *     library routine.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - Every call shares the one array, which keeps the last call's contents;
 *     the kernels write every scratch element before reading it, so nothing
 *     has to be cleared between calls.  Calls that overlap on the GPU (for
 *     example on two streams) race on the array: the caller must order them.
 */
#define DW_NOALLOC_SCRATCH_BYTES (16u << 20)
DW_API dw_status_t dwconv2d_bwd_weight_noalloc(const dw_desc_t* desc, const void* x,
                                               const void* dy, float* dw, float* db,
                                               void* stream);

/*
 * Which kernel family a call with these arguments would run (host only, no
 * launch): returns DW_ALGO_DIRECT or DW_ALGO_TILED, or -DW_ERR_* when the call
 * would fail.  op: 0 = forward (in = x, out = y), 1 = input gradient
 * (in = dy, out = dx), 2 = weight gradient (in = x, w = dy, out = dw).
 * Pointers are only inspected for alignment.
 */
DW_API int32_t dwconv2d_query_algo(const dw_desc_t* desc, int32_t op, const void* in,
                            const void* w, const void* out);

/*
 * Reads and clears the library's device error word on the current device
 * (synchronous: waits for all prior work on the device).  *code receives 0 if
 * no kernel has reported a problem since the last call, else DW_ERR_*.
 * Kernels that wait on asynchronous copies bound every wait; a wait that runs
 * out sets this word and the kernel returns early (its output is then
 * undefined).
 */
DW_API dw_status_t dwconv2d_take_device_error(int32_t* code);

/*
 * Self-test of the failure path (the pages have no counterpart: it exists so
 * that tests can check, on a GPU, what a kernel does when one of its waits
 * on an asynchronous copy never completes).  Launches one small CTA that
 * waits, with the same bounded wait every kernel uses, on a shared-memory
 * barrier that nothing completes:
 *   mode 0: one thread waits until `limit_us` microseconds have passed;
 *   mode 1: one warp waits (limit 2 s) while another raises the CTA's abort
 *           flag, as a failing warp does, and the waiting warp gives up.
 * Either way the kernel records DW_ERR_DEVICE_TIMEOUT in the device error
 * word (read it with dwconv2d_take_device_error) and returns; nothing faults,
 * and the context stays usable.  limit_us: 1 .. 10^6; mode: 0 or 1, else
 * DW_ERR_INVALID_ARG.  Asynchronous on `stream` like every call.
 */
DW_API dw_status_t dwconv2d_selftest_wait_timeout(int32_t mode, uint32_t limit_us,
                                                  void* stream);

/* Human-readable name of a status code (static string). */
DW_API const char* dwconv2d_status_string(dw_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
DW_API int32_t dwconv2d_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DWCONV2D_H_ */
