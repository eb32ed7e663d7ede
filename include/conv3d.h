/*
 * conv3d.h -- C ABI of libconv3d: implicit-GEMM 3D convolution on B200 (sm_100a).
 *
 * The operation (engineering.drawthings.ai, "Metal conv3d" post: 3D
 * convolution implemented as an implicit GEMM, the way 2D convolution is;
 * Qwen Image post, "Video VAE" section: causal 3D convolution in video-VAE
 * decoders, whose frames before the first are padding, and whose first-frame
 * case reduces to a 2D convolution with adjusted weights):
 *
 *   y[n,to,ho,wo,co] = round( bias[co] + residual[n,to,ho,wo,co]
 *       + sum_{it,ih,iw,ci} w[co,it,ih,iw,ci]
 *                           * Xpad[n, to*st+it-pf, ho*sh+ih-ph, wo*sw+iw-pw, ci] )
 *
 * computed as the GEMM  M = N*Do*Ho*Wo,  N_gemm = Cout,  K = Cin*kt*kh*kw,
 * with fp16/bf16 operands, fp32 accumulation and one round-to-nearest-even to
 * the output type.  Xpad is x extended by zeros spatially and, temporally,
 * by the rule of conv3d_tpad_t.
 *
 * Layouts (row-major, innermost last):
 *   x        [N, D, H, W, Cin]            (NDHWC)
 *   w        [Cout, kt, kh, kw, Cin]      (K-major: row co is the K vector)
 *   bias     [Cout]                        (optional)
 *   residual [N, Do, Ho, Wo, Cout]         (optional, same type as y)
 *   y        [N, Do, Ho, Wo, Cout]
 *   Do = (D + pf + pb - kt)/st + 1, Ho = (H + 2*ph - kh)/sh + 1, Wo = (W + 2*pw - kw)/sw + 1
 *   (pf/pb are the front/back temporal pads of the mode); output pixel (to, ho, wo)
 *   reads input frame to*st + it - pf, row ho*sh + ih - ph, column wo*sw + iw - pw.
 *
 * All tensor pointers are DEVICE pointers to caller-owned memory on the
 * current CUDA device; the library never frees them and keeps none after a
 * call returns.  Every call enqueues on `stream` and returns without
 * synchronising.
 */
#ifndef LIBCONV3D_CONV3D_H
#define LIBCONV3D_CONV3D_H

#include <stddef.h>

#if defined(__GNUC__)
#define CONV3D_API __attribute__((visibility("default")))
#else
#define CONV3D_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *`; NULL = legacy default stream */

typedef enum { CONV3D_F16 = 0, CONV3D_BF16 = 1 } conv3d_dtype_t;

/* Temporal padding rule (the spatial rule is always zero padding ph, pw). */
typedef enum {
  CONV3D_TPAD_ZERO = 0,             /* pad[0] zero frames in front and behind          */
  CONV3D_TPAD_CAUSAL_REPLICATE = 1, /* kt-1 copies of frame 0 in front, none behind    */
  CONV3D_TPAD_CAUSAL_ZERO = 2,      /* kt-1 zero frames in front, none behind (Wan)    */
  CONV3D_TPAD_CAUSAL_CACHED = 3     /* kt-1 cached frames of the previous chunk in front
                                       (conv3d_fwd_cached only), none behind          */
} conv3d_tpad_t;

typedef enum {
  CONV3D_OK = 0,
  CONV3D_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad enum, overlap  */
  CONV3D_ERR_UNSUPPORTED = 2,  /* valid convolution outside the supported set         */
  CONV3D_ERR_ALIGNMENT = 3,    /* a tensor pointer is not 16-byte aligned             */
  CONV3D_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (conv3d_last_error) */
  CONV3D_ERR_TIMEOUT = 5,      /* a device-side wait ran out of time                  */
  CONV3D_ERR_DEVICE_CHECK = 6, /* a device-side consistency check failed              */
  CONV3D_ERR_WORKSPACE = 7     /* workspace missing or smaller than required          */
} conv3d_status_t;

/*
 * conv3d_fwd -- y = conv3d(x, w) + bias + residual (see the top of this file).
 *
 * kernel = {kt, kh, kw}, each in [1, 8].  stride = {st, sh, sw}, each in
 * [1, 8] (larger returns CONV3D_ERR_UNSUPPORTED).  pad = {pt, ph, pw}: pt is used by
 * CONV3D_TPAD_ZERO only and must be 0 for the causal modes; pt, ph, pw in
 * [0, 127], and the output extents Do, Ho, Wo must be >= 1.
 * Supported set: Cin % 8 == 0, Cout % 8 == 0, 16-byte aligned pointers, y not
 * overlapping x, w or bias; residual may be exactly y (in-place add) but not
 * partially overlap it.  bias and residual may be NULL.
 *
 * First-frame path: with CONV3D_TPAD_CAUSAL_REPLICATE and D == 1 every
 * temporal tap reads frame 0, so the kt taps are summed (fp32) into one 2D
 * weight, kept as a high and a low 16-bit part, and a 2D convolution over
 * the two parts runs instead of kt taps (2/kt of the tensor-core work); the
 * bias is unchanged.  That fold needs conv3d_workspace_bytes() of device
 * scratch: conv3d_fwd takes it from a per-device buffer that the library
 * allocates on the first such call and keeps until conv3d_release() (calls
 * that need it and overlap on different streams race on it -- use
 * conv3d_fwd_ws for those).
 *
 * Errors: argument, alignment and support errors return before anything is
 * enqueued, with y untouched.  A failed launch returns CONV3D_ERR_CUDA.
 * Device-side timeouts are reported by conv3d_poll_status().
 */
CONV3D_API conv3d_status_t conv3d_fwd(const void* x, const void* w, const void* bias,
                                      const void* residual, void* y, int N, int Cin, int D, int H,
                                      int W, int Cout, const int kernel[3], const int stride[3],
                                      const int pad[3], conv3d_tpad_t tpad, conv3d_dtype_t dtype,
                                      struct CUstream_st* stream);

/* conv3d_fwd with caller-provided device scratch (never allocates).
 * `workspace` must be 256-byte aligned and hold conv3d_workspace_bytes();
 * it may be NULL when that is 0.  Too small -> CONV3D_ERR_WORKSPACE.  When it
 * is used, it must not overlap x, w, bias, residual or y
 * (CONV3D_ERR_INVALID_ARG). */
CONV3D_API conv3d_status_t conv3d_fwd_ws(const void* x, const void* w, const void* bias,
                                         const void* residual, void* y, int N, int Cin, int D,
                                         int H, int W, int Cout, const int kernel[3],
                                         const int stride[3], const int pad[3], conv3d_tpad_t tpad,
                                         conv3d_dtype_t dtype, void* workspace, size_t ws_bytes,
                                         struct CUstream_st* stream);

/*
 * conv3d_fwd_noalloc -- conv3d_fwd for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it is an interface
 * addition of this library.
 *
 * Some callers must not call cudaMalloc: a host framework or plug-in host
 * that owns all device memory through its own allocator and forbids any
 * other allocation, a latency-critical path where an allocation may block or
 * fail in the middle of a frame, or a deployment whose device-memory budget
 * is fixed at start-up.  This call allocates nothing.  The caller passes x, w,
 * bias, residual and y exactly as for conv3d_fwd; the only scratch the path
 * needs -- the folded first-frame weight -- lives in a fixed 16 MiB array
 * inside the library's device memory, which every GPU that loads the library
 * holds until the process exits.
 *
 * Limit: a first-frame problem (CONV3D_TPAD_CAUSAL_REPLICATE, D == 1, kt > 1)
 * must have Cout*kh*kw*Cin <= 4,194,304 (conv3d_workspace_bytes() <= 16 MiB);
 * a larger one returns CONV3D_ERR_WORKSPACE before anything is enqueued.
 * Problems that need no scratch run exactly as with conv3d_fwd.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the one array and it keeps the
 * last call's contents; every element a call's kernels read is first written
 * by the same call, so nothing has to start at zero.  Calls whose work
 * overlaps on the GPU (several streams, or several host threads) race on the
 * array: serialise them.
 */
CONV3D_API conv3d_status_t conv3d_fwd_noalloc(const void* x, const void* w, const void* bias,
                                              const void* residual, void* y, int N, int Cin,
                                              int D, int H, int W, int Cout, const int kernel[3],
                                              const int stride[3], const int pad[3],
                                              conv3d_tpad_t tpad, conv3d_dtype_t dtype,
                                              struct CUstream_st* stream);

/*
 * conv3d_fwd_cached -- one chunk of a causal convolution over a long clip.
 *
 * A video-VAE decoder that decodes a long clip chunk by chunk must give each
 * chunk the frames that precede it as its temporal front padding (Qwen Image
 * post, "Video VAE": Wan's causal convolutions pad the frames before the first
 * with zeros; after the first chunk those frames are real).  This entry point
 * computes conv3d_fwd with temporal rule CONV3D_TPAD_CAUSAL_CACHED: output
 * frame to reads input frame to + it - (kt-1), and a negative index f reads
 * prev[n, kt-1+f].  Convolving a clip in chunks -- the first with the causal
 * replicate or zero rule, each later one with prev = the last kt-1 input
 * frames of the chunk before it -- gives exactly the whole-clip result.
 *
 * prev: device pointer to [N, kt-1, H, W, Cin] of the same dtype (may be NULL
 * when kt == 1), 16-byte aligned, not overlapping y.  pad[0] must be 0;
 * Do = D.  Every other argument, the layouts and the error behaviour are
 * those of conv3d_fwd.  Needs no workspace.
 */
CONV3D_API conv3d_status_t conv3d_fwd_cached(const void* x, const void* prev, const void* w,
                                             const void* bias, const void* residual, void* y,
                                             int N, int Cin, int D, int H, int W, int Cout,
                                             const int kernel[3], const int stride[3],
                                             const int pad[3], conv3d_dtype_t dtype,
                                             struct CUstream_st* stream);

/*
 * GroupNorm (+ SiLU): the normalisation and activation in front of each
 * decoder convolution (stable-diffusion.cpp discussion "Exe Heavy Metal":
 * GROUP_NORM on the GPU; news.bugfactory.tech: a fused GroupNorm + SiLU
 * kernel).  x and y are [N, D, H, W, C] (NDHWC), C % 8 == 0, C % groups == 0,
 * C <= 2048.  A statistic set is one sample (per_frame = 0: all D*H*W pixels)
 * or one frame of one sample (per_frame = 1: H*W pixels, for causal decoders
 * whose statistics may not look ahead in time).  stats is a caller-owned
 * device buffer of sets * groups * 2 doubles (sets = N, or N*D), 8-byte
 * aligned; tensors are 16-byte aligned.
 *
 * conv3d_groupnorm_stats: stats[s][g] = {mean, 1/sqrt(var + eps)} of set s,
 *   group g (biased variance), from one read of x.  Overwrites stats.
 * conv3d_groupnorm_silu: y = silu((x - mean) * rstd * gamma[c] + beta[c])
 *   (apply_silu = 0: without the silu), one read of x and one write of y,
 *   rounded once to the dtype.  gamma/beta ([C], dtype) may be NULL (1 / 0).
 *   y may be x (in place) but must not partially overlap it.
 * Both enqueue on `stream` and return before completion.
 */
CONV3D_API conv3d_status_t conv3d_groupnorm_stats(const void* x, int N, int D, int H, int W,
                                                  int C, int groups, int per_frame, float eps,
                                                  conv3d_dtype_t dtype, double* stats,
                                                  struct CUstream_st* stream);
CONV3D_API conv3d_status_t conv3d_groupnorm_silu(const void* x, const double* stats,
                                                 const void* gamma, const void* beta, void* y,
                                                 int N, int D, int H, int W, int C, int groups,
                                                 int per_frame, int apply_silu,
                                                 conv3d_dtype_t dtype, struct CUstream_st* stream);

/*
 * conv3d_fwd_gn -- the convolution of a decoder block with the GroupNorm work
 * around it fused in (news.bugfactory.tech: a fused GroupNorm + SiLU kernel;
 * stable-diffusion.cpp discussion "Exe Heavy Metal": GROUP_NORM on the GPU;
 * the decoder block runs normalise -> activate -> convolve, and the next
 * block normalises the result again).
 *
 * In (stats non-NULL): y = conv3d(h, w) + bias + residual with
 *   h[n,f,hh,ww,c] = silu((x - mean[s][g]) * rstd[s][g] * gamma[c] + beta[c]),
 *   g = c / (Cin/groups), s = the statistic set of frame f (the sample, or the
 *   frame of the sample with per_frame = 1), rounded once to the dtype -- the
 *   value an unfused pipeline would store -- computed as the kernel reads x,
 *   so h is never written to memory; the convolution's padding (spatial
 *   zeros, the temporal rule) applies to h.  apply_silu = 0 leaves out the
 *   SiLU.  stats: {mean, rstd} from conv3d_groupnorm_stats over x with the
 *   same groups and per_frame ([sets][groups][2] doubles, 8-byte aligned);
 *   gamma, beta: [Cin] of the dtype, 16-byte aligned, or NULL (1 and 0).
 *   stats = NULL: plain x (groups, per_frame, apply_silu, gamma, beta unused).
 * Out (out_stats non-NULL): also writes the GroupNorm statistics of y itself
 *   -- what conv3d_groupnorm_stats(y, out_groups, per_frame = 0, out_eps)
 *   would give, {mean, rstd} per sample and group of the rounded outputs,
 *   [N][out_groups][2] doubles -- gathered by the kernel as it stores y, so
 *   the next block's normalisation needs no statistics pass over y.
 *   1 <= out_groups <= 64 dividing Cout; out_eps >= 0.
 *
 * Every other argument and rule is conv3d_fwd's (its workspace included);
 * the cached-frames rule is not supported (CONV3D_ERR_UNSUPPORTED).
 */
CONV3D_API conv3d_status_t conv3d_fwd_gn(const void* x, const double* stats, const void* gamma,
                                         const void* beta, int groups, int per_frame,
                                         int apply_silu, const void* w, const void* bias,
                                         const void* residual, void* y, int N, int Cin, int D,
                                         int H, int W, int Cout, const int kernel[3],
                                         const int stride[3], const int pad[3],
                                         conv3d_tpad_t tpad, conv3d_dtype_t dtype,
                                         double* out_stats, int out_groups, float out_eps,
                                         struct CUstream_st* stream);

/*
 * conv3d_bwd_data -- dx, the gradient of the convolution's input (the pages'
 * on-device fine-tuning trains convolution layers: engineering.drawthings.ai,
 * LoRA post).  For stride 1 it is itself a convolution, of dy with every tap
 * of w mirrored and the channel roles exchanged, under the complementary
 * padding (kh-1-ph, kw-1-pw spatially; kt-1-pf in front temporally); with
 * causal replicate padding the gradient of the kt-1 virtual frames in front
 * is added to frame 0.  Runs the forward kernel on dy, after a weight
 * transform into the workspace; with causal replicate padding one launch
 * covers every frame: when it has at least 4 rounds of tiles (one tile per
 * SM a round) the tiles of frame 0 also run the taps of the kt-1 virtual
 * frames, into the same fp32 accumulator (one rounding); with fewer, the
 * launch writes the kt parts of frame 0 (frames -(kt-1)..0) in fp32 into the
 * workspace beside frames 1.. in dx, and a last kernel sums them into frame 0
 * with one rounding.  A single frame
 * (D = 1) takes the forward pass's first-frame fold, its weight mirrored and
 * folded by one kernel.  Everything runs on `stream`.
 *
 * Arguments describe the FORWARD problem: dy is [N, Do, Ho, Wo, Cout] (y's
 * shape), w [Cout, kt, kh, kw, Cin], dx [N, D, H, W, Cin] (written).  Supported:
 * temporal stride 1 and spatial strides up to 8, pads <= kernel extent - 1 at
 * stride 1, temporal rules zero, causal replicate and causal zero, plus the
 * forward call's channel and alignment
 * rules.  workspace: device, 256-byte aligned, conv3d_bwd_data_workspace_bytes()
 * bytes, not overlapping the tensors (it includes about 21 MB in which a launch
 * of under 16 rounds of tiles whose last round is at most half full -- a
 * single frame, a short clip -- splits that round's tiles along K across the
 * idle SMs).  dx must not
 * overlap dy or w.  Spatial strides: dx is computed phase by phase, each phase
 * (rows h = a*sh + rh, columns a*sw + rw) a stride-1 convolution of dy with the
 * mirrored taps that reach it, stored straight to its strided positions.
 * Errors: CONV3D_ERR_UNSUPPORTED for a temporal stride other than 1, the
 * cached-frames rule (conv3d_bwd_data_cached) or pads beyond kernel extent - 1
 * at stride 1; CONV3D_ERR_WORKSPACE for a missing or
 * short workspace; otherwise as conv3d_fwd.
 */
CONV3D_API conv3d_status_t conv3d_bwd_data(const void* dy, const void* w, void* dx, int N, int Cin,
                                           int D, int H, int W, int Cout, const int kernel[3],
                                           const int stride[3], const int pad[3],
                                           conv3d_tpad_t tpad, conv3d_dtype_t dtype,
                                           void* workspace, size_t ws_bytes,
                                           struct CUstream_st* stream);
CONV3D_API size_t conv3d_bwd_data_workspace_bytes(int N, int Cin, int D, int H, int W, int Cout,
                                                  const int kernel[3], const int pad[3],
                                                  conv3d_tpad_t tpad);

/*
 * conv3d_bwd_weight -- dw (and optionally dbias), the gradients of the
 * convolution's weight and bias (the trainable parameters of the pages'
 * on-device conv-layer fine-tuning: engineering.drawthings.ai, LoRA post):
 * dw[co, tap, ci] = sum over output pixels of
 * dy[.., co] * Xpad[.., tap-shifted, ci] (the same implicit im2col matrix the
 * forward pass reads, with the same padding rules), dbias[co] = sum of dy.
 * Accumulated in fp32 in the workspace (split over pixel ranges, fp32
 * atomics: the summation order varies from run to run), rounded once: a clear
 * kernel, the weight-gradient kernel and a rounding kernel on `stream`, the
 * last two launched as programmatic dependents of the one before (each waits
 * for it on the device before touching its results).  dbias:
 * for a single tap (1x1x1) a block of the kernel itself sums dy; otherwise a
 * pass over dy runs beside the kernel on the library's auxiliary stream,
 * forked from and joined back into `stream` with events (the call still
 * orders after and before the caller's work on `stream`, and can be captured
 * in a CUDA graph).
 *
 * Arguments describe the FORWARD problem: x [N, D, H, W, Cin], dy [N, Do, Ho,
 * Wo, Cout], dw [Cout, kt, kh, kw, Cin] (written), dbias [Cout] or NULL.
 * Strides up to 8, temporal rules zero, causal replicate and causal zero.
 * workspace: device, 256-byte aligned, conv3d_bwd_weight_workspace_bytes()
 * bytes (cleared by the call).  Errors: CONV3D_ERR_UNSUPPORTED for the
 * cached-frames rule (conv3d_bwd_weight_cached), CONV3D_ERR_INVALID_ARG for a null dw or overlapping
 * buffers, CONV3D_ERR_ALIGNMENT for a dbias not 16-byte aligned,
 * CONV3D_ERR_WORKSPACE for a missing or short workspace; otherwise as conv3d_fwd.
 */
CONV3D_API conv3d_status_t conv3d_bwd_weight(const void* x, const void* dy, void* dw, void* dbias,
                                             int N, int Cin, int D, int H, int W, int Cout,
                                             const int kernel[3], const int stride[3],
                                             const int pad[3], conv3d_tpad_t tpad,
                                             conv3d_dtype_t dtype, void* workspace,
                                             size_t ws_bytes, struct CUstream_st* stream);
CONV3D_API size_t conv3d_bwd_weight_workspace_bytes(int Cin, int Cout, const int kernel[3]);

/*
 * Utilities.  The pages describe no API; these complete the convolution call
 * above.  conv3d_workspace_bytes and conv3d_output_shape restate the
 * problem's sizes (Qwen Image post, "Video VAE": the first-frame fold is the
 * only step that needs scratch; the output extents follow from the padding
 * rules at the top of this file).  conv3d_poll_status, conv3d_status_string,
 * conv3d_last_error and conv3d_release exist because every call only enqueues
 * work on the caller's stream and never synchronises (A1111 Metal discussion:
 * a native op enqueues into the host framework's command stream rather than
 * committing per call), so device-side errors must be collected separately.
 */

/*
 * The backward pass of the cached-frames chunk mode (conv3d_fwd_cached): a
 * decoder trained chunk by chunk needs the gradient of each chunk's cached
 * frames as well, to pass it back to the chunk before (Qwen Image post,
 * "Video VAE": the frames before a chunk are the previous chunk's last kt-1
 * frames; LoRA post: the conv layers are trained on device).  The chunk is the
 * zero-padded (pt = 0) convolution of the joined clip [prev; x], and these are
 * its adjoints split at the join.
 *
 * conv3d_bwd_data_cached: dx [N, D, H, W, Cin] and dprev [N, kt-1, H, W, Cin]
 *   (dprev may be NULL: not computed) for dy [N, Do, Ho, Wo, Cout]; two runs of
 *   the forward kernel over dy with the mirrored, channel-transposed weight.
 *   Stride 1 and pads <= kernel extent - 1 only (else CONV3D_ERR_UNSUPPORTED).
 *   workspace: conv3d_bwd_data_workspace_bytes(..., CONV3D_TPAD_CAUSAL_CACHED)
 *   bytes, 256-byte aligned.  No buffer may overlap another.
 * conv3d_bwd_weight_cached: dw (and dbias) as conv3d_bwd_weight, with the taps
 *   that read frames before the chunk reading prev [N, kt-1, H, W, Cin]
 *   (required when kt > 1).  Strides up to 8; workspace as conv3d_bwd_weight.
 * Otherwise the rules and errors of conv3d_bwd_data / conv3d_bwd_weight.
 */
CONV3D_API conv3d_status_t conv3d_bwd_data_cached(const void* dy, const void* w, void* dx,
                                                  void* dprev, int N, int Cin, int D, int H,
                                                  int W, int Cout, const int kernel[3],
                                                  const int stride[3], const int pad[3],
                                                  conv3d_dtype_t dtype, void* workspace,
                                                  size_t ws_bytes, struct CUstream_st* stream);
CONV3D_API conv3d_status_t conv3d_bwd_weight_cached(const void* x, const void* prev,
                                                    const void* dy, void* dw, void* dbias, int N,
                                                    int Cin, int D, int H, int W, int Cout,
                                                    const int kernel[3], const int stride[3],
                                                    const int pad[3], conv3d_dtype_t dtype,
                                                    void* workspace, size_t ws_bytes,
                                                    struct CUstream_st* stream);

/* Device scratch bytes conv3d_fwd_ws needs for this problem: the folded
 * first-frame weight for CONV3D_TPAD_CAUSAL_REPLICATE with D == 1 and kt > 1,
 * 0 otherwise (also 0 for invalid sizes or a NULL kernel). */
CONV3D_API size_t conv3d_workspace_bytes(int Cin, int Cout, const int kernel[3], int D,
                                         conv3d_tpad_t tpad);

/* Output extents {Do, Ho, Wo} for the problem (formula at the top of this
 * file).  Returns CONV3D_ERR_INVALID_ARG, leaving out_dhw untouched, for a
 * NULL array, a non-positive size, an unknown mode or an output extent < 1. */
CONV3D_API conv3d_status_t conv3d_output_shape(int D, int H, int W, const int kernel[3],
                                               const int stride[3], const int pad[3],
                                               conv3d_tpad_t tpad, int out_dhw[3]);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device (CONV3D_OK, CONV3D_ERR_TIMEOUT or CONV3D_ERR_DEVICE_CHECK). */
CONV3D_API conv3d_status_t conv3d_poll_status(struct CUstream_st* stream);

/* Static English text for a status code. */
CONV3D_API const char* conv3d_status_string(conv3d_status_t status);

/* Text of the last CONV3D_ERR_CUDA / CONV3D_ERR_UNSUPPORTED detail on this thread. */
CONV3D_API const char* conv3d_last_error(void);

/* Number of GPU kernels this library has launched in the process, on every
 * device and stream, counted when each launch is enqueued (the convolution,
 * weight-gradient and GroupNorm kernels and their small companions: weight
 * transforms, folds, roundings).  Workspace clears done with cudaMemsetAsync
 * are not kernels of the library and are not counted.  Needs no GPU (0 until
 * the first launch); never fails. */
CONV3D_API unsigned long long conv3d_kernel_launches(void);

/* Frees the cached per-device workspace, the cached tensor maps and the
 * auxiliary stream (which the weight gradient's bias pass runs on).  Not to be
 * called while work that uses them is being enqueued. */
CONV3D_API void conv3d_release(void);

/* Failure-detection self test: launches one CTA that waits, with the same
 * bounded wait the convolution uses, on an mbarrier that nothing completes,
 * limited to `timeout_ms` (1..10000).  Synchronises and returns the status
 * the device recorded: CONV3D_ERR_TIMEOUT when the mechanism works.  The
 * status word is cleared before returning. */
CONV3D_API conv3d_status_t conv3d_selftest_wait_timeout(int timeout_ms);

/* Failure-detection test hook.  Arms the next `launches` launches of the
 * convolution kernels (the forward kernel, which the data gradient also runs,
 * and the weight-gradient kernel) so that their TMA producer skips the copies
 * of its first pipeline stage: the tensor-core issuer's bounded wait on that
 * stage then runs out after timeout_ms (1..10000).  launches = 0 disarms.  An
 * armed launch aborts the way any timed-out wait does -- every role leaves its
 * loop, the copies already in flight land, tensor memory is freed and the
 * kernel returns -- so nothing faults and the context stays usable;
 * conv3d_poll_status() then reports CONV3D_ERR_TIMEOUT and the call's output
 * is unspecified.  Process-wide: arm it only while no other thread enqueues
 * convolutions.  CONV3D_ERR_INVALID_ARG for arguments out of range. */
CONV3D_API conv3d_status_t conv3d_test_arm_stall(int launches, int timeout_ms);

#ifdef __cplusplus
}
#endif

#endif /* LIBCONV3D_CONV3D_H */
