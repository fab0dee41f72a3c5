/*
 * conv_fwd.h -- C ABI of the B200 (sm_100a) implicit-GEMM convolution forward.
 *
 * The operation (the "Convolutions" tutorial, sections 1 and 4, and its
 * variants table in section 5; the MLX pull request "Add implicit matmul
 * pathway for mx.conv3d", its description and benchmark table):
 *
 *   y[n,od,oh,ow,o] = sum_{kd,kh,kw,c} x[n, od*sd-pd+kd*dd, oh*sh-ph+kh*dh,
 *                                        ow*sw-pw+kw*dw, g*C/G + c]
 *                                     * w[o, kd, kh, kw, c]
 *
 * a cross-correlation (the filter is not flipped, as the tutorial's worked
 * example fixes), with zero padding of pad[i] on both sides of spatial
 * dimension i, g = o / (O/G), and output extents
 *   Do = floor((D + 2*pd - dd*(kD-1) - 1) / sd) + 1   (likewise Ho, Wo).
 * It is computed as an implicit GEMM (tutorial section 5, "Implicit GEMM"):
 * M = N*Do*Ho*Wo output pixels by O/G output channels per group, reduced over
 * K = kD*kH*kW*C/G, with the patch ("im2col") indices computed inside the
 * kernel so that no patch matrix is ever stored.
 *
 * Layouts (all contiguous, row-major, channels last):
 *   x  [N, D, H, W, C]            (NDHWC; a 2-D convolution is D = kD = 1)
 *   w  [O, kD, kH, kW, C/groups]
 *   y  [N, Do, Ho, Wo, O]
 * Spatial parameter arrays are ordered (depth, height, width).
 *
 * Element types: CONV_F16 and CONV_BF16 run on the tcgen05 tensor cores with
 * fp32 accumulation in tensor memory and round-to-nearest-even output;
 * CONV_F32 runs an fp32 FFMA kernel (no TF32); depthwise problems of any type
 * run FP32-FMA depthwise kernels.  x, w and y share one type.
 *
 * Besides the forward pass (conv_fwd, conv_fwd_variant, conv_fwd_ex,
 * conv_fwd_host), the header declares its other two passes: the transposed
 * convolution, which is the data gradient (conv_transpose), and the weight
 * gradient (conv_wgrad), each documented at its declaration below.
 *
 * Ownership: the caller owns every buffer.  conv_fwd allocates nothing, does
 * not synchronise, and returns after queueing its work on `stream`.  Kernels
 * may read x and w in whole aligned 16-byte blocks: the block holding a
 * tensor's last element can be read in full, up to 14 bytes past the tensor's
 * end but never past that block (which, 16-byte aligned, cannot cross a page);
 * those bytes never reach y.  Nothing is written outside y.
 * Thread safety: calls may come from several host threads.
 *
 * Errors: every entry point returns CONV_OK (0) or a negative code and never
 * aborts the process; argument errors are found on the host before anything is
 * queued.  Device-side failures (a pipeline wait that timed out) are recorded
 * in a per-device status word read by conv_last_status().
 */
#ifndef CONV_FWD_H_
#define CONV_FWD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (identical to cudaStream_t / CUstream). NULL is the
 * legacy default stream. */
typedef struct CUstream_st* conv_stream_t;

typedef enum { CONV_F32 = 0, CONV_F16 = 1, CONV_BF16 = 2 } conv_dtype_t;

enum {
  CONV_OK = 0,
  CONV_EINVAL = -1,      /* a non-positive size, stride or dilation, a negative
                            pad, C or O not divisible by groups, an empty
                            output, a NULL pointer, or sizes beyond 2^31-1
                            elements per dimension product limits */
  CONV_EDTYPE = -2,      /* unknown element type */
  CONV_EALIGN = -3,      /* x, w or y not 16-byte aligned */
  CONV_EALIAS = -4,      /* y overlaps x or w */
  CONV_ELAUNCH = -5,     /* the CUDA runtime refused the launch or a copy */
  CONV_ETIMEOUT = -6,    /* a kernel's pipeline wait ran out (device status) */
  CONV_EUNSUPPORTED = -7,/* the requested kernel variant cannot run this shape */
  CONV_EDRIVER = -8,     /* the driver could not encode a TMA tensor map */
  CONV_ESCRATCH = -9     /* conv_wgrad_noalloc: the problem needs more scratch
                            than CONV_WGRAD_STATIC_SCRATCH_BYTES */
};

/* Kernel variants (for conv_fwd_variant and conv_plan). */
enum {
  CONV_VARIANT_AUTO = -1,
  CONV_VARIANT_SIMT = 0,       /* fp32 FFMA implicit GEMM (any shape, any type) */
  CONV_VARIANT_TC_TMA = 1,     /* tcgen05 + TMA im2col loads (C/G % 16 == 0) */
  CONV_VARIANT_TC_GATHER = 2, /* tcgen05 + in-kernel gather (any C, any geometry) */
  CONV_VARIANT_TC_TMA_PAIR = 3, /* TC_TMA with CTA pairs: 256-row tiles, cta_group::2 */
  CONV_VARIANT_TC_HALO = 4,     /* tcgen05, one TMA box of input halo per 16x8 output block
                                   reused by every filter tap (stride 1, C/G % 64 == 0) */
  CONV_VARIANT_TC_HALO_PAIR = 5, /* TC_HALO with CTA pairs (32x8 blocks, cta_group::2) */
  CONV_VARIANT_TC_TMA_T = 6,     /* TC_TMA in the transposed orientation: MMA M = 128
                                   output channels, N = 256 output pixels, TMA-store
                                   epilogue (C/G % 16 == 0, O/G % 128 == 0) */
  CONV_VARIANT_TC_HALO_T = 7,    /* transposed orientation with halo reuse: M = 128
                                   (or 64) output channels, N = an (up to 32) x 8
                                   output block read from one 8-wide input strip
                                   per (channel chunk, kd, kw) (stride 1,
                                   C/G % 32 == 0, O/G % 64 == 0) */
  CONV_VARIANT_TC_HALO_T_PAIR = 8, /* TC_HALO_T with CTA pairs: M = 256 output channels,
                                   cta_group::2 (O/G % 256 == 0) */
  CONV_VARIANT_TC_PHASE = 9,      /* 2-D layers with few input channels: one GEMM row =
                                   P output pixels of a row (P*sw*C a multiple of 8),
                                   its window of the flattened (w, c) input row loaded
                                   by TMA; N = P*O <= 256, a multiple of 32 (groups 1, width dilation 1,
                                   H % sh == 0, W*C*2 % 16 == 0, Wo % P == 0) */
  CONV_VARIANT_DEPTHWISE = 10,    /* depthwise (groups = C = O, C*elem % 16 == 0), any element
                                   type, FP32 FMAs: persistent CTAs, input slabs staged by TMA
                                   through an mbarrier ring (DEPTHWISE_DIRECT where the slabs do
                                   not fit); the automatic choice for these shapes */
  CONV_VARIANT_DEPTHWISE_DIRECT = 11, /* depthwise, loads straight from global memory */
  CONV_VARIANT_TC_TMA_PHASES = 12, /* conv_transpose only: one stride-1 implicit GEMM per
                                   sub-pixel phase on tcgen05 CTA pairs, A by TMA im2col of
                                   the undilated input, B straight from w as MN-major tiles
                                   (f16/bf16, dilation 1, Cin/G % 64 == 0, Cout/G % 128 == 0,
                                   strides <= 8, a geometry inside the TMA im2col limits) */
  CONV_VARIANT_TC_STAGED = 13     /* any channel count (the path for C*2 % 16 != 0): builder
                                   warps realign, per (kd, 16-channel chunk), the input
                                   region of an up-to-32 x 8 output block and the matching
                                   weights into unswizzled K-major shared-memory tiles that
                                   every (kh, kw) tap reads as a descriptor view; tcgen05
                                   MMA M = 128 output channels, N = the block's pixels
                                   (f16/bf16, groups 1, stride 1, O <= 128, no flip) */
};

/* Output extents.  stride/pad/dil: 3 ints (d, h, w).  out: 3 ints (Do, Ho, Wo).
 * Returns CONV_OK or CONV_EINVAL (non-positive input, kernel, stride or
 * dilation, negative pad, or an empty output).  Host-only; needs no GPU. */
int conv_out_dims(int D, int H, int W, int kD, int kH, int kW,
                  const int stride[3], const int pad[3], const int dil[3],
                  int out[3]);

/* Forward convolution on device buffers x, w, y (see the layouts above).
 * Queues the kernel on `stream`; returns CONV_OK or an error code (nothing is
 * queued on an error).  The variant is chosen from the type and shape:
 * f32 -> SIMT; f16/bf16 with C/G % 16 == 0 and a geometry that fits a TMA
 * im2col tensor map -> when O/G is a multiple of 64 but not of 256: TC_HALO_T
 * at stride 1 with C/G % 32 == 0, kH >= 2 and at least as many output blocks
 * as SMs, else (O/G % 128 == 0) TC_TMA for reductions of K <= 256 elements,
 * else TC_TMA_T when there are at least as many 256-pixel tiles as SMs;
 * otherwise TC_TMA_PAIR (or TC_TMA when there are fewer 256-row output tiles
 * than SM pairs); otherwise TC_PHASE where its conditions hold, else
 * TC_STAGED from 16 channels a group up where it plans, else TC_GATHER.
 * Depthwise problems (groups = C = O, C*elem % 16 == 0), of any type, run
 * DEPTHWISE.  TC_HALO, TC_HALO_PAIR and TC_HALO_T_PAIR run only when
 * requested through conv_fwd_variant.  Every kernel is launched with
 * programmatic stream serialization and waits for the previous kernel on the
 * stream before it touches global memory: results are those of stream order. */
int conv_fwd(const void* x, const void* w, void* y,
             int N, int D, int H, int W, int C, int O,
             int kD, int kH, int kW,
             const int stride[3], const int pad[3], const int dil[3],
             int groups, int dtype, conv_stream_t stream);

/* The general form: padding pad_lo[i] below and pad_hi[i] above spatial
 * dimension i (the index origin is -pad_lo; the extent is
 * floor((I + pad_lo + pad_hi - dil*(k-1) - 1) / s) + 1), and flip = 1 to read
 * the filter reversed in every spatial dimension, w[o, kD-1-kd, kH-1-kh,
 * kW-1-kw, c] (a true convolution; 0 is the cross-correlation above).  The
 * flip is the MLX pull request's "correct flip" of its input loader ("What
 * changed"); per-side padding generalises the symmetric padding.  variant is
 * CONV_VARIANT_AUTO or an explicit CONV_VARIANT_*; with flip the gather
 * kernel does not use its filter-row layouts.  Returns as conv_fwd / conv_fwd_variant; CONV_EINVAL also for a
 * negative pad or a flip other than 0 or 1. */
int conv_fwd_ex(const void* x, const void* w, void* y,
                int N, int D, int H, int W, int C, int O,
                int kD, int kH, int kW,
                const int stride[3], const int pad_lo[3], const int pad_hi[3],
                const int dil[3], int groups, int flip, int dtype, int variant,
                conv_stream_t stream);

/* conv_fwd with an explicit kernel variant (CONV_VARIANT_*).  Returns
 * CONV_EUNSUPPORTED when that variant cannot run the shape or type
 * (the tensor-core variants need f16/bf16; TC_TMA, TC_TMA_PAIR and TC_TMA_T
 * need C/G % 16 == 0 and a geometry inside the TMA im2col limits, TC_TMA_T
 * also O/G % 128 == 0; TC_HALO and TC_HALO_PAIR need stride 1 and
 * C/G % 32 == 0; TC_HALO_T also O/G % 64 == 0, TC_HALO_T_PAIR
 * O/G % 256 == 0; TC_STAGED needs one group, stride 1, O <= 128, no flip
 * and two pipeline slots in shared memory). */
int conv_fwd_variant(const void* x, const void* w, void* y,
                     int N, int D, int H, int W, int C, int O,
                     int kD, int kH, int kW,
                     const int stride[3], const int pad[3], const int dil[3],
                     int groups, int dtype, int variant, conv_stream_t stream);

/* The same computation on HOST buffers x_host, w_host, y_host.  The caller
 * also provides device buffers x_dev, w_dev, y_dev of the matching sizes
 * (the library allocates no device memory).  The batch is split into chunks
 * of whole images (up to 16, each moving at least 4 MiB): the upload of a
 * chunk, the kernel on the previous chunk (on `stream`) and the download of
 * the one before overlap, on two copy streams the library creates once per
 * device and orders against `stream` with events.  Every chunk runs the kernel
 * variant chosen for the whole batch, so y equals conv_fwd's result.  The
 * call waits for the result, so y_host holds it on return, and then reads and
 * clears the device status word: CONV_ETIMEOUT means a kernel gave up on a
 * pipeline wait and y_host is incomplete.  Host buffers should be
 * page-locked for the copies to be asynchronous.  Calls on one device take
 * turns. */
int conv_fwd_host(const void* x_host, const void* w_host, void* y_host,
                  void* x_dev, void* w_dev, void* y_dev,
                  int N, int D, int H, int W, int C, int O,
                  int kD, int kH, int kW,
                  const int stride[3], const int pad[3], const int dil[3],
                  int groups, int dtype, conv_stream_t stream);

/* Output extents with per-side padding (see conv_fwd_ex). */
int conv_out_dims_ex(int D, int H, int W, int kD, int kH, int kW,
                     const int stride[3], const int pad_lo[3], const int pad_hi[3],
                     const int dil[3], int out[3]);

/* conv_plan_variant for the general form of conv_fwd_ex (per-side padding,
 * flip).  Queues nothing. */
int conv_plan_ex(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW,
                 const int stride[3], const int pad_lo[3], const int pad_hi[3],
                 const int dil[3], int groups, int flip, int dtype, int variant,
                 int* bn, int* stages, int* ctas);

/* The variant conv_fwd would run for this shape and type (CONV_VARIANT_*), or
 * a negative error code.  Also reports the output-tile width BN, the number of
 * pipeline stages and the number of CTAs it would launch (any may be NULL);
 * for DEPTHWISE / DEPTHWISE_DIRECT, BN is the number of channels a thread
 * computes and stages is the slab ring depth (1 for the direct form).
 * Queries the current device's SM count; queues nothing. */
int conv_plan(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW,
              const int stride[3], const int pad[3], const int dil[3],
              int groups, int dtype, int* bn, int* stages, int* ctas);

/* conv_plan for an explicit variant (CONV_VARIANT_*; AUTO behaves as
 * conv_plan).  Returns that variant, CONV_EUNSUPPORTED when it cannot run the
 * shape or type (the same rule as conv_fwd_variant), or another negative
 * error code.  Queues nothing. */
int conv_plan_variant(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW,
                      const int stride[3], const int pad[3], const int dil[3],
                      int groups, int dtype, int variant, int* bn, int* stages, int* ctas);

/* ---- transposed ("upsampling") convolution ----------------------------
 *
 * "Convolutions" tutorial, "Convolution variants worth knowing": the
 * transposed convolution of decoders and diffusion models, read as the
 * adjoint (data gradient) of conv_fwd with the same weights:
 *
 *   y[n, q, g*Cout/G + c] = sum over taps k and input channels ci of group g
 *                           with q = i*s - p + k*d (per dimension) of
 *                           x[n, i, ci] * w[ci, k, c]
 *
 * x: [N, D, H, W, Cin]; w: [Cin, kD, kH, kW, Cout/groups] (conv_fwd's weight
 * layout with O = Cin, C = Cout); y: [N, Qd, Qh, Qw, Cout] with
 * Q = (I-1)*s - 2p + d*(k-1) + 1 + op per dimension, the output padding op in
 * [0, max(s, d)).  Requires p <= d*(k-1) per dimension (CONV_EUNSUPPORTED
 * otherwise).  It runs as a forward convolution over the input zero-dilated
 * by the stride (the inserted zeros are never stored: the gather producers and
 * the FP32 kernel skip them when computing addresses) with the mirrored,
 * channel-exchanged filter, or, where it fits, by sub-pixel phases
 * (CONV_VARIANT_TC_TMA_PHASES): output q = s*t + r takes only the taps
 * k = (r + p) mod s (mod s), a stride-1 convolution of the undilated input per
 * phase, fed by TMA.  Variants: AUTO (TC_TMA_PHASES where it fits, else
 * TC_GATHER for f16/bf16; SIMT for f32), TC_TMA_PHASES, TC_GATHER and SIMT;
 * any other variant returns CONV_EUNSUPPORTED.
 * Buffers, alignment, streams and errors as for conv_fwd. */

/* Extents (Qd, Qh, Qw) of the transposed convolution. */
int conv_transpose_out_dims(int D, int H, int W, int kD, int kH, int kW, const int stride[3],
                            const int pad[3], const int out_pad[3], const int dil[3], int out[3]);

/* Queues the transposed convolution on `stream`; allocates nothing. */
int conv_transpose(const void* x, const void* w, void* y, int N, int D, int H, int W, int Cin, int Cout,
                   int kD, int kH, int kW, const int stride[3], const int pad[3], const int out_pad[3],
                   const int dil[3], int groups, int dtype, int variant, conv_stream_t stream);

/* conv_plan_variant for the transposed convolution.  Queues nothing. */
int conv_transpose_plan(int N, int D, int H, int W, int Cin, int Cout, int kD, int kH, int kW,
                        const int stride[3], const int pad[3], const int out_pad[3], const int dil[3],
                        int groups, int dtype, int variant, int* bn, int* stages, int* ctas);

/* ---- weight gradient ----------------------------------------------------
 *
 * The gradient of conv_fwd's weights given the gradient dy of its output
 * (the forward pass with padding pad_lo below and pad_hi above, no flip):
 *
 *   dw[o, kd, kh, kw, c] = sum over n, od, oh, ow of dy[n, od, oh, ow, o] *
 *       x[n, od*sd - pd + kd*dd, oh*sh - ph + kh*dh, ow*sw - pw + kw*dw, g*C/G + c]
 *
 * x: [N, D, H, W, C]; dy: [N, Do, Ho, Wo, O] (the forward output's extents);
 * dw: [O, kD, kH, kW, C/groups], written (not accumulated into).  As a GEMM
 * per group: M = O/G output channels, N = taps * C/G weight columns, and a
 * reduction over the output pixels, split into ranges.  Two kernels compute
 * the ranges' fp32 partial sums:
 *  - CONV_WGRAD_TENSOR_CORES (f16/bf16, C/G % 64 == 0, O/G % 256 == 0, an
 *    input geometry the TMA im2col unit describes): tcgen05 CTA pairs, 256
 *    output channels x 256 columns per unit, dy rows and im2col rows of x
 *    staged by TMA as in the forward pass and read as MN-major operands;
 *  - CONV_WGRAD_FP32 (everything else): FP32 FMAs.
 * Each range's partial sums go to their own slice of a caller-provided
 * workspace of conv_wgrad_workspace_size bytes (16-byte aligned, disjoint
 * from x, dy, dw); a second kernel adds the slices in range order and rounds
 * to nearest into dw.  No atomics, and the split depends on the shape alone,
 * so a result is the same bits on every run and every device.  Queues two
 * kernels on `stream`; allocates nothing.  Errors as for conv_fwd;
 * CONV_EINVAL also for a missing or short workspace. */

enum { CONV_WGRAD_FP32 = 0, CONV_WGRAD_TENSOR_CORES = 1 };

/* The path conv_wgrad takes for these shapes (CONV_WGRAD_*) and the number of
 * ranges of its pixel reduction (either may be NULL).  Host-only. */
int conv_wgrad_plan(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW, const int stride[3],
                    const int pad_lo[3], const int pad_hi[3], const int dil[3], int groups, int dtype, int* path,
                    int* nsplit);

/* Bytes of fp32 workspace conv_wgrad needs (any element type). */
int conv_wgrad_workspace_size(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW,
                              const int stride[3], const int pad_lo[3], const int pad_hi[3],
                              const int dil[3], int groups, int dtype, unsigned long long* bytes);

int conv_wgrad(const void* x, const void* dy, void* dw, int N, int D, int H, int W, int C, int O,
               int kD, int kH, int kW, const int stride[3], const int pad_lo[3], const int pad_hi[3],
               const int dil[3], int groups, int dtype, void* workspace,
               unsigned long long workspace_bytes, conv_stream_t stream);

/* ---- weight gradient without allocation -------------------------------
 *
 * No counterpart in the pages: this entry point exists for callers that cannot
 * allocate device memory.  Examples are a plugin inside a framework whose
 * caching allocator owns all of the device's memory, a real-time loop that
 * forbids cudaMalloc/cudaFree because they can block or synchronise the
 * device, and a runtime that reserved its whole memory budget at start-up.
 * Such callers cannot provide conv_wgrad's workspace.
 *
 * conv_wgrad_noalloc computes what conv_wgrad computes, with the same
 * arguments minus the workspace.  Its fp32 scratch is a fixed array of
 * CONV_WGRAD_STATIC_SCRATCH_BYTES inside the library's device image.  Every
 * device that loads the library holds that array until the process exits.
 * The call allocates nothing and calls no allocating routine.
 *
 *  - Limit: each range of the split pixel reduction needs a slice of
 *    O * kD*kH*kW * C/groups * 4 bytes.  The call splits the reduction as
 *    conv_wgrad does when those slices fit in the array, else into as many
 *    ranges as fit (the two entry points may then differ in the last bits).
 *    A problem whose one slice exceeds CONV_WGRAD_STATIC_SCRATCH_BYTES
 *    returns CONV_ESCRATCH and queues nothing.
 *  - Set-up: the first call on a device (with that device current) looks up
 *    the array's device address once.  Make that first call before any stream
 *    capture.
 *  - Sharing: every call on a device uses the same array, which keeps the
 *    last call's contents.  Each call writes every element of the slices it
 *    uses before reading them, so nothing of an earlier call reaches its
 *    result.  Calls whose work overlaps on the GPU (two streams, or two host
 *    threads on different streams) race on the array and give wrong results;
 *    order them on one stream or with events.
 *
 * Returns as conv_wgrad, plus CONV_ESCRATCH. */
#define CONV_WGRAD_STATIC_SCRATCH_BYTES (16ull << 20)

int conv_wgrad_noalloc(const void* x, const void* dy, void* dw, int N, int D, int H, int W, int C, int O,
                       int kD, int kH, int kW, const int stride[3], const int pad_lo[3], const int pad_hi[3],
                       const int dil[3], int groups, int dtype, conv_stream_t stream);

/* Waits for `stream`, then reads and clears the current device's status word.
 * Returns CONV_OK, or CONV_ETIMEOUT if a kernel since the last call gave up on
 * a pipeline wait (the kernel then wrote no further output and returned), or
 * CONV_ELAUNCH if the stream itself reports an error. */
int conv_last_status(conv_stream_t stream);

/* Human-readable text for a return code (static storage). */
const char* conv_strerror(int code);

/* Library version as major*10000 + minor*100 + patch. */
int conv_version(void);

/* Failure-detection test hook.  The next launch on this process of a kernel
 * with pipeline waits (the tensor-core kernels, including the weight
 * gradient's, and the TMA depthwise kernel) makes its MMA thread (depthwise:
 * its first consumer warp) wait on a pipeline barrier that nothing arrives at,
 * with a limit of `timeout_ns` (1 ns .. 10 s) instead of the usual 2 s: the
 * wait runs out, the kernel raises its abort flag, every role drains what it
 * has in flight, tensor memory is freed, the kernel returns without writing
 * further output, and conv_last_status() then reports CONV_ETIMEOUT.  Nothing
 * faults or hangs; the context stays usable.  One-shot.  Returns CONV_OK or
 * CONV_EINVAL. */
int conv_debug_inject_stall(unsigned long long timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* CONV_FWD_H_ */
