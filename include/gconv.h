/*
 * gconv.h -- C ABI of libgconv.so: grouped / depthwise convolution on NVIDIA B200 (sm_100a).
 *
 * The operations, and the passages that define them:
 *
 *  gconv2d_fwd  Grouped 2-D convolution. Input channels, filters and output channels are
 *               divided into `groups` equal blocks with no connections between blocks
 *               ("Grouped convolutions", neon issue #296, thestew42's first reply); output
 *               channels come out group-major, 111122223333... (same thread, ibmua's post on
 *               output orderings). groups == C_in is the fully-grouped (depthwise) case of
 *               that thread. The arithmetic is F.conv2d's cross-correlation with zero padding,
 *               as called with padding and groups in "F.conv2d runs x15 slower in
 *               mixed-precision/half-precision mode" (the timing script), where the weight is
 *               [C_out, C_in/groups, kH, kW]:
 *                 y[n,co,ho,wo] = bias[co] + sum_{ci<C_in/g, kh<kH, kw<kW}
 *                     w[co,ci,kh,kw] * x[n, (co / (C_out/g))*(C_in/g) + ci,
 *                                        ho*stride - pad + kh*dilation,
 *                                        wo*stride - pad + kw*dilation]
 *               with x = 0 outside the image and
 *                 Ho = floor((H + 2*pad - dilation*(kH-1) - 1) / stride) + 1 (same for Wo).
 *
 *  gconv2d_bwd_*  The grouped conv2d's data and weight gradients (declared below with their
 *               sums).
 *
 *  dwconv1d_*   Depthwise conv1d over (batch, steps, channels) with groups = channels, the
 *               Conformer convolution module's depthwise layer ("Investigate custom Triton
 *               kernels for depthwise-separable convolutions in Conformer", speechbrain #2733:
 *               the issue text and the Oct 27 comment on the layout), with its backward pass
 *               (Oct 30 comment):
 *                 fwd    y[b,t,c]  = sum_{k<K} w[c,k] * x[b, t+k-pad_left, c]
 *                 dgrad  dx[b,s,c] = sum_{k<K} w[c,k] * dy[b, s-k+pad_left, c]
 *                 wgrad  dw[c,k]   = sum_{b,t} dy[b,t,c] * x[b, t+k-pad_left, c]
 *               with x = 0 outside [0, T), dy = 0 outside [0, T_out),
 *               T_out = T + pad_left + pad_right - K + 1.
 *
 * Layouts (dense, row-major, no strides):
 *   GCONV_NCHW  x[N][C_in][H][W], w[C_out][C_in/g][kH][kW], y[N][C_out][Ho][Wo]
 *   GCONV_NHWC  x[N][H][W][C_in], w[C_out][kH][kW][C_in/g], y[N][Ho][Wo][C_out]
 *               (PyTorch's channels_last for activations and weights)
 *   conv1d      x, dx: [B][T][C]; y, dy: [B][T_out][C]; w, dw: [C][K]
 *   bias        [C_out] in the data dtype, or NULL.
 *
 * Numerics: GCONV_F32 accumulates in fp32 FMA (no TF32); GCONV_F16 / GCONV_BF16 read 16-bit
 * inputs, accumulate in fp32 (tensor-core TMEM accumulators or CUDA-core FMA) and round the
 * result once to the data dtype, round-to-nearest-even. dw is written in the data dtype.
 *
 * Ownership and calling convention: every pointer is device memory owned by the caller. The
 * library allocates nothing; scratch comes from the caller's workspace, sized by the
 * *_workspace_size queries (0 means none is needed). Outputs are overwritten, never
 * accumulated into. Inputs and outputs must not overlap. All calls validate on the host
 * first; on any error they return a status, launch nothing and leave the outputs untouched.
 * Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default stream)
 * on the current device; the call returns without synchronising. There is no mutable global
 * state apart from the device error word read by gconv_get_device_error() and the fixed
 * scratch of dwconv1d_bwd_weight_noalloc, so calls on different streams may be made from
 * different threads (that one entry point excepted, see its comment).
 *
 * Stream order: the tensor-core kernels, the depthwise 3x3 kernel and the second kernel of
 * two-kernel calls are launched with programmatic stream serialization. Their setup (barrier
 * initialisation, tensor-memory allocation) may overlap the tail of the previous kernel in
 * the stream, whoever launched it, but they wait for that kernel to complete before their
 * first global-memory access, so stream order holds for every byte they read or write. Calls
 * may be captured into CUDA graphs.
 */
#ifndef GCONV_H_
#define GCONV_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GCONV_OK = 0,
  GCONV_ERR_INVALID_ARG = 1,    /* NULL pointer, non-positive size, groups not dividing C_in
                                   and C_out, window larger than the padded input, bad enum */
  GCONV_ERR_UNSUPPORTED = 2,    /* a forced path that cannot run this problem */
  GCONV_ERR_MISALIGNED = 3,     /* a forced vector/tensor-core path whose pointers or channel
                                   strides are not 16-byte aligned */
  GCONV_ERR_WORKSPACE = 4,      /* workspace NULL or smaller than the query returned */
  GCONV_ERR_CUDA = 5,           /* a CUDA runtime/driver call or a kernel launch failed */
  GCONV_ERR_DEVICE_TIMEOUT = 6  /* a kernel's bounded wait gave up (see gconv_get_device_error) */
} gconv_status;

typedef enum { GCONV_NCHW = 0, GCONV_NHWC = 1 } gconv_layout;

typedef enum { GCONV_F32 = 0, GCONV_F16 = 1, GCONV_BF16 = 2 } gconv_dtype;

/* Which kernel family runs a gconv2d_fwd problem. AUTO picks one by shape (see
 * gconv2d_select_path); the others force a family and fail with UNSUPPORTED / MISALIGNED
 * if it cannot run the problem. */
typedef enum {
  GCONV_PATH_AUTO = 0,
  GCONV_PATH_DIRECT = 1,   /* CUDA-core direct convolution (the depthwise or narrow-group
                              kernel when one applies, otherwise the generic direct kernel) */
  GCONV_PATH_IGEMM = 2,    /* per-group implicit GEMM on tcgen05 tensor cores (F16 / BF16) */
  GCONV_PATH_GENERIC = 3   /* the generic direct kernel (any shape, layout and dtype) */
} gconv_path;

/* Kernels reported by gconv2d_select_path. */
typedef enum {
  GCONV_KERNEL_DIRECT_GENERIC = 1,    /* one thread per output, fp32 FMA, any problem */
  GCONV_KERNEL_DEPTHWISE_NHWC = 2,    /* 8-channel vectors, sliding window, 16-bit NHWC */
  GCONV_KERNEL_IGEMM_TC = 3,          /* tcgen05 implicit GEMM, NHWC */
  GCONV_KERNEL_IGEMM_TC_NCHW = 4,     /* NCHW -> NHWC staging in the workspace + tcgen05 */
  GCONV_KERNEL_CONV1D_GENERIC = 5,    /* dwconv1d: one thread per output, fp32 FMA, any problem */
  GCONV_KERNEL_CONV1D_RING = 6,       /* dwconv1d: CUDA-core TMA-ring kernel; 16-bit, C % 8 == 0,
                                         K in {3, 5, 7, 9, 15, 31} */
  GCONV_KERNEL_CONV1D_TC = 7,         /* dwconv1d: tcgen05 banded product; 16-bit, C % 16 == 0,
                                         K <= 49 */
  GCONV_KERNEL_GROUPED_NHWC = 8,      /* conv2d, 2 / 4 / 8 channels per group in and out, 3x3,
                                         dilation 1, stride 1 or 2, 16-bit NHWC: CUDA cores */
  GCONV_KERNEL_DGRAD_GENERIC = 9,     /* conv2d data gradient: one thread per dx element, fp32
                                         FMA, any problem */
  GCONV_KERNEL_WGRAD_GENERIC = 10,    /* conv2d weight gradient: one thread per (dw entry,
                                         slice), fp32 FMA, any problem */
  GCONV_KERNEL_WGRAD_DEPTHWISE_NHWC = 11, /* conv2d weight gradient, depthwise 3x3 / 5x5,
                                         dilation 1, stride 1 or 2, 16-bit NHWC, C even */
  GCONV_KERNEL_DGRAD_DEPTHWISE_NHWC = 12, /* conv2d data gradient, depthwise 3x3 / 5x5 / 7x7,
                                         dilation 1, stride 1 or 2, 16-bit NHWC, C a multiple
                                         of 8 / 4 / 2: 16- / 8- / 4-byte channel vectors */
  GCONV_KERNEL_WGRAD_TILED_NHWC = 13, /* conv2d weight gradient, 16-bit NHWC, C_in/g and
                                         C_out/g >= 32 and multiples of 8: shared-memory tiled
                                         outer products on the CUDA cores */
  GCONV_KERNEL_WGRAD_DW3_TMA = 14,    /* conv2d weight gradient, depthwise 3x3, dilation 1,
                                         stride 1 or 2, pad <= 2, 16-bit NHWC, C % 8 == 0:
                                         x and dy staged by TMA */
  GCONV_KERNEL_WGRAD_TILED_NCHW = 15, /* GCONV_KERNEL_WGRAD_TILED_NHWC for NCHW tensors: x and
                                         dy transposed to NHWC in the workspace first */
  GCONV_KERNEL_DWSEP1D_FUSED = 16,    /* depthwise-separable block in one kernel: depthwise
                                         conv1d on the CUDA cores into shared memory, pointwise
                                         GEMM on tcgen05; 16-bit, C % 64 == 0, C_out % 16 == 0
                                         and <= 512, K in {3, 5, 7, 9, 15, 31} */
  GCONV_KERNEL_DWSEP_UNFUSED = 17,    /* depthwise-separable block as two launches: the
                                         depthwise output in the workspace, then the pointwise
                                         convolution */
  GCONV_KERNEL_WGRAD_TC_NHWC = 18,    /* conv2d weight gradient on tcgen05 tensor cores: per
                                         group and tap a GEMM over output positions, dy and x
                                         read as MN-major TMA tiles; 16-bit NHWC, stride 1,
                                         C_out/g % 128 == 0, C_in/g % 64 == 0,
                                         (kW-1)*dilation <= 8, Wo >= 32 */
  GCONV_KERNEL_WGRAD_TC_NCHW = 19,    /* GCONV_KERNEL_WGRAD_TC_NHWC for NCHW tensors: x and dy
                                         transposed to NHWC in the workspace first */
  GCONV_KERNEL_CONV1D_STRIP = 20,     /* dwconv1d: CUDA-core kernel on 128-byte input rows
                                         (64-channel tiles, taps in registers); 16-bit,
                                         C % 64 == 0, K in {3, 5, 7, 9, 15, 31} */
  GCONV_KERNEL_DWSEP2D_FUSED = 21,    /* 2-D depthwise-separable block in one kernel: 16-bit
                                         NHWC, depthwise 3x3 / 5x5, stride 1 / 2, dilation 1,
                                         C % 64 == 0, C_out % 16 == 0 and <= 512 */
  GCONV_KERNEL_DGRAD_DW3S2_TMA = 22,  /* conv2d data gradient, depthwise 3x3, stride 2, pad 1,
                                         dilation 1, 16-bit NHWC, C % 8 == 0: dy staged by TMA,
                                         dx written by TMA stores */
  GCONV_KERNEL_MERGE_MAX_TWO_PASS = 23 /* conv2d with the max merge across groups: the
                                         group-major output in the workspace on the transposed
                                         row-strip kernel (NCHW: through the NHWC staging), then
                                         the maximum over groups, 16-byte vectors */
} gconv_kernel;

/* Order and merging of the output channels ("Grouped convolutions", neon issue #296, ibmua's
 * post on output orderings: the group-major order 111122223333..., the interleaved order
 * 1234123412341234, and pulling the groups' results together by average or max pooling
 * across groups). With cpg_out = C_out / groups, filter j of group i is group-major channel
 * i*cpg_out + j:
 *   GROUP_MAJOR  y has C_out channels; channel i*cpg_out + j = filter j of group i (bias
 *                [i*cpg_out + j] added); what gconv2d_fwd writes.
 *   INTERLEAVED  y has C_out channels; channel j*groups + i = filter j of group i.
 *   MERGE_AVG    y has cpg_out channels; channel j = mean over groups i of group-major channel
 *                i*cpg_out + j (each with its bias).
 *   MERGE_MAX    y has cpg_out channels; channel j = maximum over i of the same. */
typedef enum {
  GCONV_OUT_GROUP_MAJOR = 0,
  GCONV_OUT_INTERLEAVED = 1,
  GCONV_OUT_MERGE_AVG = 2,
  GCONV_OUT_MERGE_MAX = 3
} gconv_out_mode;

/* Output shape of a gconv2d problem: validates the arguments exactly as gconv2d_fwd_out does
 * and writes *C_y (C_out, or C_out/groups for the merges), *Ho, *Wo by F.conv2d's rule
 * (Ho = floor((H + 2*pad - dilation*(kH-1) - 1) / stride) + 1, same for Wo; the output-size
 * rule of the timing script in "F.conv2d runs x15 slower in mixed-precision/half-precision
 * mode"). y is [N][C_y][Ho][Wo] (NCHW) or [N][Ho][Wo][C_y] (NHWC); dy of the backward calls
 * has the GROUP_MAJOR shape. Host-only, launches nothing.
 * Errors: INVALID_ARG (also for NULL outputs, a bad out_mode, or Ho / Wo < 1); the outputs are
 * untouched then. */
gconv_status gconv2d_out_shape(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                               int stride, int pad, int dilation, int groups,
                               gconv_layout layout, gconv_dtype dtype, gconv_out_mode out_mode,
                               int* C_y, int* Ho, int* Wo);

/* gconv2d_fwd_path writing the output in `out_mode` (above); y has the shape
 * gconv2d_out_shape reports. The order or the merge is applied in the kernel's epilogue, on
 * the fp32 accumulators (a merge adds or compares the groups' fp32 values, then rounds once),
 * so no second pass over y is made -- except for MERGE_MAX on problems that the transposed
 * row-strip kernel takes (GCONV_KERNEL_MERGE_MAX_TWO_PASS): the group-major output is written
 * to the workspace, rounded, and a second kernel takes the maximum over groups; rounding is
 * monotonic, so the maximum of the rounded values is the rounded maximum, bit for bit the
 * one-pass result. GROUP_MAJOR, and the modes that equal it (one filter per group for
 * INTERLEAVED, one group for the merges), run exactly as gconv2d_fwd_path. Other variants:
 * AUTO runs the tensor-core implicit GEMM for 16-bit problems it takes (the transposed
 * row-strip kernel for INTERLEAVED and MERGE_AVG where that tiling applies, the two passes
 * above for MERGE_MAX, otherwise the tile kernel; a merge there covers all groups of a
 * 16..64-filter block in one tile) and the generic direct kernel otherwise; DIRECT and
 * GENERIC run the generic direct kernel; IGEMM forces the tensor cores (UNSUPPORTED /
 * MISALIGNED as for gconv2d_fwd_path). The workspace (16-byte aligned) holds the two-pass
 * group-major output (N * C_out * Ho * Wo elements) and, for NCHW tensor-core runs, the NHWC
 * staging; gconv2d_fwd_out_workspace_size reports it.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA. */
gconv_status gconv2d_fwd_out(const void* x, const void* w, const void* bias, void* y, int N,
                             int C_in, int H, int W, int C_out, int kH, int kW, int stride,
                             int pad, int dilation, int groups, gconv_layout layout,
                             gconv_dtype dtype, gconv_out_mode out_mode, gconv_path path,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes gconv2d_fwd_out needs (0 if none or invalid), and the gconv_kernel it would
 * run for 16-byte aligned pointers (a negative gconv_status if it would fail). */
size_t gconv2d_fwd_out_workspace_size(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                      int stride, int pad, int dilation, int groups,
                                      gconv_layout layout, gconv_dtype dtype,
                                      gconv_out_mode out_mode, gconv_path path);
int gconv2d_fwd_out_select_path(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                int stride, int pad, int dilation, int groups,
                                gconv_layout layout, gconv_dtype dtype, gconv_out_mode out_mode,
                                gconv_path path);

/* Bytes of workspace gconv2d_fwd needs for this problem under `path` (0 if none; also 0 for
 * invalid arguments, which gconv2d_fwd then rejects). */
size_t gconv2d_fwd_workspace_size(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                  int stride, int pad, int dilation, int groups,
                                  gconv_layout layout, gconv_dtype dtype, gconv_path path);

/* Grouped conv2d forward (definition above), kernel chosen automatically. `y` is written in
 * full. `workspace` may be NULL when gconv2d_fwd_workspace_size(..., GCONV_PATH_AUTO) is 0.
 * Errors: INVALID_ARG, WORKSPACE, CUDA. Never MISALIGNED: unaligned problems run on a
 * kernel without the vector requirement. */
gconv_status gconv2d_fwd(const void* x, const void* w, const void* bias, void* y,
                         int N, int C_in, int H, int W, int C_out, int kH, int kW,
                         int stride, int pad, int dilation, int groups,
                         gconv_layout layout, gconv_dtype dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

/* gconv2d_fwd with an explicit kernel family (for path sweeps and tests). */
gconv_status gconv2d_fwd_path(const void* x, const void* w, const void* bias, void* y,
                              int N, int C_in, int H, int W, int C_out, int kH, int kW,
                              int stride, int pad, int dilation, int groups,
                              gconv_layout layout, gconv_dtype dtype, gconv_path path,
                              void* workspace, size_t workspace_bytes, void* stream);

/* The gconv_kernel that gconv2d_fwd_path would run for this problem, assuming 16-byte
 * aligned pointers; a negative gconv_status (e.g. -GCONV_ERR_INVALID_ARG) if it would fail. */
int gconv2d_select_path(int N, int C_in, int H, int W, int C_out, int kH, int kW, int stride,
                        int pad, int dilation, int groups, gconv_layout layout,
                        gconv_dtype dtype, gconv_path path);

/* ---- grouped conv2d backward. Sizes and layouts are those of the forward problem: x
 * [N][C_in][H][W] / [N][H][W][C_in], w as for gconv2d_fwd, dy with y's shape and layout.
 * These are the gradients of the forward sum above (the grouped layers on the pages are
 * trained: the Adam-trained ensemble of "Optimize convolution batching rule performance",
 * the backward passes timed in the Conformer thread):
 *   dx[n,c,h,w]      = sum over co in c's group and taps (kh, kw) with
 *                      h + pad - kh*dilation = ho*stride, w + pad - kw*dilation = wo*stride
 *                      (0 <= ho < Ho, 0 <= wo < Wo) of w[co, c mod (C_in/g), kh, kw]*dy[n,co,ho,wo]
 *   dw[co,ci,kh,kw]  = sum over (n, ho, wo) of dy[n,co,ho,wo] *
 *                      x[n, (co / (C_out/g))*(C_in/g) + ci, ho*stride-pad+kh*dilation,
 *                        wo*stride-pad+kw*dilation]
 * with x = 0 outside the image. No bias gradient (it is a plain sum of dy). */

/* Bytes of workspace gconv2d_bwd_data_path needs under `path` (0 if none or invalid). When
 * the data gradient runs as a forward convolution, this holds the flipped, transposed filter
 * (C_out * C_in/g * kH * kW elements, rounded up to 256 bytes) followed by the forward
 * kernel's own workspace. */
size_t gconv2d_bwd_data_workspace_size(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                       int stride, int pad, int dilation, int groups,
                                       gconv_layout layout, gconv_dtype dtype, gconv_path path);

/* Data gradient dy, w -> dx (written in full). With stride 1, a square kernel and
 * pad <= dilation*(k-1) it is computed as the forward convolution of dy with the per-group
 * transposed, 180-degree-rotated filter and pad' = dilation*(k-1) - pad, on the forward
 * kernels (AUTO / DIRECT / IGEMM choose among them as gconv2d_fwd_path does, F32 under AUTO
 * excepted). Under AUTO / DIRECT, depthwise NHWC problems that do not run that way take the
 * TMA-staged kernel for 3x3, stride 2, pad 1 (GCONV_KERNEL_DGRAD_DW3S2_TMA; dy and dx 16-byte
 * aligned), else a vectorised depthwise gather kernel (GCONV_KERNEL_DGRAD_DEPTHWISE_NHWC);
 * other problems, fp32 under AUTO and GENERIC run the one-thread-per-element gather kernel. IGEMM on a problem that cannot run as a forward convolution on the tensor
 * cores is UNSUPPORTED (or MISALIGNED). The workspace must be 16-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA. */
gconv_status gconv2d_bwd_data(const void* dy, const void* w, void* dx, int N, int C_in, int H,
                              int W, int C_out, int kH, int kW, int stride, int pad,
                              int dilation, int groups, gconv_layout layout, gconv_dtype dtype,
                              void* workspace, size_t workspace_bytes, void* stream);
gconv_status gconv2d_bwd_data_path(const void* dy, const void* w, void* dx, int N, int C_in,
                                   int H, int W, int C_out, int kH, int kW, int stride, int pad,
                                   int dilation, int groups, gconv_layout layout,
                                   gconv_dtype dtype, gconv_path path, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* The gconv_kernel gconv2d_bwd_data_path would run (a forward kernel code, run on the
 * exchanged problem, or GCONV_KERNEL_DGRAD_GENERIC), assuming aligned pointers; a negative
 * gconv_status if it would fail. */
int gconv2d_bwd_data_select_path(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                 int stride, int pad, int dilation, int groups,
                                 gconv_layout layout, gconv_dtype dtype, gconv_path path);

/* Bytes of workspace gconv2d_bwd_weight_path needs: fp32 partial sums, one per dw entry and
 * slice of the work (0 if none or invalid). The size is that of the kernel chosen for
 * 16-byte aligned x and dy; a call whose pointers select another kernel may need more (and
 * then returns GCONV_ERR_WORKSPACE). */
size_t gconv2d_bwd_weight_workspace_size(int N, int C_in, int H, int W, int C_out, int kH,
                                         int kW, int stride, int pad, int dilation, int groups,
                                         gconv_layout layout, gconv_dtype dtype,
                                         gconv_path path);

/* Weight gradient x, dy -> dw (w's shape, layout and dtype; written in full, zeros when
 * N == 0). Deterministic: the N*Ho output rows are cut into slices fixed by the problem's
 * sizes alone, each slice's partial sums are added in a fixed order and the slices are added
 * in slice order (no float atomics), so repeated calls -- on any GPU -- give bitwise-identical
 * dw. AUTO runs the TMA-staged depthwise 3x3 kernel where it applies
 * (GCONV_KERNEL_WGRAD_DW3_TMA; x and dy 16-byte aligned), else the depthwise kernel
 * (GCONV_KERNEL_WGRAD_DEPTHWISE_NHWC; x and dy 4-byte aligned), else the tensor-core kernel
 * for wide groups (GCONV_KERNEL_WGRAD_TC_NHWC with x and dy 16-byte aligned, or
 * GCONV_KERNEL_WGRAD_TC_NCHW, which stages NCHW x and dy as NHWC in the workspace), else the
 * CUDA-core tiled kernel (GCONV_KERNEL_WGRAD_TILED_NHWC / _NCHW, same staging), else the
 * generic kernel. DIRECT runs the same list without the tensor-core kernel; IGEMM forces the
 * tensor-core kernel (UNSUPPORTED where it does not apply, MISALIGNED for unaligned NHWC x or
 * dy); GENERIC forces the generic kernel. N*Ho > 2^30 is UNSUPPORTED.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
gconv_status gconv2d_bwd_weight(const void* x, const void* dy, void* dw, int N, int C_in, int H,
                                int W, int C_out, int kH, int kW, int stride, int pad,
                                int dilation, int groups, gconv_layout layout, gconv_dtype dtype,
                                void* workspace, size_t workspace_bytes, void* stream);
gconv_status gconv2d_bwd_weight_path(const void* x, const void* dy, void* dw, int N, int C_in,
                                     int H, int W, int C_out, int kH, int kW, int stride,
                                     int pad, int dilation, int groups, gconv_layout layout,
                                     gconv_dtype dtype, gconv_path path, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* The gconv_kernel gconv2d_bwd_weight_path would run, or a negative gconv_status. */
int gconv2d_bwd_weight_select_path(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                   int stride, int pad, int dilation, int groups,
                                   gconv_layout layout, gconv_dtype dtype, gconv_path path);

/* Output steps of a depthwise conv1d problem: validates the arguments as dwconv1d_fwd does
 * and writes *T_out = T + pad_left + pad_right - K + 1 (the steps of y and dy; x and dx have
 * T). Host-only. Errors: INVALID_ARG (also for NULL T_out, or T_out < 1). */
gconv_status dwconv1d_out_steps(int B, int T, int C, int K, int pad_left, int pad_right,
                                gconv_dtype dtype, int* T_out);

/* Depthwise conv1d forward: x [B][T][C], w [C][K] -> y [B][T_out][C].
 * Errors: INVALID_ARG (incl. T_out < 1), CUDA. */
gconv_status dwconv1d_fwd(const void* x, const void* w, void* y, int B, int T, int C, int K,
                          int pad_left, int pad_right, gconv_dtype dtype, void* stream);

/* Depthwise conv1d data gradient: dy [B][T_out][C], w [C][K] -> dx [B][T][C].
 * Computed as the forward kernel with the filter reversed and pads (K-1-pad_left,
 * K-1-pad_right). Errors as dwconv1d_fwd. */
gconv_status dwconv1d_bwd_data(const void* dy, const void* w, void* dx, int B, int T, int C,
                               int K, int pad_left, int pad_right, gconv_dtype dtype,
                               void* stream);

/* dwconv1d_fwd / dwconv1d_bwd_data with an explicit kernel family: DIRECT forces the
 * CUDA-core ring kernel (else the generic kernel), IGEMM the tensor-core kernel, GENERIC the
 * generic kernel; AUTO is what dwconv1d_fwd / dwconv1d_bwd_data run. The pages define one
 * operation; the families are this library's kernels for it (for path comparisons and tests).
 * Errors as dwconv1d_fwd, plus UNSUPPORTED (IGEMM on a problem it cannot run: 32-bit data,
 * C % 16 != 0, K > 49) and MISALIGNED (IGEMM with x, w or y not 16-byte aligned). */
gconv_status dwconv1d_fwd_path(const void* x, const void* w, void* y, int B, int T, int C, int K,
                               int pad_left, int pad_right, gconv_dtype dtype, gconv_path path,
                               void* stream);
gconv_status dwconv1d_bwd_data_path(const void* dy, const void* w, void* dx, int B, int T, int C,
                                    int K, int pad_left, int pad_right, gconv_dtype dtype,
                                    gconv_path path, void* stream);

/* The gconv_kernel (GCONV_KERNEL_CONV1D_*) that dwconv1d_fwd_path / dwconv1d_bwd_data_path
 * would run, assuming 16-byte aligned pointers; a negative gconv_status if it would fail. */
int dwconv1d_select_path(int B, int T, int C, int K, int pad_left, int pad_right,
                         gconv_dtype dtype, gconv_path path);

/* Bytes of workspace dwconv1d_bwd_weight needs (fp32 partial sums of fixed slices of B*T_out;
 * 0 for invalid arguments). */
size_t dwconv1d_bwd_weight_workspace_size(int B, int T, int C, int K, int pad_left,
                                          int pad_right, gconv_dtype dtype);

/* Depthwise conv1d weight gradient: x [B][T][C], dy [B][T_out][C] -> dw [C][K].
 * Deterministic: fixed slices of B*T_out are reduced in a fixed order (no float atomics),
 * so repeated calls give bitwise-identical dw. Errors: INVALID_ARG, WORKSPACE, CUDA. */
gconv_status dwconv1d_bwd_weight(const void* x, const void* dy, void* dw, void* workspace,
                                 size_t workspace_bytes, int B, int T, int C, int K,
                                 int pad_left, int pad_right, gconv_dtype dtype, void* stream);

/* Size of the fixed device scratch used by dwconv1d_bwd_weight_noalloc (4 MiB). */
#define GCONV_WGRAD_NOALLOC_SCRATCH_BYTES (4u * 1024u * 1024u)

/* dwconv1d_bwd_weight without a workspace argument, for callers that cannot allocate device
 * memory: runtimes that forbid device allocation once they are running (fixed memory budgets
 * in long-lived speech / streaming servers), and plugins or foreign-language callers that have
 * no handle on the host application's device allocator. The pages have no counterpart: it is
 * a calling convention of this library, not part of the method.
 * Same arguments, result and errors as dwconv1d_bwd_weight, and bitwise the same dw. The
 * partial sums go to a file-scope device array of GCONV_WGRAD_NOALLOC_SCRATCH_BYTES that is
 * part of the library image, so every GPU that loads the library holds it until the process
 * exits; problems whose dwconv1d_bwd_weight_workspace_size exceeds it are rejected with
 * GCONV_ERR_WORKSPACE before any launch. Nothing is allocated: no cudaMalloc, cudaFree or
 * allocating library call. The first call on a device looks up the array's device address
 * with that device current (a cudaGetSymbolAddress); make that first call before any stream
 * capture. All calls share the one array: calls that overlap on the GPU (on different
 * streams without ordering between them) race and may return wrong dw. No part of the array
 * has to start at zero; each call writes every slot it reads. */
gconv_status dwconv1d_bwd_weight_noalloc(const void* x, const void* dy, void* dw, int B, int T,
                                         int C, int K, int pad_left, int pad_right,
                                         gconv_dtype dtype, void* stream);

/* ---- depthwise-separable block on (batch, steps, channels): a depthwise conv1d followed by a
 * pointwise (1x1) convolution over channels, the block of the Conformer convolution module
 * ("Investigate custom Triton kernels for depthwise-separable convolutions in Conformer",
 * speechbrain #2733: the issue text; the Oct 30 comment on the Fast Conformer downsampler,
 * built the same way):
 *   d[b,t,c] = sum_{k<K} w_dw[c,k] * x[b, t+k-pad_left, c]      (dwconv1d_fwd)
 *   z[b,t,o] = bias[o] + sum_{c<C} w_pw[o,c] * d[b,t,c]
 * x [B][T][C], w_dw [C][K], w_pw [C_out][C], bias [C_out] or NULL, z [B][T_out][C_out],
 * T_out = T + pad_left + pad_right - K + 1. Nothing sits between the two convolutions
 * (normalisation and activation are separate layers). For 16-bit data the intermediate d is
 * rounded once to the data type (the tensor-core operand); the accumulations are fp32.
 * AUTO runs the fused kernel (GCONV_KERNEL_DWSEP1D_FUSED: d never leaves the SM) where it
 * applies, otherwise the composition (GCONV_KERNEL_DWSEP_UNFUSED: d in the workspace, then
 * the pointwise convolution on the library's own kernels); IGEMM forces the fused kernel
 * (UNSUPPORTED / MISALIGNED if it cannot run), DIRECT forces the composition, GENERIC the
 * composition on the generic kernels. The workspace (16-byte aligned) holds d for the
 * composition; 0 bytes for the fused kernel.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA. */
size_t dwsep1d_fwd_workspace_size(int B, int T, int C, int K, int pad_left, int pad_right,
                                  int C_out, gconv_dtype dtype, gconv_path path);
int dwsep1d_select_path(int B, int T, int C, int K, int pad_left, int pad_right, int C_out,
                        gconv_dtype dtype, gconv_path path);
gconv_status dwsep1d_fwd(const void* x, const void* w_dw, const void* w_pw, const void* bias,
                         void* z, int B, int T, int C, int K, int pad_left, int pad_right,
                         int C_out, gconv_dtype dtype, gconv_path path, void* workspace,
                         size_t workspace_bytes, void* stream);

/* ---- 2-D depthwise-separable block: a depthwise conv2d (groups = C, kernel kH x kW, stride,
 * pad, dilation as for gconv2d_fwd) followed by a pointwise 1x1 convolution C -> C_out, the
 * strided layers of the Fast Conformer downsampler (same thread, Oct 30 comment):
 *   z[n,o,ho,wo] = bias[o] + sum_c w_pw[o,c] * d[n,c,ho,wo],  d = gconv2d_fwd(x, w_dw, groups=C)
 * x in `layout` with C channels; w_dw the depthwise weight of that layout ([C][1][kH][kW] or
 * [C][kH][kW][1], the same bytes); w_pw [C_out][C]; bias [C_out] or NULL; z in `layout`
 * with C_out channels and the depthwise output's Ho x Wo. AUTO runs the fused kernel
 * (GCONV_KERNEL_DWSEP2D_FUSED) where it applies, otherwise the composition
 * (GCONV_KERNEL_DWSEP_UNFUSED: d in the workspace, then the pointwise convolution, each on
 * the kernel gconv2d_fwd would pick); IGEMM / DIRECT / GENERIC as for dwsep1d_fwd. The 16-bit
 * intermediate is rounded once to the data type. The workspace (16-byte aligned) holds d and
 * the two convolutions' own workspaces for the composition; 0 bytes for the fused kernel.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA. */
size_t dwsep2d_fwd_workspace_size(int N, int C, int H, int W, int kH, int kW, int stride,
                                  int pad, int dilation, int C_out, gconv_layout layout,
                                  gconv_dtype dtype, gconv_path path);
int dwsep2d_select_path(int N, int C, int H, int W, int kH, int kW, int stride, int pad,
                        int dilation, int C_out, gconv_layout layout, gconv_dtype dtype,
                        gconv_path path);
gconv_status dwsep2d_fwd(const void* x, const void* w_dw, const void* w_pw, const void* bias,
                         void* z, int N, int C, int H, int W, int kH, int kW, int stride,
                         int pad, int dilation, int C_out, gconv_layout layout,
                         gconv_dtype dtype, gconv_path path, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the device error word that kernels with
 * bounded waits set when a wait gives up. *code receives 0 if none gave up. Returns
 * GCONV_ERR_DEVICE_TIMEOUT if one did, GCONV_ERR_CUDA if synchronisation failed. */
gconv_status gconv_get_device_error(void* stream, int* code);

/* Test hook for the bounded waits. From the next call on, the generic tensor-core tile kernel
 * (GCONV_KERNEL_IGEMM_TC on shapes that no specialised tiling takes, e.g. output rows narrower
 * than 128 pixels and not a multiple of 8) declares `bytes` more per pipeline stage to its
 * mbarrier than its TMA copies deliver, so that stage never completes: its waits give up after
 * their 1 s limit, the CTA drains its copies and MMAs (each drain bounded by the same limit),
 * frees its tensor memory and exits, and gconv_get_device_error then returns
 * GCONV_ERR_DEVICE_TIMEOUT. No fault, trap or unbounded wait is involved; the context stays
 * usable, and outputs of such a call are undefined. 0 (the default) restores normal
 * operation. Process-wide, not thread-safe against concurrent launches; for tests only.
 * Errors: INVALID_ARG unless bytes is a multiple of 16 and at most 65536. */
gconv_status gconv_debug_set_tx_surplus(unsigned int bytes);

/* Human-readable name of a status. Never NULL. */
const char* gconv_status_string(gconv_status status);

/* Library version, major*10000 + minor*100 + patch. */
int gconv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GCONV_H_ */
