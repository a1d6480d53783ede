// Internal declarations shared by the CUDA translation units of libgconv.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include <cuda.h>   // CUtensorMap types (the driver entry point is resolved at run time)

#include "gconv.h"

namespace gconv {

// A validated conv2d problem (all derived sizes filled in by the host dispatcher).
struct Conv2d {
  int N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups;
  int Ho, Wo, cpg_in, cpg_out;
  int layout;  // GCONV_NCHW / GCONV_NHWC
  int dtype;   // GCONV_F32 / GCONV_F16 / GCONV_BF16
  int out_mode = GCONV_OUT_GROUP_MAJOR;   // gconv_out_mode of the output
};

// Channels of y: C_out, or C_out / groups when the groups are merged.
__host__ __device__ __forceinline__ int out_channels(const Conv2d& p) {
  return (p.out_mode == GCONV_OUT_MERGE_AVG || p.out_mode == GCONV_OUT_MERGE_MAX) ? p.cpg_out
                                                                                  : p.C_out;
}

// A validated depthwise conv1d problem on (batch, steps, channels).
struct Conv1d {
  int B, T, C, K, pad_left, pad_right, T_out;
  int dtype;
};

// ------------------------------------------------------------------ element conversions
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float v) { return v; }
  static __device__ __forceinline__ float from_f32(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float v) { return __float2bfloat16_rn(v); }
};
template <> struct Elem<__half> {
  static __device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }
  static __device__ __forceinline__ __half from_f32(float v) { return __float2half_rn(v); }
};

// Two packed 16-bit values (low half = lower address) -> float2.
template <typename T> __device__ __forceinline__ float2 unpack2(uint32_t u);
template <> __device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t u) {
  // bf16 is the upper half of an fp32 bit pattern
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
template <> __device__ __forceinline__ float2 unpack2<__half>(uint32_t u) {
  __half2 h = *reinterpret_cast<__half2*>(&u);
  return __half22float2(h);
}

// float2 -> two packed 16-bit values, each rounded to nearest even.
template <typename T> __device__ __forceinline__ uint32_t pack2(float2 v);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float2 v) {
  __nv_bfloat162 h = __float22bfloat162_rn(v);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float2 v) {
  __half2 h = __float22half2_rn(v);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  return __ffma2_rn(a, b, c);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Raise a kernel's dynamic shared-memory limit once per device (bit i of `mask` = device i).
inline cudaError_t set_max_dynamic_smem(const void* func, size_t bytes,
                                        std::atomic<unsigned int>& mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned int bit = 1u << (dev & 31);
  if (mask.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  // ask for the largest shared-memory carveout, so that occupancy is not cut by an L1/shared
  // split sized for a single block
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) mask.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ------------------------------------------------------------------ launchers
// Each returns cudaSuccess or the launch error. Host-side checks have been done.

cudaError_t launch_direct_generic(const Conv2d& p, const void* x, const void* w, const void* bias,
                                  void* y, cudaStream_t s);

bool depthwise_nhwc_supported(const Conv2d& p);
cudaError_t launch_depthwise_nhwc(const Conv2d& p, const void* x, const void* w,
                                  const void* bias, void* y, cudaStream_t s);
// The stride-1 3x3 depthwise kernel reading each filter rotated by 180 degrees: the data
// gradient of a stride-1 depthwise layer as a forward pass over dy, with no flipped copy of
// the filter.
bool depthwise_nhwc_flipped_supported(const Conv2d& p);
cudaError_t launch_depthwise_nhwc_flipped(const Conv2d& p, const void* x, const void* w, void* y,
                                          cudaStream_t s);

// Narrow groups (2 / 4 / 8 channels per group), 3x3, NHWC, 16-bit, C % 8 == 0, aligned x, y.
bool grouped_nhwc_supported(const Conv2d& p);
cudaError_t launch_grouped_nhwc(const Conv2d& p, const void* x, const void* w,
                                const void* bias, void* y, cudaStream_t s);

bool igemm_supported(const Conv2d& p);      // shape/dtype eligibility, layout-independent
size_t igemm_nchw_workspace(const Conv2d& p);
cudaError_t launch_igemm_nhwc(const Conv2d& p, const void* x, const void* w, const void* bias,
                              void* y, cudaStream_t s);
cudaError_t launch_igemm_nchw(const Conv2d& p, const void* x, const void* w, const void* bias,
                              void* y, void* workspace, cudaStream_t s);
// Transposed row-strip kernel (igemm_rowt.cu): NHWC x, [C_out][kH][kW][C_in/g] weights,
// 16-bit data; y in p.layout. Supported: outputs >= 128 wide, 64-channel input blocks,
// filters per group a multiple of 128, kW halo <= 8 rows, any output mode but the max merge.
bool igemm_rowt_supported(const Conv2d& p);
cudaError_t launch_igemm_rowt(const Conv2d& p, const void* x, const void* w, const void* bias,
                              void* y, cudaStream_t s);
// y (p's MERGE_MAX shape) = the maximum over groups of g, p's group-major output in p.layout.
cudaError_t launch_merge_max_groups(const Conv2d& p, const void* g, void* y, cudaStream_t s);

// Grouped conv2d backward. dgrad_as_forward: stride 1, square kernel, pad <= dil*(k-1), so the
// data gradient is the forward conv of the exchanged problem with the flipped, transposed
// filter that launch_flip_transpose_weight writes (C_out * C_in/g * kH * kW elements).
bool dgrad_as_forward(const Conv2d& p);
cudaError_t launch_flip_transpose_weight(const Conv2d& p, const void* w, void* wt,
                                         cudaStream_t s);
cudaError_t launch_dgrad_generic(const Conv2d& p, const void* dy, const void* w, void* dx,
                                 cudaStream_t s);
// Depthwise NHWC data gradient (16-bit, dilation 1, 3x3 / 5x5 / 7x7, stride 1 or 2); dy and dx
// aligned to dgrad_depthwise_vec_bytes.
bool dgrad_depthwise_supported(const Conv2d& p);
int dgrad_depthwise_vec_bytes(const Conv2d& p);
cudaError_t launch_dgrad_depthwise(const Conv2d& p, const void* dy, const void* w, void* dx,
                                   cudaStream_t s);
// Depthwise 3x3, stride 2, pad 1 data gradient on a TMA ring (16-bit NHWC, C % 8 == 0; dy and
// dx 16-byte aligned).
bool dgrad_dw3s2_tma_supported(const Conv2d& p);
cudaError_t launch_dgrad_dw3s2_tma(const Conv2d& p, const void* dy, const void* w, void* dx,
                                   cudaStream_t s);
bool wgrad_depthwise_supported(const Conv2d& p);
// Depthwise 3x3 weight gradient on a TMA ring (16-bit NHWC, dilation 1, stride 1 or 2, pad <= 2,
// C % 8 == 0; x and dy 16-byte aligned).
bool wgrad_dw3_tma_supported(const Conv2d& p);
// Wide-group NHWC weight gradient (16-bit, C_in/g and C_out/g >= 32 and multiples of 8; x and
// dy 16-byte aligned).
bool wgrad_tiled_supported(const Conv2d& p);
// Wide-group weight gradient on the tensor cores (16-bit, stride 1, C_out/g % 128 == 0,
// C_in/g % 64 == 0, (kW-1)*dil <= 8, Wo >= 32); NHWC operands, fp32 partials [S][E].
bool wgrad_tc_supported(const Conv2d& p);
int wgrad_tc_slices(const Conv2d& p);
cudaError_t launch_wgrad_tc(const Conv2d& p, const void* x, const void* dy, float* part,
                            cudaStream_t s);
size_t wgrad_workspace(const Conv2d& p, int kernel);
cudaError_t launch_wgrad(const Conv2d& p, const void* x, const void* dy, void* dw, void* ws,
                         int kernel, cudaStream_t s);

// [N][C][HW] -> [N][HW][C] for 16-bit elements (NCHW -> NHWC staging): 64 x 64 tiles through
// shared memory, 16-byte loads and stores when HW and C are multiples of 8.
cudaError_t launch_nchw_to_nhwc16(const void* x, void* xt, int N, int C, long long HW,
                                  cudaStream_t s);

bool conv1d_vector_supported(const Conv1d& p);
// Kernel (GCONV_KERNEL_CONV1D_*) for a forward / data-gradient call under `path`; x, w, y null
// = a query that assumes aligned pointers. -1 with *why set when the forced family cannot run.
int conv1d_choose_kernel(const Conv1d& p, int path, const void* x, const void* w, const void* y,
                         gconv_status* why);
cudaError_t launch_dwconv1d_fwd(const Conv1d& p, const void* x, const void* w, void* y,
                                bool flip, int pad_left, int T_in, int T_out, int kernel,
                                cudaStream_t s);
// Tensor-core forward / data gradient: 16-bit data, C % 8 == 0, K <= 49, 16-byte aligned x, w, y.
bool conv1d_tc_supported(const Conv1d& p);
cudaError_t launch_dwconv1d_tc(const Conv1d& p, const void* x, const void* w, void* y, bool flip,
                               int pad_left, int T_in, int T_out, cudaStream_t s);
// Conv1d with 128-byte input rows on the CUDA cores (16-bit, C % 64 == 0, K in {3, 5, 7, 9,
// 15, 31}): forward / data gradient, and the weight gradient with its fixed-order partials.
bool conv1d_strip_supported(const Conv1d& p);
cudaError_t launch_dwconv1d_strip(const Conv1d& p, const void* x, const void* w, void* y,
                                  bool flip, int pad_left, int T_in, int T_out, cudaStream_t s);
size_t dwconv1d_wgrad_strip_workspace(const Conv1d& p);
cudaError_t launch_dwconv1d_wgrad_strip(const Conv1d& p, const void* x, const void* dy, void* dw,
                                        void* workspace, cudaStream_t s);
size_t dwconv1d_wgrad_workspace(const Conv1d& p);
cudaError_t launch_dwconv1d_wgrad(const Conv1d& p, const void* x, const void* dy, void* dw,
                                  void* workspace, cudaStream_t s);
size_t dwconv1d_wgrad_noalloc_limit();
cudaError_t launch_dwconv1d_wgrad_noalloc(const Conv1d& p, const void* x, const void* dy,
                                          void* dw, cudaStream_t s);

// Fused depthwise-separable block (dwconv1d then pointwise 1x1): 16-bit, C % 64 == 0,
// C_out % 16 == 0 and <= 512, K in {3, 5, 7, 9, 15, 31}; x, w_pw, z 16-byte aligned.
bool dwsep1d_fused_supported(const Conv1d& p, int C_out);
cudaError_t launch_dwsep1d_fused(const Conv1d& p, int C_out, const void* x, const void* wdw,
                                 const void* wpw, const void* bias, void* z, cudaStream_t s);

// Fused 2-D depthwise-separable block (depthwise KxK, K in {3, 5}, stride 1 or 2, then
// pointwise): 16-bit NHWC, C % 64 == 0, C_out % 16 == 0 and <= 512; `p` is the depthwise
// problem (groups = C_in = C_out); x, w_pw, z 16-byte aligned.
bool dwsep2d_fused_supported(const Conv2d& p, int C_out);
cudaError_t launch_dwsep2d_fused(const Conv2d& p, int C_out, const void* x, const void* wdw,
                                 const void* wpw, const void* bias, void* z, cudaStream_t s);

// cuTensorMapEncodeTiled, resolved through the runtime (null if unavailable).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();
int sm_count();                       // SMs of the current device (cached)

// Test hook (gconv_debug_set_tx_surplus): extra bytes per stage that the generic tensor-core
// tile kernel's producer declares to its barrier; 0 unless a test set it.
unsigned int debug_tx_surplus();

// Launch with programmatic stream serialization: the kernel may start before the previous
// kernel in the stream has finished (its setup overlapping that kernel's tail) and must call
// ptx::pdl_wait() before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned int grid, unsigned int block,
                       size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Device error word (set by kernels whose bounded waits give up).
cudaError_t read_and_clear_device_error(cudaStream_t s, int* code);
unsigned int* device_error_word();

}  // namespace gconv
