// Depthwise conv1d on (batch, steps, channels): forward, data gradient, weight gradient.
//
// The layer is the Conformer convolution module's depthwise convolution (groups = channels)
// as laid out in "Investigate custom Triton kernels for depthwise-separable convolutions in
// Conformer" (speechbrain #2733: (batch, steps, channels), the Oct 27 comment), including the
// backward pass of the Oct 30 comment:
//   fwd    y[b,t,c]  = sum_k w[c,k] * x[b, t+k-pl, c]
//   dgrad  dx[b,s,c] = sum_k w[c,k] * dy[b, s-k+pl, c]
//                    = the forward with the filter reversed and pads (K-1-pl, K-1-pr)
//   wgrad  dw[c,k]   = sum_{b,t} dy[b,t,c] * x[b, t+k-pl, c]
//
// Vector kernels (16-bit data, C % 8 == 0, 16-byte aligned x / dy, K in the instantiated set):
//  * fwd / dgrad: a block stages a [128 + K - 1 steps] x [64 channels] input tile in shared
//    memory as fp32 pairs (16-byte global loads, zero fill outside [0, T)). A thread owns a
//    channel pair and 16 consecutive outputs; its K filter taps stay in registers and each
//    staged input step is read once and applied to every output it touches (packed fp32x2
//    FMA). The loop over the kernel size is fully unrolled.
//  * wgrad: a block owns 64 channels and a fixed slice of one batch's steps; a thread keeps K
//    fp32-pair partial sums for its channel pair over 16-step strips; strips are summed in a
//    fixed order in shared memory and the per-slice partials go to the caller's workspace. A
//    second kernel sums the slices in a fixed order. No float atomics: bitwise reproducible.
// Generic kernels cover every other shape, one thread per output (fwd/dgrad) or one warp per
// (c, k) with a fixed-order shuffle reduction (wgrad).
#include <type_traits>

#include "internal.cuh"

namespace gconv {
namespace {

constexpr int TS = 16;            // outputs (steps) per thread
constexpr int STRIPS = 8;         // warps per block, one strip of TS steps each
constexpr int CP = 32;            // channel pairs per block
constexpr int CH = 2 * CP;        // channels per block
constexpr int TB = TS * STRIPS;   // steps per block tile
constexpr int NTHREADS = CP * STRIPS;

// Stage steps [s0, s0 + rows) x channels [c0, c0 + 64) of a [.., T, C] tensor as fp32 pairs
// dst[r * CP + pair]; zero outside [0, T) and beyond C.
template <typename T>
__device__ __forceinline__ void stage_rows(float2* dst, const T* src, int T_len, int C, int s0,
                                           int rows, int c0) {
  for (int i = threadIdx.x; i < rows * 8; i += NTHREADS) {
    const int r = i >> 3, q = i & 7;
    const int s = s0 + r, c = c0 + q * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (s >= 0 && s < T_len && c < C) v = __ldg(reinterpret_cast<const uint4*>(src + (long long)s * C + c));
    float2* d = dst + r * CP + q * 4;
    d[0] = unpack2<T>(v.x);
    d[1] = unpack2<T>(v.y);
    d[2] = unpack2<T>(v.z);
    d[3] = unpack2<T>(v.w);
  }
}

template <typename T, int K, bool FLIP>
__global__ void __launch_bounds__(NTHREADS, 2) dwconv1d_fwd_kernel(const T* __restrict__ x,
                                                                    const T* __restrict__ w,
                                                                    T* __restrict__ y, int T_in,
                                                                    int C, int T_out, int pl) {
  extern __shared__ float2 smem[];
  constexpr int ROWS = TB + K - 1;
  float2* xs = smem;               // [ROWS][CP]
  float* wsm = reinterpret_cast<float*>(smem + ROWS * CP);   // [K][CH]
  const int tid = threadIdx.x, cp = tid % CP, strip = tid / CP;
  const int c0 = blockIdx.x * CH, t0 = blockIdx.y * TB, b = blockIdx.z;

  for (int i = tid; i < CH * K; i += NTHREADS) {
    const int cc = i / K, k = i % K;
    const float v = (c0 + cc < C) ? Elem<T>::to_f32(w[(long long)(c0 + cc) * K + k]) : 0.0f;
    wsm[(FLIP ? K - 1 - k : k) * CH + cc] = v;
  }
  stage_rows<T>(xs, x + (long long)b * T_in * C, T_in, C, t0 - pl, ROWS, c0);
  __syncthreads();

  float2 wk[K];
#pragma unroll
  for (int k = 0; k < K; ++k) wk[k] = reinterpret_cast<const float2*>(wsm + k * CH)[cp];
  float2 acc[TS];
#pragma unroll
  for (int i = 0; i < TS; ++i) acc[i] = make_float2(0.f, 0.f);
  const float2* xr = xs + strip * TS * CP + cp;
#pragma unroll
  for (int j = 0; j < TS + K - 1; ++j) {
    const float2 xv = xr[j * CP];
#pragma unroll
    for (int i = 0; i < TS; ++i) {
      const int k = j - i;
      if (k >= 0 && k < K) acc[i] = ffma2(wk[k], xv, acc[i]);
    }
  }
  const int c = c0 + 2 * cp;
  if (c < C) {
    T* yp = y + ((long long)b * T_out + t0 + strip * TS) * C + c;
#pragma unroll
    for (int i = 0; i < TS; ++i)
      if (t0 + strip * TS + i < T_out)
        *reinterpret_cast<uint32_t*>(yp + (long long)i * C) = pack2<T>(acc[i]);
  }
}

template <typename T, int K>
__global__ void __launch_bounds__(NTHREADS, 2) dwconv1d_wgrad_kernel(
    const T* __restrict__ x, const T* __restrict__ dy, float* __restrict__ partial, int T_in,
    int C, int T_out, int pl, int slice_len, int n_tslices) {
  extern __shared__ float2 smem[];
  float2* dys = smem;              // [TB][CP]
  float2* xs = smem + TB * CP;     // [TB + K - 1][CP]
  const int tid = threadIdx.x, cp = tid % CP, strip = tid / CP;
  const int c0 = blockIdx.x * CH;
  const int slice = blockIdx.y, b = slice / n_tslices, ts = slice % n_tslices;
  const int t_begin = ts * slice_len;
  const int t_end = min(T_out, t_begin + slice_len);
  const T* xb = x + (long long)b * T_in * C;
  const T* dyb = dy + (long long)b * T_out * C;

  float2 acc[K];
#pragma unroll
  for (int k = 0; k < K; ++k) acc[k] = make_float2(0.f, 0.f);

  for (int tb = t_begin; tb < t_end; tb += TB) {
    stage_rows<T>(dys, dyb, t_end, C, tb, TB, c0);          // zero at and beyond t_end
    stage_rows<T>(xs, xb, T_in, C, tb - pl, TB + K - 1, c0);
    __syncthreads();
    float2 dv[TS];
#pragma unroll
    for (int i = 0; i < TS; ++i) dv[i] = dys[(strip * TS + i) * CP + cp];
    const float2* xr = xs + strip * TS * CP + cp;
#pragma unroll
    for (int j = 0; j < TS + K - 1; ++j) {
      const float2 xv = xr[j * CP];
#pragma unroll
      for (int i = 0; i < TS; ++i) {
        const int k = j - i;
        if (k >= 0 && k < K) acc[k] = ffma2(dv[i], xv, acc[k]);
      }
    }
    __syncthreads();
  }
  // fixed-order sum over the block's strips
  float2* red = smem;              // [STRIPS][K][CP], fits in the staging area
#pragma unroll
  for (int k = 0; k < K; ++k) red[(strip * K + k) * CP + cp] = acc[k];
  __syncthreads();
  for (int i = tid; i < K * CP; i += NTHREADS) {
    const int k = i / CP, pp = i % CP;
    float2 s = red[k * CP + pp];
    for (int st = 1; st < STRIPS; ++st) {
      const float2 v = red[(st * K + k) * CP + pp];
      s.x += v.x;
      s.y += v.y;
    }
    const int c = c0 + 2 * pp;
    if (c < C) {
      float* dst = partial + ((long long)slice * C + c) * K + k;
      dst[0] = s.x;
      dst[K] = s.y;
    }
  }
}

template <typename T>
__global__ void wgrad_finalize_kernel(const float* __restrict__ partial, T* __restrict__ dw,
                                      int n_slices, int CK) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= CK) return;
  float s = 0.f;
  for (int q = 0; q < n_slices; ++q) s += partial[(long long)q * CK + i];
  dw[i] = Elem<T>::from_f32(s);
}

// ---------------------------------------------------------------- generic kernels

template <typename T, bool FLIP>
__global__ void dwconv1d_fwd_generic(const T* __restrict__ x, const T* __restrict__ w,
                                     T* __restrict__ y, int B, int T_in, int C, int K, int T_out,
                                     int pl) {
  const long long total = (long long)B * T_out * C;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(i % C);
    const long long bt = i / C;
    const int t = (int)(bt % T_out), b = (int)(bt / T_out);
    float acc = 0.f;
    for (int k = 0; k < K; ++k) {
      const int s = t + k - pl;
      if (s < 0 || s >= T_in) continue;
      const float wv = Elem<T>::to_f32(w[(long long)c * K + (FLIP ? K - 1 - k : k)]);
      acc = fmaf(wv, Elem<T>::to_f32(x[((long long)b * T_in + s) * C + c]), acc);
    }
    y[i] = Elem<T>::from_f32(acc);
  }
}

template <typename T>
__global__ void dwconv1d_wgrad_generic(const T* __restrict__ x, const T* __restrict__ dy,
                                       T* __restrict__ dw, int B, int T_in, int C, int K,
                                       int T_out, int pl) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= C * K) return;
  const int c = warp / K, k = warp % K;
  float s = 0.f;
  const long long n = (long long)B * T_out;
  for (long long i = lane; i < n; i += 32) {
    const int t = (int)(i % T_out), b = (int)(i / T_out);
    const int src = t + k - pl;
    if (src < 0 || src >= T_in) continue;
    s = fmaf(Elem<T>::to_f32(dy[i * C + c]), Elem<T>::to_f32(x[((long long)b * T_in + src) * C + c]), s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) dw[(long long)c * K + k] = Elem<T>::from_f32(s);
}

// ---------------------------------------------------------------- host side

bool k_instantiated(int K) {
  return K == 3 || K == 5 || K == 7 || K == 9 || K == 15 || K == 31;
}

template <typename T, int K, bool FLIP>
cudaError_t fwd_vec(const T* x, const T* w, T* y, int B, int T_in, int C, int T_out, int pl,
                    cudaStream_t s) {
  const size_t smem = (size_t)(TB + K - 1) * CP * sizeof(float2) + (size_t)K * CH * sizeof(float);
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)dwconv1d_fwd_kernel<T, K, FLIP>, smem,
                                       configured);
  if (e != cudaSuccess) return e;
  dim3 grid((C + CH - 1) / CH, (T_out + TB - 1) / TB, B);
  dwconv1d_fwd_kernel<T, K, FLIP><<<grid, NTHREADS, smem, s>>>(x, w, y, T_in, C, T_out, pl);
  return cudaGetLastError();
}

template <typename T, bool FLIP>
cudaError_t fwd_dispatch(const Conv1d& p, const void* x, const void* w, void* y, int pl,
                         int T_in, int T_out, bool vec, cudaStream_t s) {
  const T* xx = (const T*)x;
  const T* ww = (const T*)w;
  T* yy = (T*)y;
  if constexpr (!std::is_same<T, float>::value) {
    if (vec) switch (p.K) {
      case 3: return fwd_vec<T, 3, FLIP>(xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 5: return fwd_vec<T, 5, FLIP>(xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 7: return fwd_vec<T, 7, FLIP>(xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 9: return fwd_vec<T, 9, FLIP>(xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 15: return fwd_vec<T, 15, FLIP>(xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 31: return fwd_vec<T, 31, FLIP>(xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      default: break;
    }
  }
  const long long total = (long long)p.B * T_out * p.C;
  long long blocks = (total + 255) / 256;
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  if (blocks < 1) blocks = 1;
  dwconv1d_fwd_generic<T, FLIP><<<(unsigned)blocks, 256, 0, s>>>(xx, ww, yy, p.B, T_in, p.C, p.K,
                                                                  T_out, pl);
  return cudaGetLastError();
}

template <typename T>
cudaError_t fwd_any_dtype(const Conv1d& p, const void* x, const void* w, void* y, bool flip,
                          int pl, int T_in, int T_out, bool vec, cudaStream_t s) {
  return flip ? fwd_dispatch<T, true>(p, x, w, y, pl, T_in, T_out, vec, s)
              : fwd_dispatch<T, false>(p, x, w, y, pl, T_in, T_out, vec, s);
}

// Slicing of B*T_out for the weight gradient: n_tslices slices per batch of slice_len steps
// (a multiple of the block tile), enough blocks to fill the GPU about twice.
void wgrad_slicing(const Conv1d& p, int* slice_len, int* n_tslices) {
  const int n_ctiles = (p.C + CH - 1) / CH;
  const int tiles_per_batch = (p.T_out + TB - 1) / TB;
  int want = (2 * 148 + n_ctiles * p.B - 1) / (n_ctiles * p.B);
  if (want < 1) want = 1;
  if (want > tiles_per_batch) want = tiles_per_batch;
  const int tiles_per_slice = (tiles_per_batch + want - 1) / want;
  *slice_len = tiles_per_slice * TB;
  *n_tslices = (p.T_out + *slice_len - 1) / *slice_len;
}

template <typename T, int K>
cudaError_t wgrad_vec(const Conv1d& p, const T* x, const T* dy, T* dw, float* partial,
                      cudaStream_t s) {
  int slice_len, n_tslices;
  wgrad_slicing(p, &slice_len, &n_tslices);
  const size_t stage = (size_t)(2 * TB + K - 1) * CP * sizeof(float2);
  const size_t red = (size_t)STRIPS * K * CP * sizeof(float2);
  const size_t smem = stage > red ? stage : red;
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)dwconv1d_wgrad_kernel<T, K>, smem, configured);
  if (e != cudaSuccess) return e;
  const int n_slices = p.B * n_tslices;
  dim3 grid((p.C + CH - 1) / CH, n_slices);
  dwconv1d_wgrad_kernel<T, K><<<grid, NTHREADS, smem, s>>>(x, dy, partial, p.T, p.C, p.T_out,
                                                            p.pad_left, slice_len, n_tslices);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int CK = p.C * p.K;
  wgrad_finalize_kernel<T><<<(CK + 255) / 256, 256, 0, s>>>(partial, dw, n_slices, CK);
  return cudaGetLastError();
}

template <typename T>
cudaError_t wgrad_any(const Conv1d& p, const void* x, const void* dy, void* dw, void* ws,
                      bool vec, cudaStream_t s) {
  const T* xx = (const T*)x;
  const T* dd = (const T*)dy;
  T* out = (T*)dw;
  float* partial = (float*)ws;
  if constexpr (!std::is_same<T, float>::value) {
    if (vec) switch (p.K) {
      case 3: return wgrad_vec<T, 3>(p, xx, dd, out, partial, s);
      case 5: return wgrad_vec<T, 5>(p, xx, dd, out, partial, s);
      case 7: return wgrad_vec<T, 7>(p, xx, dd, out, partial, s);
      case 9: return wgrad_vec<T, 9>(p, xx, dd, out, partial, s);
      case 15: return wgrad_vec<T, 15>(p, xx, dd, out, partial, s);
      case 31: return wgrad_vec<T, 31>(p, xx, dd, out, partial, s);
      default: break;
    }
  }
  const long long warps = (long long)p.C * p.K;
  dwconv1d_wgrad_generic<T><<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(
      xx, dd, out, p.B, p.T, p.C, p.K, p.T_out, p.pad_left);
  return cudaGetLastError();
}

}  // namespace

// Vector kernels: 16-bit data, channels a multiple of 8 (16-byte channel vectors) and a
// filter length with an unrolled instantiation.
bool conv1d_vector_supported(const Conv1d& p) {
  const int t_max = p.T > p.T_out ? p.T : p.T_out;
  return p.dtype != GCONV_F32 && p.C % 8 == 0 && k_instantiated(p.K) && p.B <= 65535 &&
         (t_max + TB - 1) / TB <= 65535;   // grid.z = B, grid.y = step tiles
}

cudaError_t launch_dwconv1d_fwd(const Conv1d& p, const void* x, const void* w, void* y, bool flip,
                                int pad_left, int T_in, int T_out, cudaStream_t s) {
  const bool vec = conv1d_vector_supported(p) && aligned16(x) && aligned16(y);
  if (p.B == 0) return cudaSuccess;
  switch (p.dtype) {
    case GCONV_F32: return fwd_any_dtype<float>(p, x, w, y, flip, pad_left, T_in, T_out, false, s);
    case GCONV_F16: return fwd_any_dtype<__half>(p, x, w, y, flip, pad_left, T_in, T_out, vec, s);
    default: return fwd_any_dtype<__nv_bfloat16>(p, x, w, y, flip, pad_left, T_in, T_out, vec, s);
  }
}

size_t dwconv1d_wgrad_workspace(const Conv1d& p) {
  if (!conv1d_vector_supported(p) || p.B == 0) return 0;
  int slice_len, n_tslices;
  wgrad_slicing(p, &slice_len, &n_tslices);
  return (size_t)p.B * n_tslices * p.C * p.K * sizeof(float);
}

cudaError_t launch_dwconv1d_wgrad(const Conv1d& p, const void* x, const void* dy, void* dw,
                                  void* workspace, cudaStream_t s) {
  const bool vec = conv1d_vector_supported(p) && aligned16(x) && aligned16(dy) &&
                   workspace != nullptr && p.B > 0;
  switch (p.dtype) {
    case GCONV_F32: return wgrad_any<float>(p, x, dy, dw, workspace, false, s);
    case GCONV_F16: return wgrad_any<__half>(p, x, dy, dw, workspace, vec, s);
    default: return wgrad_any<__nv_bfloat16>(p, x, dy, dw, workspace, vec, s);
  }
}

}  // namespace gconv

// ---------------------------------------------------------------- allocation-free variant
//
// dwconv1d_bwd_weight_noalloc runs the same weight-gradient kernels with their partial-sum
// scratch taken from the fixed device array below instead of a caller workspace, for
// callers that cannot allocate device memory. The array is part of the library image: every
// GPU that loads the library holds it until the process exits. Calls share it, so two such
// calls that overlap on the GPU (different streams, no ordering) race on it. Nothing in it
// needs to start at zero: the partial kernel writes every slot the reduction reads.

namespace gconv {
namespace {

constexpr size_t kNoallocScratchBytes = GCONV_WGRAD_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) float g_wgrad_noalloc_scratch[kNoallocScratchBytes / sizeof(float)];

// Device address of the scratch array for the current device, looked up (with that device
// current) on the first call made on it and cached. The host-side symbol is only a handle.
cudaError_t noalloc_scratch(float** out) {
  static std::atomic<float*> cached[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  float* p = cached[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_wgrad_noalloc_scratch);
    if (e != cudaSuccess) return e;
    p = static_cast<float*>(addr);
    cached[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

size_t dwconv1d_wgrad_noalloc_limit() { return kNoallocScratchBytes; }

cudaError_t launch_dwconv1d_wgrad_noalloc(const Conv1d& p, const void* x, const void* dy,
                                          void* dw, cudaStream_t s) {
  float* scratch = nullptr;
  if (dwconv1d_wgrad_workspace(p) > 0) {
    const cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return e;
  }
  return launch_dwconv1d_wgrad(p, x, dy, dw, scratch, s);
}

}  // namespace gconv
