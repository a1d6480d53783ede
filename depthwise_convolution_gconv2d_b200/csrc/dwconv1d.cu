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
// Vector kernels (16-bit data, C % 8 == 0, 16-byte aligned x / dy, K in the instantiated set)
// stream their inputs with TMA through shared-memory rings filled by a producer warp (the
// tensor map's zero fill outside [0, T) is the padding), so bytes in flight come from the copy
// engine rather than from thread count:
//  * fwd / dgrad: persistent CTAs walk a contiguous chunk of [112 steps x 64 channels] output
//    tiles; a box of 112 + K - 1 input steps per tile. A thread owns a channel pair and 16
//    consecutive outputs; all K filter taps stay in registers as fp32 pairs (reloaded only when
//    the chunk moves to the next channel tile) and each staged input step is read once from
//    shared memory and applied to every output it touches (packed fp32x2 FMA, loop over the
//    kernel size fully unrolled, one pass over the filter).
//  * wgrad: a block owns 64 channels and a fixed slice of one batch's steps and streams
//    (dy, x) box pairs of 112 steps through its ring; a thread keeps K fp32-pair partial sums
//    for its channel pair over 16-step strips; strips are summed in a fixed order in shared
//    memory and the per-slice partials go to the caller's workspace. A second kernel sums the
//    slices in a fixed order. No float atomics: bitwise reproducible.
// Both run 8-warp CTAs, two per SM, at up to 128 registers a thread.
// Generic kernels cover every other shape, one thread per output (fwd/dgrad) or one warp per
// (c, k) with a fixed-order shuffle reduction (wgrad).
#include <type_traits>

#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

constexpr int TS = 16;            // outputs (steps) per thread
constexpr int STRIPS = 8;         // warps per block, one strip of TS steps each
constexpr int CP = 32;            // channel pairs per block
constexpr int CH = 2 * CP;        // channels per block
constexpr int TB = TS * STRIPS;   // steps per block tile
constexpr int NTHREADS = CP * STRIPS;

// Ring kernels: 1 producer warp + RSTRIPS compute warps = 8 warps, so that two CTAs share an
// SM (the register file is split across the four SM sub-partitions; a ninth warp would put
// three warps of each CTA on one of them)
constexpr int RSTRIPS = 7;
constexpr int RCOMPUTE = 32 * RSTRIPS;
constexpr int RING_THREADS = 32 + RCOMPUTE;
constexpr int TBF = TS * RSTRIPS;               // forward: steps per tile
constexpr int MAX_STAGES = 6;

struct Ring1d {
  int B, T_in, C, T_out, pl;
  int n_ct, n_tt, num_tiles, stages;
  unsigned int stage_bytes, tx_bytes;
};

// tile t -> (step tile, batch, channel tile), channel tile slowest
struct Coord1d {
  int tt, b, ct;
  __device__ __forceinline__ void set(const Ring1d& P, long long t) {
    tt = (int)(t % P.n_tt);
    const long long r = t / P.n_tt;
    b = (int)(r % P.B);
    ct = (int)(r / P.B);
  }
  __device__ __forceinline__ void next(const Ring1d& P) {
    if (++tt < P.n_tt) return;
    tt = 0;
    if (++b < P.B) return;
    b = 0;
    ++ct;
  }
};

template <typename T, int K, bool FLIP>
__global__ void __maxnreg__(128)
    dwconv1d_fwd_kernel(const __grid_constant__ CUtensorMap tmx, const T* __restrict__ w,
                        T* __restrict__ y, const Ring1d P, unsigned int* err) {
  using namespace ptx;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 128u);
  unsigned long long* full =
      reinterpret_cast<unsigned long long*>(smem + (size_t)P.stages * P.stage_bytes);
  unsigned long long* empty = full + MAX_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + MAX_STAGES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long t_begin = (long long)P.num_tiles * blockIdx.x / gridDim.x;
  const long long t_end = (long long)P.num_tiles * (blockIdx.x + 1) / gridDim.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], RSTRIPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      Coord1d c;
      c.set(P, t_begin);
      int s = 0;
      unsigned int ph = 0;
      long long issued = 0;
      for (long long t = t_begin; t < t_end; ++t) {
        if (!mbar_try_wait(&empty[s], ph ^ 1u) &&
            !mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, 32u))
          break;
        mbar_arrive_expect_tx(&full[s], P.tx_bytes);
        tma_load_3d(smem + (size_t)s * P.stage_bytes, &tmx, &full[s], c.ct * CH,
                    c.tt * TBF - P.pl, c.b);
        ++issued;
        c.next(P);
        if (++s == P.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      const unsigned long long dl = drain_deadline();
      for (long long q = (issued > P.stages ? issued - P.stages : 0); q < issued; ++q)
        mbar_wait_until(&full[q % P.stages], (unsigned int)((q / P.stages) & 1), dl, err,
                        ERR_DRAIN);
    }
  } else {
    const int cp = lane, strip = warp - 1;
    float2 wk[K];                                   // the pair's taps, fp32, in registers
    Coord1d c;
    c.set(P, t_begin);
    int prev_ct = -1;
    int s = 0;
    unsigned int ph = 0;
    for (long long t = t_begin; t < t_end; ++t) {
      const int ch = c.ct * CH + 2 * cp;
      if (c.ct != prev_ct) {
        prev_ct = c.ct;
#pragma unroll
        for (int k = 0; k < K; ++k) {
          const int kk = FLIP ? K - 1 - k : k;
          wk[k] = ch < P.C ? make_float2(Elem<T>::to_f32(w[(long long)ch * K + kk]),
                                         Elem<T>::to_f32(w[(long long)(ch + 1) * K + kk]))
                           : make_float2(0.f, 0.f);
        }
      }
      bool got = mbar_try_wait(&full[s], ph);
      if (!got) got = mbar_wait(&full[s], ph, abort_flag, err, 32u);
      if (!__all_sync(0xffffffffu, got)) break;
      // staged box: row r (input step tt*TB - pl + r) holds 64 channels = 32 packed pairs;
      // each input step is read and widened once and applied to every output it touches
      const uint32_t* xr =
          reinterpret_cast<const uint32_t*>(smem + (size_t)s * P.stage_bytes) + strip * TS * CP +
          cp;
      float2 acc[TS];
#pragma unroll
      for (int i = 0; i < TS; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < TS + K - 1; ++j) {
        const float2 xv = unpack2<T>(xr[j * CP]);
#pragma unroll
        for (int i = 0; i < TS; ++i) {
          const int k = j - i;
          if (k >= 0 && k < K) acc[i] = ffma2(wk[k], xv, acc[i]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (ch < P.C) {
        const int t0 = c.tt * TBF + strip * TS;
        T* yp = y + ((long long)c.b * P.T_out + t0) * P.C + ch;
#pragma unroll
        for (int i = 0; i < TS; ++i)
          if (t0 + i < P.T_out)
            *reinterpret_cast<uint32_t*>(yp + (long long)i * P.C) = pack2<T>(acc[i]);
      }
      c.next(P);
      if (++s == P.stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
  __syncthreads();
}

constexpr int WTS = 16;            // weight gradient: steps per thread strip
constexpr int WTB = WTS * RSTRIPS; // steps per sub-tile

struct WgradRing {
  int T_in, C, T_out, pl, slice_len, n_tslices, stages;
  unsigned int stage_bytes, dy_bytes, x_bytes;
};

template <typename T, int K>
__global__ void __maxnreg__(128)
    dwconv1d_wgrad_kernel(const __grid_constant__ CUtensorMap tmx,
                          const __grid_constant__ CUtensorMap tmdy, float* __restrict__ partial,
                          const WgradRing P, unsigned int* err) {
  using namespace ptx;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 128u);
  unsigned long long* full =
      reinterpret_cast<unsigned long long*>(smem + (size_t)P.stages * P.stage_bytes);
  unsigned long long* empty = full + MAX_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + MAX_STAGES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ct = blockIdx.x;
  const int slice = blockIdx.y, b = slice / P.n_tslices, ts = slice % P.n_tslices;
  const int t_begin = ts * P.slice_len;
  const int t_end = min(P.T_out, t_begin + P.slice_len);
  const int n_sub = (t_end - t_begin + WTB - 1) / WTB;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], RSTRIPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmdy);
  }
  __syncthreads();
  float2 acc[K];
#pragma unroll
  for (int k = 0; k < K; ++k) acc[k] = make_float2(0.f, 0.f);
  if (warp == 0) {
    if (lane == 0) {
      // the last sub-tile may reach into the next slice: those dy steps are masked to zero by
      // the compute warps; past T_out the boxes read the tensor map's zero fill
      int s = 0;
      unsigned int ph = 0;
      long long issued = 0;
      for (int i = 0; i < n_sub; ++i) {
        if (!mbar_try_wait(&empty[s], ph ^ 1u) &&
            !mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, 64u))
          break;
        const int tb = t_begin + i * WTB;
        unsigned char* st = smem + (size_t)s * P.stage_bytes;
        mbar_arrive_expect_tx(&full[s], P.dy_bytes + P.x_bytes);
        tma_load_3d(st, &tmdy, &full[s], ct * CH, tb, b);
        tma_load_3d(st + P.dy_bytes, &tmx, &full[s], ct * CH, tb - P.pl, b);
        ++issued;
        if (++s == P.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      const unsigned long long dl = drain_deadline();
      for (long long q = (issued > P.stages ? issued - P.stages : 0); q < issued; ++q)
        mbar_wait_until(&full[q % P.stages], (unsigned int)((q / P.stages) & 1), dl, err,
                        ERR_DRAIN);
    }
  } else {
    const int cp = lane, strip = warp - 1;
    int s = 0;
    unsigned int ph = 0;
    for (int i = 0; i < n_sub; ++i) {
      bool got = mbar_try_wait(&full[s], ph);
      if (!got) got = mbar_wait(&full[s], ph, abort_flag, err, 64u);
      if (!__all_sync(0xffffffffu, got)) break;
      const uint32_t* dyr = reinterpret_cast<const uint32_t*>(smem + (size_t)s * P.stage_bytes) +
                            strip * WTS * CP + cp;
      const uint32_t* xr =
          reinterpret_cast<const uint32_t*>(smem + (size_t)s * P.stage_bytes + P.dy_bytes) +
          strip * WTS * CP + cp;
      const int tq0 = t_begin + i * WTB + strip * WTS;   // step of dv[0]
      float2 dv[WTS];
#pragma unroll
      for (int q = 0; q < WTS; ++q)
        dv[q] = tq0 + q < t_end ? unpack2<T>(dyr[q * CP]) : make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < WTS + K - 1; ++j) {
        const float2 xv = unpack2<T>(xr[j * CP]);
#pragma unroll
        for (int q = 0; q < WTS; ++q) {
          const int k = j - q;
          if (k >= 0 && k < K) acc[k] = ffma2(dv[q], xv, acc[k]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == P.stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
  __syncthreads();   // ring drained: reuse it for the fixed-order sum over strips
  float2* red = reinterpret_cast<float2*>(smem);     // [RSTRIPS][K][CP]
  if (warp > 0) {
#pragma unroll
    for (int k = 0; k < K; ++k) red[((warp - 1) * K + k) * CP + lane] = acc[k];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < K * CP; i += blockDim.x) {
    const int k = i / CP, pp = i % CP;
    float2 sum = red[k * CP + pp];
    for (int st = 1; st < RSTRIPS; ++st) {
      const float2 v = red[(st * K + k) * CP + pp];
      sum.x += v.x;
      sum.y += v.y;
    }
    const int c = ct * CH + 2 * pp;
    if (c < P.C) {
      float* dst = partial + ((long long)slice * P.C + c) * K + k;
      dst[0] = sum.x;
      dst[K] = sum.y;
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

bool make_tensor_map_btc(CUtensorMap* m, int dtype, const void* base, int C, int T_len, int B,
                         int rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const CUtensorMapDataType dt =
      dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T_len, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)C * 2, (cuuint64_t)T_len * C * 2};
  const cuuint32_t box[3] = {CH, (cuuint32_t)rows, 1};
  const cuuint32_t ones[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, ones,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int K, bool FLIP>
cudaError_t fwd_vec(const Conv1d& p, const T* x, const T* w, T* y, int B, int T_in, int C,
                    int T_out, int pl, cudaStream_t s) {
  Ring1d P;
  P.B = B; P.T_in = T_in; P.C = C; P.T_out = T_out; P.pl = pl;
  P.n_ct = (C + CH - 1) / CH;
  P.n_tt = (T_out + TBF - 1) / TBF;
  const long long tiles = (long long)P.n_ct * B * P.n_tt;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  P.num_tiles = (int)tiles;
  P.tx_bytes = (unsigned int)(TBF + K - 1) * CH * 2;
  P.stage_bytes = (P.tx_bytes + 127u) & ~127u;
  P.stages = 4;
  const size_t smem = 128 + (size_t)P.stages * P.stage_bytes + 2 * MAX_STAGES * 8 + 16;
  CUtensorMap tm;
  if (!make_tensor_map_btc(&tm, p.dtype, x, C, T_in, B, TBF + K - 1)) return cudaErrorInvalidValue;
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)dwconv1d_fwd_kernel<T, K, FLIP>, smem,
                                       configured);
  if (e != cudaSuccess) return e;
  int fit = 2;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, dwconv1d_fwd_kernel<T, K, FLIP>,
                                                    RING_THREADS, smem) != cudaSuccess ||
      fit < 1)
    fit = 1;
  long long grid = (long long)sm_count() * fit;
  if (grid > P.num_tiles) grid = P.num_tiles;
  dwconv1d_fwd_kernel<T, K, FLIP><<<(unsigned)grid, RING_THREADS, smem, s>>>(tm, w, y, P,
                                                                           device_error_word());
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
      case 3: return fwd_vec<T, 3, FLIP>(p, xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 5: return fwd_vec<T, 5, FLIP>(p, xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 7: return fwd_vec<T, 7, FLIP>(p, xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 9: return fwd_vec<T, 9, FLIP>(p, xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 15: return fwd_vec<T, 15, FLIP>(p, xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
      case 31: return fwd_vec<T, 31, FLIP>(p, xx, ww, yy, p.B, T_in, p.C, T_out, pl, s);
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
  WgradRing P;
  P.T_in = p.T; P.C = p.C; P.T_out = p.T_out; P.pl = p.pad_left;
  P.slice_len = slice_len; P.n_tslices = n_tslices;
  P.dy_bytes = (unsigned int)WTB * CH * 2;
  P.x_bytes = (unsigned int)(WTB + K - 1) * CH * 2;
  P.stage_bytes = (P.dy_bytes + P.x_bytes + 127u) & ~127u;
  // as deep a ring as lets two CTAs share an SM (<= 110 KB each), 2 to 4 stages
  P.stages = (int)((110u * 1024u) / P.stage_bytes);
  if (P.stages > 4) P.stages = 4;
  if (P.stages < 2) P.stages = 2;
  const size_t red = (size_t)RSTRIPS * K * CP * sizeof(float2);
  size_t ring = (size_t)P.stages * P.stage_bytes;
  if (ring < red) ring = red;
  const size_t smem = 128 + ring + 2 * MAX_STAGES * 8 + 16;
  CUtensorMap tx, tdy;
  if (!make_tensor_map_btc(&tx, p.dtype, x, p.C, p.T, p.B, WTB + K - 1) ||
      !make_tensor_map_btc(&tdy, p.dtype, dy, p.C, p.T_out, p.B, WTB))
    return cudaErrorInvalidValue;
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)dwconv1d_wgrad_kernel<T, K>, smem, configured);
  if (e != cudaSuccess) return e;
  const int n_slices = p.B * n_tslices;
  dim3 grid((p.C + CH - 1) / CH, n_slices);
  dwconv1d_wgrad_kernel<T, K><<<grid, RING_THREADS, smem, s>>>(tx, tdy, partial, P,
                                                               device_error_word());
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

int conv1d_choose_kernel(const Conv1d& p, int path, const void* x, const void* w, const void* y,
                         gconv_status* why) {
  *why = GCONV_OK;
  const bool query = (x == nullptr && w == nullptr && y == nullptr);
  const bool ring_ok = conv1d_vector_supported(p);
  const bool ring_al = query || (aligned16(x) && aligned16(y));
  const bool tc_ok = conv1d_tc_supported(p);
  const bool tc_al = query || (aligned16(x) && aligned16(y) && aligned16(w));
  const bool strip_ok = conv1d_strip_supported(p) && (query || (aligned16(x) && aligned16(y)));
  switch (path) {
    case GCONV_PATH_GENERIC:
      return GCONV_KERNEL_CONV1D_GENERIC;
    case GCONV_PATH_DIRECT:
      if (strip_ok) return GCONV_KERNEL_CONV1D_STRIP;
      return (ring_ok && ring_al) ? GCONV_KERNEL_CONV1D_RING : GCONV_KERNEL_CONV1D_GENERIC;
    case GCONV_PATH_IGEMM:
      if (!tc_ok) { *why = GCONV_ERR_UNSUPPORTED; return -1; }
      if (!tc_al) { *why = GCONV_ERR_MISALIGNED; return -1; }
      return GCONV_KERNEL_CONV1D_TC;
    case GCONV_PATH_AUTO:
      // the tensor-core kernel (Conformer layer: 22.5 us against 26.6 us for the 128-byte-row
      // CUDA-core kernel and 30.6 us for the ring kernel), else the 128-byte-row kernel, the
      // 16-byte-vector ring kernel, the generic kernel
      if (tc_ok && tc_al) return GCONV_KERNEL_CONV1D_TC;
      if (strip_ok) return GCONV_KERNEL_CONV1D_STRIP;
      if (ring_ok && ring_al) return GCONV_KERNEL_CONV1D_RING;
      return GCONV_KERNEL_CONV1D_GENERIC;
    default:
      *why = GCONV_ERR_INVALID_ARG;
      return -1;
  }
}

cudaError_t launch_dwconv1d_fwd(const Conv1d& p, const void* x, const void* w, void* y, bool flip,
                                int pad_left, int T_in, int T_out, int kernel, cudaStream_t s) {
  if (p.B == 0) return cudaSuccess;
  if (kernel == GCONV_KERNEL_CONV1D_TC)
    return launch_dwconv1d_tc(p, x, w, y, flip, pad_left, T_in, T_out, s);
  if (kernel == GCONV_KERNEL_CONV1D_STRIP)
    return launch_dwconv1d_strip(p, x, w, y, flip, pad_left, T_in, T_out, s);
  const bool vec = kernel == GCONV_KERNEL_CONV1D_RING;
  switch (p.dtype) {
    case GCONV_F32: return fwd_any_dtype<float>(p, x, w, y, flip, pad_left, T_in, T_out, false, s);
    case GCONV_F16: return fwd_any_dtype<__half>(p, x, w, y, flip, pad_left, T_in, T_out, vec, s);
    default: return fwd_any_dtype<__nv_bfloat16>(p, x, w, y, flip, pad_left, T_in, T_out, vec, s);
  }
}

// The 128-byte-row weight gradient where it applies (its partials: one fp32 value per
// channel, tap and run of tiles), else the ring kernel's slices.
bool wgrad_strip_ok(const Conv1d& p) { return conv1d_strip_supported(p); }

size_t dwconv1d_wgrad_workspace(const Conv1d& p) {
  if (p.B == 0) return 0;
  // the strip kernel's size, or the ring kernel's, whichever the call's pointers select: the
  // larger of the two when both apply
  const size_t strip = wgrad_strip_ok(p) ? dwconv1d_wgrad_strip_workspace(p) : 0;
  if (!conv1d_vector_supported(p)) return strip;
  int slice_len, n_tslices;
  wgrad_slicing(p, &slice_len, &n_tslices);
  const size_t ring = (size_t)p.B * n_tslices * p.C * p.K * sizeof(float);
  return ring > strip ? ring : strip;
}

cudaError_t launch_dwconv1d_wgrad(const Conv1d& p, const void* x, const void* dy, void* dw,
                                  void* workspace, cudaStream_t s) {
  if (p.B > 0 && wgrad_strip_ok(p) && aligned16(x) && aligned16(dy) && workspace != nullptr)
    return launch_dwconv1d_wgrad_strip(p, x, dy, dw, workspace, s);
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
