// Depthwise conv1d on (batch, steps, channels) with 128-byte input rows, on the CUDA cores.
//
// The Conformer convolution module's depthwise layer ("Investigate custom Triton kernels for
// depthwise-separable convolutions in Conformer", speechbrain #2733; the Oct 27 comment fixes
// the (batch, steps, channels) layout, the Oct 30 comment the backward pass):
//   forward          y[b,t,c]  = sum_{k<K} w[c,k] * x[b, t+k-pl, c]
//   data gradient    the same sum with the filter reversed and the left pad K-1-pl, on dy
//   weight gradient  dw[c,k]   = sum_{b,t} dy[b,t,c] * x[b, t+k-pl, c]
//
// A tile is 64 channels (one 128-byte row per step, a whole L2 line) x 112 output steps of one
// batch. A CTA owns one 64-channel block and a fixed run of that block's tiles, so the filter
// taps of a thread's channel pair are loaded once per CTA and stay in registers:
//   * warp 0 (one thread) streams each tile's input rows -- 112 + K - 1 of them, TMA zero fill
//     outside [0, T) -- into a ring of shared-memory stages (and, for the weight gradient, the
//     tile's 112 rows of dy);
//   * warps 1-7 each own 16 consecutive steps of the tile for all 32 channel pairs: a lane's
//     channel pair is one 32-bit word of every row, so a warp reads whole 128-byte rows with
//     no bank conflict, each input word once, and runs 16*K fp32x2 multiply-adds on it;
//   * forward / data gradient: each warp writes its 16 x 64 outputs, rounded once, into its
//     own 2 KB staging slab (128-byte swizzle) and issues one TMA store (clipped at T_out);
//   * weight gradient: the K fp32x2 tap sums of a thread accumulate over all of the CTA's
//     tiles; at the end the 7 warps' sums are added in warp order and the CTA writes one fp32
//     partial per (channel, tap); a second kernel adds the CTAs' partials in a fixed order. The
//     runs of tiles are a function of the shape only, so dw is bitwise reproducible.
// Every mbarrier wait is bounded (1 s); a wait that gives up sets the library's device error
// word, and the CTA drains its copies (bounded too) and exits.
#include <cuda.h>

#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

using namespace ptx;

constexpr int SP_CB = 64;             // channels per tile (128-byte rows)
// 7 compute warps + the producer: two 8-warp CTAs put 4 warps on each SM sub-partition, which
// leaves 128 registers a thread (the K = 31 taps and 16 accumulators are 94 of them)
constexpr int SP_WARPS = 7;           // compute warps; 16 steps each
constexpr int SP_TS = 16 * SP_WARPS;  // output steps per tile
constexpr int SP_THREADS = 32 * (SP_WARPS + 1);
constexpr int SP_STAGES = 3;
// The weight gradient runs 8 compute warps and no producer warp (thread 0 issues the copies):
// a 7 + 1 warp CTA left one SM sub-partition with half the FMA work of the others, and
// 128-step tiles divide T = 2048 with no ragged tile.
constexpr int SPW_WARPS = 8;
constexpr int SPW_TS = 16 * SPW_WARPS;
constexpr int SPW_THREADS = 32 * SPW_WARPS;
constexpr int SP_TARGET_CTAS = 296;   // runs of tiles are sized for about this many CTAs
constexpr unsigned int ERR_SP = 1u << 20;

struct SpParams {
  int B, T_in, T_out, C, pl;          // pl: left zero padding of the input in this pass
  int n_cb, n_tb, tiles_per_cb;       // tiles_per_cb = B * n_tb
  int runs;                           // CTAs per channel block
  unsigned int x_bytes, dy_bytes, stage_bytes;
};

__host__ __device__ inline int sp_tile_steps(bool wgrad) { return wgrad ? SPW_TS : SP_TS; }

__host__ __device__ inline unsigned int sp_stage_bytes(int K, bool wgrad) {
  const int ts = sp_tile_steps(wgrad);
  const unsigned int x = (unsigned int)(ts + K - 1) * 128u;
  const unsigned int d = wgrad ? (unsigned int)ts * 128u : 0u;
  return (x + d + 1023u) & ~1023u;
}

// One tile run: tiles [t_begin, t_end) of channel block cb (tile = b * n_tb + tb).
struct Run {
  int cb, t_begin, t_end;
  __device__ __forceinline__ Run(const SpParams& P) {
    cb = blockIdx.x / P.runs;
    const int r = blockIdx.x - cb * P.runs;
    t_begin = (int)((long long)P.tiles_per_cb * r / P.runs);
    t_end = (int)((long long)P.tiles_per_cb * (r + 1) / P.runs);
  }
};

// Forward / data gradient. FLIP reverses the filter (data gradient).
template <typename T, int K, bool FLIP>
__global__ void __launch_bounds__(SP_THREADS, 2)
    dwconv1d_strip_kernel(const __grid_constant__ CUtensorMap tmx,
                          const __grid_constant__ CUtensorMap tmy, const T* __restrict__ w,
                          const SpParams P, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem(smem_raw, 1024u);
  unsigned char* ring = smem;
  unsigned char* slabs = smem + SP_STAGES * P.stage_bytes;        // 7 warps x 2 x 2 KB
  float2* wsm = reinterpret_cast<float2*>(slabs + SP_WARPS * 4096);  // taps [K][32 pairs]
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(wsm + K * 32);
  unsigned long long* full = bars;
  unsigned long long* empty = full + SP_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + SP_STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Run run(P);
  if (threadIdx.x == 0) {
    for (int s = 0; s < SP_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], SP_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmy);
  }
  __syncthreads();
  if (warp != 0) {
    // the compute warps lay out the block's taps as fp32 pairs [tap][pair] (reversed for the
    // data gradient) while the producer already streams the first tiles; consecutive threads
    // write consecutive channels, so the table is written without bank conflicts (a
    // channel-major walk of w wrote 32 threads into one bank and held every CTA ~3 us before
    // its first load was issued, measured)
    const T* wb = w + (long long)run.cb * SP_CB * K;
    float* wf = reinterpret_cast<float*>(wsm);
    for (int e = threadIdx.x - 32; e < SP_CB * K; e += SP_THREADS - 32) {
      const int k = e / SP_CB, c = e - k * SP_CB;
      const int kk = FLIP ? K - 1 - k : k;
      wf[(kk * 32 + (c >> 1)) * 2 + (c & 1)] = Elem<T>::to_f32(wb[c * K + k]);
    }
    named_sync(1, SP_THREADS - 32);
  }

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      unsigned int ph = 0;
      long long issued = 0;
      for (int t = run.t_begin; t < run.t_end; ++t) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, ERR_SP | 1u)) break;
        const int b = t / P.n_tb, tb = t - b * P.n_tb;
        mbar_arrive_expect_tx(&full[s], P.x_bytes);
        tma_load_3d(ring + (size_t)s * P.stage_bytes, &tmx, &full[s], run.cb * SP_CB,
                    tb * SP_TS - P.pl, b);
        ++issued;
        if (++s == SP_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      const unsigned long long dl = drain_deadline();
      for (long long q = (issued > SP_STAGES ? issued - SP_STAGES : 0); q < issued; ++q)
        mbar_wait_until(&full[q % SP_STAGES], (unsigned int)((q / SP_STAGES) & 1), dl, err,
                        ERR_DRAIN);
    }
  } else {
    const int w2 = warp - 1;
    // the taps of this lane's channel pair, fp32 pairs (reversed for the data gradient)
    float2 wk[K];
#pragma unroll
    for (int k = 0; k < K; ++k) wk[k] = wsm[k * 32 + lane];
    unsigned char* slab0 = slabs + w2 * 4096;
    int s = 0;
    unsigned int ph = 0;
    int nslab = 0;
    for (int t = run.t_begin; t < run.t_end; ++t) {
      bool got = mbar_try_wait(&full[s], ph);
      if (!got) got = mbar_wait(&full[s], ph, abort_flag, err, ERR_SP | 2u);
      if (!__all_sync(0xffffffffu, got)) break;
      const uint32_t* xr =
          reinterpret_cast<const uint32_t*>(ring + (size_t)s * P.stage_bytes) + w2 * 16 * 32 +
          lane;
      float2 acc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 16 + K - 1; ++i) {
        const float2 xv = unpack2<T>(xr[i * 32]);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int k = i - j;
          if (k >= 0 && k < K) acc[j] = ffma2(wk[k], xv, acc[j]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == SP_STAGES) {
        s = 0;
        ph ^= 1u;
      }
      // outputs: 16 rows of 128 bytes, 16-byte chunk q of row r at (q ^ (r & 7))
      unsigned char* slab = slab0 + (nslab & 1) * 2048;
      if (nslab >= 2) {
        if (lane == 0) bulk_wait_read1();
        __syncwarp();
      }
      const int q = lane >> 2;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        *reinterpret_cast<uint32_t*>(slab + j * 128 + ((q ^ (j & 7)) << 4) + ((lane & 3) << 2)) =
            pack2<T>(acc[j]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int b = t / P.n_tb, tb = t - b * P.n_tb;
        tma_store_3d(&tmy, slab, run.cb * SP_CB, tb * SP_TS + w2 * 16, b);
        bulk_commit();
      }
      ++nslab;
    }
    if (lane == 0) bulk_wait_read0();
    __syncwarp();
  }
}

// Weight gradient: fp32 partials part[cb][run][64 channels][K] (channel-major within a block).
template <typename T, int K>
__global__ void __launch_bounds__(SPW_THREADS, 2)
    dwconv1d_wgrad_strip_kernel(const __grid_constant__ CUtensorMap tmx,
                                const __grid_constant__ CUtensorMap tmd,
                                float* __restrict__ part, const SpParams P, unsigned int* err) {
  pdl_launch_dependents();   // the run sum may be scheduled as this grid's CTAs finish
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem(smem_raw, 1024u);
  unsigned char* ring = smem;
  unsigned long long* bars =
      reinterpret_cast<unsigned long long*>(smem + SP_STAGES * P.stage_bytes);
  unsigned long long* full = bars;
  unsigned long long* empty = full + SP_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + SP_STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Run run(P);
  const int n = run.t_end - run.t_begin;
  const bool producer = threadIdx.x == 0;
  if (producer) {
    for (int s = 0; s < SP_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], SPW_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmd);
  }
  __syncthreads();

  // thread 0 fills the ring at the start and refills stage s with tile i + SP_STAGES once
  // every warp has released tile i
  int issued = 0, consumed = 0;
  auto issue = [&](int i) {
    const int s = i % SP_STAGES;
    const int t = run.t_begin + i;
    const int b = t / P.n_tb, tb = t - b * P.n_tb;
    unsigned char* st = ring + (size_t)s * P.stage_bytes;
    mbar_arrive_expect_tx(&full[s], P.x_bytes + P.dy_bytes);
    tma_load_3d(st, &tmx, &full[s], run.cb * SP_CB, tb * SPW_TS - P.pl, b);
    tma_load_3d(st + P.x_bytes, &tmd, &full[s], run.cb * SP_CB, tb * SPW_TS, b);
  };
  if (producer) {
    for (int q = 0; q < SP_STAGES && q < n; ++q) issue(q);
    issued = n < SP_STAGES ? n : SP_STAGES;
  }

  float2 acc[K];
#pragma unroll
  for (int k = 0; k < K; ++k) acc[k] = make_float2(0.0f, 0.0f);
  bool ok = true;
  for (int i = 0; i < n; ++i) {
    const int s = i % SP_STAGES;
    const unsigned int ph = (unsigned int)(i / SP_STAGES) & 1u;
    bool got = mbar_try_wait(&full[s], ph);
    if (!got) got = mbar_wait(&full[s], ph, abort_flag, err, ERR_SP | 8u);
    if (!__all_sync(0xffffffffu, got)) {
      ok = false;
      break;
    }
    if (producer) consumed = i + 1;
    const unsigned char* st = ring + (size_t)s * P.stage_bytes;
    const uint32_t* xr = reinterpret_cast<const uint32_t*>(st) + warp * 16 * 32 + lane;
    const uint32_t* dr = reinterpret_cast<const uint32_t*>(st + P.x_bytes) + warp * 16 * 32 +
                         lane;
    float2 g[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) g[j] = unpack2<T>(dr[j * 32]);
    // dy rows past T_out read as zeros (TMA fill), so they add nothing
#pragma unroll
    for (int r = 0; r < 16 + K - 1; ++r) {
      const float2 xv = unpack2<T>(xr[r * 32]);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int k = r - j;
        if (k >= 0 && k < K) acc[k] = ffma2(g[j], xv, acc[k]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    bool refill_ok = true;
    if (producer && i + SP_STAGES < n) {
      refill_ok = mbar_wait(&empty[s], ph, abort_flag, err, ERR_SP | 4u);
      if (refill_ok) {
        issue(i + SP_STAGES);
        issued = i + SP_STAGES + 1;
      }
    }
    if (!__all_sync(0xffffffffu, refill_ok)) {
      ok = false;
      break;
    }
  }
  if (producer) {
    const unsigned long long dl = drain_deadline();
    for (int q = consumed; q < issued; ++q)
      mbar_wait_until(&full[q % SP_STAGES], (unsigned int)((q / SP_STAGES) & 1), dl, err,
                      ERR_DRAIN);
  }
  // the 8 warps' sums, added in warp order through the (now idle) ring
  ok = __syncthreads_and(ok ? 1 : 0) != 0 && !*abort_flag;
  if (!ok) return;
  float2* red = reinterpret_cast<float2*>(ring);      // [warp][k][lane]
#pragma unroll
  for (int k = 0; k < K; ++k) red[(warp * K + k) * 32 + lane] = acc[k];
  __syncthreads();
  float* out = part + ((long long)blockIdx.x) * SP_CB * K;   // [cb][run] blocks of 64 x K
  for (int e = threadIdx.x; e < 32 * K; e += SPW_THREADS) {
    const int k = e / 32, l = e - k * 32;
    float2 v = red[k * 32 + l];
#pragma unroll
    for (int wv = 1; wv < SPW_WARPS; ++wv) {
      const float2 u = red[(wv * K + k) * 32 + l];
      v.x += u.x;
      v.y += u.y;
    }
    out[(2 * l) * K + k] = v.x;
    out[(2 * l + 1) * K + k] = v.y;
  }
}

// dw[c][k] = sum over runs r of part[cb][r][c - 64 cb][k], rounded once. A CTA takes 32
// consecutive dw entries (one per lane: coalesced loads) and its 8 warps split the runs (warp
// j adds runs j, j+8, ... in that order, starting from 0; runs past the count add 0); the 8
// warp sums are then added in warp order -- a fixed order, so the result is bitwise
// reproducible.
template <typename T>
__global__ void __launch_bounds__(256) dwconv1d_wgrad_strip_sum(const float* __restrict__ part,
                                                                T* __restrict__ dw, int C, int K,
                                                                int runs) {
  pdl_wait();   // the partials of the kernel before (launch_pdl)
  __shared__ float acc8[8][33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  float v = 0.0f;
  if (e < C * K) {
    const int c = e / K, k = e - c * K;
    const int cb = c / SP_CB, cl = c - cb * SP_CB;
    const float* p = part + ((long long)cb * runs * SP_CB + cl) * K + k;
    // the warp's first 8 runs are loaded together, then added in run order (one dependent
    // load after another took ~4 us for the Conformer layer's 37 runs, measured)
    float r8[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int r = warp + 8 * q;
      r8[q] = r < runs ? p[(long long)r * SP_CB * K] : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) v += r8[q];
    for (int r = warp + 64; r < runs; r += 8) v += p[(long long)r * SP_CB * K];
  }
  acc8[warp][lane] = v;
  __syncthreads();
  if (warp == 0 && e < C * K) {
    float t = acc8[0][lane];
#pragma unroll
    for (int j = 1; j < 8; ++j) t += acc8[j][lane];
    dw[e] = Elem<T>::from_f32(t);
  }
}

bool sp_k_supported(int K) {
  return K == 3 || K == 5 || K == 7 || K == 9 || K == 15 || K == 31;
}

// Parameters of a pass over T_in input steps producing T_out output steps (pl: left pad).
bool make_sp_params(const Conv1d& p, int T_in, int T_out, int pl, bool wgrad, SpParams* P) {
  if (p.dtype != GCONV_BF16 && p.dtype != GCONV_F16) return false;
  const int ts = sp_tile_steps(wgrad);
  if (p.C % SP_CB != 0 || !sp_k_supported(p.K) || ts + p.K - 1 > 256) return false;
  P->B = p.B; P->T_in = T_in; P->T_out = T_out; P->C = p.C; P->pl = pl;
  P->n_cb = p.C / SP_CB;
  P->n_tb = (T_out + ts - 1) / ts;
  const long long tpc = (long long)p.B * P->n_tb;
  if (tpc > INT32_MAX || tpc < 1) return false;
  P->tiles_per_cb = (int)tpc;
  long long runs = (SP_TARGET_CTAS + P->n_cb - 1) / P->n_cb;
  if (runs > tpc) runs = tpc;
  if ((long long)P->n_cb * runs > INT32_MAX) return false;
  P->runs = (int)runs;
  P->x_bytes = (unsigned int)(ts + p.K - 1) * 128u;
  P->dy_bytes = wgrad ? (unsigned int)ts * 128u : 0u;
  P->stage_bytes = sp_stage_bytes(p.K, wgrad);
  return true;
}

size_t sp_smem(const SpParams& P, int K, bool wgrad) {
  return 1024 + SP_STAGES * (size_t)P.stage_bytes +
         (wgrad ? 0 : SP_WARPS * 4096 + (size_t)K * 32 * 8) + 64;
}

bool encode_rows(EncodeTiledFn enc, CUtensorMap* m, int dtype, const void* base, int C, int T,
                 int B, int box_rows, bool swizzle) {
  const CUtensorMapDataType dt =
      dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dim[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t str[2] = {(cuuint64_t)C * 2, (cuuint64_t)T * C * 2};
  const cuuint32_t box[3] = {(cuuint32_t)SP_CB, (cuuint32_t)box_rows, 1};
  const cuuint32_t ones[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(base), dim, str, box, ones,
             CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <typename T, int K>
cudaError_t launch_fwd_k(const SpParams& P, const CUtensorMap& tx, const CUtensorMap& ty,
                         const void* w, bool flip, cudaStream_t s) {
  static std::atomic<unsigned int> conf0{0}, conf1{0};
  const size_t smem = sp_smem(P, K, false);
  const void* fn = flip ? (const void*)dwconv1d_strip_kernel<T, K, true>
                        : (const void*)dwconv1d_strip_kernel<T, K, false>;
  cudaError_t e = set_max_dynamic_smem(fn, smem, flip ? conf1 : conf0);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(P.n_cb * P.runs);
  if (flip)
    dwconv1d_strip_kernel<T, K, true><<<grid, SP_THREADS, smem, s>>>(tx, ty, (const T*)w, P,
                                                                     device_error_word());
  else
    dwconv1d_strip_kernel<T, K, false><<<grid, SP_THREADS, smem, s>>>(tx, ty, (const T*)w, P,
                                                                      device_error_word());
  return cudaGetLastError();
}

template <typename T, int K>
cudaError_t launch_wgrad_k(const SpParams& P, const CUtensorMap& tx, const CUtensorMap& td,
                           float* part, void* dw, cudaStream_t s) {
  static std::atomic<unsigned int> conf{0};
  const size_t smem = sp_smem(P, K, true);
  cudaError_t e = set_max_dynamic_smem((const void*)dwconv1d_wgrad_strip_kernel<T, K>, smem, conf);
  if (e != cudaSuccess) return e;
  dwconv1d_wgrad_strip_kernel<T, K><<<(unsigned)(P.n_cb * P.runs), SPW_THREADS, smem, s>>>(
      tx, td, part, P, device_error_word());
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int E = P.C * K;
  return launch_pdl(dwconv1d_wgrad_strip_sum<T>, (unsigned)((E + 31) / 32), 256u, 0, s, part,
                    (T*)dw, P.C, K, P.runs);
}

template <typename T>
cudaError_t dispatch_fwd(const SpParams& P, int K, const CUtensorMap& tx, const CUtensorMap& ty,
                         const void* w, bool flip, cudaStream_t s) {
  switch (K) {
    case 3: return launch_fwd_k<T, 3>(P, tx, ty, w, flip, s);
    case 5: return launch_fwd_k<T, 5>(P, tx, ty, w, flip, s);
    case 7: return launch_fwd_k<T, 7>(P, tx, ty, w, flip, s);
    case 9: return launch_fwd_k<T, 9>(P, tx, ty, w, flip, s);
    case 15: return launch_fwd_k<T, 15>(P, tx, ty, w, flip, s);
    case 31: return launch_fwd_k<T, 31>(P, tx, ty, w, flip, s);
    default: return cudaErrorNotSupported;
  }
}

template <typename T>
cudaError_t dispatch_wgrad(const SpParams& P, int K, const CUtensorMap& tx,
                           const CUtensorMap& td, float* part, void* dw, cudaStream_t s) {
  switch (K) {
    case 3: return launch_wgrad_k<T, 3>(P, tx, td, part, dw, s);
    case 5: return launch_wgrad_k<T, 5>(P, tx, td, part, dw, s);
    case 7: return launch_wgrad_k<T, 7>(P, tx, td, part, dw, s);
    case 9: return launch_wgrad_k<T, 9>(P, tx, td, part, dw, s);
    case 15: return launch_wgrad_k<T, 15>(P, tx, td, part, dw, s);
    case 31: return launch_wgrad_k<T, 31>(P, tx, td, part, dw, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

bool conv1d_strip_supported(const Conv1d& p) {
  SpParams P;
  const int t_max = p.T > p.T_out ? p.T : p.T_out;
  return p.B > 0 && p.B <= 65535 && t_max <= (1 << 30) &&
         make_sp_params(p, p.T, p.T_out, p.pad_left, false, &P) &&
         make_sp_params(p, p.T_out, p.T, p.K - 1 - p.pad_left, false, &P);
}

cudaError_t launch_dwconv1d_strip(const Conv1d& p, const void* x, const void* w, void* y,
                                  bool flip, int pad_left, int T_in, int T_out, cudaStream_t s) {
  SpParams P;
  if (!make_sp_params(p, T_in, T_out, pad_left, false, &P)) return cudaErrorNotSupported;
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tx, ty;
  if (!encode_rows(enc, &tx, p.dtype, x, p.C, T_in, p.B, SP_TS + p.K - 1, false) ||
      !encode_rows(enc, &ty, p.dtype, y, p.C, T_out, p.B, 16, true))
    return cudaErrorInvalidValue;
  if (p.dtype == GCONV_BF16) return dispatch_fwd<__nv_bfloat16>(P, p.K, tx, ty, w, flip, s);
  return dispatch_fwd<__half>(P, p.K, tx, ty, w, flip, s);
}

size_t dwconv1d_wgrad_strip_workspace(const Conv1d& p) {
  SpParams P;
  if (!make_sp_params(p, p.T, p.T_out, p.pad_left, true, &P)) return 0;
  return (size_t)P.n_cb * P.runs * SP_CB * p.K * sizeof(float);
}

cudaError_t launch_dwconv1d_wgrad_strip(const Conv1d& p, const void* x, const void* dy, void* dw,
                                        void* workspace, cudaStream_t s) {
  SpParams P;
  if (!make_sp_params(p, p.T, p.T_out, p.pad_left, true, &P)) return cudaErrorNotSupported;
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tx, td;
  if (!encode_rows(enc, &tx, p.dtype, x, p.C, p.T, p.B, SPW_TS + p.K - 1, false) ||
      !encode_rows(enc, &td, p.dtype, dy, p.C, p.T_out, p.B, SPW_TS, false))
    return cudaErrorInvalidValue;
  if (p.dtype == GCONV_BF16)
    return dispatch_wgrad<__nv_bfloat16>(P, p.K, tx, td, (float*)workspace, dw, s);
  return dispatch_wgrad<__half>(P, p.K, tx, td, (float*)workspace, dw, s);
}

}  // namespace gconv
