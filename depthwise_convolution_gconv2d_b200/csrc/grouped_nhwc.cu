// Narrow-group conv2d (2, 4 or 8 channels per group in and out), 3x3, NHWC, 16-bit.
//
// Grouped convolution as "Grouped convolutions" (neon issue #296) defines it: output channel co
// of group g sums over the group's own input channels only. With so few channels per group the
// per-group GEMM is narrower than a tensor-core MMA's K and N (16), so the layer runs on the
// CUDA cores; like the depthwise kernel it is bound by HBM unless the instruction count per
// output is kept near the multiply-adds themselves (9 * cpg per output).
//
// Persistent CTAs stream (rows x 28 + halo columns x 64 channels) input boxes through a TMA
// ring filled by a producer warp (zero fill = the padding; 64-channel tiles hold whole groups).
// Seven compute warps each own 4 output columns of the tile; a thread owns one output-channel
// pair of its group over 4 columns x BH rows (accumulators in registers). It walks the group's
// input channels one at a time: that channel's 9 filter taps for the pair come from a per-tile
// table of fp32 pairs in shared memory, each staged input value is widened once into a
// broadcast fp32 pair and feeds, by packed fp32x2 FMA, every output row and column it touches.
// Each warp stages its outputs in shared memory and writes them with one TMA store per tile.
#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

constexpr int NG_CH = 64;                   // channels per tile (128-byte box rows)
constexpr int NG_R = 4;                     // output columns per thread
constexpr int NG_WARPS = 7;                 // compute warps
constexpr int NG_BW = NG_R * NG_WARPS;      // output columns per tile
constexpr int NG_THREADS = 32 + 32 * NG_WARPS;
constexpr int NG_MAX_STAGES = 8;
constexpr size_t NG_SMEM_PER_SM = 220 * 1024;

struct NgParams {
  int N, H, W, C, Ho, Wo, pad;
  int IW, IH;                               // input box columns and rows
  int n_ct, n_wt, n_ht, num_tiles, stages;
  unsigned int stage_bytes, tx_bytes;
};

// tile t -> (column tile, row tile, image, channel tile), channel tile slowest
struct NgCoord {
  int ct, n, th, tw;
  __device__ __forceinline__ void set(const NgParams& P, int t) {
    tw = t % P.n_wt;
    int r = t / P.n_wt;
    th = r % P.n_ht;
    r /= P.n_ht;
    n = r % P.N;
    ct = r / P.N;
  }
  __device__ __forceinline__ void next(const NgParams& P) {
    if (++tw < P.n_wt) return;
    tw = 0;
    if (++th < P.n_ht) return;
    th = 0;
    if (++n < P.N) return;
    n = 0;
    ++ct;
  }
};

template <int S> __host__ __device__ constexpr int ng_iw() { return (NG_BW - 1) * S + 3; }

template <typename T, int S, int BH, int CPG>
__global__ void __launch_bounds__(NG_THREADS, 2)
    grouped3x3_tma_kernel(const __grid_constant__ CUtensorMap tmx,
                          const __grid_constant__ CUtensorMap tmy, const T* __restrict__ w,
                          const T* __restrict__ bias, const NgParams P, unsigned int* err) {
  using namespace ptx;
  constexpr int NCT = 32 * NG_WARPS;                // compute threads (named barrier 1)
  constexpr int NIN = (NG_R - 1) * S + 3;           // input columns a thread reads per row
  constexpr int RIN = (BH - 1) * S + 3;             // input rows per tile
  constexpr int ROW_W = ng_iw<S>() * (NG_CH / 2);   // 32-bit words per box row
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem(smem_raw, 128u);
  // [ring][per-warp output staging][filter table: CPG x 9 taps x 32 pairs of fp32][barriers]
  unsigned char* ostage = smem + (size_t)P.stages * P.stage_bytes;
  float2* wtab = reinterpret_cast<float2*>(ostage + (size_t)NG_WARPS * BH * NG_R * NG_CH * 2);
  unsigned long long* full = reinterpret_cast<unsigned long long*>(wtab + CPG * 9 * 32);
  unsigned long long* empty = full + NG_MAX_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NG_MAX_STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = (int)((long long)P.num_tiles * blockIdx.x / gridDim.x);
  const int t_end = (int)((long long)P.num_tiles * (blockIdx.x + 1) / gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NG_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmy);
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      NgCoord c;
      c.set(P, t_begin);
      int s = 0;
      unsigned int ph = 0;
      int issued = 0;
      for (int t = t_begin; t < t_end; ++t) {
        if (!mbar_try_wait(&empty[s], ph ^ 1u) &&
            !mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, 16u))
          break;
        mbar_arrive_expect_tx(&full[s], P.tx_bytes);
        tma_load_4d(smem + (size_t)s * P.stage_bytes, &tmx, &full[s], c.ct * NG_CH,
                    c.tw * NG_BW * S - P.pad, c.th * BH * S - P.pad, c.n);
        ++issued;
        c.next(P);
        if (++s == P.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      // copies in flight must land before the CTA exits
      const unsigned long long dl = drain_deadline();
      for (int q = (issued > P.stages ? issued - P.stages : 0); q < issued; ++q)
        mbar_wait_until(&full[q % P.stages], (unsigned int)((q / P.stages) & 1), dl, err,
                        ERR_DRAIN);
    }
  } else {
    // ------------------------------------------------------------ compute warps
    const int cp = lane, g = warp - 1, ctid = threadIdx.x - 32;
    const int gbase = ((2 * cp) / CPG) * CPG;       // first input channel of the pair's group
    unsigned char* wstage = ostage + (size_t)g * BH * NG_R * NG_CH * 2;
    unsigned int* orow = reinterpret_cast<unsigned int*>(wstage) + cp;
    NgCoord c;
    c.set(P, t_begin);
    int prev_ct = -1;
    float2 bv = make_float2(0.f, 0.f);
    int s = 0;
    unsigned int ph = 0;
    for (int t = t_begin; t < t_end; ++t) {
      bool got = mbar_try_wait(&full[s], ph);
      if (!got) got = mbar_wait(&full[s], ph, abort_flag, err, 16u);
      // also the point where every compute warp has finished the previous tile
      if (!named_all(1, NCT, got)) break;
      const int co0 = c.ct * NG_CH + 2 * cp;
      const bool ch_ok = co0 < P.C;
      if (c.ct != prev_ct) {
        prev_ct = c.ct;
        // filter table of this channel tile: wtab[ci][tap][pair] = taps of (co, co + 1)
        for (int i = ctid; i < CPG * 9 * 32; i += NCT) {
          const int ci = i / (9 * 32), rem = i % (9 * 32), tap = rem / 32, pp = rem % 32;
          const int co = c.ct * NG_CH + 2 * pp;
          wtab[i] = co < P.C
                        ? make_float2(Elem<T>::to_f32(w[((long long)co * 9 + tap) * CPG + ci]),
                                      Elem<T>::to_f32(w[((long long)(co + 1) * 9 + tap) * CPG + ci]))
                        : make_float2(0.f, 0.f);
        }
        bv = (bias && ch_ok) ? make_float2(Elem<T>::to_f32(bias[co0]),
                                           Elem<T>::to_f32(bias[co0 + 1]))
                             : make_float2(0.f, 0.f);
        named_sync(1, NCT);
      }
      // box word (row, column, pair) = (row * IW + column) * 32 + pair
      const uint32_t* px = reinterpret_cast<const uint32_t*>(smem + (size_t)s * P.stage_bytes) +
                           (g * NG_R * S) * (NG_CH / 2);
      float2 acc[BH][NG_R];
#pragma unroll
      for (int j = 0; j < BH; ++j)
#pragma unroll
        for (int r = 0; r < NG_R; ++r) acc[j][r] = bv;
#pragma unroll
      for (int ci = 0; ci < CPG; ++ci) {
        float2 wr[9];
#pragma unroll
        for (int tap = 0; tap < 9; ++tap) wr[tap] = wtab[(ci * 9 + tap) * 32 + cp];
        const int chin = gbase + ci;                 // input channel within the tile
        const uint32_t* pc = px + (chin >> 1);
        // bf16 / fp16 half of the word -> fp32 bits in the upper half (bf16) or converted
        const bool hi = (chin & 1) != 0;
#pragma unroll
        for (int rr = 0; rr < RIN; ++rr) {
          float2 v[NIN];
#pragma unroll
          for (int i = 0; i < NIN; ++i) {
            const float2 two = unpack2<T>(pc[rr * ROW_W + i * (NG_CH / 2)]);
            const float x = hi ? two.y : two.x;
            v[i] = make_float2(x, x);
          }
#pragma unroll
          for (int j = 0; j < BH; ++j) {
            const int kh = rr - j * S;
            if (kh < 0 || kh > 2) continue;
#pragma unroll
            for (int kw = 0; kw < 3; ++kw)
#pragma unroll
              for (int r = 0; r < NG_R; ++r)
                acc[j][r] = ffma2(wr[kh * 3 + kw], v[r * S + kw], acc[j][r]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s]);                      // the input box is consumed
        bulk_wait_read0();                           // this warp's previous store has read
      }
      __syncwarp();
#pragma unroll
      for (int j = 0; j < BH; ++j)
#pragma unroll
        for (int r = 0; r < NG_R; ++r)
          orow[(j * NG_R + r) * (NG_CH / 2)] = pack2<T>(acc[j][r]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0 && c.tw * NG_BW + g * NG_R < P.Wo) {
        // the TMA store clips the box at the tensor's edges (rows, columns, channels); a box
        // wholly right of the image is not issued
        tma_store_4d(&tmy, wstage, c.ct * NG_CH, c.tw * NG_BW + g * NG_R, c.th * BH, c.n);
        bulk_commit();
      }
      (void)ch_ok;
      c.next(P);
      if (++s == P.stages) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (lane == 0) bulk_wait0();
  }
  __syncthreads();
}

template <typename T, int S, int BH, int CPG>
cudaError_t launch_ng(const Conv2d& p, const void* x, const void* w, const void* bias, void* y,
                      cudaStream_t s) {
  NgParams P;
  P.N = p.N; P.H = p.H; P.W = p.W; P.C = p.C_in; P.Ho = p.Ho; P.Wo = p.Wo; P.pad = p.pad;
  P.IW = ng_iw<S>();
  P.IH = (BH - 1) * S + 3;
  P.n_ct = (p.C_in + NG_CH - 1) / NG_CH;
  P.n_wt = (p.Wo + NG_BW - 1) / NG_BW;
  P.n_ht = (p.Ho + BH - 1) / BH;
  const long long tiles = (long long)P.n_ct * p.N * P.n_ht * P.n_wt;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  P.num_tiles = (int)tiles;
  P.tx_bytes = (unsigned int)(NG_CH * P.IW * P.IH * 2);
  P.stage_bytes = (P.tx_bytes + 127u) & ~127u;
  const size_t fixed = 128 + (size_t)NG_WARPS * BH * NG_R * NG_CH * 2 +
                       (size_t)CPG * 9 * 32 * sizeof(float2) + 2 * NG_MAX_STAGES * 8 + 16;
  // two CTAs per SM when two rings of >= 2 stages fit, else one
  int per_sm = 2;
  int stages = (int)((NG_SMEM_PER_SM / 2 - fixed) / P.stage_bytes);
  if (stages < 2) {
    per_sm = 1;
    stages = (int)((NG_SMEM_PER_SM - fixed) / P.stage_bytes);
  }
  if (stages > NG_MAX_STAGES) stages = NG_MAX_STAGES;
  if (stages < 2) return cudaErrorInvalidValue;
  P.stages = stages;
  const size_t smem = fixed + (size_t)stages * P.stage_bytes;

  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  CUtensorMap tmx, tmy;
  const cuuint64_t dims[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t strides[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                                 (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t box[4] = {NG_CH, (cuuint32_t)P.IW, (cuuint32_t)P.IH, 1};
  if (enc(&tmx, dt, 4, const_cast<void*>(x), dims, strides, box, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t ydims[4] = {(cuuint64_t)p.C_out, (cuuint64_t)p.Wo, (cuuint64_t)p.Ho,
                               (cuuint64_t)p.N};
  const cuuint64_t ystrides[3] = {(cuuint64_t)p.C_out * 2, (cuuint64_t)p.Wo * p.C_out * 2,
                                  (cuuint64_t)p.Ho * p.Wo * p.C_out * 2};
  const cuuint32_t ybox[4] = {NG_CH, NG_R, BH, 1};
  if (enc(&tmy, dt, 4, y, ydims, ystrides, ybox, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)grouped3x3_tma_kernel<T, S, BH, CPG>,
                                       NG_SMEM_PER_SM / 2 > smem ? NG_SMEM_PER_SM / 2 : smem,
                                       configured);
  if (e != cudaSuccess) return e;
  int fit = per_sm;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
          &fit, grouped3x3_tma_kernel<T, S, BH, CPG>, NG_THREADS, smem) != cudaSuccess ||
      fit < 1)
    fit = 1;
  if (fit > per_sm) fit = per_sm;
  long long grid = (long long)sm_count() * fit;
  if (grid > P.num_tiles) grid = P.num_tiles;
  grouped3x3_tma_kernel<T, S, BH, CPG><<<(unsigned)grid, NG_THREADS, smem, s>>>(
      tmx, tmy, (const T*)w, (const T*)bias, P, device_error_word());
  return cudaGetLastError();
}

template <typename T, int CPG>
cudaError_t launch_ng_cpg(const Conv2d& p, const void* x, const void* w, const void* bias,
                          void* y, cudaStream_t s) {
  return p.stride == 1 ? launch_ng<T, 1, 4, CPG>(p, x, w, bias, y, s)
                       : launch_ng<T, 2, 2, CPG>(p, x, w, bias, y, s);
}

template <typename T>
cudaError_t launch_ng_typed(const Conv2d& p, const void* x, const void* w, const void* bias,
                            void* y, cudaStream_t s) {
  switch (p.cpg_in) {
    case 2: return launch_ng_cpg<T, 2>(p, x, w, bias, y, s);
    case 4: return launch_ng_cpg<T, 4>(p, x, w, bias, y, s);
    default: return launch_ng_cpg<T, 8>(p, x, w, bias, y, s);
  }
}

}  // namespace

bool grouped_nhwc_supported(const Conv2d& p) {
  return p.layout == GCONV_NHWC && p.dtype != GCONV_F32 && p.kH == 3 && p.kW == 3 &&
         p.dil == 1 && (p.stride == 1 || p.stride == 2) && p.pad <= 2 &&
         p.cpg_in == p.cpg_out && (p.cpg_in == 2 || p.cpg_in == 4 || p.cpg_in == 8) &&
         p.C_in % 8 == 0;
}

cudaError_t launch_grouped_nhwc(const Conv2d& p, const void* x, const void* w, const void* bias,
                                void* y, cudaStream_t s) {
  if (p.N == 0) return cudaSuccess;
  if (p.dtype == GCONV_F16) return launch_ng_typed<__half>(p, x, w, bias, y, s);
  return launch_ng_typed<__nv_bfloat16>(p, x, w, bias, y, s);
}

}  // namespace gconv
