// Depthwise (fully-grouped, groups == C_in == C_out) conv2d, NHWC, 16-bit data.
//
// The fully-grouped case of "Grouped convolutions" (neon issue #296; TensorFlow's
// depthwise_conv2d in the same thread), in the channels-last layout the half-precision
// thread points to ("F.conv2d runs x15 slower ...", the NHWC replies). Memory-bound: each
// output needs kH*kW multiply-adds per channel and one read of its inputs.
//
// 3x3, dilation 1, stride 1 or 2 (the depthwise layers of the workloads) run on a TMA-staged
// kernel: persistent CTAs stream (rows x columns x 64 channels) input boxes through a ring of
// shared-memory stages with one TMA load per tile (the tensor map's zero fill is the padding),
// so the bytes in flight per SM come from the copy engine rather than from thread count.
// Each thread owns one channel pair across 4 adjacent output columns: every staged input word
// it needs is read and widened to fp32 once and then feeds all of its outputs (3 rows of 6 or
// 9 fp32 pairs rotate by renaming as the fully unrolled row loop moves down); the 3x3 filter
// of its pair stays in registers; the multiply-adds are fp32x2 packed, 4 independent chains.
// Other shapes run the register-window kernel: a thread owns VEC consecutive channels (one 16-,
// 8- or 4-byte vector) of one output column (n, wo) and walks down a chunk of output rows. Its
// kH x kW input window sits in registers as packed 16-bit vectors; moving one output row down
// shifts the window by `stride` input rows, so only `stride` new rows of kW vectors are loaded
// per output (when dilation == 1), and those loads are issued one row ahead of the arithmetic.
// The filter of the thread's VEC channels stays in fp32 registers. Consecutive threads take
// consecutive channel vectors, so a warp's loads and stores are contiguous runs of the channel
// dim.
#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

template <int NW> struct VecT;
template <> struct VecT<4> { using type = uint4; };
template <> struct VecT<2> { using type = uint2; };
template <> struct VecT<1> { using type = unsigned int; };

template <int NW>
__device__ __forceinline__ typename VecT<NW>::type ldg_vec(const void* p) {
  return __ldg(reinterpret_cast<const typename VecT<NW>::type*>(p));
}
template <int NW>
__device__ __forceinline__ typename VecT<NW>::type zero_vec() {
  typename VecT<NW>::type v;
  unsigned int* u = reinterpret_cast<unsigned int*>(&v);
#pragma unroll
  for (int i = 0; i < NW; ++i) u[i] = 0u;
  return v;
}

template <typename T, int K, int S, int VEC, bool SLIDE>
__global__ void __launch_bounds__(256) depthwise_nhwc_kernel(
    const T* __restrict__ x, const T* __restrict__ w, const T* __restrict__ bias,
    T* __restrict__ y, Conv2d p, int CV, int WB, int n_cblk, int HCH, int n_hch) {
  constexpr int NW = VEC / 2;              // 32-bit words per channel vector
  using Vec = typename VecT<NW>::type;
  constexpr int NEW = SLIDE ? (S < K ? S : K) : K;   // rows loaded per output row
  constexpr int KEEP = K - NEW;

  const int tid = threadIdx.x;
  const int cv = tid % CV, wl = tid / CV;
  const int cb = blockIdx.x % n_cblk, wb = blockIdx.x / n_cblk;
  const int c = (cb * CV + cv) * VEC;
  const int wo = wb * WB + wl;
  const int n = blockIdx.y / n_hch, hc = blockIdx.y % n_hch;
  if (wl >= WB || c >= p.C_in || wo >= p.Wo) return;  // no block-wide barrier below
  const int ho0 = hc * HCH;
  const int ho1 = min(p.Ho, ho0 + HCH);
  if (ho0 >= ho1) return;

  float wr[K][K][VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v)
#pragma unroll
    for (int kh = 0; kh < K; ++kh)
#pragma unroll
      for (int kw = 0; kw < K; ++kw)
        wr[kh][kw][v] = Elem<T>::to_f32(w[(long long)(c + v) * K * K + kh * K + kw]);
  float bv[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) bv[v] = bias ? Elem<T>::to_f32(bias[c + v]) : 0.0f;

  const long long rowC = (long long)p.W * p.C_in;
  const T* xn = x + (long long)n * p.H * rowC + c;
  long long woff[K];
  bool wok[K];
#pragma unroll
  for (int kw = 0; kw < K; ++kw) {
    const int wi = wo * S - p.pad + kw * p.dil;
    wok[kw] = (wi >= 0 && wi < p.W);
    woff[kw] = (long long)wi * p.C_in;
  }
  auto load_row = [&](Vec (&dst)[K], int hi) {
    const bool hok = (hi >= 0 && hi < p.H);
#pragma unroll
    for (int kw = 0; kw < K; ++kw)
      dst[kw] = (hok && wok[kw]) ? ldg_vec<NW>(xn + hi * rowC + woff[kw]) : zero_vec<NW>();
  };

  Vec win[K][K];
#pragma unroll
  for (int r = 0; r < K; ++r) load_row(win[r], ho0 * S - p.pad + r * p.dil);

  T* yp = y + (((long long)n * p.Ho + ho0) * p.Wo + wo) * p.C_out + c;
  const long long ystep = (long long)p.Wo * p.C_out;
  for (int ho = ho0; ho < ho1; ++ho) {
    // prefetch the rows the next output row adds to the window
    Vec nxt[NEW][K];
    if (ho + 1 < ho1) {
#pragma unroll
      for (int r = 0; r < NEW; ++r)
        load_row(nxt[r], (ho + 1) * S - p.pad + (KEEP + r) * p.dil);
    }
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = bv[v];
#pragma unroll
    for (int kh = 0; kh < K; ++kh)
#pragma unroll
      for (int kw = 0; kw < K; ++kw) {
        const unsigned int* u = reinterpret_cast<const unsigned int*>(&win[kh][kw]);
#pragma unroll
        for (int q = 0; q < NW; ++q) {
          const float2 xv = unpack2<T>(u[q]);
          acc[2 * q] = fmaf(wr[kh][kw][2 * q], xv.x, acc[2 * q]);
          acc[2 * q + 1] = fmaf(wr[kh][kw][2 * q + 1], xv.y, acc[2 * q + 1]);
        }
      }
    Vec out;
    unsigned int* o = reinterpret_cast<unsigned int*>(&out);
#pragma unroll
    for (int q = 0; q < NW; ++q) o[q] = pack2<T>(make_float2(acc[2 * q], acc[2 * q + 1]));
    *reinterpret_cast<Vec*>(yp) = out;
    yp += ystep;
    if (ho + 1 < ho1) {
#pragma unroll
      for (int r = 0; r < KEEP; ++r)
#pragma unroll
        for (int kw = 0; kw < K; ++kw) win[r][kw] = win[r + NEW][kw];
#pragma unroll
      for (int r = 0; r < NEW; ++r)
#pragma unroll
        for (int kw = 0; kw < K; ++kw) win[KEEP + r][kw] = nxt[r][kw];
    }
  }
}

// ---------------------------------------------------------------- 3x3 TMA-staged kernel

constexpr int DW3_MAX_STAGES = 8;
constexpr int DW3_CH = 64;                 // channels per tile (128-byte box rows)
constexpr size_t DW3_SMEM_BUDGET = 220 * 1024;   // per SM: two CTAs of <= 110 KB

struct Dw3Params {
  int N, H, W, C, Ho, Wo, pad;
  int BW, IW, IH;                          // output tile columns; input box columns and rows
  int n_ct, n_wt, n_ht, num_tiles, stages;
  unsigned int stage_bytes, tx_bytes;
  int flip;   // 1: read each 3x3 filter rotated by 180 degrees (the data gradient)
};

// Tile coordinates, channel tile slowest: tw -> th -> n -> ct. A CTA walks a contiguous chunk
// of tiles, so its filter registers change only when the chunk crosses a channel tile.
struct Dw3Coord {
  int ct, n, th, tw;
  __device__ __forceinline__ void set(const Dw3Params& P, long long t) {
    tw = (int)(t % P.n_wt);
    long long r = t / P.n_wt;
    th = (int)(r % P.n_ht);
    r /= P.n_ht;
    n = (int)(r % P.N);
    ct = (int)(r / P.N);
  }
  __device__ __forceinline__ void next(const Dw3Params& P) {
    if (++tw < P.n_wt) return;
    tw = 0;
    if (++th < P.n_ht) return;
    th = 0;
    if (++n < P.N) return;
    n = 0;
    ++ct;
  }
};

constexpr int DW3_R = 4;                   // output columns per thread
constexpr int DW3_NG = 7;                  // column groups (one compute warp each)
constexpr int DW3_BW = DW3_R * DW3_NG;     // output columns per tile
constexpr int DW3_THREADS = 32 + 32 * DW3_NG;
template <int S> __host__ __device__ constexpr int DW3_IW() { return (DW3_BW - 1) * S + 3; }

// Warp 0 lane 0 is the TMA producer; warps 1.. compute. Stage s is handed over through
// full[s] (TMA transaction bytes) and empty[s] (one arrival per compute warp).
template <typename T, int S, int BH>
__global__ void __launch_bounds__(DW3_THREADS, 2)
    dw3x3_tma_kernel(const __grid_constant__ CUtensorMap tmx,
                     const __grid_constant__ CUtensorMap tmy, const T* __restrict__ w,
                     const T* __restrict__ bias, const Dw3Params P, unsigned int* err) {
  using namespace ptx;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 128u);
  // output staging after the input ring: compute warp g owns [BH][DW3_R][64 ch], the box of
  // its own TMA store
  unsigned char* ostage = smem + (size_t)P.stages * P.stage_bytes;
  unsigned long long* full =
      reinterpret_cast<unsigned long long*>(ostage + (size_t)BH * DW3_BW * DW3_CH * 2);
  unsigned long long* empty = full + DW3_MAX_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + DW3_MAX_STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_compute_warps = (int)(blockDim.x >> 5) - 1;
  const int t_begin = (int)((long long)P.num_tiles * blockIdx.x / gridDim.x);
  const int t_end = (int)((long long)P.num_tiles * (blockIdx.x + 1) / gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], (unsigned int)n_compute_warps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmy);
  }
  __syncthreads();
  // the setup above may overlap the previous kernel in the stream (launch_pdl)
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      Dw3Coord c;
      c.set(P, t_begin);
      int s = 0;
      unsigned int ph = 0;
      long long issued = 0;
      for (int t = t_begin; t < t_end; ++t) {
        if (!mbar_try_wait(&empty[s], ph ^ 1u) &&
            !mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, 16u))
          break;
        mbar_arrive_expect_tx(&full[s], P.tx_bytes);
        tma_load_4d(smem + (size_t)s * P.stage_bytes, &tmx, &full[s], c.ct * DW3_CH,
                    c.tw * P.BW * S - P.pad, c.th * BH * S - P.pad, c.n);
        ++issued;
        c.next(P);
        if (++s == P.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      // copies in flight must land before the CTA exits (instant on the normal path)
      const unsigned long long dl = drain_deadline();
      for (long long q = (issued > P.stages ? issued - P.stages : 0); q < issued; ++q)
        mbar_wait_until(&full[q % P.stages], (unsigned int)((q / P.stages) & 1), dl, err,
                        ERR_DRAIN);
    }
  } else {
    constexpr int NIN = (DW3_R - 1) * S + 3;        // input columns a thread reads per row
    constexpr int row_w = DW3_IW<S>() * (DW3_CH / 2);  // 32-bit words per box row
    const int cp = lane, g = warp - 1;
    Dw3Coord c;
    c.set(P, t_begin);
    int prev_ct = -1;
    float2 wv[3][3];
    float2 bv = make_float2(0.f, 0.f);
    int s = 0;
    unsigned int ph = 0;
    unsigned char* wstage = ostage + (size_t)g * BH * DW3_R * DW3_CH * 2;
    unsigned int* orow = reinterpret_cast<unsigned int*>(wstage) + cp;
    for (int t = t_begin; t < t_end; ++t) {
      bool got = mbar_try_wait(&full[s], ph);
      if (!got) got = mbar_wait(&full[s], ph, abort_flag, err, 16u);
      if (!__all_sync(0xffffffffu, got)) break;
      if (lane == 0) bulk_wait_read0();              // this warp's previous store has read it
      __syncwarp();
      const int ch = c.ct * DW3_CH + 2 * cp;
      const bool ch_ok = ch < P.C;
      if (c.ct != prev_ct) {
        prev_ct = c.ct;
#pragma unroll
        for (int kh = 0; kh < 3; ++kh)
#pragma unroll
          for (int kw = 0; kw < 3; ++kw) {
            const int tp = P.flip ? 8 - (kh * 3 + kw) : kh * 3 + kw;
            wv[kh][kw] = ch_ok ? make_float2(Elem<T>::to_f32(w[ch * 9 + tp]),
                                             Elem<T>::to_f32(w[(ch + 1) * 9 + tp]))
                               : make_float2(0.f, 0.f);
          }
        bv = (bias && ch_ok) ? make_float2(Elem<T>::to_f32(bias[ch]), Elem<T>::to_f32(bias[ch + 1]))
                             : make_float2(0.f, 0.f);
      }
      // box word (row, column, pair) = (row * IW + column) * 32 + pair
      const uint32_t* px = reinterpret_cast<const uint32_t*>(smem + (size_t)s * P.stage_bytes) +
                           (g * DW3_R * S) * (DW3_CH / 2) + cp;
      float2 in[3][NIN];                               // input row r lives in slot r % 3
      auto load_row = [&](int r, float2 (&dst)[NIN]) {
#pragma unroll
        for (int i = 0; i < NIN; ++i) dst[i] = unpack2<T>(px[r * row_w + i * (DW3_CH / 2)]);
      };
      load_row(0, in[0]);
      if (S == 1) load_row(1, in[1]);
#pragma unroll
      for (int j = 0; j < BH; ++j) {
        if (S == 1) {
          load_row(j + 2, in[(j + 2) % 3]);
        } else {
          load_row(2 * j + 1, in[(2 * j + 1) % 3]);
          load_row(2 * j + 2, in[(2 * j + 2) % 3]);
        }
        float2 acc[DW3_R];
#pragma unroll
        for (int r = 0; r < DW3_R; ++r) acc[r] = bv;
#pragma unroll
        for (int kh = 0; kh < 3; ++kh) {
          const int slot = (j * S + kh) % 3;
#pragma unroll
          for (int kw = 0; kw < 3; ++kw)
#pragma unroll
            for (int r = 0; r < DW3_R; ++r)
              acc[r] = ffma2(wv[kh][kw], in[slot][r * S + kw], acc[r]);
        }
        // staged output word (row j, column r, pair cp); the TMA store clips the box at the
        // tensor's edges (rows past Ho, columns past Wo, channels past C)
#pragma unroll
        for (int r = 0; r < DW3_R; ++r)
          orow[(j * DW3_R + r) * (DW3_CH / 2)] = pack2<T>(acc[r]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s]);
        if (c.tw * DW3_BW + g * DW3_R < P.Wo) {   // a box wholly right of the image is skipped
          tma_store_4d(&tmy, wstage, c.ct * DW3_CH, c.tw * DW3_BW + g * DW3_R, c.th * BH, c.n);
          bulk_commit();
        }
      }
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

template <typename T, int S, int BH>
cudaError_t launch_dw3_tma(const Conv2d& p, const void* x, const void* w, const void* bias,
                           void* y, cudaStream_t s, bool flip = false) {
  Dw3Params P;
  P.flip = flip ? 1 : 0;
  P.N = p.N; P.H = p.H; P.W = p.W; P.C = p.C_in; P.Ho = p.Ho; P.Wo = p.Wo; P.pad = p.pad;
  P.BW = DW3_BW;
  P.IW = DW3_IW<S>();
  P.IH = (BH - 1) * S + 3;
  P.n_ct = (p.C_in + DW3_CH - 1) / DW3_CH;
  P.n_wt = (p.Wo + P.BW - 1) / P.BW;
  P.n_ht = (p.Ho + BH - 1) / BH;
  const long long tiles = (long long)P.n_ct * p.N * P.n_ht * P.n_wt;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  P.num_tiles = (int)tiles;
  P.tx_bytes = (unsigned int)(DW3_CH * P.IW * P.IH * 2);
  P.stage_bytes = (P.tx_bytes + 127u) & ~127u;
  // as many CTAs per SM (up to 3) as can each hold a ring of >= 2 stages
  const size_t ostage = (size_t)BH * DW3_BW * DW3_CH * 2;
  int per_sm = 3, stages = 0;
  for (; per_sm >= 1; --per_sm) {
    const size_t share = DW3_SMEM_BUDGET / per_sm;
    stages = share > ostage ? (int)((share - ostage) / P.stage_bytes) : 0;
    if (stages >= 2) break;
  }
  if (stages > DW3_MAX_STAGES) stages = DW3_MAX_STAGES;
  if (stages < 2) return cudaErrorInvalidValue;
  P.stages = stages;
  const size_t smem =
      128 + (size_t)stages * P.stage_bytes + ostage + 2 * DW3_MAX_STAGES * 8 + 16;

  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tm;
  const cuuint64_t dims[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t strides[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                                 (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t box[4] = {DW3_CH, (cuuint32_t)P.IW, (cuuint32_t)P.IH, 1};
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  // 128-byte promotion: a box row is one pixel's 64 channels; wider promotion would pull in
  // the next channel tile, which this CTA order reaches only much later
  if (enc(&tm, dt, 4, const_cast<void*>(x), dims, strides, box, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  CUtensorMap tmy;
  const cuuint64_t ydims[4] = {(cuuint64_t)p.C_out, (cuuint64_t)p.Wo, (cuuint64_t)p.Ho,
                               (cuuint64_t)p.N};
  const cuuint64_t ystrides[3] = {(cuuint64_t)p.C_out * 2, (cuuint64_t)p.Wo * p.C_out * 2,
                                  (cuuint64_t)p.Ho * p.Wo * p.C_out * 2};
  const cuuint32_t ybox[4] = {DW3_CH, DW3_R, BH, 1};
  if (enc(&tmy, dt, 4, y, ydims, ystrides, ybox, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)dw3x3_tma_kernel<T, S, BH>,
                                       DW3_SMEM_BUDGET + 1024, configured);
  if (e != cudaSuccess) return e;
  const int threads = DW3_THREADS;
  int fit = per_sm;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
          &fit, dw3x3_tma_kernel<T, S, BH>, threads, smem) != cudaSuccess || fit < 1)
    fit = 1;
  if (fit > per_sm) fit = per_sm;
  long long grid = (long long)sm_count() * fit;
  if (grid > P.num_tiles) grid = P.num_tiles;
  return launch_pdl(dw3x3_tma_kernel<T, S, BH>, (unsigned)grid, (unsigned)threads, smem, s, tm,
                    tmy, (const T*)w, (const T*)bias, P, device_error_word());
}

bool dw3_tma_eligible(const Conv2d& p) {
  return p.kH == 3 && p.kW == 3 && p.dil == 1 && (p.stride == 1 || p.stride == 2) &&
         p.C_in % 8 == 0 && p.pad <= 2;
}

template <int K> constexpr int vec_for() { return K <= 3 ? 8 : (K <= 5 ? 4 : 2); }

template <typename T, int K, int S>
cudaError_t launch_ks(const Conv2d& p, const void* x, const void* w, const void* bias, void* y,
                      cudaStream_t s) {
  constexpr int VEC = vec_for<K>();
  const int nvec = p.C_in / VEC;
  const int CV = nvec < 32 ? nvec : 32;
  const int WB = 256 / CV;
  const int n_cblk = (nvec + CV - 1) / CV;
  const int n_wblk = (p.Wo + WB - 1) / WB;
  // rows per thread: enough blocks for ~8 waves of 2 blocks per SM, at least 4 rows each
  const long long base = (long long)n_cblk * n_wblk * p.N;
  int n_hch = (int)((148LL * 2 * 8 + base - 1) / base);
  if (n_hch < 1) n_hch = 1;
  if (n_hch > (p.Ho + 3) / 4) n_hch = (p.Ho + 3) / 4;
  if (n_hch > 65535 / p.N) n_hch = 65535 / p.N;     // grid.y = N * n_hch
  if (n_hch < 1) n_hch = 1;
  const int HCH = (p.Ho + n_hch - 1) / n_hch;
  n_hch = (p.Ho + HCH - 1) / HCH;
  dim3 grid((unsigned)(n_cblk * n_wblk), (unsigned)(p.N * n_hch));
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
  if (p.dil == 1)
    depthwise_nhwc_kernel<T, K, S, VEC, true><<<grid, 256, 0, s>>>(
        (const T*)x, (const T*)w, (const T*)bias, (T*)y, p, CV, WB, n_cblk, HCH, n_hch);
  else
    depthwise_nhwc_kernel<T, K, S, VEC, false><<<grid, 256, 0, s>>>(
        (const T*)x, (const T*)w, (const T*)bias, (T*)y, p, CV, WB, n_cblk, HCH, n_hch);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const Conv2d& p, const void* x, const void* w, const void* bias, void* y,
                         cudaStream_t s) {
  if (dw3_tma_eligible(p))
    return p.stride == 1 ? launch_dw3_tma<T, 1, 8>(p, x, w, bias, y, s)
                         : launch_dw3_tma<T, 2, 2>(p, x, w, bias, y, s);
  const int K = p.kH;
  if (p.stride == 1) {
    if (K == 3) return launch_ks<T, 3, 1>(p, x, w, bias, y, s);
    if (K == 5) return launch_ks<T, 5, 1>(p, x, w, bias, y, s);
    return launch_ks<T, 7, 1>(p, x, w, bias, y, s);
  }
  if (K == 3) return launch_ks<T, 3, 2>(p, x, w, bias, y, s);
  if (K == 5) return launch_ks<T, 5, 2>(p, x, w, bias, y, s);
  return launch_ks<T, 7, 2>(p, x, w, bias, y, s);
}

}  // namespace

// Eligibility, excluding pointer alignment (checked by the dispatcher): 16-bit NHWC,
// one input and one output channel per group, square 3/5/7 filters, stride 1 or 2, and a
// channel count that is a multiple of the vector width.
bool depthwise_nhwc_supported(const Conv2d& p) {
  if (p.layout != GCONV_NHWC || p.dtype == GCONV_F32) return false;
  if (p.groups != p.C_in || p.C_out != p.C_in) return false;
  if (p.kH != p.kW || (p.kH != 3 && p.kH != 5 && p.kH != 7)) return false;
  if (p.stride != 1 && p.stride != 2) return false;
  const int vec = p.kH <= 3 ? 8 : (p.kH <= 5 ? 4 : 2);
  return p.C_in % vec == 0;
}

cudaError_t launch_depthwise_nhwc(const Conv2d& p, const void* x, const void* w,
                                  const void* bias, void* y, cudaStream_t s) {
  if (p.dtype == GCONV_F16) return launch_typed<__half>(p, x, w, bias, y, s);
  return launch_typed<__nv_bfloat16>(p, x, w, bias, y, s);
}

bool depthwise_nhwc_flipped_supported(const Conv2d& p) {
  return depthwise_nhwc_supported(p) && dw3_tma_eligible(p) && p.stride == 1;
}

cudaError_t launch_depthwise_nhwc_flipped(const Conv2d& p, const void* x, const void* w, void* y,
                                          cudaStream_t s) {
  if (!depthwise_nhwc_flipped_supported(p)) return cudaErrorInvalidValue;
  if (p.dtype == GCONV_F16) return launch_dw3_tma<__half, 1, 8>(p, x, w, nullptr, y, s, true);
  return launch_dw3_tma<__nv_bfloat16, 1, 8>(p, x, w, nullptr, y, s, true);
}

}  // namespace gconv
