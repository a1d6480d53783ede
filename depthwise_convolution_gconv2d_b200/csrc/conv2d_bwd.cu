// Backward pass of the grouped conv2d: data gradient and weight gradient.
//
// The grouped layers on the pages are trained (the Adam-trained ensemble of "Optimize
// convolution batching rule performance", whose vmap'd grouped conv is differentiated; the
// backward timings of the Conformer thread), so the layer's two gradients follow from the
// forward sum y[n,co,ho,wo] = sum_{ci,kh,kw} w[co,ci,kh,kw] x[n, g*cpg_in+ci, h, w] with
// h = ho*stride - pad + kh*dil, w = wo*stride - pad + kw*dil (g = co / cpg_out):
//   dx[n, g*cpg_in+ci, h, w] = sum over (co in group g, kh, kw) with h + pad - kh*dil and
//                              w + pad - kw*dil multiples of stride of
//                              w[co,ci,kh,kw] * dy[n, co, (h+pad-kh*dil)/stride, (w+pad-kw*dil)/stride]
//   dw[co,ci,kh,kw]          = sum over (n, ho, wo) of dy[n,co,ho,wo] * x[n, g*cpg_in+ci, h, w]
//
// At stride 1 the data gradient is itself a grouped convolution: the forward problem with the
// roles of C_in and C_out exchanged, input dy (Ho x Wo), pad' = dil*(k-1) - pad, and per group
// the filter transposed (ci <-> co) and rotated by 180 degrees. `flip_transpose_weight_kernel`
// writes that filter into the caller's workspace and the forward kernels (tensor cores,
// depthwise, narrow groups) run the rest. Other depthwise shapes (stride 2, larger pads) take a
// gather kernel on 16-byte channel vectors, everything else a one-thread-per-element gather.
//
// The weight gradient is a reduction over N*Ho*Wo positions per filter tap. It is
// deterministic: the work is cut into fixed slices (a function of the shape only), each
// slice's partial sums are accumulated in a fixed order into fp32 workspace slots, and a
// second kernel adds the slices in slice order and rounds once to the data type. No float
// atomics, so repeated calls give bitwise-identical dw on any GPU. Kernels, most specific
// first: depthwise 3x3 on a TMA ring (the forward 3x3 kernel's data path with filter and
// output exchanged), depthwise 3x3 / 5x5 with register chunks, wide groups as shared-memory
// tiled outer products per (group, tap) on the CUDA cores (NCHW through an NHWC staging copy),
// and a one-thread-per-entry generic kernel.
#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

// Target CTA count of the weight-gradient kernels (8 per SM of a 148-SM part); a fixed
// constant rather than a device query, so the slicing -- and the rounding -- never depends on
// the device.
constexpr long long WGRAD_TARGET_CTAS = 1184;

__device__ __forceinline__ long long w_index(const Conv2d& p, int layout, int co, int ci,
                                             int kh, int kw) {
  if (layout == GCONV_NCHW) return (((long long)co * p.cpg_in + ci) * p.kH + kh) * p.kW + kw;
  return (((long long)co * p.kH + kh) * p.kW + kw) * p.cpg_in + ci;
}

// ------------------------------------------------------------------ weight for dgrad-as-conv
// wt is the weight of the exchanged problem (C_out' = C_in, C_in'/g = cpg_out):
//   wt[c][kh'][kw'][col] (NHWC) or wt[c][col][kh'][kw'] (NCHW)
//     = w[g*cpg_out + col][c - g*cpg_in][kH-1-kh'][kW-1-kw'],  g = c / cpg_in.
template <typename T, int LAYOUT>
__global__ void __launch_bounds__(256) flip_transpose_weight_kernel(const T* __restrict__ w,
                                                                     T* __restrict__ wt,
                                                                     Conv2d p, long long total) {
  const long long step = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += step) {
    long long r = i;
    int col, kh2, kw2, c;
    if (LAYOUT == GCONV_NHWC) {
      col = (int)(r % p.cpg_out); r /= p.cpg_out;
      kw2 = (int)(r % p.kW); r /= p.kW;
      kh2 = (int)(r % p.kH); c = (int)(r / p.kH);
    } else {
      kw2 = (int)(r % p.kW); r /= p.kW;
      kh2 = (int)(r % p.kH); r /= p.kH;
      col = (int)(r % p.cpg_out); c = (int)(r / p.cpg_out);
    }
    const int g = c / p.cpg_in;
    wt[i] = w[w_index(p, LAYOUT, g * p.cpg_out + col, c - g * p.cpg_in, p.kH - 1 - kh2,
                      p.kW - 1 - kw2)];
  }
}

// The NHWC case as a tiled transpose: w is [C_out][kH][kW][cpg_in], so per group g the
// [cpg_out] x [kH * kW * cpg_in] block of w (row col, column e = tap * cpg_in + ci, contiguous)
// becomes rows (ci, reversed tap) x columns col of wt; 64 x 64 tiles through shared memory, so both the loads (along e) and the
// stores (along col) are contiguous. (The element-wise gather above, one 2-byte load per
// output from filters 2.3 KB apart, took several microseconds for the wide-group layer's
// 1.2 MB of weights.)
template <typename T>
__global__ void __launch_bounds__(256) flip_weight_nhwc_tiled_kernel(const T* __restrict__ w,
                                                                      T* __restrict__ wt,
                                                                      int cpg_in, int cpg_out,
                                                                      int taps) {
  __shared__ unsigned short tile[64][66];
  const unsigned short* ws = reinterpret_cast<const unsigned short*>(w);
  unsigned short* wd = reinterpret_cast<unsigned short*>(wt);
  const int g = blockIdx.z, e0 = blockIdx.x * 64, c0 = blockIdx.y * 64;
  const long long E = (long long)cpg_in * taps;
  const unsigned short* src = ws + (long long)g * cpg_out * E;
  // a thread's 16 loads are issued before any of them is stored (a load -> store chain per
  // element left each thread waiting out 16 DRAM latencies: 12 us for 1.2 MB, measured)
  unsigned short v[16];
#pragma unroll
  for (int it = 0; it < 16; ++it) {
    const int i = threadIdx.x + 256 * it;
    const int r = i >> 6, q = i & 63;              // r: filter col, q: e (contiguous)
    const int col = c0 + r, e = e0 + q;
    v[it] = (col < cpg_out && e < E) ? src[(long long)col * E + e] : (unsigned short)0;
  }
#pragma unroll
  for (int it = 0; it < 16; ++it) {
    const int i = threadIdx.x + 256 * it;
    tile[i >> 6][i & 63] = v[it];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int q = i >> 6, r = i & 63;              // r: filter col (contiguous in wt)
    const int col = c0 + r, e = e0 + q;
    if (col < cpg_out && e < E) {
      const int tap = e / cpg_in, ci = e - tap * cpg_in;
      const long long c = (long long)g * cpg_in + ci;
      wd[(c * taps + (taps - 1 - tap)) * cpg_out + col] = tile[r][q];
    }
  }
}

// ------------------------------------------------------------------ generic data gradient
// One thread per dx element (decoded in dx's memory order, so stores are contiguous); fp32
// FMA over the group's output channels and the taps whose window reads this input.
template <typename T, int LAYOUT>
__global__ void __launch_bounds__(256) dgrad_generic_kernel(const T* __restrict__ dy,
                                                             const T* __restrict__ w,
                                                             T* __restrict__ dx, Conv2d p,
                                                             long long total) {
  const long long step = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += step) {
    int n, c, h, wi;
    long long r = i;
    if (LAYOUT == GCONV_NCHW) {
      wi = (int)(r % p.W); r /= p.W;
      h = (int)(r % p.H); r /= p.H;
      c = (int)(r % p.C_in); n = (int)(r / p.C_in);
    } else {
      c = (int)(r % p.C_in); r /= p.C_in;
      wi = (int)(r % p.W); r /= p.W;
      h = (int)(r % p.H); n = (int)(r / p.H);
    }
    const int g = c / p.cpg_in, ci = c - g * p.cpg_in;
    const int co0 = g * p.cpg_out;
    float acc = 0.0f;
    for (int kh = 0; kh < p.kH; ++kh) {
      const int th = h + p.pad - kh * p.dil;       // = ho * stride
      if (th < 0 || th % p.stride != 0) continue;
      const int ho = th / p.stride;
      if (ho >= p.Ho) continue;
      for (int kw = 0; kw < p.kW; ++kw) {
        const int tw = wi + p.pad - kw * p.dil;
        if (tw < 0 || tw % p.stride != 0) continue;
        const int wo = tw / p.stride;
        if (wo >= p.Wo) continue;
        if (LAYOUT == GCONV_NCHW) {
          const T* d = dy + (((long long)n * p.C_out + co0) * p.Ho + ho) * p.Wo + wo;
          const long long dstep = (long long)p.Ho * p.Wo;
          for (int j = 0; j < p.cpg_out; ++j)
            acc = fmaf(Elem<T>::to_f32(w[w_index(p, LAYOUT, co0 + j, ci, kh, kw)]),
                       Elem<T>::to_f32(d[j * dstep]), acc);
        } else {
          const T* d = dy + (((long long)n * p.Ho + ho) * p.Wo + wo) * p.C_out + co0;
          for (int j = 0; j < p.cpg_out; ++j)
            acc = fmaf(Elem<T>::to_f32(w[w_index(p, LAYOUT, co0 + j, ci, kh, kw)]),
                       Elem<T>::to_f32(d[j]), acc);
        }
      }
    }
    dx[i] = Elem<T>::from_f32(acc);
  }
}

// ------------------------------------------------------------------ generic weight gradient
// One thread per (dw entry, slice): entry e in dw's memory order, slice = (n, ho) rows
// [r0, r1). Partial sum in (row, wo) order -> ws[slice][e].
template <typename T, int LAYOUT>
__global__ void __launch_bounds__(256) wgrad_generic_kernel(const T* __restrict__ x,
                                                             const T* __restrict__ dy,
                                                             float* __restrict__ ws, Conv2d p,
                                                             long long E, int rows) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  int co, ci, kh, kw;
  long long r = e;
  if (LAYOUT == GCONV_NCHW) {
    kw = (int)(r % p.kW); r /= p.kW;
    kh = (int)(r % p.kH); r /= p.kH;
    ci = (int)(r % p.cpg_in); co = (int)(r / p.cpg_in);
  } else {
    ci = (int)(r % p.cpg_in); r /= p.cpg_in;
    kw = (int)(r % p.kW); r /= p.kW;
    kh = (int)(r % p.kH); co = (int)(r / p.kH);
  }
  const int c = (co / p.cpg_out) * p.cpg_in + ci;
  const int R = p.N * p.Ho;
  const int r0 = blockIdx.y * rows, r1 = min(R, r0 + rows);
  float acc = 0.0f;
  for (int row = r0; row < r1; ++row) {
    const int n = row / p.Ho, ho = row - n * p.Ho;
    const int h = ho * p.stride - p.pad + kh * p.dil;
    if (h < 0 || h >= p.H) continue;
    for (int wo = 0; wo < p.Wo; ++wo) {
      const int wi = wo * p.stride - p.pad + kw * p.dil;
      if (wi < 0 || wi >= p.W) continue;
      long long xi, yi;
      if (LAYOUT == GCONV_NCHW) {
        xi = (((long long)n * p.C_in + c) * p.H + h) * p.W + wi;
        yi = (((long long)n * p.C_out + co) * p.Ho + ho) * p.Wo + wo;
      } else {
        xi = (((long long)n * p.H + h) * p.W + wi) * p.C_in + c;
        yi = (((long long)n * p.Ho + ho) * p.Wo + wo) * p.C_out + co;
      }
      acc = fmaf(Elem<T>::to_f32(dy[yi]), Elem<T>::to_f32(x[xi]), acc);
    }
  }
  ws[(long long)blockIdx.y * E + e] = acc;
}

// ------------------------------------------------------------------ depthwise weight gradient
// NHWC, 16-bit, K x K (K = 3 or 5), dilation 1, stride S = 1 or 2. A thread owns one channel
// pair and one slice of (n, ho) rows, with its K x K fp32-pair accumulators in registers. It
// walks each output row in chunks of U columns: first every load of the chunk is issued -- the
// U dy pairs and the K x ((U-1)*S + K) input pairs they meet (4 bytes a lane, a warp reading
// 128 contiguous bytes) -- so that a warp has ~40 independent loads in flight, then the chunk's
// U*K*K packed multiply-adds run. Partials go to ws[slice][tap][C] (coalesced float2 stores).
template <typename T, int K, int S, int U>
__global__ void __launch_bounds__(128) wgrad_depthwise_nhwc_kernel(const T* __restrict__ x,
                                                                    const T* __restrict__ dy,
                                                                    float* __restrict__ ws,
                                                                    Conv2d p, int rows) {
  constexpr int NC = (U - 1) * S + K;         // input columns a chunk reads
  const int CW = p.C_in / 2;                  // channel pairs = 32-bit words per pixel
  const int cp = blockIdx.x * blockDim.x + threadIdx.x;
  if (cp >= CW) return;
  const unsigned int* xw = reinterpret_cast<const unsigned int*>(x);
  const unsigned int* dyw = reinterpret_cast<const unsigned int*>(dy);
  const int R = p.N * p.Ho;
  const int r0 = blockIdx.y * rows, r1 = min(R, r0 + rows);

  float2 acc[K][K];
#pragma unroll
  for (int kh = 0; kh < K; ++kh)
#pragma unroll
    for (int kw = 0; kw < K; ++kw) acc[kh][kw] = make_float2(0.0f, 0.0f);

  for (int row = r0; row < r1; ++row) {
    const int n = row / p.Ho, ho = row - n * p.Ho;
    const int h0 = ho * S - p.pad;
    long long rb[K];   // word index of (n, h0 + kh, 0, cp); -1 when the row is padding
#pragma unroll
    for (int kh = 0; kh < K; ++kh) {
      const int h = h0 + kh;
      rb[kh] = (h >= 0 && h < p.H) ? ((long long)n * p.H + h) * p.W * CW + cp : -1;
    }
    const unsigned int* drow = dyw + ((long long)n * p.Ho + ho) * p.Wo * CW + cp;
    for (int wo0 = 0; wo0 < p.Wo; wo0 += U) {
      const int c0 = wo0 * S - p.pad;
      float2 d[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        d[u] = wo0 + u < p.Wo ? unpack2<T>(__ldg(drow + (long long)(wo0 + u) * CW))
                              : make_float2(0.0f, 0.0f);
      float2 xv[K][NC];
#pragma unroll
      for (int kh = 0; kh < K; ++kh)
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const int col = c0 + j;
          xv[kh][j] = (rb[kh] >= 0 && col >= 0 && col < p.W)
                          ? unpack2<T>(__ldg(xw + rb[kh] + (long long)col * CW))
                          : make_float2(0.0f, 0.0f);
        }
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int kh = 0; kh < K; ++kh)
#pragma unroll
          for (int kw = 0; kw < K; ++kw)
            acc[kh][kw] = ffma2(d[u], xv[kh][u * S + kw], acc[kh][kw]);
    }
  }
  float2* out = reinterpret_cast<float2*>(ws + (long long)blockIdx.y * K * K * p.C_in) + cp;
#pragma unroll
  for (int kh = 0; kh < K; ++kh)
#pragma unroll
    for (int kw = 0; kw < K; ++kw) out[(long long)(kh * K + kw) * CW] = acc[kh][kw];
}

// ------------------------------------------------------------------ depthwise 3x3 weight gradient, TMA-staged
// NHWC, 16-bit, 3x3, dilation 1, stride S = 1 or 2, pad <= 2, C % 8 == 0. The data path of the
// forward 3x3 kernel with the roles of filter and output exchanged: a producer thread streams,
// per tile of BH output rows x 28 output columns x 64 channels, the input box
// ((BH-1)*S+3 rows x 27*S+3 columns, zero fill as the padding) and the matching dy box (zero
// fill past Ho / Wo) through a shared-memory ring; seven compute warps each take 4 output
// columns, a thread one channel pair, and add dy(pair) * x(pair) into 9 fp32-pair accumulators
// with the input rows rolling through registers as in the forward. A CTA owns one channel tile
// and a fixed slice of that tile's spatial tiles (a function of the shape only); at the end the
// seven warps' accumulators are added in warp order in shared memory and written as the CTA's
// partial ws[slice][tap][C]. Every wait is bounded (1 s); on expiry the CTA sets the device
// error word, drains its copies and writes nothing.
constexpr int DWW_CH = 64;                  // channels per tile (128-byte box rows)
constexpr int DWW_R = 4;                    // output columns per thread
constexpr int DWW_NG = 7;                   // compute warps (column groups)
constexpr int DWW_BW = DWW_R * DWW_NG;      // output columns per tile
constexpr int DWW_THREADS = 32 + 32 * DWW_NG;
constexpr int DWW_MAX_STAGES = 4;
constexpr int DWW_CTAS = 296;               // two CTAs on each of 148 SMs; a fixed constant
                                            // so the summation order never depends on the device
constexpr size_t DWW_SMEM_CTA = 110 * 1024; // two CTAs per SM

template <int S> __host__ __device__ constexpr int dww_iw() { return (DWW_BW - 1) * S + 3; }
template <int S> __host__ __device__ constexpr int dww_bh() { return S == 1 ? 4 : 2; }

struct DwwParams {
  int N, C, Ho, Wo, pad;
  int n_ct, n_ht, n_wt, tiles_per_ct, slices, stages;
  unsigned int x_bytes, stage_bytes, tx_bytes;
};

template <typename T, int S>
__global__ void __launch_bounds__(DWW_THREADS, 2)
    wgrad_dw3_tma_kernel(const __grid_constant__ CUtensorMap tmx,
                         const __grid_constant__ CUtensorMap tmd, float* __restrict__ ws,
                         const DwwParams P, unsigned int* err) {
  using namespace ptx;
  pdl_launch_dependents();   // the slice sum may be scheduled as this grid's CTAs finish
  constexpr int BH = dww_bh<S>();
  constexpr int IW = dww_iw<S>();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 128u);
  unsigned long long* full =
      reinterpret_cast<unsigned long long*>(smem + (size_t)P.stages * P.stage_bytes);
  unsigned long long* empty = full + DWW_MAX_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + DWW_MAX_STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ct = blockIdx.x / P.slices, sl = blockIdx.x - ct * P.slices;
  const int t_begin = (int)((long long)P.tiles_per_ct * sl / P.slices);
  const int t_end = (int)((long long)P.tiles_per_ct * (sl + 1) / P.slices);
  if (threadIdx.x == 0) {
    for (int i = 0; i < P.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], (unsigned int)DWW_NG);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmd);
  }
  __syncthreads();

  float2 acc[3][3];
#pragma unroll
  for (int kh = 0; kh < 3; ++kh)
#pragma unroll
    for (int kw = 0; kw < 3; ++kw) acc[kh][kw] = make_float2(0.0f, 0.0f);

  if (warp == 0) {
    if (lane == 0) {
      int st = 0;
      unsigned int ph = 0;
      long long issued = 0;
      for (int t = t_begin; t < t_end; ++t) {
        const int tw = t % P.n_wt;
        const int r = t / P.n_wt;
        const int th = r % P.n_ht, n = r / P.n_ht;
        if (!mbar_try_wait(&empty[st], ph ^ 1u) &&
            !mbar_wait(&empty[st], ph ^ 1u, abort_flag, err, 32u))
          break;
        unsigned char* dst = smem + (size_t)st * P.stage_bytes;
        mbar_arrive_expect_tx(&full[st], P.tx_bytes);
        tma_load_4d(dst, &tmx, &full[st], ct * DWW_CH, tw * DWW_BW * S - P.pad,
                    th * BH * S - P.pad, n);
        tma_load_4d(dst + P.x_bytes, &tmd, &full[st], ct * DWW_CH, tw * DWW_BW, th * BH, n);
        ++issued;
        if (++st == P.stages) {
          st = 0;
          ph ^= 1u;
        }
      }
      // copies in flight land before the ring is reused below (instant on the normal path)
      const unsigned long long dl = drain_deadline();
      for (long long q = (issued > P.stages ? issued - P.stages : 0); q < issued; ++q)
        mbar_wait_until(&full[q % P.stages], (unsigned int)((q / P.stages) & 1), dl, err,
                        ERR_DRAIN);
    }
  } else {
    constexpr int NIN = (DWW_R - 1) * S + 3;     // input columns a thread reads per row
    constexpr int row_w = IW * (DWW_CH / 2);     // 32-bit words per input box row
    constexpr int drow_w = DWW_BW * (DWW_CH / 2);
    const int g = warp - 1;
    int st = 0;
    unsigned int ph = 0;
    for (int t = t_begin; t < t_end; ++t) {
      bool got = mbar_try_wait(&full[st], ph);
      if (!got) got = mbar_wait(&full[st], ph, abort_flag, err, 32u);
      if (!__all_sync(0xffffffffu, got)) break;
      const uint32_t* px = reinterpret_cast<const uint32_t*>(smem + (size_t)st * P.stage_bytes) +
                           (g * DWW_R * S) * (DWW_CH / 2) + lane;
      const uint32_t* pd =
          reinterpret_cast<const uint32_t*>(smem + (size_t)st * P.stage_bytes + P.x_bytes) +
          (g * DWW_R) * (DWW_CH / 2) + lane;
      float2 in[3][NIN];                         // input row r lives in slot r % 3
      auto load_row = [&](int r, float2 (&dst)[NIN]) {
#pragma unroll
        for (int i = 0; i < NIN; ++i) dst[i] = unpack2<T>(px[r * row_w + i * (DWW_CH / 2)]);
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
        float2 d[DWW_R];
#pragma unroll
        for (int r = 0; r < DWW_R; ++r) d[r] = unpack2<T>(pd[j * drow_w + r * (DWW_CH / 2)]);
#pragma unroll
        for (int kh = 0; kh < 3; ++kh) {
          const int slot = (j * S + kh) % 3;
#pragma unroll
          for (int kw = 0; kw < 3; ++kw)
#pragma unroll
            for (int r = 0; r < DWW_R; ++r)
              acc[kh][kw] = ffma2(d[r], in[slot][r * S + kw], acc[kh][kw]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == P.stages) {
        st = 0;
        ph ^= 1u;
      }
    }
  }
  __syncthreads();
  if (*abort_flag) return;
  // the ring is idle (every copy has landed and been read): add the warps' sums in warp order
  float2* red = reinterpret_cast<float2*>(smem);   // [warp][tap][lane]
  if (warp >= 1) {
#pragma unroll
    for (int kh = 0; kh < 3; ++kh)
#pragma unroll
      for (int kw = 0; kw < 3; ++kw) red[((warp - 1) * 9 + kh * 3 + kw) * 32 + lane] = acc[kh][kw];
  }
  __syncthreads();
  if (warp == 1) {
    const int ch = ct * DWW_CH + 2 * lane;
    if (ch < P.C) {
      float2* out = reinterpret_cast<float2*>(ws + (long long)sl * 9 * P.C) + ch / 2;
#pragma unroll
      for (int tap = 0; tap < 9; ++tap) {
        float2 v = red[tap * 32 + lane];
#pragma unroll
        for (int gg = 1; gg < DWW_NG; ++gg) {
          const float2 u = red[(gg * 9 + tap) * 32 + lane];
          v.x += u.x;
          v.y += u.y;
        }
        out[(long long)tap * (P.C / 2)] = v;
      }
    }
  }
}

DwwParams dww_params(const Conv2d& p) {
  DwwParams P{};
  const int S = p.stride;
  const int BH = S == 1 ? dww_bh<1>() : dww_bh<2>();
  const int IW = S == 1 ? dww_iw<1>() : dww_iw<2>();
  const int IH = (BH - 1) * S + 3;
  P.N = p.N; P.C = p.C_in; P.Ho = p.Ho; P.Wo = p.Wo; P.pad = p.pad;
  P.n_ct = (p.C_in + DWW_CH - 1) / DWW_CH;
  P.n_ht = (p.Ho + BH - 1) / BH;
  P.n_wt = (p.Wo + DWW_BW - 1) / DWW_BW;
  P.tiles_per_ct = (int)((long long)p.N * P.n_ht * P.n_wt);   // < 2^31: checked on support
  int sl = DWW_CTAS / P.n_ct;
  if (sl < 1) sl = 1;
  P.slices = sl;
  P.x_bytes = (unsigned int)((DWW_CH * IW * IH * 2 + 127) & ~127);
  const unsigned int d_bytes = (unsigned int)(DWW_CH * DWW_BW * BH * 2);
  P.tx_bytes = (unsigned int)(DWW_CH * IW * IH * 2) + d_bytes;
  P.stage_bytes = (P.x_bytes + d_bytes + 127u) & ~127u;
  int stages = (int)((DWW_SMEM_CTA - 1024) / P.stage_bytes);
  if (stages > DWW_MAX_STAGES) stages = DWW_MAX_STAGES;
  P.stages = stages;
  return P;
}

size_t dww_smem(const DwwParams& P) {
  return 128 + (size_t)P.stages * P.stage_bytes + 2 * DWW_MAX_STAGES * 8 + 16;
}

template <typename T, int S>
cudaError_t launch_dww(const Conv2d& p, const void* x, const void* dy, float* ws,
                       const DwwParams& P, cudaStream_t s) {
  constexpr int BH = dww_bh<S>();
  constexpr int IW = dww_iw<S>();
  if (P.stages < 2 || (long long)P.n_ct * P.slices > 0x7fffffffLL) return cudaErrorInvalidValue;
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  CUtensorMap tmx, tmd;
  const cuuint64_t xd[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                            (cuuint64_t)p.N};
  const cuuint64_t xs[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                            (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t xb[4] = {DWW_CH, (cuuint32_t)IW, (cuuint32_t)((BH - 1) * S + 3), 1};
  if (enc(&tmx, dt, 4, const_cast<void*>(x), xd, xs, xb, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t dd[4] = {(cuuint64_t)p.C_out, (cuuint64_t)p.Wo, (cuuint64_t)p.Ho,
                            (cuuint64_t)p.N};
  const cuuint64_t ds[3] = {(cuuint64_t)p.C_out * 2, (cuuint64_t)p.Wo * p.C_out * 2,
                            (cuuint64_t)p.Ho * p.Wo * p.C_out * 2};
  const cuuint32_t db[4] = {DWW_CH, DWW_BW, BH, 1};
  if (enc(&tmd, dt, 4, const_cast<void*>(dy), dd, ds, db, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  static std::atomic<unsigned int> configured{0};
  const size_t smem = dww_smem(P);
  cudaError_t e = set_max_dynamic_smem((const void*)wgrad_dw3_tma_kernel<T, S>, smem, configured);
  if (e != cudaSuccess) return e;
  wgrad_dw3_tma_kernel<T, S><<<(unsigned)(P.n_ct * P.slices), DWW_THREADS, smem, s>>>(
      tmx, tmd, ws, P, device_error_word());
  return cudaGetLastError();
}

// ------------------------------------------------------------------ depthwise data gradient
// NHWC, 16-bit, groups == C_in == C_out, C % VEC == 0, dilation 1, K x K, any stride and pad
// (the shapes that are not a stride-1 forward convolution). A thread owns VEC channels (one
// 16-, 8- or 4-byte vector) and keeps their K x K filter in fp32 registers; it walks dx pixels
// (n, h, w) and for each adds the taps (kh, kw) with h + pad - kh and w + pad - kw multiples of
// the stride -- on average K*K/S^2 of them -- as vector loads of dy, then stores one vector.
// Consecutive threads take consecutive channel vectors (contiguous loads and stores).
template <int VEC> struct DVec;
template <> struct DVec<8> { using type = uint4; };
template <> struct DVec<4> { using type = uint2; };
template <> struct DVec<2> { using type = unsigned int; };

template <typename T, int K, int S, int VEC>
__global__ void __launch_bounds__(256) dgrad_depthwise_nhwc_kernel(const T* __restrict__ dy,
                                                                    const T* __restrict__ w,
                                                                    T* __restrict__ dx,
                                                                    Conv2d p) {
  using V = typename DVec<VEC>::type;
  constexpr int NW = VEC / 2;
  const int CV = p.C_in / VEC;
  const int cv = blockIdx.x * blockDim.x + threadIdx.x;
  if (cv >= CV) return;
  const int c = cv * VEC;
  float wr[K * K][VEC];
#pragma unroll
  for (int t = 0; t < K * K; ++t)
#pragma unroll
    for (int v = 0; v < VEC; ++v) wr[t][v] = Elem<T>::to_f32(w[(long long)(c + v) * K * K + t]);
  const int rows = p.N * p.H;
  for (int r = blockIdx.y; r < rows; r += gridDim.y) {      // dx rows (n, h)
    const int n = r / p.H, h = r - n * p.H;
    const T* drow[K];                                       // dy row of tap kh, or null
#pragma unroll
    for (int kh = 0; kh < K; ++kh) {
      const int th = h + p.pad - kh;
      drow[kh] = (th >= 0 && th % S == 0 && th / S < p.Ho)
                     ? dy + ((long long)n * p.Ho + th / S) * p.Wo * p.C_out + c
                     : nullptr;
    }
    T* xrow = dx + (long long)r * p.W * p.C_in + c;
    for (int wi = threadIdx.y; wi < p.W; wi += blockDim.y) {
      float2 acc[NW];
#pragma unroll
      for (int i = 0; i < NW; ++i) acc[i] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int kw = 0; kw < K; ++kw) {
        const int tw = wi + p.pad - kw;
        if (tw < 0 || tw % S != 0 || tw / S >= p.Wo) continue;
        const int col = tw / S;
#pragma unroll
        for (int kh = 0; kh < K; ++kh) {
          if (drow[kh] == nullptr) continue;
          const V d = __ldg(reinterpret_cast<const V*>(drow[kh] + (long long)col * p.C_out));
          const unsigned int* du = reinterpret_cast<const unsigned int*>(&d);
#pragma unroll
          for (int i = 0; i < NW; ++i)
            acc[i] = ffma2(unpack2<T>(du[i]),
                           make_float2(wr[kh * K + kw][2 * i], wr[kh * K + kw][2 * i + 1]),
                           acc[i]);
        }
      }
      V o;
      unsigned int* ou = reinterpret_cast<unsigned int*>(&o);
#pragma unroll
      for (int i = 0; i < NW; ++i) ou[i] = pack2<T>(acc[i]);
      *reinterpret_cast<V*>(xrow + (long long)wi * p.C_in) = o;
    }
  }
}

// ------------------------------------------------------------------ stride-2 depthwise 3x3 dgrad
// The data gradient of a depthwise 3x3, stride 2, pad 1 layer is an upsampling: dx pixel (h, w)
// collects w[kh][kw] * dy[(h + 1 - kh) / 2][(w + 1 - kw) / 2] over the taps whose numerators are
// even -- one tap at (even h, even w), two at mixed parities, four at (odd, odd). A tile is
// DGS_BH dx rows x 28 dx columns x 64 channels (h0, w0 even); its dy box is rows
// [h0/2, h0/2 + BH/2] x columns [w0/2, w0/2 + 14] x 64 channels (TMA, zero fill past the
// edges), in a ring of stages filled by a producer warp. Seven compute warps own 4 dx columns
// each for all 32 channel pairs: a thread's 4 columns read dy columns 2g .. 2g+2 of the box,
// so each dy word it needs is read once per tile, and the 9 taps of its channel pair stay in
// registers. Each warp stages its [BH][4][64] dx box in shared memory and writes it with one
// TMA store (clipped at the image's edges), as in the forward 3x3 kernel.
constexpr int DGS_R = 4;                    // dx columns per thread
constexpr int DGS_NG = 7;                   // compute warps
constexpr int DGS_BW = DGS_R * DGS_NG;      // dx columns per tile (even)
constexpr int DGS_BH = 8;                   // dx rows per tile (even)
constexpr int DGS_IW = DGS_BW / 2 + 1;      // dy box columns
constexpr int DGS_IH = DGS_BH / 2 + 1;      // dy box rows
constexpr int DGS_CH = 64;
constexpr int DGS_THREADS = 32 + 32 * DGS_NG;
constexpr int DGS_MAX_STAGES = 6;
constexpr size_t DGS_SMEM_CTA = 72 * 1024;  // three CTAs per SM

struct DgsParams {
  int N, H, W, C, Ho, Wo;
  int n_ct, n_wt, n_ht, num_tiles, stages;
  unsigned int stage_bytes, tx_bytes;
};

template <typename T>
__global__ void __launch_bounds__(DGS_THREADS, 3)
    dgrad_dw3s2_tma_kernel(const __grid_constant__ CUtensorMap tmd,
                           const __grid_constant__ CUtensorMap tmx, const T* __restrict__ w,
                           const DgsParams P, unsigned int* err) {
  using namespace ptx;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 128u);
  unsigned char* ostage = smem + (size_t)P.stages * P.stage_bytes;
  unsigned long long* full =
      reinterpret_cast<unsigned long long*>(ostage + (size_t)DGS_BH * DGS_BW * DGS_CH * 2);
  unsigned long long* empty = full + DGS_MAX_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + DGS_MAX_STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = (int)((long long)P.num_tiles * blockIdx.x / gridDim.x);
  const int t_end = (int)((long long)P.num_tiles * (blockIdx.x + 1) / gridDim.x);
  // tile t: tw fastest, then th, n, channel tile
  auto decode = [&](int t, int& ct, int& n, int& th, int& tw) {
    tw = t % P.n_wt;
    int r = t / P.n_wt;
    th = r % P.n_ht;
    r /= P.n_ht;
    n = r % P.N;
    ct = r / P.N;
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], DGS_NG);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmd);
    prefetch_tmap(&tmx);
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      unsigned int ph = 0;
      long long issued = 0;
      for (int t = t_begin; t < t_end; ++t) {
        if (!mbar_try_wait(&empty[s], ph ^ 1u) &&
            !mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, 128u))
          break;
        int ct, n, th, tw;
        decode(t, ct, n, th, tw);
        mbar_arrive_expect_tx(&full[s], P.tx_bytes);
        tma_load_4d(smem + (size_t)s * P.stage_bytes, &tmd, &full[s], ct * DGS_CH,
                    tw * (DGS_BW / 2), th * (DGS_BH / 2), n);
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
    const int cp = lane, g = warp - 1;
    int prev_ct = -1;
    float2 wv[3][3];
    int s = 0;
    unsigned int ph = 0;
    unsigned char* wstage = ostage + (size_t)g * DGS_BH * DGS_R * DGS_CH * 2;
    unsigned int* orow = reinterpret_cast<unsigned int*>(wstage) + cp;
    for (int t = t_begin; t < t_end; ++t) {
      bool got = mbar_try_wait(&full[s], ph);
      if (!got) got = mbar_wait(&full[s], ph, abort_flag, err, 128u);
      if (!__all_sync(0xffffffffu, got)) break;
      if (lane == 0) bulk_wait_read0();              // this warp's previous store has read it
      __syncwarp();
      int ct, n, th, tw;
      decode(t, ct, n, th, tw);
      const int ch = ct * DGS_CH + 2 * cp;
      const bool ch_ok = ch < P.C;
      if (ct != prev_ct) {
        prev_ct = ct;
#pragma unroll
        for (int kh = 0; kh < 3; ++kh)
#pragma unroll
          for (int kw = 0; kw < 3; ++kw)
            wv[kh][kw] = ch_ok ? make_float2(Elem<T>::to_f32(w[ch * 9 + kh * 3 + kw]),
                                             Elem<T>::to_f32(w[(ch + 1) * 9 + kh * 3 + kw]))
                               : make_float2(0.f, 0.f);
      }
      // box word (row, column, pair) = (row * IW + column) * 32 + pair; this thread's dy
      // columns are 2g .. 2g + 2
      const uint32_t* pd = reinterpret_cast<const uint32_t*>(smem + (size_t)s * P.stage_bytes) +
                           (2 * g) * (DGS_CH / 2) + cp;
      float2 d[DGS_IH][3];
#pragma unroll
      for (int r = 0; r < DGS_IH; ++r)
#pragma unroll
        for (int m = 0; m < 3; ++m) d[r][m] = unpack2<T>(pd[(r * DGS_IW + m) * (DGS_CH / 2)]);
#pragma unroll
      for (int j = 0; j < DGS_BH; ++j) {
        float2 acc[DGS_R];
#pragma unroll
        for (int r = 0; r < DGS_R; ++r) acc[r] = make_float2(0.f, 0.f);
        // (kh, dy box row) pairs of dx row j: kh = 1 from row j/2 (even j); kh = 0 from row
        // (j+1)/2 and kh = 2 from row (j-1)/2 (odd j)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int kh = (j % 2 == 0) ? 1 : (q == 0 ? 0 : 2);
          if (j % 2 == 0 && q == 1) continue;
          const int row = (j % 2 == 0) ? j / 2 : (q == 0 ? (j + 1) / 2 : (j - 1) / 2);
          // dx column 4g + r: even r: kw = 1 from dy column r/2; odd r: kw = 0 from
          // (r+1)/2 and kw = 2 from (r-1)/2
          acc[0] = ffma2(wv[kh][1], d[row][0], acc[0]);
          acc[1] = ffma2(wv[kh][0], d[row][1], acc[1]);
          acc[1] = ffma2(wv[kh][2], d[row][0], acc[1]);
          acc[2] = ffma2(wv[kh][1], d[row][1], acc[2]);
          acc[3] = ffma2(wv[kh][0], d[row][2], acc[3]);
          acc[3] = ffma2(wv[kh][2], d[row][1], acc[3]);
        }
#pragma unroll
        for (int r = 0; r < DGS_R; ++r)
          orow[(j * DGS_R + r) * (DGS_CH / 2)] = pack2<T>(acc[r]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s]);
        if (tw * DGS_BW + g * DGS_R < P.W) {   // a box wholly right of the image is skipped
          tma_store_4d(&tmx, wstage, ct * DGS_CH, tw * DGS_BW + g * DGS_R, th * DGS_BH, n);
          bulk_commit();
        }
      }
      if (++s == P.stages) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (lane == 0) bulk_wait0();
  }
  __syncthreads();
}

// ------------------------------------------------------------------ wide-group weight gradient
// NHWC, 16-bit, C_in/g and C_out/g multiples of 8 and at least 32. Per group and tap (kh, kw),
// dw[co][kh][kw][ci] over the group's filters and channels is a sum over output positions p of
// the outer product dy[p][co] * x[tap-shifted p][ci]. A CTA owns one 128 x 128 (co, ci) tile of
// one (group, tap) and one fixed slice of positions; its 256 threads own 8 x 8 fp32
// accumulators each. Each step stages 16 positions' dy row segment ([16][128 co]) and their
// tap-shifted input segment ([16][128 ci], zero where the tap falls in the padding) in shared
// memory as fp32 -- one 16-byte load per thread per operand, issued before the previous step's
// multiply-adds -- and every thread then reads two 4-float vectors of each per position.
constexpr int WT_TILE = 128;
constexpr int WT_K = 16;

template <typename T>
__global__ void __launch_bounds__(256) wgrad_tiled_nhwc_kernel(const T* __restrict__ x,
                                                                const T* __restrict__ dy,
                                                                float* __restrict__ ws,
                                                                Conv2d p, int n_mt, int n_nt,
                                                                long long E, int per_slice) {
  __shared__ __align__(16) float sA[2][WT_K][WT_TILE + 4];   // dy: [position][co]
  __shared__ __align__(16) float sB[2][WT_K][WT_TILE + 4];   // x:  [position][ci]
  const int taps = p.kH * p.kW;
  int t = blockIdx.x;
  const int nt = t % n_nt; t /= n_nt;
  const int mt = t % n_mt; t /= n_mt;
  const int tap = t % taps;
  const int g = t / taps;
  const int kh = tap / p.kW, kw = tap - kh * p.kW;
  const long long P = (long long)p.N * p.Ho * p.Wo;
  const long long p0 = (long long)blockIdx.y * per_slice;
  const long long p1 = min(P, p0 + per_slice);

  const int tid = threadIdx.x;
  const int lk = tid / 16, lv = tid % 16;          // loader: position lk, 8-channel vector lv
  const int co_l = mt * WT_TILE + lv * 8;          // within the group
  const int ci_l = nt * WT_TILE + lv * 8;
  const bool co_ok = co_l < p.cpg_out, ci_ok = ci_l < p.cpg_in;
  const T* dyg = dy + (long long)g * p.cpg_out + co_l;
  const T* xg = x + (long long)g * p.cpg_in + ci_l;

  auto fetch = [&](long long pos, uint4& va, uint4& vb) {
    va = make_uint4(0, 0, 0, 0);
    vb = make_uint4(0, 0, 0, 0);
    if (pos >= p1) return;
    if (co_ok) va = __ldg(reinterpret_cast<const uint4*>(dyg + pos * p.C_out));
    if (!ci_ok) return;
    const int pi = (int)pos;                       // N*Ho*Wo < 2^31 (checked on the host)
    const int wo = pi % p.Wo;
    const int r = pi / p.Wo;
    const int ho = r % p.Ho, n = r / p.Ho;
    const int h = ho * p.stride - p.pad + kh * p.dil;
    const int w = wo * p.stride - p.pad + kw * p.dil;
    if (h < 0 || h >= p.H || w < 0 || w >= p.W) return;
    vb = __ldg(reinterpret_cast<const uint4*>(xg + (((long long)n * p.H + h) * p.W + w) * p.C_in));
  };
  auto stage = [&](int buf, const uint4& va, const uint4& vb) {
    const unsigned int* ua = reinterpret_cast<const unsigned int*>(&va);
    const unsigned int* ub = reinterpret_cast<const unsigned int*>(&vb);
    float4* da = reinterpret_cast<float4*>(&sA[buf][lk][lv * 8]);
    float4* db = reinterpret_cast<float4*>(&sB[buf][lk][lv * 8]);
    float2 a0 = unpack2<T>(ua[0]), a1 = unpack2<T>(ua[1]), a2 = unpack2<T>(ua[2]),
           a3 = unpack2<T>(ua[3]);
    float2 b0 = unpack2<T>(ub[0]), b1 = unpack2<T>(ub[1]), b2 = unpack2<T>(ub[2]),
           b3 = unpack2<T>(ub[3]);
    da[0] = make_float4(a0.x, a0.y, a1.x, a1.y);
    da[1] = make_float4(a2.x, a2.y, a3.x, a3.y);
    db[0] = make_float4(b0.x, b0.y, b1.x, b1.y);
    db[1] = make_float4(b2.x, b2.y, b3.x, b3.y);
  };

  const int ty = tid / 16, tx = tid % 16;          // compute: rows ty*4 (+64), cols tx*4 (+64)
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  uint4 va, vb;
  fetch(p0 + lk, va, vb);
  stage(0, va, vb);
  __syncthreads();
  int buf = 0;
  for (long long base = p0; base < p1; base += WT_K) {
    const bool more = base + WT_K < p1;
    if (more) fetch(base + WT_K + lk, va, vb);     // next step's loads fly during the math
#pragma unroll
    for (int k = 0; k < WT_K; ++k) {
      const float4 a_lo = *reinterpret_cast<const float4*>(&sA[buf][k][ty * 4]);
      const float4 a_hi = *reinterpret_cast<const float4*>(&sA[buf][k][64 + ty * 4]);
      const float4 b_lo = *reinterpret_cast<const float4*>(&sB[buf][k][tx * 4]);
      const float4 b_hi = *reinterpret_cast<const float4*>(&sB[buf][k][64 + tx * 4]);
      const float a[8] = {a_lo.x, a_lo.y, a_lo.z, a_lo.w, a_hi.x, a_hi.y, a_hi.z, a_hi.w};
      const float b[8] = {b_lo.x, b_lo.y, b_lo.z, b_lo.w, b_hi.x, b_hi.y, b_hi.z, b_hi.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) {
      stage(buf ^ 1, va, vb);
      __syncthreads();
      buf ^= 1;
    }
  }
  // partial of this slice for dw[g*cpg_out + co][kh][kw][ci]
  float* out = ws + (long long)blockIdx.y * E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int co = mt * WT_TILE + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (co >= p.cpg_out) continue;
    float* row = out + (((long long)(g * p.cpg_out + co) * p.kH + kh) * p.kW + kw) * p.cpg_in;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int ci = nt * WT_TILE + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (ci < p.cpg_in) row[ci] = acc[i][j];
    }
  }
}

size_t staged_bytes(long long elems) { return ((size_t)elems * 2 + 255) / 256 * 256; }

// dw from the slice partials: dw[e(q)] = sum over slices s of ws[s][q], q the partial index.
// A CTA takes 32 consecutive q (one per lane, so each warp load is 128 contiguous bytes) and its
// 8 warps split the slices: warp j adds slices j, j+8, j+16, ... in that order, then the 8 warp
// sums are added in warp order -- a fixed order, so the result is bitwise reproducible.
// Partial order -> dw index e: SUM_SAME e = q; SUM_TAP_MAJOR partials are [s][tap][C] and
// e = c * taps + tap (the depthwise kernels); SUM_TO_NCHW partials are in the NHWC weight order
// (co, kh, kw, ci) and e is the NCHW weight order (co, ci, kh, kw).
enum { SUM_SAME = 0, SUM_TAP_MAJOR = 1, SUM_TO_NCHW = 2 };

template <typename T, int MODE>
__global__ void __launch_bounds__(256) wgrad_sum_kernel(const float* __restrict__ ws,
                                                         T* __restrict__ dw, long long E,
                                                         int S, int taps, int cpg_in, int kW) {
  ptx::pdl_wait();   // the partials of the kernel before (launch_pdl)
  __shared__ float part[8][33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long q = (long long)blockIdx.x * 32 + lane;
  float acc = 0.0f;
  if (q < E) {
#pragma unroll 4
    for (int s = warp; s < S; s += 8) acc += ws[(long long)s * E + q];
  }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && q < E) {
    float t = part[0][lane];
#pragma unroll
    for (int j = 1; j < 8; ++j) t += part[j][lane];
    long long e = q;
    if (MODE == SUM_TAP_MAJOR) {
      const long long C = E / taps;
      e = (q % C) * taps + q / C;
    } else if (MODE == SUM_TO_NCHW) {
      const long long ci = q % cpg_in, r = q / cpg_in;   // r = (co * kH + kh) * kW + kw
      const long long tap = r % taps, co = r / taps;     // tap = kh * kW + kw
      e = (co * cpg_in + ci) * taps + tap;
      (void)kW;
    }
    dw[e] = Elem<T>::from_f32(t);
  }
}

unsigned sum_grid(long long E) { return (unsigned)((E + 31) / 32); }

unsigned grid_for(long long total, int threads) {
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148LL * 64) blocks = 148LL * 64;   // grid-stride beyond 64 blocks per SM
  return (unsigned)(blocks < 1 ? 1 : blocks);
}

template <typename T>
cudaError_t flip_typed(const Conv2d& p, const void* w, void* wt, cudaStream_t s) {
  const long long total = (long long)p.C_out * p.cpg_in * p.kH * p.kW;
  const long long E = (long long)p.cpg_in * p.kH * p.kW;
  // the tiled transpose where its 64 x 64 tiles are mostly full (wide groups); narrow groups
  // (a depthwise filter is 9 elements) keep the element-wise kernel, which launches no
  // mostly idle tiles
  if (p.layout == GCONV_NHWC && sizeof(T) == 2 && p.cpg_out >= 32 && E >= 32 &&
      (E + 63) / 64 <= INT32_MAX && (p.cpg_out + 63) / 64 <= 65535 && p.groups <= 65535) {
    const dim3 grid((unsigned)((E + 63) / 64), (unsigned)((p.cpg_out + 63) / 64),
                    (unsigned)p.groups);
    flip_weight_nhwc_tiled_kernel<T><<<grid, 256, 0, s>>>((const T*)w, (T*)wt, p.cpg_in,
                                                          p.cpg_out, p.kH * p.kW);
    return cudaGetLastError();
  }
  if (p.layout == GCONV_NHWC)
    flip_transpose_weight_kernel<T, GCONV_NHWC><<<grid_for(total, 256), 256, 0, s>>>(
        (const T*)w, (T*)wt, p, total);
  else
    flip_transpose_weight_kernel<T, GCONV_NCHW><<<grid_for(total, 256), 256, 0, s>>>(
        (const T*)w, (T*)wt, p, total);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dgrad_typed(const Conv2d& p, const void* dy, const void* w, void* dx,
                        cudaStream_t s) {
  const long long total = (long long)p.N * p.C_in * p.H * p.W;
  if (total == 0) return cudaSuccess;
  if (p.layout == GCONV_NHWC)
    dgrad_generic_kernel<T, GCONV_NHWC><<<grid_for(total, 256), 256, 0, s>>>(
        (const T*)dy, (const T*)w, (T*)dx, p, total);
  else
    dgrad_generic_kernel<T, GCONV_NCHW><<<grid_for(total, 256), 256, 0, s>>>(
        (const T*)dy, (const T*)w, (T*)dx, p, total);
  return cudaGetLastError();
}

int dgrad_depthwise_vec(const Conv2d& p) { return p.kH <= 3 ? 8 : (p.kH <= 5 ? 4 : 2); }

template <typename T, int K, int VEC>
cudaError_t dgrad_dw_k(const Conv2d& p, const void* dy, const void* w, void* dx,
                       cudaStream_t s) {
  const int CV = p.C_in / VEC;
  const dim3 block(32, 8);
  const unsigned gx = (unsigned)((CV + 31) / 32);
  long long gy = (long long)p.N * p.H;                       // one dx row per CTA row step
  const long long cap = (WGRAD_TARGET_CTAS + gx - 1) / gx;   // ~8 CTAs per SM in all
  if (gy > cap) gy = cap;
  const dim3 grid(gx, (unsigned)gy);
  if (p.stride == 1)
    dgrad_depthwise_nhwc_kernel<T, K, 1, VEC><<<grid, block, 0, s>>>((const T*)dy, (const T*)w,
                                                                     (T*)dx, p);
  else
    dgrad_depthwise_nhwc_kernel<T, K, 2, VEC><<<grid, block, 0, s>>>((const T*)dy, (const T*)w,
                                                                     (T*)dx, p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dgs(const Conv2d& p, const void* dy, const void* w, void* dx, cudaStream_t s) {
  DgsParams P;
  P.N = p.N; P.H = p.H; P.W = p.W; P.C = p.C_in; P.Ho = p.Ho; P.Wo = p.Wo;
  P.n_ct = (p.C_in + DGS_CH - 1) / DGS_CH;
  P.n_wt = (p.W + DGS_BW - 1) / DGS_BW;
  P.n_ht = (p.H + DGS_BH - 1) / DGS_BH;
  const long long tiles = (long long)P.n_ct * p.N * P.n_ht * P.n_wt;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  P.num_tiles = (int)tiles;
  P.tx_bytes = (unsigned int)(DGS_CH * DGS_IW * DGS_IH * 2);
  P.stage_bytes = (P.tx_bytes + 127u) & ~127u;
  const size_t ostage = (size_t)DGS_BH * DGS_BW * DGS_CH * 2;
  const size_t fixed = 128 + ostage + 2 * DGS_MAX_STAGES * 8 + 16;
  int stages = (int)((DGS_SMEM_CTA - fixed) / P.stage_bytes);
  if (stages > DGS_MAX_STAGES) stages = DGS_MAX_STAGES;
  if (stages < 2) return cudaErrorInvalidValue;
  P.stages = stages;
  const size_t smem = fixed + (size_t)stages * P.stage_bytes;
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  CUtensorMap tmd, tmx;
  const cuuint64_t ddim[4] = {(cuuint64_t)p.C_out, (cuuint64_t)p.Wo, (cuuint64_t)p.Ho,
                              (cuuint64_t)p.N};
  const cuuint64_t dstr[3] = {(cuuint64_t)p.C_out * 2, (cuuint64_t)p.Wo * p.C_out * 2,
                              (cuuint64_t)p.Ho * p.Wo * p.C_out * 2};
  const cuuint32_t dbox[4] = {DGS_CH, DGS_IW, DGS_IH, 1};
  if (enc(&tmd, dt, 4, const_cast<void*>(dy), ddim, dstr, dbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t xdim[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t xstr[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                              (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t xbox[4] = {DGS_CH, DGS_R, DGS_BH, 1};
  if (enc(&tmx, dt, 4, dx, xdim, xstr, xbox, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)dgrad_dw3s2_tma_kernel<T>, DGS_SMEM_CTA,
                                       configured);
  if (e != cudaSuccess) return e;
  long long grid = (long long)sm_count() * 3;
  if (grid > P.num_tiles) grid = P.num_tiles;
  dgrad_dw3s2_tma_kernel<T><<<(unsigned)grid, DGS_THREADS, smem, s>>>(
      tmd, tmx, (const T*)w, P, device_error_word());
  return cudaGetLastError();
}

template <typename T>
cudaError_t dgrad_dw_typed(const Conv2d& p, const void* dy, const void* w, void* dx,
                           cudaStream_t s) {
  switch (p.kH) {
    case 3: return dgrad_dw_k<T, 3, 8>(p, dy, w, dx, s);
    case 5: return dgrad_dw_k<T, 5, 4>(p, dy, w, dx, s);
    default: return dgrad_dw_k<T, 7, 2>(p, dy, w, dx, s);
  }
}

// Slices of the N*Ho rows for a weight-gradient launch with `blocks_x` CTAs per slice.
void wgrad_slices(const Conv2d& p, long long blocks_x, int* S, int* rows) {
  const long long R = (long long)p.N * p.Ho;
  long long want = (WGRAD_TARGET_CTAS + blocks_x - 1) / blocks_x;
  if (want < 1) want = 1;
  if (want > R) want = R;
  if (want > 65535) want = 65535;
  long long per = (R + want - 1) / want;
  *rows = (int)per;
  *S = (int)((R + per - 1) / per);
}

void tiled_tiles(const Conv2d& p, int* n_mt, int* n_nt) {
  *n_mt = (p.cpg_out + WT_TILE - 1) / WT_TILE;
  *n_nt = (p.cpg_in + WT_TILE - 1) / WT_TILE;
}

// Position slices of the tiled weight gradient: a multiple of WT_K positions each, enough
// slices for ~WGRAD_TARGET_CTAS CTAs in all (a function of the shape only).
void tiled_slices(const Conv2d& p, long long tiles, int* S, int* per) {
  const long long P = (long long)p.N * p.Ho * p.Wo;
  long long want = (WGRAD_TARGET_CTAS + tiles - 1) / tiles;
  const long long max_s = (P + WT_K - 1) / WT_K;
  if (want > max_s) want = max_s;
  if (want > 65535) want = 65535;
  if (want < 1) want = 1;
  long long q = (P + want - 1) / want;
  q = (q + WT_K - 1) / WT_K * WT_K;
  *per = (int)q;
  *S = (int)((P + q - 1) / q);
}

long long tiled_count(const Conv2d& p) {
  int n_mt, n_nt;
  tiled_tiles(p, &n_mt, &n_nt);
  return (long long)p.groups * p.kH * p.kW * n_mt * n_nt;
}

long long wgrad_blocks_x(const Conv2d& p, int kernel) {
  if (kernel == GCONV_KERNEL_WGRAD_DEPTHWISE_NHWC) return (p.C_in / 2 + 127) / 128;
  const long long E = (long long)p.C_out * p.cpg_in * p.kH * p.kW;
  return (E + 255) / 256;
}

template <typename T>
cudaError_t wgrad_typed(const Conv2d& p, const void* x, const void* dy, void* dw, void* ws,
                        int kernel, cudaStream_t s) {
  const long long E = (long long)p.C_out * p.cpg_in * p.kH * p.kW;
  if constexpr (sizeof(T) == 2) {
    if (kernel == GCONV_KERNEL_WGRAD_DW3_TMA) {
      const DwwParams P = dww_params(p);
      cudaError_t e = p.stride == 1 ? launch_dww<T, 1>(p, x, dy, (float*)ws, P, s)
                                    : launch_dww<T, 2>(p, x, dy, (float*)ws, P, s);
      if (e != cudaSuccess) return e;
      return launch_pdl(wgrad_sum_kernel<T, SUM_TAP_MAJOR>, (unsigned)sum_grid(E), 256u, 0, s,
                        (const float*)ws, (T*)dw, E, P.slices, 9, 1, 3);
    }
    const bool tc = kernel == GCONV_KERNEL_WGRAD_TC_NHWC || kernel == GCONV_KERNEL_WGRAD_TC_NCHW;
    const bool to_nchw = kernel == GCONV_KERNEL_WGRAD_TILED_NCHW ||
                         kernel == GCONV_KERNEL_WGRAD_TC_NCHW;
    if (kernel == GCONV_KERNEL_WGRAD_TILED_NHWC || kernel == GCONV_KERNEL_WGRAD_TILED_NCHW || tc) {
      Conv2d q = p;
      q.layout = GCONV_NHWC;
      const T* xt = (const T*)x;
      const T* dt = (const T*)dy;
      float* part = (float*)ws;
      if (to_nchw) {
        // stage x and dy as NHWC at the front of the workspace, partials after them
        const size_t xb = staged_bytes((long long)p.N * p.C_in * p.H * p.W);
        const size_t db = staged_bytes((long long)p.N * p.C_out * p.Ho * p.Wo);
        T* xs = (T*)ws;
        T* ds = (T*)((char*)ws + xb);
        part = (float*)((char*)ws + xb + db);
        cudaError_t e = launch_nchw_to_nhwc16(x, xs, p.N, p.C_in, (long long)p.H * p.W, s);
        if (e == cudaSuccess)
          e = launch_nchw_to_nhwc16(dy, ds, p.N, p.C_out, (long long)p.Ho * p.Wo, s);
        if (e != cudaSuccess) return e;
        xt = xs;
        dt = ds;
      }
      int S;
      cudaError_t e;
      if (tc) {
        S = wgrad_tc_slices(q);
        e = launch_wgrad_tc(q, xt, dt, part, s);
      } else {
        int n_mt, n_nt, per;
        tiled_tiles(q, &n_mt, &n_nt);
        const long long tiles = tiled_count(q);
        tiled_slices(q, tiles, &S, &per);
        wgrad_tiled_nhwc_kernel<T><<<dim3((unsigned)tiles, (unsigned)S), 256, 0, s>>>(
            xt, dt, part, q, n_mt, n_nt, E, per);
        e = cudaGetLastError();
      }
      if (e != cudaSuccess) return e;
      if (to_nchw)
        return launch_pdl(wgrad_sum_kernel<T, SUM_TO_NCHW>, (unsigned)sum_grid(E), 256u, 0, s,
                          part, (T*)dw, E, S, p.kH * p.kW, p.cpg_in, p.kW);
      return launch_pdl(wgrad_sum_kernel<T, SUM_SAME>, (unsigned)sum_grid(E), 256u, 0, s, part,
                        (T*)dw, E, S, 1, 1, 1);
    }
  }
  int S, rows;
  const long long bx = wgrad_blocks_x(p, kernel);
  wgrad_slices(p, bx, &S, &rows);
  float* part = (float*)ws;
  const dim3 grid((unsigned)bx, (unsigned)S);
  if constexpr (sizeof(T) == 2) {
   if (kernel == GCONV_KERNEL_WGRAD_DEPTHWISE_NHWC) {
    const T* xt = (const T*)x;
    const T* dt = (const T*)dy;
    if (p.kH == 3 && p.stride == 1)
      wgrad_depthwise_nhwc_kernel<T, 3, 1, 8><<<grid, 128, 0, s>>>(xt, dt, part, p, rows);
    else if (p.kH == 3)
      wgrad_depthwise_nhwc_kernel<T, 3, 2, 4><<<grid, 128, 0, s>>>(xt, dt, part, p, rows);
    else if (p.stride == 1)
      wgrad_depthwise_nhwc_kernel<T, 5, 1, 4><<<grid, 128, 0, s>>>(xt, dt, part, p, rows);
    else
      wgrad_depthwise_nhwc_kernel<T, 5, 2, 2><<<grid, 128, 0, s>>>(xt, dt, part, p, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_pdl(wgrad_sum_kernel<T, SUM_TAP_MAJOR>, (unsigned)sum_grid(E), 256u, 0, s,
                      part, (T*)dw, E, S, p.kH * p.kW, 1, p.kW);
   }
  }
  if (p.layout == GCONV_NHWC)
    wgrad_generic_kernel<T, GCONV_NHWC><<<grid, 256, 0, s>>>((const T*)x, (const T*)dy, part, p,
                                                            E, rows);
  else
    wgrad_generic_kernel<T, GCONV_NCHW><<<grid, 256, 0, s>>>((const T*)x, (const T*)dy, part, p,
                                                            E, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_pdl(wgrad_sum_kernel<T, SUM_SAME>, (unsigned)sum_grid(E), 256u, 0, s, part,
                    (T*)dw, E, S, 1, 1, 1);
}

}  // namespace

bool dgrad_as_forward(const Conv2d& p) {
  return p.stride == 1 && p.kH == p.kW && p.pad <= p.dil * (p.kH - 1);
}

cudaError_t launch_flip_transpose_weight(const Conv2d& p, const void* w, void* wt,
                                         cudaStream_t s) {
  switch (p.dtype) {
    case GCONV_F32: return flip_typed<float>(p, w, wt, s);
    case GCONV_F16: return flip_typed<__half>(p, w, wt, s);
    default: return flip_typed<__nv_bfloat16>(p, w, wt, s);
  }
}

cudaError_t launch_dgrad_generic(const Conv2d& p, const void* dy, const void* w, void* dx,
                                 cudaStream_t s) {
  switch (p.dtype) {
    case GCONV_F32: return dgrad_typed<float>(p, dy, w, dx, s);
    case GCONV_F16: return dgrad_typed<__half>(p, dy, w, dx, s);
    default: return dgrad_typed<__nv_bfloat16>(p, dy, w, dx, s);
  }
}

bool dgrad_depthwise_supported(const Conv2d& p) {
  return p.layout == GCONV_NHWC && p.dtype != GCONV_F32 && p.groups == p.C_in &&
         p.C_out == p.C_in && p.kH == p.kW && (p.kH == 3 || p.kH == 5 || p.kH == 7) &&
         p.dil == 1 && (p.stride == 1 || p.stride == 2) && p.C_in % dgrad_depthwise_vec(p) == 0 &&
         (long long)p.N * p.H <= 0x7fffffffLL;
}

int dgrad_depthwise_vec_bytes(const Conv2d& p) { return 2 * dgrad_depthwise_vec(p); }

bool dgrad_dw3s2_tma_supported(const Conv2d& p) {
  return p.layout == GCONV_NHWC && p.dtype != GCONV_F32 && p.groups == p.C_in &&
         p.C_out == p.C_in && p.kH == 3 && p.kW == 3 && p.dil == 1 && p.stride == 2 &&
         p.pad == 1 && p.C_in % 8 == 0 && p.N <= 65535 &&
         (long long)((p.C_in + DGS_CH - 1) / DGS_CH) * p.N * ((p.H + DGS_BH - 1) / DGS_BH) *
                 ((p.W + DGS_BW - 1) / DGS_BW) <= 0x7fffffffLL;
}

cudaError_t launch_dgrad_dw3s2_tma(const Conv2d& p, const void* dy, const void* w, void* dx,
                                   cudaStream_t s) {
  if ((long long)p.N * p.H * p.W == 0) return cudaSuccess;
  if (p.dtype == GCONV_F16) return launch_dgs<__half>(p, dy, w, dx, s);
  return launch_dgs<__nv_bfloat16>(p, dy, w, dx, s);
}

cudaError_t launch_dgrad_depthwise(const Conv2d& p, const void* dy, const void* w, void* dx,
                                   cudaStream_t s) {
  if ((long long)p.N * p.H * p.W == 0) return cudaSuccess;
  if (p.dtype == GCONV_F16) return dgrad_dw_typed<__half>(p, dy, w, dx, s);
  return dgrad_dw_typed<__nv_bfloat16>(p, dy, w, dx, s);
}

bool wgrad_dw3_tma_supported(const Conv2d& p) {
  return p.layout == GCONV_NHWC && p.dtype != GCONV_F32 && p.groups == p.C_in &&
         p.C_out == p.C_in && p.kH == 3 && p.kW == 3 && p.dil == 1 &&
         (p.stride == 1 || p.stride == 2) && p.pad <= 2 && p.C_in % 8 == 0 &&
         (long long)p.N * ((p.Ho + dww_bh<2>() - 1) / dww_bh<2>()) *
                 ((p.Wo + DWW_BW - 1) / DWW_BW) <= 0x7fffffffLL;   // tiles of a channel tile
}

bool wgrad_depthwise_supported(const Conv2d& p) {
  return p.layout == GCONV_NHWC && p.dtype != GCONV_F32 && p.groups == p.C_in &&
         p.C_out == p.C_in && p.C_in % 2 == 0 && p.kH == p.kW && (p.kH == 3 || p.kH == 5) &&
         p.dil == 1 && (p.stride == 1 || p.stride == 2);
}

bool wgrad_tiled_supported(const Conv2d& p) {
  // NCHW is staged as NHWC by launch_nchw_to_nhwc16 (grid: HW / 64 x C / 64 x N)
  const bool staging_ok = p.layout == GCONV_NHWC ||
                          (p.N <= 65535 && (long long)p.H * p.W <= 0x7fffffffLL &&
                           (long long)p.Ho * p.Wo <= 0x7fffffffLL &&
                           (p.C_in + 63) / 64 <= 65535 && (p.C_out + 63) / 64 <= 65535);
  return staging_ok && p.dtype != GCONV_F32 && p.cpg_in >= 32 && p.cpg_out >= 32 &&
         p.cpg_in % 8 == 0 && p.cpg_out % 8 == 0 && tiled_count(p) <= 0x7fffffffLL &&
         (long long)p.N * p.Ho * p.Wo <= 0x7fffffffLL;
}

size_t wgrad_workspace(const Conv2d& p, int kernel) {
  if ((long long)p.N * p.Ho == 0) return 0;
  if (kernel == GCONV_KERNEL_WGRAD_DW3_TMA)
    return (size_t)dww_params(p).slices * 9 * (size_t)p.C_in * sizeof(float);
  if (kernel == GCONV_KERNEL_WGRAD_TILED_NHWC || kernel == GCONV_KERNEL_WGRAD_TILED_NCHW ||
      kernel == GCONV_KERNEL_WGRAD_TC_NHWC || kernel == GCONV_KERNEL_WGRAD_TC_NCHW) {
    int S, per;
    if (kernel == GCONV_KERNEL_WGRAD_TC_NHWC || kernel == GCONV_KERNEL_WGRAD_TC_NCHW)
      S = wgrad_tc_slices(p);
    else
      tiled_slices(p, tiled_count(p), &S, &per);
    size_t b = (size_t)S * (size_t)p.C_out * p.cpg_in * p.kH * p.kW * sizeof(float);
    if (kernel == GCONV_KERNEL_WGRAD_TILED_NCHW || kernel == GCONV_KERNEL_WGRAD_TC_NCHW)
      b += staged_bytes((long long)p.N * p.C_in * p.H * p.W) +
           staged_bytes((long long)p.N * p.C_out * p.Ho * p.Wo);
    return b;
  }
  int S, rows;
  wgrad_slices(p, wgrad_blocks_x(p, kernel), &S, &rows);
  const long long E = (long long)p.C_out * p.cpg_in * p.kH * p.kW;
  return (size_t)S * (size_t)E * sizeof(float);
}

cudaError_t launch_wgrad(const Conv2d& p, const void* x, const void* dy, void* dw, void* ws,
                         int kernel, cudaStream_t s) {
  if (p.N == 0) {
    const size_t es = p.dtype == GCONV_F32 ? 4 : 2;
    return cudaMemsetAsync(dw, 0, (size_t)p.C_out * p.cpg_in * p.kH * p.kW * es, s);
  }
  switch (p.dtype) {
    case GCONV_F32: return wgrad_typed<float>(p, x, dy, dw, ws, kernel, s);
    case GCONV_F16: return wgrad_typed<__half>(p, x, dy, dw, ws, kernel, s);
    default: return wgrad_typed<__nv_bfloat16>(p, x, dy, dw, ws, kernel, s);
  }
}

}  // namespace gconv
