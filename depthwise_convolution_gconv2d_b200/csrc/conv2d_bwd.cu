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
// depthwise, narrow groups) run the rest. Other shapes take the gather kernel below.
//
// The weight gradient is a reduction over N*Ho*Wo positions per filter tap. It is
// deterministic: the (n, ho) rows are cut into fixed slices (a function of the shape only),
// each slice's partial sums are accumulated in a fixed order into fp32 workspace slots, and a
// second kernel adds the slices in slice order and rounds once to the data type. No float
// atomics, so repeated calls give bitwise-identical dw on any GPU.
#include "internal.cuh"

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
// pair and one slice of (n, ho) rows; its K x K fp32-pair accumulators and the K x K window of
// input pairs live in registers. Walking along an output row, the window moves S columns:
// K - S columns are kept and S new ones loaded (one 4-byte load per input row and column, a
// warp reading 128 contiguous bytes), and one dy pair feeds K*K packed multiply-adds.
// Partials go to ws[slice][tap][C] (coalesced float2 stores).
template <typename T, int K, int S>
__global__ void __launch_bounds__(128) wgrad_depthwise_nhwc_kernel(const T* __restrict__ x,
                                                                    const T* __restrict__ dy,
                                                                    float* __restrict__ ws,
                                                                    Conv2d p, int rows) {
  static_assert(S < K, "the window keeps K - S columns");
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
    auto load = [&](int kh, int col) -> float2 {
      if (rb[kh] < 0 || col < 0 || col >= p.W) return make_float2(0.0f, 0.0f);
      return unpack2<T>(__ldg(xw + rb[kh] + (long long)col * CW));
    };
    float2 win[K][K];
#pragma unroll
    for (int kh = 0; kh < K; ++kh)
#pragma unroll
      for (int kw = 0; kw < K; ++kw) win[kh][kw] = load(kh, kw - p.pad);
    const unsigned int* drow = dyw + ((long long)n * p.Ho + ho) * p.Wo * CW + cp;
    for (int wo = 0; wo < p.Wo; ++wo) {
      if (wo > 0) {
        const int w0 = wo * S - p.pad;
#pragma unroll
        for (int kh = 0; kh < K; ++kh) {
#pragma unroll
          for (int kw = 0; kw < K - S; ++kw) win[kh][kw] = win[kh][kw + S];
#pragma unroll
          for (int kw = K - S; kw < K; ++kw) win[kh][kw] = load(kh, w0 + kw);
        }
      }
      const float2 d = unpack2<T>(__ldg(drow + (long long)wo * CW));
#pragma unroll
      for (int kh = 0; kh < K; ++kh)
#pragma unroll
        for (int kw = 0; kw < K; ++kw) acc[kh][kw] = ffma2(d, win[kh][kw], acc[kh][kw]);
    }
  }
  float2* out = reinterpret_cast<float2*>(ws + (long long)blockIdx.y * K * K * p.C_in) + cp;
#pragma unroll
  for (int kh = 0; kh < K; ++kh)
#pragma unroll
    for (int kw = 0; kw < K; ++kw) out[(long long)(kh * K + kw) * CW] = acc[kh][kw];
}

// dw[e] = sum over slices s (in order) of the partial of entry e. TAP_MAJOR: partials are laid
// out [s][tap][C] and e = c * taps + tap (the depthwise kernel); otherwise [s][e].
template <typename T, bool TAP_MAJOR>
__global__ void __launch_bounds__(256) wgrad_sum_kernel(const float* __restrict__ ws,
                                                         T* __restrict__ dw, long long E,
                                                         int S, int taps) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  long long src = e;
  if (TAP_MAJOR) {
    const long long C = E / taps;
    src = (e % taps) * C + e / taps;
  }
  float acc = 0.0f;
  for (int s = 0; s < S; ++s) acc += ws[(long long)s * E + src];
  dw[e] = Elem<T>::from_f32(acc);
}

unsigned grid_for(long long total, int threads) {
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148LL * 64) blocks = 148LL * 64;   // grid-stride beyond 64 blocks per SM
  return (unsigned)(blocks < 1 ? 1 : blocks);
}

template <typename T>
cudaError_t flip_typed(const Conv2d& p, const void* w, void* wt, cudaStream_t s) {
  const long long total = (long long)p.C_out * p.cpg_in * p.kH * p.kW;
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

long long wgrad_blocks_x(const Conv2d& p, int kernel) {
  if (kernel == GCONV_KERNEL_WGRAD_DEPTHWISE_NHWC) return (p.C_in / 2 + 127) / 128;
  const long long E = (long long)p.C_out * p.cpg_in * p.kH * p.kW;
  return (E + 255) / 256;
}

template <typename T>
cudaError_t wgrad_typed(const Conv2d& p, const void* x, const void* dy, void* dw, void* ws,
                        int kernel, cudaStream_t s) {
  const long long E = (long long)p.C_out * p.cpg_in * p.kH * p.kW;
  int S, rows;
  const long long bx = wgrad_blocks_x(p, kernel);
  wgrad_slices(p, bx, &S, &rows);
  float* part = (float*)ws;
  const dim3 grid((unsigned)bx, (unsigned)S);
  if constexpr (sizeof(T) == 2) {
   if (kernel == GCONV_KERNEL_WGRAD_DEPTHWISE_NHWC) {
    const T* xt = (const T*)x;
    const T* dt = (const T*)dy;
    if (p.kH == 3 && p.stride == 1) wgrad_depthwise_nhwc_kernel<T, 3, 1><<<grid, 128, 0, s>>>(xt, dt, part, p, rows);
    else if (p.kH == 3) wgrad_depthwise_nhwc_kernel<T, 3, 2><<<grid, 128, 0, s>>>(xt, dt, part, p, rows);
    else if (p.stride == 1) wgrad_depthwise_nhwc_kernel<T, 5, 1><<<grid, 128, 0, s>>>(xt, dt, part, p, rows);
    else wgrad_depthwise_nhwc_kernel<T, 5, 2><<<grid, 128, 0, s>>>(xt, dt, part, p, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wgrad_sum_kernel<T, true><<<(unsigned)((E + 255) / 256), 256, 0, s>>>(part, (T*)dw, E, S,
                                                                          p.kH * p.kW);
    return cudaGetLastError();
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
  wgrad_sum_kernel<T, false><<<(unsigned)((E + 255) / 256), 256, 0, s>>>(part, (T*)dw, E, S, 1);
  return cudaGetLastError();
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

bool wgrad_depthwise_supported(const Conv2d& p) {
  return p.layout == GCONV_NHWC && p.dtype != GCONV_F32 && p.groups == p.C_in &&
         p.C_out == p.C_in && p.C_in % 2 == 0 && p.kH == p.kW && (p.kH == 3 || p.kH == 5) &&
         p.dil == 1 && (p.stride == 1 || p.stride == 2);
}

size_t wgrad_workspace(const Conv2d& p, int kernel) {
  if ((long long)p.N * p.Ho == 0) return 0;
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
