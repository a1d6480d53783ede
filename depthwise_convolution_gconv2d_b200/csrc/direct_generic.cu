// Generic direct grouped convolution: one thread per output element, fp32 FMA accumulation.
//
// Runs any problem the ABI accepts (any groups, kernel size, stride, dilation, padding,
// layout and dtype). It is the kernel for fp32 (no TF32 rounding anywhere) and the path for
// shapes the specialised kernels do not take. The group of output channel co is
// co / (C_out/g) and it reads input channels [g*cpg_in, (g+1)*cpg_in): the grouping of
// "Grouped convolutions" (neon issue #296), output channels group-major. The group offset is
// added once per thread to the input and weight bases -- the "stride the pointer by the group"
// idea from the same thread -- with the group taken from the output index, so all groups run
// in one launch.
#include "internal.cuh"

namespace gconv {
namespace {

// One output element of the group-major convolution: output channel co, pixel (n, ho, wo),
// bias included, fp32 FMA accumulation.
template <typename T, int LAYOUT>
__device__ __forceinline__ float conv_point(const T* __restrict__ x, const T* __restrict__ w,
                                            const T* __restrict__ bias, const Conv2d& p, int n,
                                            int co, int ho, int wo) {
  const int g = co / p.cpg_out;
  const int h0 = ho * p.stride - p.pad;
  const int w0 = wo * p.stride - p.pad;
  float acc = bias ? Elem<T>::to_f32(bias[co]) : 0.0f;
  if (LAYOUT == GCONV_NCHW) {
    // x[n][g*cpg_in + ci][h][w], w[co][ci][kh][kw]
    const T* xg = x + ((long long)n * p.C_in + (long long)g * p.cpg_in) * p.H * p.W;
    const T* wc = w + (long long)co * p.cpg_in * p.kH * p.kW;
    for (int ci = 0; ci < p.cpg_in; ++ci) {
      const T* xc = xg + (long long)ci * p.H * p.W;
      const T* wk = wc + ci * p.kH * p.kW;
      for (int kh = 0; kh < p.kH; ++kh) {
        const int h = h0 + kh * p.dil;
        if (h < 0 || h >= p.H) continue;
        for (int kw = 0; kw < p.kW; ++kw) {
          const int ww = w0 + kw * p.dil;
          if (ww < 0 || ww >= p.W) continue;
          acc = fmaf(Elem<T>::to_f32(wk[kh * p.kW + kw]),
                     Elem<T>::to_f32(xc[(long long)h * p.W + ww]), acc);
        }
      }
    }
  } else {
    // x[n][h][w][g*cpg_in + ci], w[co][kh][kw][ci]
    const T* xn = x + (long long)n * p.H * p.W * p.C_in + (long long)g * p.cpg_in;
    const T* wc = w + (long long)co * p.kH * p.kW * p.cpg_in;
    for (int kh = 0; kh < p.kH; ++kh) {
      const int h = h0 + kh * p.dil;
      if (h < 0 || h >= p.H) continue;
      for (int kw = 0; kw < p.kW; ++kw) {
        const int ww = w0 + kw * p.dil;
        if (ww < 0 || ww >= p.W) continue;
        const T* xp = xn + ((long long)h * p.W + ww) * p.C_in;
        const T* wk = wc + (kh * p.kW + kw) * p.cpg_in;
        for (int ci = 0; ci < p.cpg_in; ++ci)
          acc = fmaf(Elem<T>::to_f32(wk[ci]), Elem<T>::to_f32(xp[ci]), acc);
      }
    }
  }
  return acc;
}

// One thread per element of y, which has out_channels(p) channels. Output variants of the
// same thread's post on orderings: position pos of the interleaved order holds filter
// pos / g of group pos % g; a merged channel j is the mean or the maximum over the groups of
// group-major channel i * cpg_out + j (each group's bias added before the merge).
template <typename T, int LAYOUT>
__global__ void __launch_bounds__(256) direct_generic_kernel(const T* __restrict__ x,
                                                              const T* __restrict__ w,
                                                              const T* __restrict__ bias,
                                                              T* __restrict__ y, Conv2d p,
                                                              long long total) {
  const int oc = out_channels(p);
  const long long step = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += step) {
    int n, c, ho, wo;
    long long r = i;
    // decode in the output's memory order, so consecutive threads write consecutive addresses
    if (LAYOUT == GCONV_NCHW) {
      wo = (int)(r % p.Wo); r /= p.Wo;
      ho = (int)(r % p.Ho); r /= p.Ho;
      c = (int)(r % oc); n = (int)(r / oc);
    } else {
      c = (int)(r % oc); r /= oc;
      wo = (int)(r % p.Wo); r /= p.Wo;
      ho = (int)(r % p.Ho); n = (int)(r / p.Ho);
    }
    float v;
    if (p.out_mode == GCONV_OUT_MERGE_AVG || p.out_mode == GCONV_OUT_MERGE_MAX) {
      v = conv_point<T, LAYOUT>(x, w, bias, p, n, c, ho, wo);
      for (int gi = 1; gi < p.groups; ++gi) {
        const float u = conv_point<T, LAYOUT>(x, w, bias, p, n, gi * p.cpg_out + c, ho, wo);
        v = p.out_mode == GCONV_OUT_MERGE_AVG ? v + u : fmaxf(v, u);
      }
      if (p.out_mode == GCONV_OUT_MERGE_AVG) v *= 1.0f / (float)p.groups;
    } else {
      const int co = p.out_mode == GCONV_OUT_INTERLEAVED
                         ? (c % p.groups) * p.cpg_out + c / p.groups : c;
      v = conv_point<T, LAYOUT>(x, w, bias, p, n, co, ho, wo);
    }
    y[i] = Elem<T>::from_f32(v);
  }
}

template <typename T>
cudaError_t launch_typed(const Conv2d& p, const void* x, const void* w, const void* bias, void* y,
                         cudaStream_t s) {
  const long long total = (long long)p.N * out_channels(p) * p.Ho * p.Wo;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148LL * 64) blocks = 148LL * 64;  // grid-stride beyond 64 blocks per SM
  if (p.layout == GCONV_NCHW)
    direct_generic_kernel<T, GCONV_NCHW><<<(unsigned)blocks, threads, 0, s>>>(
        (const T*)x, (const T*)w, (const T*)bias, (T*)y, p, total);
  else
    direct_generic_kernel<T, GCONV_NHWC><<<(unsigned)blocks, threads, 0, s>>>(
        (const T*)x, (const T*)w, (const T*)bias, (T*)y, p, total);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_direct_generic(const Conv2d& p, const void* x, const void* w, const void* bias,
                                  void* y, cudaStream_t s) {
  switch (p.dtype) {
    case GCONV_F32: return launch_typed<float>(p, x, w, bias, y, s);
    case GCONV_F16: return launch_typed<__half>(p, x, w, bias, y, s);
    default: return launch_typed<__nv_bfloat16>(p, x, w, bias, y, s);
  }
}

}  // namespace gconv
