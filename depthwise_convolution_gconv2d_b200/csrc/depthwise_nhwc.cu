// Depthwise (fully-grouped, groups == C_in == C_out) conv2d, NHWC, 16-bit data.
//
// The fully-grouped case of "Grouped convolutions" (neon issue #296; TensorFlow's
// depthwise_conv2d in the same thread), in the channels-last layout the half-precision
// thread points to ("F.conv2d runs x15 slower ...", the NHWC replies). Memory-bound: each
// output needs kH*kW multiply-adds per channel and one read of its inputs.
//
// Mapping: a thread owns VEC consecutive channels (one 16-, 8- or 4-byte vector) of one
// output column (n, wo) and walks down a chunk of output rows. Its kH x kW input window sits
// in registers as packed 16-bit vectors; moving one output row down shifts the window by
// `stride` input rows, so only `stride` new rows of kW vectors are loaded per output (when
// dilation == 1), and those loads are issued one row ahead of the arithmetic. The filter of
// the thread's VEC channels stays in fp32 registers. Consecutive threads take consecutive
// channel vectors, so a warp's loads and stores are contiguous runs of the channel dim.
#include "internal.cuh"

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

}  // namespace gconv
