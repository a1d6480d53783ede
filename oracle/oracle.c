/*
 * Oracle for grouped / depthwise convolution -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 nested loops that state the definitions directly. Only the
 * test-suite, the package smoke check and the benchmark's CPU-baseline leg use
 * this file. The CUDA library shares no code, header or table with it.
 *
 * What is computed, and where it is defined:
 *  - Grouped 2-D convolution: input channels, filters and output channels are
 *    split into `groups` equal blocks with no connection between blocks
 *    ("Grouped convolutions", neon issue #296, thestew42's first reply), in
 *    the usual group-major channel order 1111 2222 3333 ... (same thread,
 *    ibmua's post on output orderings). The arithmetic is cross-correlation with
 *    zero padding, i.e. the semantics of `F.conv2d(input, weight, padding,
 *    groups)` as called in "F.conv2d runs x15 slower in mixed-precision/
 *    half-precision mode" (the timing script in the first post). groups == C_in
 *    is the fully-grouped (depthwise) case of the neon thread.
 *  - Depthwise conv1d over (batch, steps, channels) with groups = channels, as
 *    in "Investigate custom Triton kernels for depthwise-separable convolutions
 *    in Conformer" (speechbrain #2733, the issue text and the Oct 27 comment on
 *    the (batch, steps, channels) layout), plus its backward pass (the Oct 30
 *    comment): data gradient and weight gradient, written as the literal
 *    adjoint (scatter form) of the forward sum.
 *  - The grouped conv2d's own data and weight gradients, in the same scatter /
 *    direct-sum forms, for the training uses of grouped layers on the pages.
 *  - The depthwise-separable block of the Conformer thread: a depthwise
 *    convolution followed by a pointwise (1x1) convolution over channels.
 *  - The neon thread's output variants: interleaved (1234...) output order and
 *    average / max merges across groups.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - output size  Ho = floor((H + 2*pad - dil*(kH-1) - 1)/stride) + 1 (PyTorch's
 *    rule for F.conv2d; symmetric scalar stride/pad/dilation);
 *  - weight layouts: NCHW uses w[C_out][C_in/g][kH][kW] (the shape printed in
 *    the timing script), NHWC uses w[C_out][kH][kW][C_in/g];
 *  - conv1d: T_out = T + pad_left + pad_right - K + 1, zero outside [0, T).
 *
 * All buffers are dense, row-major, fp64. Parallelism: OpenMP over the
 * outermost independent output loop only; each output is one sequential sum.
 */
#include <stddef.h>
#include <stdint.h>

#define ORACLE_NCHW 0
#define ORACLE_NHWC 1

typedef struct {
  long N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, Ho, Wo;
  int layout;
} conv2d_shape;

static long out_extent(long in, long k, long stride, long pad, long dil) {
  long span = in + 2 * pad - dil * (k - 1) - 1;
  if (span < 0) return 0;
  return span / stride + 1;
}

static long x_index(const conv2d_shape* s, long n, long c, long h, long w) {
  if (s->layout == ORACLE_NCHW) return ((n * s->C_in + c) * s->H + h) * s->W + w;
  return ((n * s->H + h) * s->W + w) * s->C_in + c;
}

static long w_index(const conv2d_shape* s, long co, long ci, long kh, long kw) {
  long cpg_in = s->C_in / s->groups;
  if (s->layout == ORACLE_NCHW) return ((co * cpg_in + ci) * s->kH + kh) * s->kW + kw;
  return ((co * s->kH + kh) * s->kW + kw) * cpg_in + ci;
}

static long y_index(const conv2d_shape* s, long n, long co, long ho, long wo) {
  if (s->layout == ORACLE_NCHW) return ((n * s->C_out + co) * s->Ho + ho) * s->Wo + wo;
  return ((n * s->Ho + ho) * s->Wo + wo) * s->C_out + co;
}

/* One output element of the grouped convolution: the whole definition. */
static double conv2d_point(const conv2d_shape* s, const double* x, const double* w,
                           const double* bias, long n, long co, long ho, long wo) {
  long cpg_in = s->C_in / s->groups;
  long cpg_out = s->C_out / s->groups;
  long g = co / cpg_out;            /* group-major: output channel co is in group co / cpg_out */
  double acc = bias ? bias[co] : 0.0;
  for (long ci = 0; ci < cpg_in; ++ci) {
    long c = g * cpg_in + ci;         /* the group reads only its own block of input channels */
    for (long kh = 0; kh < s->kH; ++kh) {
      long h = ho * s->stride - s->pad + kh * s->dil;
      if (h < 0 || h >= s->H) continue;   /* zero padding */
      for (long kw = 0; kw < s->kW; ++kw) {
        long wi = wo * s->stride - s->pad + kw * s->dil;
        if (wi < 0 || wi >= s->W) continue;
        acc += w[w_index(s, co, ci, kh, kw)] * x[x_index(s, n, c, h, wi)];
      }
    }
  }
  return acc;
}

static int make_shape(conv2d_shape* s, long N, long C_in, long H, long W, long C_out, long kH,
                      long kW, long stride, long pad, long dil, long groups, int layout) {
  if (N < 0 || C_in <= 0 || H <= 0 || W <= 0 || C_out <= 0 || kH <= 0 || kW <= 0) return -1;
  if (stride <= 0 || pad < 0 || dil <= 0 || groups <= 0) return -1;
  if (C_in % groups != 0 || C_out % groups != 0) return -1;
  if (layout != ORACLE_NCHW && layout != ORACLE_NHWC) return -1;
  s->N = N; s->C_in = C_in; s->H = H; s->W = W; s->C_out = C_out; s->kH = kH; s->kW = kW;
  s->stride = stride; s->pad = pad; s->dil = dil; s->groups = groups; s->layout = layout;
  s->Ho = out_extent(H, kH, stride, pad, dil);
  s->Wo = out_extent(W, kW, stride, pad, dil);
  if (s->Ho <= 0 || s->Wo <= 0) return -1;
  return 0;
}

/* Output spatial size for the given input size; 0 when the window does not fit. */
long oracle_conv_out_extent(long in, long k, long stride, long pad, long dil) {
  if (stride <= 0 || dil <= 0 || k <= 0 || pad < 0) return 0;
  return out_extent(in, k, stride, pad, dil);
}

/* Full grouped conv2d. Returns 0 on success, -1 on an invalid shape. */
int oracle_conv2d(const double* x, const double* w, const double* bias, double* y, long N,
                  long C_in, long H, long W, long C_out, long kH, long kW, long stride, long pad,
                  long dil, long groups, int layout) {
  conv2d_shape s;
  if (make_shape(&s, N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, layout)) return -1;
  long outer = N * C_out;
#pragma omp parallel for schedule(dynamic, 1)
  for (long nc = 0; nc < outer; ++nc) {
    long n = nc / C_out, co = nc % C_out;
    for (long ho = 0; ho < s.Ho; ++ho)
      for (long wo = 0; wo < s.Wo; ++wo)
        y[y_index(&s, n, co, ho, wo)] = conv2d_point(&s, x, w, bias, n, co, ho, wo);
  }
  return 0;
}

/* Selected outputs of grouped conv2d: out[i] = y at the 4-tuple idx[4i..4i+3] =
 * (n, co, ho, wo). Used to check full-size launches on sampled outputs. */
int oracle_conv2d_points(const double* x, const double* w, const double* bias, double* out,
                         const int64_t* idx, long npts, long N, long C_in, long H, long W,
                         long C_out, long kH, long kW, long stride, long pad, long dil,
                         long groups, int layout) {
  conv2d_shape s;
  if (make_shape(&s, N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, layout)) return -1;
  for (long i = 0; i < npts; ++i) {
    long n = idx[4 * i], co = idx[4 * i + 1], ho = idx[4 * i + 2], wo = idx[4 * i + 3];
    if (n < 0 || n >= N || co < 0 || co >= C_out || ho < 0 || ho >= s.Ho || wo < 0 || wo >= s.Wo)
      return -1;
  }
#pragma omp parallel for schedule(static)
  for (long i = 0; i < npts; ++i)
    out[i] = conv2d_point(&s, x, w, bias, idx[4 * i], idx[4 * i + 1], idx[4 * i + 2],
                          idx[4 * i + 3]);
  return 0;
}

/* ---------------- grouped conv2d backward ---------------- */
/* The gradients of L = sum over outputs of dy * y for the forward sum of conv2d_point (the
 * training use of grouped layers on the pages: the Adam-trained ensemble of "Optimize
 * convolution batching rule performance" and the backward passes timed in the Conformer
 * thread). dy has the forward output's shape and layout, dx the input's, dw the weight's. */

/* Data gradient, scatter form: each forward term w[co,ci,kh,kw] * x[n,c,h,wi] of output
 * (n,co,ho,wo) sends w[co,ci,kh,kw] * dy[n,co,ho,wo] back to dx[n,c,h,wi]. Parallel over n,
 * so the scatter is race-free. */
int oracle_conv2d_bwd_data(const double* dy, const double* w, double* dx, long N, long C_in,
                           long H, long W, long C_out, long kH, long kW, long stride, long pad,
                           long dil, long groups, int layout) {
  conv2d_shape s;
  if (make_shape(&s, N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, layout)) return -1;
  long cpg_in = C_in / groups, cpg_out = C_out / groups;
#pragma omp parallel for schedule(dynamic, 1)
  for (long n = 0; n < N; ++n) {
    for (long c = 0; c < C_in; ++c)
      for (long h = 0; h < H; ++h)
        for (long wi = 0; wi < W; ++wi) dx[x_index(&s, n, c, h, wi)] = 0.0;
    for (long co = 0; co < C_out; ++co) {
      long g = co / cpg_out;
      for (long ho = 0; ho < s.Ho; ++ho)
        for (long wo = 0; wo < s.Wo; ++wo) {
          double d = dy[y_index(&s, n, co, ho, wo)];
          for (long ci = 0; ci < cpg_in; ++ci)
            for (long kh = 0; kh < kH; ++kh) {
              long h = ho * stride - pad + kh * dil;
              if (h < 0 || h >= H) continue;
              for (long kw = 0; kw < kW; ++kw) {
                long wi = wo * stride - pad + kw * dil;
                if (wi < 0 || wi >= W) continue;
                dx[x_index(&s, n, g * cpg_in + ci, h, wi)] += w[w_index(&s, co, ci, kh, kw)] * d;
              }
            }
        }
    }
  }
  return 0;
}

/* dx at selected input positions idx[4i..4i+3] = (n, c, h, w), gathered: the sum over the
 * outputs (co in c's group, ho, wo) and taps (kh, kw) whose window reads x[n,c,h,w], i.e.
 * ho*stride - pad + kh*dil == h and wo*stride - pad + kw*dil == w. */
int oracle_conv2d_bwd_data_points(const double* dy, const double* w, double* out,
                                  const int64_t* idx, long npts, long N, long C_in, long H,
                                  long W, long C_out, long kH, long kW, long stride, long pad,
                                  long dil, long groups, int layout) {
  conv2d_shape s;
  if (make_shape(&s, N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, layout)) return -1;
  for (long i = 0; i < npts; ++i) {
    long n = idx[4 * i], c = idx[4 * i + 1], h = idx[4 * i + 2], wi = idx[4 * i + 3];
    if (n < 0 || n >= N || c < 0 || c >= C_in || h < 0 || h >= H || wi < 0 || wi >= W) return -1;
  }
  long cpg_in = C_in / groups, cpg_out = C_out / groups;
#pragma omp parallel for schedule(static)
  for (long i = 0; i < npts; ++i) {
    long n = idx[4 * i], c = idx[4 * i + 1], h = idx[4 * i + 2], wi = idx[4 * i + 3];
    long g = c / cpg_in, ci = c % cpg_in;
    double acc = 0.0;
    for (long co = g * cpg_out; co < (g + 1) * cpg_out; ++co)
      for (long kh = 0; kh < kH; ++kh) {
        long th = h + pad - kh * dil;          /* = ho * stride */
        if (th < 0 || th % stride != 0 || th / stride >= s.Ho) continue;
        for (long kw = 0; kw < kW; ++kw) {
          long tw = wi + pad - kw * dil;       /* = wo * stride */
          if (tw < 0 || tw % stride != 0 || tw / stride >= s.Wo) continue;
          acc += w[w_index(&s, co, ci, kh, kw)] * dy[y_index(&s, n, co, th / stride, tw / stride)];
        }
      }
    out[i] = acc;
  }
  return 0;
}

/* One weight-gradient entry: dw[co,ci,kh,kw] = sum over (n, ho, wo) of
 * dy[n,co,ho,wo] * x[n, g*cpg_in + ci, ho*stride - pad + kh*dil, wo*stride - pad + kw*dil],
 * summed in (n, ho, wo) order; taps that fall in the padding contribute nothing. */
static double conv2d_wgrad_entry(const conv2d_shape* s, const double* x, const double* dy,
                                 long co, long ci, long kh, long kw) {
  long cpg_in = s->C_in / s->groups, cpg_out = s->C_out / s->groups;
  long c = (co / cpg_out) * cpg_in + ci;
  double acc = 0.0;
  for (long n = 0; n < s->N; ++n)
    for (long ho = 0; ho < s->Ho; ++ho) {
      long h = ho * s->stride - s->pad + kh * s->dil;
      if (h < 0 || h >= s->H) continue;
      for (long wo = 0; wo < s->Wo; ++wo) {
        long wi = wo * s->stride - s->pad + kw * s->dil;
        if (wi < 0 || wi >= s->W) continue;
        acc += dy[y_index(s, n, co, ho, wo)] * x[x_index(s, n, c, h, wi)];
      }
    }
  return acc;
}

/* Full weight gradient, dw in the weight layout of `layout`. */
int oracle_conv2d_bwd_weight(const double* x, const double* dy, double* dw, long N, long C_in,
                             long H, long W, long C_out, long kH, long kW, long stride, long pad,
                             long dil, long groups, int layout) {
  conv2d_shape s;
  if (make_shape(&s, N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, layout)) return -1;
  long cpg_in = C_in / groups;
#pragma omp parallel for schedule(dynamic, 1)
  for (long co = 0; co < C_out; ++co)
    for (long ci = 0; ci < cpg_in; ++ci)
      for (long kh = 0; kh < kH; ++kh)
        for (long kw = 0; kw < kW; ++kw)
          dw[w_index(&s, co, ci, kh, kw)] = conv2d_wgrad_entry(&s, x, dy, co, ci, kh, kw);
  return 0;
}

/* Selected weight-gradient entries idx[4i..4i+3] = (co, ci, kh, kw). */
int oracle_conv2d_bwd_weight_points(const double* x, const double* dy, double* out,
                                    const int64_t* idx, long npts, long N, long C_in, long H,
                                    long W, long C_out, long kH, long kW, long stride, long pad,
                                    long dil, long groups, int layout) {
  conv2d_shape s;
  if (make_shape(&s, N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, layout)) return -1;
  long cpg_in = C_in / groups;
  for (long i = 0; i < npts; ++i) {
    long co = idx[4 * i], ci = idx[4 * i + 1], kh = idx[4 * i + 2], kw = idx[4 * i + 3];
    if (co < 0 || co >= C_out || ci < 0 || ci >= cpg_in || kh < 0 || kh >= kH || kw < 0 || kw >= kW)
      return -1;
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (long i = 0; i < npts; ++i)
    out[i] = conv2d_wgrad_entry(&s, x, dy, idx[4 * i], idx[4 * i + 1], idx[4 * i + 2],
                                idx[4 * i + 3]);
  return 0;
}

/* ---------------- output orderings and merges across groups ---------------- */
/* Interleaved output order: ibmua's post on output orderings in "Grouped convolutions" (neon
 * issue #296) asks for the feature maps as 1234123412341234 instead of the usual group-major
 * 111122223333444. Output position p = j * groups + i holds filter j of group i, i.e. the
 * group-major output channel i * cpg_out + j. y has the forward output's shape. */
int oracle_conv2d_interleaved(const double* x, const double* w, const double* bias, double* y,
                              long N, long C_in, long H, long W, long C_out, long kH, long kW,
                              long stride, long pad, long dil, long groups, int layout) {
  conv2d_shape s;
  if (make_shape(&s, N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, layout)) return -1;
  long cpg_out = C_out / groups;
#pragma omp parallel for schedule(dynamic, 1)
  for (long np = 0; np < N * C_out; ++np) {
    long n = np / C_out, pos = np % C_out;
    long i = pos % groups, j = pos / groups;
    long co = i * cpg_out + j;
    for (long ho = 0; ho < s.Ho; ++ho)
      for (long wo = 0; wo < s.Wo; ++wo)
        y[y_index(&s, n, pos, ho, wo)] = conv2d_point(&s, x, w, bias, n, co, ho, wo);
  }
  return 0;
}

/* Merge across groups: the same post wants the groups' results pulled together by average or
 * max pooling across groups (volumetric pooling over the interleaved order), and the next
 * post combines groups through a 1x1 layer for want of Avg / Max. Output channel j < cpg_out
 * is the mean (mode 0) or the maximum (mode 1) over groups i of group-major channel
 * i * cpg_out + j; y is [N][cpg_out][Ho][Wo] (NCHW) or [N][Ho][Wo][cpg_out] (NHWC). */
int oracle_conv2d_group_merge(const double* x, const double* w, const double* bias, double* y,
                              long N, long C_in, long H, long W, long C_out, long kH, long kW,
                              long stride, long pad, long dil, long groups, int layout,
                              int mode) {
  conv2d_shape s;
  if (mode != 0 && mode != 1) return -1;
  if (make_shape(&s, N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups, layout)) return -1;
  long cpg_out = C_out / groups;
#pragma omp parallel for schedule(dynamic, 1)
  for (long nj = 0; nj < N * cpg_out; ++nj) {
    long n = nj / cpg_out, j = nj % cpg_out;
    for (long ho = 0; ho < s.Ho; ++ho)
      for (long wo = 0; wo < s.Wo; ++wo) {
        double m = 0.0;
        for (long i = 0; i < groups; ++i) {
          double v = conv2d_point(&s, x, w, bias, n, i * cpg_out + j, ho, wo);
          if (mode == 0) m += v;
          else if (i == 0 || v > m) m = v;
        }
        if (mode == 0) m /= (double)groups;
        long yi = layout == ORACLE_NCHW ? ((n * cpg_out + j) * s.Ho + ho) * s.Wo + wo
                                        : ((n * s.Ho + ho) * s.Wo + wo) * cpg_out + j;
        y[yi] = m;
      }
  }
  return 0;
}

/* ---------------- depthwise conv1d over (batch, steps, channels) ---------------- */

static int conv1d_ok(long B, long T, long C, long K, long pl, long pr) {
  if (B < 0 || T <= 0 || C <= 0 || K <= 0 || pl < 0 || pr < 0) return 0;
  return T + pl + pr - K + 1 > 0;
}

/* y[b][t][c] = sum_k w[c][k] * x[b][t + k - pl][c], x = 0 outside [0, T). */
int oracle_dwconv1d_fwd(const double* x, const double* w, double* y, long B, long T, long C,
                        long K, long pl, long pr) {
  if (!conv1d_ok(B, T, C, K, pl, pr)) return -1;
  long T_out = T + pl + pr - K + 1;
#pragma omp parallel for schedule(static)
  for (long b = 0; b < B; ++b)
    for (long t = 0; t < T_out; ++t)
      for (long c = 0; c < C; ++c) {
        double acc = 0.0;
        for (long k = 0; k < K; ++k) {
          long s = t + k - pl;
          if (s < 0 || s >= T) continue;
          acc += w[c * K + k] * x[(b * T + s) * C + c];
        }
        y[(b * T_out + t) * C + c] = acc;
      }
  return 0;
}

/* Data gradient: each forward term w[c][k]*x[b][s][c] (s = t + k - pl) sends
 * w[c][k]*dy[b][t][c] back to dx[b][s][c]. Written in that scatter form; the
 * per-batch loop keeps the scatter race-free under OpenMP. */
int oracle_dwconv1d_bwd_data(const double* dy, const double* w, double* dx, long B, long T,
                             long C, long K, long pl, long pr) {
  if (!conv1d_ok(B, T, C, K, pl, pr)) return -1;
  long T_out = T + pl + pr - K + 1;
#pragma omp parallel for schedule(static)
  for (long b = 0; b < B; ++b) {
    for (long s = 0; s < T; ++s)
      for (long c = 0; c < C; ++c) dx[(b * T + s) * C + c] = 0.0;
    for (long t = 0; t < T_out; ++t)
      for (long k = 0; k < K; ++k) {
        long s = t + k - pl;
        if (s < 0 || s >= T) continue;
        for (long c = 0; c < C; ++c)
          dx[(b * T + s) * C + c] += w[c * K + k] * dy[(b * T_out + t) * C + c];
      }
  }
  return 0;
}

/* Weight gradient: dw[c][k] = sum over (b, t) of dy[b][t][c] * x[b][t + k - pl][c],
 * summed in (b, t) order. */
int oracle_dwconv1d_bwd_weight(const double* x, const double* dy, double* dw, long B, long T,
                               long C, long K, long pl, long pr) {
  if (!conv1d_ok(B, T, C, K, pl, pr)) return -1;
  long T_out = T + pl + pr - K + 1;
#pragma omp parallel for schedule(static)
  for (long c = 0; c < C; ++c)
    for (long k = 0; k < K; ++k) {
      double acc = 0.0;
      for (long b = 0; b < B; ++b)
        for (long t = 0; t < T_out; ++t) {
          long s = t + k - pl;
          if (s < 0 || s >= T) continue;
          acc += dy[(b * T_out + t) * C + c] * x[(b * T + s) * C + c];
        }
      dw[c * K + k] = acc;
    }
  return 0;
}

/* ---------------- depthwise-separable block ---------------- */
/* A depthwise convolution followed by a pointwise (1x1, dense) convolution over channels: the
 * "depthwise-separable convolutions in Conformer" of the Conformer thread (the convolution
 * module's depthwise conv1d on (batch, steps, channels), and the strided depthwise-separable
 * Conv2D of Fast Conformer's downsampler named in its Oct 30 comment):
 *   y[..., c] = depthwise(x)[..., c]        (the dwconv1d / depthwise conv2d above)
 *   z[..., o] = bpw[o] + sum_c wpw[o][c] * y[..., c]
 * computed as that composition in fp64 (no rounding of y). wpw is [C_out][C]. */

/* 1-D: x [B][T][C], wdw [C][K], wpw [C_out][C], z [B][T_out][C_out]; y is caller scratch
 * [B][T_out][C]. */
int oracle_dwsep1d_fwd(const double* x, const double* wdw, const double* wpw, const double* bpw,
                       double* y, double* z, long B, long T, long C, long K, long pl, long pr,
                       long C_out) {
  if (C_out <= 0) return -1;
  if (oracle_dwconv1d_fwd(x, wdw, y, B, T, C, K, pl, pr)) return -1;
  long rows = B * (T + pl + pr - K + 1);
#pragma omp parallel for schedule(static)
  for (long r = 0; r < rows; ++r)
    for (long o = 0; o < C_out; ++o) {
      double acc = bpw ? bpw[o] : 0.0;
      for (long c = 0; c < C; ++c) acc += wpw[o * C + c] * y[r * C + c];
      z[r * C_out + o] = acc;
    }
  return 0;
}

/* One output z[b][t][o] of the 1-D block, summed directly over (c, k). */
static double dwsep1d_point(const double* x, const double* wdw, const double* wpw,
                            const double* bpw, long T, long C, long K, long pl, long b, long t,
                            long o) {
  double acc = bpw ? bpw[o] : 0.0;
  for (long c = 0; c < C; ++c) {
    double yc = 0.0;
    for (long k = 0; k < K; ++k) {
      long s = t + k - pl;
      if (s < 0 || s >= T) continue;
      yc += wdw[c * K + k] * x[(b * T + s) * C + c];
    }
    acc += wpw[o * C + c] * yc;
  }
  return acc;
}

/* Selected outputs idx[3i..3i+2] = (b, t, o) of the 1-D block. */
int oracle_dwsep1d_points(const double* x, const double* wdw, const double* wpw,
                          const double* bpw, double* out, const int64_t* idx, long npts, long B,
                          long T, long C, long K, long pl, long pr, long C_out) {
  if (!conv1d_ok(B, T, C, K, pl, pr) || C_out <= 0) return -1;
  long T_out = T + pl + pr - K + 1;
  for (long i = 0; i < npts; ++i) {
    long b = idx[3 * i], t = idx[3 * i + 1], o = idx[3 * i + 2];
    if (b < 0 || b >= B || t < 0 || t >= T_out || o < 0 || o >= C_out) return -1;
  }
#pragma omp parallel for schedule(static)
  for (long i = 0; i < npts; ++i)
    out[i] = dwsep1d_point(x, wdw, wpw, bpw, T, C, K, pl, idx[3 * i], idx[3 * i + 1],
                           idx[3 * i + 2]);
  return 0;
}

/* 2-D: x in `layout` with C channels, wdw the depthwise weight ([C][1][kH][kW] or
 * [C][kH][kW][1]), wpw [C_out][C], z in `layout` with C_out channels; y is caller scratch with
 * the depthwise output's shape. */
int oracle_dwsep2d_fwd(const double* x, const double* wdw, const double* wpw, const double* bpw,
                       double* y, double* z, long N, long C, long H, long W, long kH, long kW,
                       long stride, long pad, long dil, long C_out, int layout) {
  conv2d_shape s;
  if (C_out <= 0) return -1;
  if (make_shape(&s, N, C, H, W, C, kH, kW, stride, pad, dil, C, layout)) return -1;
  if (oracle_conv2d(x, wdw, NULL, y, N, C, H, W, C, kH, kW, stride, pad, dil, C, layout))
    return -1;
  long HW = s.Ho * s.Wo;
#pragma omp parallel for schedule(static)
  for (long np = 0; np < N * HW; ++np) {
    long n = np / HW, hw = np % HW;
    for (long o = 0; o < C_out; ++o) {
      double acc = bpw ? bpw[o] : 0.0;
      for (long c = 0; c < C; ++c) {
        long yi = layout == ORACLE_NCHW ? (n * C + c) * HW + hw : (n * HW + hw) * C + c;
        acc += wpw[o * C + c] * y[yi];
      }
      long zi = layout == ORACLE_NCHW ? (n * C_out + o) * HW + hw : (n * HW + hw) * C_out + o;
      z[zi] = acc;
    }
  }
  return 0;
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
