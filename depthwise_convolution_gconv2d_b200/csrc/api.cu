// C ABI of libgconv.so: argument validation, kernel selection and launch.
//
// Shape logic (all integer, checked before any launch): C_in and C_out must be multiples of
// `groups` (the equal split of channels and filters into groups of "Grouped convolutions",
// neon issue #296), Ho/Wo follow F.conv2d's output-size rule and must be >= 1, and a group
// index is never stored per element -- it is derived from the output channel in every kernel,
// so all groups run in one launch (the thread's argument against one launch per group).
#include <limits.h>

#include <atomic>

#include "internal.cuh"

namespace gconv {

__device__ unsigned int g_device_error;   // set by kernels whose bounded waits give up

unsigned int* device_error_word() {
  static std::atomic<unsigned int*> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  unsigned int* p = cached[dev].load(std::memory_order_acquire);
  if (p) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_device_error) != cudaSuccess) return nullptr;
  cached[dev].store((unsigned int*)addr, std::memory_order_release);
  return (unsigned int*)addr;
}

// Test hook: bytes the generic tensor-core tile kernel's producer declares per stage on top of
// what its copies deliver (0 on every normal run).
static std::atomic<unsigned int> g_tx_surplus{0};

unsigned int debug_tx_surplus() { return g_tx_surplus.load(std::memory_order_relaxed); }

cudaError_t read_and_clear_device_error(cudaStream_t s, int* code) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  }
  *code = (int)v;
  return e;
}

namespace {

long long out_extent(long long in, long long k, long long stride, long long pad, long long dil) {
  const long long span = in + 2 * pad - dil * (k - 1) - 1;
  return span < 0 ? 0 : span / stride + 1;
}

// Fills `p`; returns GCONV_OK or GCONV_ERR_INVALID_ARG.
gconv_status make_conv2d(Conv2d* p, int N, int C_in, int H, int W, int C_out, int kH, int kW,
                         int stride, int pad, int dil, int groups, int layout, int dtype,
                         int out_mode = GCONV_OUT_GROUP_MAJOR) {
  if (out_mode < GCONV_OUT_GROUP_MAJOR || out_mode > GCONV_OUT_MERGE_MAX)
    return GCONV_ERR_INVALID_ARG;
  if (N < 0 || C_in <= 0 || H <= 0 || W <= 0 || C_out <= 0 || kH <= 0 || kW <= 0)
    return GCONV_ERR_INVALID_ARG;
  if (stride <= 0 || pad < 0 || dil <= 0 || groups <= 0) return GCONV_ERR_INVALID_ARG;
  if (C_in % groups != 0 || C_out % groups != 0) return GCONV_ERR_INVALID_ARG;
  if (layout != GCONV_NCHW && layout != GCONV_NHWC) return GCONV_ERR_INVALID_ARG;
  if (dtype != GCONV_F32 && dtype != GCONV_F16 && dtype != GCONV_BF16) return GCONV_ERR_INVALID_ARG;
  const long long Ho = out_extent(H, kH, stride, pad, dil);
  const long long Wo = out_extent(W, kW, stride, pad, dil);
  if (Ho < 1 || Wo < 1 || Ho > INT_MAX || Wo > INT_MAX) return GCONV_ERR_INVALID_ARG;
  // element counts must be addressable with 64-bit offsets and sane grid sizes
  const long long xs = (long long)N * C_in * H * W;
  const long long ys = (long long)N * C_out * Ho * Wo;
  if (xs < 0 || ys < 0 || xs > (1LL << 40) || ys > (1LL << 40)) return GCONV_ERR_INVALID_ARG;
  p->N = N; p->C_in = C_in; p->H = H; p->W = W; p->C_out = C_out; p->kH = kH; p->kW = kW;
  p->stride = stride; p->pad = pad; p->dil = dil; p->groups = groups;
  p->Ho = (int)Ho; p->Wo = (int)Wo;
  p->cpg_in = C_in / groups; p->cpg_out = C_out / groups;
  p->layout = layout; p->dtype = dtype;
  p->out_mode = out_mode;
  return GCONV_OK;
}

int depthwise_vec_bytes(const Conv2d& p) { return 2 * (p.kH <= 3 ? 8 : (p.kH <= 5 ? 4 : 2)); }

bool aligned_to(const void* ptr, int bytes) {
  return ptr == nullptr || (reinterpret_cast<uintptr_t>(ptr) % (uintptr_t)bytes) == 0;
}

// Kernel choice. `x`/`w`/`y` may all be null (query mode: alignment assumed).
int choose_kernel(const Conv2d& p, int path, const void* x, const void* w, const void* y,
                  gconv_status* why) {
  *why = GCONV_OK;
  const bool query = (x == nullptr && w == nullptr && y == nullptr);
  const bool dw_ok = depthwise_nhwc_supported(p) && p.N <= 65535;
  const bool dw_al = query || (aligned_to(x, depthwise_vec_bytes(p)) &&
                               aligned_to(y, depthwise_vec_bytes(p)));
  // narrow groups: TMA boxes and stores need 16-byte aligned x and y
  const bool ng_ok = grouped_nhwc_supported(p) && (query || (aligned16(x) && aligned16(y)));
  const bool tc_ok = igemm_supported(p);
  // tensor maps need 16-byte aligned bases (x, and w when it is used in place: NHWC)
  const bool tc_al = query || (aligned16(x) && aligned16(y) &&
                               (p.layout == GCONV_NCHW || aligned16(w)));
  const int tc_kernel = p.layout == GCONV_NHWC ? GCONV_KERNEL_IGEMM_TC : GCONV_KERNEL_IGEMM_TC_NCHW;
  switch (path) {
    case GCONV_PATH_GENERIC:
      return GCONV_KERNEL_DIRECT_GENERIC;
    case GCONV_PATH_DIRECT:
      if (dw_ok && dw_al) return GCONV_KERNEL_DEPTHWISE_NHWC;
      return ng_ok ? GCONV_KERNEL_GROUPED_NHWC : GCONV_KERNEL_DIRECT_GENERIC;
    case GCONV_PATH_IGEMM:
      if (!tc_ok) { *why = GCONV_ERR_UNSUPPORTED; return -1; }
      if (!tc_al) { *why = GCONV_ERR_MISALIGNED; return -1; }
      return tc_kernel;
    case GCONV_PATH_AUTO:
      if (p.dtype == GCONV_F32) return GCONV_KERNEL_DIRECT_GENERIC;
      if (dw_ok && dw_al) return GCONV_KERNEL_DEPTHWISE_NHWC;
      if (ng_ok) return GCONV_KERNEL_GROUPED_NHWC;
      if (tc_ok && tc_al) return tc_kernel;
      return GCONV_KERNEL_DIRECT_GENERIC;
    default:
      *why = GCONV_ERR_INVALID_ARG;
      return -1;
  }
}

// Output variants. The interleaved order equals the group-major one when each group has one
// filter or there is one group, and a merge over one group is the plain output: those run on
// the ordinary kernels. Otherwise the variant runs in the epilogue of the tensor-core tile
// kernels (16-bit data the implicit GEMM takes) or in the generic direct kernel.
bool out_mode_is_plain(const Conv2d& p) {
  if (p.out_mode == GCONV_OUT_GROUP_MAJOR || p.groups == 1) return true;
  return p.out_mode == GCONV_OUT_INTERLEAVED && p.cpg_out == 1;
}

// The max merge in two passes (GCONV_KERNEL_MERGE_MAX_TWO_PASS): the plain problem, written
// group-major to the workspace by the transposed row-strip kernel, then the maximum over
// groups. Taken where that kernel runs the plain problem (16-bit).
bool merge_max_two_pass_ok(const Conv2d& p) {
  if (p.out_mode != GCONV_OUT_MERGE_MAX || p.dtype == GCONV_F32) return false;
  Conv2d q = p;
  q.out_mode = GCONV_OUT_GROUP_MAJOR;
  return igemm_supported(q) && igemm_rowt_supported(q);
}

size_t merge_max_group_major_bytes(const Conv2d& p) {
  return ((size_t)p.N * p.C_out * p.Ho * p.Wo * 2 + 255) / 256 * 256;
}

int choose_kernel_out(const Conv2d& p, int path, const void* x, const void* w, const void* y,
                      gconv_status* why) {
  if (out_mode_is_plain(p)) {
    Conv2d q = p;
    q.out_mode = GCONV_OUT_GROUP_MAJOR;
    return choose_kernel(q, path, x, w, y, why);
  }
  *why = GCONV_OK;
  const bool query = (x == nullptr && w == nullptr && y == nullptr);
  if (merge_max_two_pass_ok(p) && (path == GCONV_PATH_AUTO || path == GCONV_PATH_IGEMM) &&
      (query || (aligned16(x) && aligned16(y) && (p.layout == GCONV_NCHW || aligned16(w)))))
    return GCONV_KERNEL_MERGE_MAX_TWO_PASS;
  const bool tc_ok = igemm_supported(p);
  const bool tc_al = query || (aligned16(x) && aligned16(y) &&
                               (p.layout == GCONV_NCHW || aligned16(w)));
  const int tc_kernel = p.layout == GCONV_NHWC ? GCONV_KERNEL_IGEMM_TC : GCONV_KERNEL_IGEMM_TC_NCHW;
  switch (path) {
    case GCONV_PATH_GENERIC:
    case GCONV_PATH_DIRECT:
      return GCONV_KERNEL_DIRECT_GENERIC;
    case GCONV_PATH_IGEMM:
      if (!tc_ok) { *why = GCONV_ERR_UNSUPPORTED; return -1; }
      if (!tc_al) { *why = GCONV_ERR_MISALIGNED; return -1; }
      return tc_kernel;
    case GCONV_PATH_AUTO:
      if (p.dtype != GCONV_F32 && tc_ok && tc_al) return tc_kernel;
      return GCONV_KERNEL_DIRECT_GENERIC;
    default:
      *why = GCONV_ERR_INVALID_ARG;
      return -1;
  }
}

gconv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GCONV_OK : GCONV_ERR_CUDA; }

// Launches forward kernel `kernel` on a validated problem (workspace checked here for NCHW
// tensor-core staging).
gconv_status launch_forward(int kernel, const Conv2d& p, const void* x, const void* w,
                            const void* bias, void* y, void* workspace, size_t workspace_bytes,
                            cudaStream_t s) {
  switch (kernel) {
    case GCONV_KERNEL_DEPTHWISE_NHWC:
      return cuda_status(launch_depthwise_nhwc(p, x, w, bias, y, s));
    case GCONV_KERNEL_GROUPED_NHWC:
      return cuda_status(launch_grouped_nhwc(p, x, w, bias, y, s));
    case GCONV_KERNEL_IGEMM_TC:
      return cuda_status(launch_igemm_nhwc(p, x, w, bias, y, s));
    case GCONV_KERNEL_IGEMM_TC_NCHW: {
      const size_t need = igemm_nchw_workspace(p);
      if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))
        return GCONV_ERR_WORKSPACE;
      return cuda_status(launch_igemm_nchw(p, x, w, bias, y, workspace, s));
    }
    default:
      return cuda_status(launch_direct_generic(p, x, w, bias, y, s));
  }
}

// ------------------------------------------------------------------ conv2d backward dispatch
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

size_t weight_bytes(const Conv2d& p) {
  return (size_t)p.C_out * p.cpg_in * p.kH * p.kW * (p.dtype == GCONV_F32 ? 4 : 2);
}

// The forward problem whose output is the data gradient (valid when dgrad_as_forward(p)):
// input dy (C_out channels, Ho x Wo), output dx (C_in channels, H x W), stride 1,
// pad' = dil*(k-1) - pad.
gconv_status exchanged_problem(const Conv2d& p, Conv2d* q) {
  return make_conv2d(q, p.N, p.C_out, p.Ho, p.Wo, p.C_in, p.kH, p.kW, 1,
                     p.dil * (p.kH - 1) - p.pad, p.dil, p.groups, p.layout, p.dtype);
}

// Kernel for a data-gradient call: a forward kernel code (run on the exchanged problem with
// the flipped, transposed filter) or GCONV_KERNEL_DGRAD_GENERIC. `wt` is where that filter
// will be (the workspace); all of dy, wt, dx null = query mode.
int dgrad_choose(const Conv2d& p, int path, const void* dy, const void* wt, const void* dx,
                 gconv_status* why, Conv2d* q) {
  *why = GCONV_OK;
  const bool via = dgrad_as_forward(p) && exchanged_problem(p, q) == GCONV_OK;
  const bool query = dy == nullptr && wt == nullptr && dx == nullptr;
  const int vb = dgrad_depthwise_vec_bytes(p);
  const bool dwk = dgrad_depthwise_supported(p) &&
                   (query || (aligned_to(dy, vb) && aligned_to(dx, vb)));
  const bool dgs = dgrad_dw3s2_tma_supported(p) && (query || (aligned16(dy) && aligned16(dx)));
  switch (path) {
    case GCONV_PATH_GENERIC:
      return GCONV_KERNEL_DGRAD_GENERIC;
    case GCONV_PATH_AUTO:
    case GCONV_PATH_DIRECT: {
      int k = -1;
      if (via && !(path == GCONV_PATH_AUTO && p.dtype == GCONV_F32))
        k = choose_kernel(*q, path, dy, wt, dx, why);
      *why = GCONV_OK;
      if (k >= 0 && k != GCONV_KERNEL_DIRECT_GENERIC) return k;
      if (dgs) return GCONV_KERNEL_DGRAD_DW3S2_TMA;
      return dwk ? GCONV_KERNEL_DGRAD_DEPTHWISE_NHWC : GCONV_KERNEL_DGRAD_GENERIC;
    }
    case GCONV_PATH_IGEMM:
      if (!via) { *why = GCONV_ERR_UNSUPPORTED; return -1; }
      return choose_kernel(*q, path, dy, wt, dx, why);
    default:
      *why = GCONV_ERR_INVALID_ARG;
      return -1;
  }
}

size_t dgrad_workspace(const Conv2d& p, const Conv2d& q, int kernel) {
  if (kernel == GCONV_KERNEL_DGRAD_GENERIC || kernel == GCONV_KERNEL_DGRAD_DEPTHWISE_NHWC ||
      kernel == GCONV_KERNEL_DGRAD_DW3S2_TMA)
    return 0;
  const size_t fwd = kernel == GCONV_KERNEL_IGEMM_TC_NCHW ? igemm_nchw_workspace(q) : 0;
  return round_up(weight_bytes(p), 256) + fwd;
}

bool aligned4(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

int wgrad_choose(const Conv2d& p, int path, const void* x, const void* dy, gconv_status* why) {
  *why = GCONV_OK;
  const bool query = x == nullptr && dy == nullptr;
  const bool dw_ok = wgrad_depthwise_supported(p) && (query || (aligned4(x) && aligned4(dy)));
  // wide groups: NHWC reads x and dy in place (16-byte vectors); NCHW stages them as NHWC
  const bool tl_ok = wgrad_tiled_supported(p) &&
                     (p.layout == GCONV_NCHW || query || (aligned16(x) && aligned16(dy)));
  const int tl_kernel = p.layout == GCONV_NHWC ? GCONV_KERNEL_WGRAD_TILED_NHWC
                                               : GCONV_KERNEL_WGRAD_TILED_NCHW;
  const bool tma_ok = wgrad_dw3_tma_supported(p) && (query || (aligned16(x) && aligned16(dy)));
  // tensor cores: NHWC operands read by TMA in place (16-byte aligned), NCHW staged as NHWC
  const bool tc_ok = wgrad_tc_supported(p) && wgrad_tiled_supported(p) &&
                     (p.layout == GCONV_NCHW || query || (aligned16(x) && aligned16(dy)));
  const int tc_kernel = p.layout == GCONV_NHWC ? GCONV_KERNEL_WGRAD_TC_NHWC
                                               : GCONV_KERNEL_WGRAD_TC_NCHW;
  switch (path) {
    case GCONV_PATH_GENERIC:
      return GCONV_KERNEL_WGRAD_GENERIC;
    case GCONV_PATH_AUTO:
      if (tma_ok) return GCONV_KERNEL_WGRAD_DW3_TMA;
      if (dw_ok) return GCONV_KERNEL_WGRAD_DEPTHWISE_NHWC;
      if (tc_ok) return tc_kernel;
      return tl_ok ? tl_kernel : GCONV_KERNEL_WGRAD_GENERIC;
    case GCONV_PATH_DIRECT:
      if (tma_ok) return GCONV_KERNEL_WGRAD_DW3_TMA;
      if (dw_ok) return GCONV_KERNEL_WGRAD_DEPTHWISE_NHWC;
      return tl_ok ? tl_kernel : GCONV_KERNEL_WGRAD_GENERIC;
    case GCONV_PATH_IGEMM:
      if (!wgrad_tc_supported(p) || !wgrad_tiled_supported(p)) {
        *why = GCONV_ERR_UNSUPPORTED;
        return -1;
      }
      if (!tc_ok) {
        *why = GCONV_ERR_MISALIGNED;
        return -1;
      }
      return tc_kernel;
    default:
      *why = GCONV_ERR_INVALID_ARG;
      return -1;
  }
}

// The weight gradient's row slices are ints on the device.
bool wgrad_rows_ok(const Conv2d& p) { return (long long)p.N * p.Ho <= (1LL << 30); }

gconv_status make_conv1d(Conv1d* p, int B, int T, int C, int K, int pl, int pr, int dtype) {
  if (B < 0 || T <= 0 || C <= 0 || K <= 0 || pl < 0 || pr < 0) return GCONV_ERR_INVALID_ARG;
  if (dtype != GCONV_F32 && dtype != GCONV_F16 && dtype != GCONV_BF16) return GCONV_ERR_INVALID_ARG;
  const long long T_out = (long long)T + pl + pr - K + 1;
  if (T_out < 1 || T_out > INT_MAX) return GCONV_ERR_INVALID_ARG;
  const long long n = (long long)B * (T > T_out ? T : T_out) * C;
  if (n > (1LL << 40)) return GCONV_ERR_INVALID_ARG;
  p->B = B; p->T = T; p->C = C; p->K = K; p->pad_left = pl; p->pad_right = pr;
  p->T_out = (int)T_out; p->dtype = dtype;
  return GCONV_OK;
}

// ------------------------------------------------------------------ depthwise-separable block
size_t elem_bytes(int dtype) { return dtype == GCONV_F32 ? 4 : 2; }

// Kernel for a dwsep1d_fwd call: the fused kernel, or the two-kernel composition (depthwise
// into the workspace, then the pointwise GEMM). x / wdw / wpw / z null = query mode.
int dwsep1d_choose(const Conv1d& p, int C_out, int path, const void* x, const void* wdw,
                   const void* wpw, const void* z, gconv_status* why) {
  *why = GCONV_OK;
  const bool query = x == nullptr && wdw == nullptr && wpw == nullptr && z == nullptr;
  const bool fused_ok = dwsep1d_fused_supported(p, C_out);
  const bool fused_al = query || (aligned16(x) && aligned16(wdw) && aligned16(wpw) &&
                                  aligned16(z));
  switch (path) {
    case GCONV_PATH_AUTO:
      return fused_ok && fused_al ? GCONV_KERNEL_DWSEP1D_FUSED : GCONV_KERNEL_DWSEP_UNFUSED;
    case GCONV_PATH_IGEMM:
      if (!fused_ok) { *why = GCONV_ERR_UNSUPPORTED; return -1; }
      if (!fused_al) { *why = GCONV_ERR_MISALIGNED; return -1; }
      return GCONV_KERNEL_DWSEP1D_FUSED;
    case GCONV_PATH_DIRECT:
    case GCONV_PATH_GENERIC:
      return GCONV_KERNEL_DWSEP_UNFUSED;
    default:
      *why = GCONV_ERR_INVALID_ARG;
      return -1;
  }
}

// Depthwise outputs up to this size stay in the 126 MB L2 between two launches.
constexpr double kDwsepL2Bytes = 96.0 * 1024 * 1024;

// The 2-D block: `p` is its depthwise problem (groups = C_in = C_out = C).
int dwsep2d_choose(const Conv2d& p, int C_out, int path, const void* x, const void* wdw,
                   const void* wpw, const void* z, gconv_status* why) {
  *why = GCONV_OK;
  const bool query = x == nullptr && wdw == nullptr && wpw == nullptr && z == nullptr;
  const bool fused_ok = dwsep2d_fused_supported(p, C_out);
  const bool fused_al = query || (aligned16(x) && aligned16(wdw) && aligned16(wpw) &&
                                  aligned16(z));
  // AUTO takes the fused kernel only when the depthwise output would not stay in L2 between
  // the two launches of the composition: with it resident, the composition moves no more
  // HBM bytes than the fused kernel and ran faster (stride-2 block x[8,512,128,256]: 122 us
  // against 142 us, measured from a clean cold L2)
  const bool d_in_l2 =
      (double)p.N * p.Ho * p.Wo * p.C_out * elem_bytes(p.dtype) <= kDwsepL2Bytes;
  switch (path) {
    case GCONV_PATH_AUTO:
      return fused_ok && fused_al && !d_in_l2 ? GCONV_KERNEL_DWSEP2D_FUSED
                                              : GCONV_KERNEL_DWSEP_UNFUSED;
    case GCONV_PATH_IGEMM:
      if (!fused_ok) { *why = GCONV_ERR_UNSUPPORTED; return -1; }
      if (!fused_al) { *why = GCONV_ERR_MISALIGNED; return -1; }
      return GCONV_KERNEL_DWSEP2D_FUSED;
    case GCONV_PATH_DIRECT:
    case GCONV_PATH_GENERIC:
      return GCONV_KERNEL_DWSEP_UNFUSED;
    default:
      *why = GCONV_ERR_INVALID_ARG;
      return -1;
  }
}

// Composition workspace of the 2-D block: the depthwise output, then the depthwise call's and
// the pointwise call's own workspaces (NCHW tensor-core staging).
struct Dwsep2dWs {
  size_t d_bytes, dw_ws, pw_ws, total;
};

Dwsep2dWs dwsep2d_ws(const Conv2d& p, const Conv2d& q, int path) {
  Dwsep2dWs w{};
  w.d_bytes = round_up((size_t)p.N * p.C_out * p.Ho * p.Wo * elem_bytes(p.dtype), 256);
  gconv_status why;
  const int part = path == GCONV_PATH_GENERIC ? GCONV_PATH_GENERIC : GCONV_PATH_AUTO;
  const int k1 = choose_kernel(p, part, nullptr, nullptr, nullptr, &why);
  const int k2 = choose_kernel(q, part, nullptr, nullptr, nullptr, &why);
  w.dw_ws = k1 == GCONV_KERNEL_IGEMM_TC_NCHW ? round_up(igemm_nchw_workspace(p), 256) : 0;
  w.pw_ws = k2 == GCONV_KERNEL_IGEMM_TC_NCHW ? round_up(igemm_nchw_workspace(q), 256) : 0;
  w.total = w.d_bytes + (w.dw_ws > w.pw_ws ? w.dw_ws : w.pw_ws);
  return w;
}

size_t dwsep1d_workspace(const Conv1d& p, int kernel) {
  if (kernel != GCONV_KERNEL_DWSEP_UNFUSED) return 0;
  return round_up((size_t)p.B * p.T_out * p.C * elem_bytes(p.dtype), 256);
}

}  // namespace
}  // namespace gconv

using namespace gconv;

extern "C" {

gconv_status gconv2d_out_shape(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                               int stride, int pad, int dilation, int groups,
                               gconv_layout layout, gconv_dtype dtype, gconv_out_mode out_mode,
                               int* C_y, int* Ho, int* Wo) {
  if (C_y == nullptr || Ho == nullptr || Wo == nullptr) return GCONV_ERR_INVALID_ARG;
  Conv2d p;
  const gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation,
                                      groups, layout, dtype, out_mode);
  if (st != GCONV_OK) return st;
  *C_y = out_channels(p);
  *Ho = p.Ho;
  *Wo = p.Wo;
  return GCONV_OK;
}

size_t gconv2d_fwd_out_workspace_size(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                      int stride, int pad, int dilation, int groups,
                                      gconv_layout layout, gconv_dtype dtype,
                                      gconv_out_mode out_mode, gconv_path path) {
  Conv2d p;
  if (make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups, layout,
                  dtype, out_mode) != GCONV_OK)
    return 0;
  gconv_status why;
  const int k = choose_kernel_out(p, path, nullptr, nullptr, nullptr, &why);
  if (k == GCONV_KERNEL_MERGE_MAX_TWO_PASS) {
    Conv2d q = p;
    q.out_mode = GCONV_OUT_GROUP_MAJOR;
    return merge_max_group_major_bytes(p) +
           (p.layout == GCONV_NCHW ? igemm_nchw_workspace(q) : 0);
  }
  return k == GCONV_KERNEL_IGEMM_TC_NCHW ? igemm_nchw_workspace(p) : 0;
}

int gconv2d_fwd_out_select_path(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                int stride, int pad, int dilation, int groups,
                                gconv_layout layout, gconv_dtype dtype, gconv_out_mode out_mode,
                                gconv_path path) {
  Conv2d p;
  gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups,
                                layout, dtype, out_mode);
  if (st != GCONV_OK) return -(int)st;
  const int k = choose_kernel_out(p, path, nullptr, nullptr, nullptr, &st);
  return k < 0 ? -(int)st : k;
}

gconv_status gconv2d_fwd_out(const void* x, const void* w, const void* bias, void* y, int N,
                             int C_in, int H, int W, int C_out, int kH, int kW, int stride,
                             int pad, int dilation, int groups, gconv_layout layout,
                             gconv_dtype dtype, gconv_out_mode out_mode, gconv_path path,
                             void* workspace, size_t workspace_bytes, void* stream) {
  Conv2d p;
  gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups,
                                layout, dtype, out_mode);
  if (st != GCONV_OK) return st;
  if (N > 0 && (x == nullptr || w == nullptr || y == nullptr)) return GCONV_ERR_INVALID_ARG;
  const int kernel = choose_kernel_out(p, path, x, w, y, &st);
  if (kernel < 0) return st;
  if (N == 0) return GCONV_OK;
  if (kernel == GCONV_KERNEL_MERGE_MAX_TWO_PASS) {
    Conv2d q = p;
    q.out_mode = GCONV_OUT_GROUP_MAJOR;
    const size_t g_bytes = merge_max_group_major_bytes(p);
    const size_t stage = p.layout == GCONV_NCHW ? igemm_nchw_workspace(q) : 0;
    if (workspace == nullptr || workspace_bytes < g_bytes + stage || !aligned16(workspace))
      return GCONV_ERR_WORKSPACE;
    const int k1 = p.layout == GCONV_NHWC ? GCONV_KERNEL_IGEMM_TC : GCONV_KERNEL_IGEMM_TC_NCHW;
    st = launch_forward(k1, q, x, w, bias, workspace, (char*)workspace + g_bytes, stage,
                        (cudaStream_t)stream);
    if (st != GCONV_OK) return st;
    return cuda_status(launch_merge_max_groups(p, workspace, y, (cudaStream_t)stream));
  }
  if (out_mode_is_plain(p)) p.out_mode = GCONV_OUT_GROUP_MAJOR;
  return launch_forward(kernel, p, x, w, bias, y, workspace, workspace_bytes,
                        (cudaStream_t)stream);
}

gconv_status dwconv1d_out_steps(int B, int T, int C, int K, int pad_left, int pad_right,
                                gconv_dtype dtype, int* T_out) {
  if (T_out == nullptr) return GCONV_ERR_INVALID_ARG;
  Conv1d p;
  const gconv_status st = make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype);
  if (st != GCONV_OK) return st;
  *T_out = p.T_out;
  return GCONV_OK;
}

size_t gconv2d_fwd_workspace_size(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                  int stride, int pad, int dilation, int groups,
                                  gconv_layout layout, gconv_dtype dtype, gconv_path path) {
  Conv2d p;
  if (make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups, layout,
                  dtype) != GCONV_OK)
    return 0;
  gconv_status why;
  const int k = choose_kernel(p, path, nullptr, nullptr, nullptr, &why);
  return k == GCONV_KERNEL_IGEMM_TC_NCHW ? igemm_nchw_workspace(p) : 0;
}

int gconv2d_select_path(int N, int C_in, int H, int W, int C_out, int kH, int kW, int stride,
                        int pad, int dilation, int groups, gconv_layout layout,
                        gconv_dtype dtype, gconv_path path) {
  Conv2d p;
  gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups,
                                layout, dtype);
  if (st != GCONV_OK) return -(int)st;
  const int k = choose_kernel(p, path, nullptr, nullptr, nullptr, &st);
  return k < 0 ? -(int)st : k;
}

gconv_status gconv2d_fwd_path(const void* x, const void* w, const void* bias, void* y, int N,
                              int C_in, int H, int W, int C_out, int kH, int kW, int stride,
                              int pad, int dilation, int groups, gconv_layout layout,
                              gconv_dtype dtype, gconv_path path, void* workspace,
                              size_t workspace_bytes, void* stream) {
  Conv2d p;
  gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups,
                                layout, dtype);
  if (st != GCONV_OK) return st;
  if (N > 0 && (x == nullptr || w == nullptr || y == nullptr)) return GCONV_ERR_INVALID_ARG;
  const int kernel = choose_kernel(p, path, x, w, y, &st);
  if (kernel < 0) return st;
  if (N == 0) return GCONV_OK;
  return launch_forward(kernel, p, x, w, bias, y, workspace, workspace_bytes,
                        (cudaStream_t)stream);
}

gconv_status gconv2d_fwd(const void* x, const void* w, const void* bias, void* y, int N,
                         int C_in, int H, int W, int C_out, int kH, int kW, int stride, int pad,
                         int dilation, int groups, gconv_layout layout, gconv_dtype dtype,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return gconv2d_fwd_path(x, w, bias, y, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation,
                          groups, layout, dtype, GCONV_PATH_AUTO, workspace, workspace_bytes,
                          stream);
}

size_t gconv2d_bwd_data_workspace_size(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                       int stride, int pad, int dilation, int groups,
                                       gconv_layout layout, gconv_dtype dtype, gconv_path path) {
  Conv2d p, q;
  if (make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups, layout,
                  dtype) != GCONV_OK)
    return 0;
  gconv_status why;
  const int k = dgrad_choose(p, path, nullptr, nullptr, nullptr, &why, &q);
  return k < 0 ? 0 : dgrad_workspace(p, q, k);
}

int gconv2d_bwd_data_select_path(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                 int stride, int pad, int dilation, int groups,
                                 gconv_layout layout, gconv_dtype dtype, gconv_path path) {
  Conv2d p, q;
  gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups,
                                layout, dtype);
  if (st != GCONV_OK) return -(int)st;
  const int k = dgrad_choose(p, path, nullptr, nullptr, nullptr, &st, &q);
  return k < 0 ? -(int)st : k;
}

gconv_status gconv2d_bwd_data_path(const void* dy, const void* w, void* dx, int N, int C_in,
                                   int H, int W, int C_out, int kH, int kW, int stride, int pad,
                                   int dilation, int groups, gconv_layout layout,
                                   gconv_dtype dtype, gconv_path path, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  Conv2d p, q;
  gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups,
                                layout, dtype);
  if (st != GCONV_OK) return st;
  if (N > 0 && (dy == nullptr || w == nullptr || dx == nullptr)) return GCONV_ERR_INVALID_ARG;
  // the flipped filter goes to the start of the workspace; a forward staging area follows it
  const bool ws_al = workspace != nullptr && aligned16(workspace);
  const void* wt = ws_al ? workspace : nullptr;
  const int kernel = N > 0 ? dgrad_choose(p, path, dy, wt, dx, &st, &q)
                           : dgrad_choose(p, path, nullptr, nullptr, nullptr, &st, &q);
  if (kernel < 0) return st;
  if (N == 0) return GCONV_OK;
  const size_t need = dgrad_workspace(p, q, kernel);
  if (need > 0 && (!ws_al || workspace_bytes < need)) return GCONV_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (kernel == GCONV_KERNEL_DGRAD_GENERIC)
    return cuda_status(launch_dgrad_generic(p, dy, w, dx, s));
  if (kernel == GCONV_KERNEL_DGRAD_DEPTHWISE_NHWC)
    return cuda_status(launch_dgrad_depthwise(p, dy, w, dx, s));
  if (kernel == GCONV_KERNEL_DGRAD_DW3S2_TMA)
    return cuda_status(launch_dgrad_dw3s2_tma(p, dy, w, dx, s));
  if (kernel == GCONV_KERNEL_DEPTHWISE_NHWC && depthwise_nhwc_flipped_supported(q))
    return cuda_status(launch_depthwise_nhwc_flipped(q, dy, w, dx, s));
  st = cuda_status(launch_flip_transpose_weight(p, w, workspace, s));
  if (st != GCONV_OK) return st;
  const size_t off = round_up(weight_bytes(p), 256);
  return launch_forward(kernel, q, dy, workspace, nullptr, dx, (char*)workspace + off,
                        workspace_bytes - off, s);
}

gconv_status gconv2d_bwd_data(const void* dy, const void* w, void* dx, int N, int C_in, int H,
                              int W, int C_out, int kH, int kW, int stride, int pad,
                              int dilation, int groups, gconv_layout layout, gconv_dtype dtype,
                              void* workspace, size_t workspace_bytes, void* stream) {
  return gconv2d_bwd_data_path(dy, w, dx, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation,
                               groups, layout, dtype, GCONV_PATH_AUTO, workspace,
                               workspace_bytes, stream);
}

size_t gconv2d_bwd_weight_workspace_size(int N, int C_in, int H, int W, int C_out, int kH,
                                         int kW, int stride, int pad, int dilation, int groups,
                                         gconv_layout layout, gconv_dtype dtype,
                                         gconv_path path) {
  Conv2d p;
  if (make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups, layout,
                  dtype) != GCONV_OK || !wgrad_rows_ok(p))
    return 0;
  gconv_status why;
  const int k = wgrad_choose(p, path, nullptr, nullptr, &why);
  return k < 0 ? 0 : wgrad_workspace(p, k);
}

int gconv2d_bwd_weight_select_path(int N, int C_in, int H, int W, int C_out, int kH, int kW,
                                   int stride, int pad, int dilation, int groups,
                                   gconv_layout layout, gconv_dtype dtype, gconv_path path) {
  Conv2d p;
  gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups,
                                layout, dtype);
  if (st != GCONV_OK) return -(int)st;
  if (!wgrad_rows_ok(p)) return -(int)GCONV_ERR_UNSUPPORTED;
  const int k = wgrad_choose(p, path, nullptr, nullptr, &st);
  return k < 0 ? -(int)st : k;
}

gconv_status gconv2d_bwd_weight_path(const void* x, const void* dy, void* dw, int N, int C_in,
                                     int H, int W, int C_out, int kH, int kW, int stride,
                                     int pad, int dilation, int groups, gconv_layout layout,
                                     gconv_dtype dtype, gconv_path path, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  Conv2d p;
  gconv_status st = make_conv2d(&p, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation, groups,
                                layout, dtype);
  if (st != GCONV_OK) return st;
  if (dw == nullptr || (N > 0 && (x == nullptr || dy == nullptr))) return GCONV_ERR_INVALID_ARG;
  if (!wgrad_rows_ok(p)) return GCONV_ERR_UNSUPPORTED;
  const int kernel = N > 0 ? wgrad_choose(p, path, x, dy, &st)
                           : wgrad_choose(p, path, nullptr, nullptr, &st);
  if (kernel < 0) return st;
  const size_t need = wgrad_workspace(p, kernel);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return GCONV_ERR_WORKSPACE;
  return cuda_status(launch_wgrad(p, x, dy, dw, workspace, kernel, (cudaStream_t)stream));
}

gconv_status gconv2d_bwd_weight(const void* x, const void* dy, void* dw, int N, int C_in, int H,
                                int W, int C_out, int kH, int kW, int stride, int pad,
                                int dilation, int groups, gconv_layout layout, gconv_dtype dtype,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return gconv2d_bwd_weight_path(x, dy, dw, N, C_in, H, W, C_out, kH, kW, stride, pad, dilation,
                                 groups, layout, dtype, GCONV_PATH_AUTO, workspace,
                                 workspace_bytes, stream);
}

gconv_status dwconv1d_fwd_path(const void* x, const void* w, void* y, int B, int T, int C, int K,
                               int pad_left, int pad_right, gconv_dtype dtype, gconv_path path,
                               void* stream) {
  Conv1d p;
  gconv_status st = make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype);
  if (st != GCONV_OK) return st;
  if (B > 0 && (x == nullptr || w == nullptr || y == nullptr)) return GCONV_ERR_INVALID_ARG;
  const int kernel = conv1d_choose_kernel(p, path, x, w, y, &st);
  if (kernel < 0) return st;
  if (B == 0) return GCONV_OK;
  return cuda_status(launch_dwconv1d_fwd(p, x, w, y, false, pad_left, T, p.T_out, kernel,
                                         (cudaStream_t)stream));
}

gconv_status dwconv1d_fwd(const void* x, const void* w, void* y, int B, int T, int C, int K,
                          int pad_left, int pad_right, gconv_dtype dtype, void* stream) {
  return dwconv1d_fwd_path(x, w, y, B, T, C, K, pad_left, pad_right, dtype, GCONV_PATH_AUTO,
                           stream);
}

gconv_status dwconv1d_bwd_data_path(const void* dy, const void* w, void* dx, int B, int T, int C,
                                    int K, int pad_left, int pad_right, gconv_dtype dtype,
                                    gconv_path path, void* stream) {
  Conv1d p;
  gconv_status st = make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype);
  if (st != GCONV_OK) return st;
  if (B > 0 && (dy == nullptr || w == nullptr || dx == nullptr)) return GCONV_ERR_INVALID_ARG;
  const int kernel = conv1d_choose_kernel(p, path, dy, w, dx, &st);
  if (kernel < 0) return st;
  if (B == 0) return GCONV_OK;
  // dx = forward of dy (T_out steps) with the reversed filter and left pad K-1-pad_left
  return cuda_status(launch_dwconv1d_fwd(p, dy, w, dx, true, K - 1 - pad_left, p.T_out, T,
                                         kernel, (cudaStream_t)stream));
}

gconv_status dwconv1d_bwd_data(const void* dy, const void* w, void* dx, int B, int T, int C,
                               int K, int pad_left, int pad_right, gconv_dtype dtype,
                               void* stream) {
  return dwconv1d_bwd_data_path(dy, w, dx, B, T, C, K, pad_left, pad_right, dtype,
                                GCONV_PATH_AUTO, stream);
}

int dwconv1d_select_path(int B, int T, int C, int K, int pad_left, int pad_right,
                         gconv_dtype dtype, gconv_path path) {
  Conv1d p;
  gconv_status st = make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype);
  if (st != GCONV_OK) return -(int)st;
  const int k = conv1d_choose_kernel(p, path, nullptr, nullptr, nullptr, &st);
  return k < 0 ? -(int)st : k;
}

size_t dwconv1d_bwd_weight_workspace_size(int B, int T, int C, int K, int pad_left,
                                          int pad_right, gconv_dtype dtype) {
  Conv1d p;
  if (make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype) != GCONV_OK) return 0;
  return dwconv1d_wgrad_workspace(p);
}

gconv_status dwconv1d_bwd_weight(const void* x, const void* dy, void* dw, void* workspace,
                                 size_t workspace_bytes, int B, int T, int C, int K,
                                 int pad_left, int pad_right, gconv_dtype dtype, void* stream) {
  Conv1d p;
  gconv_status st = make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype);
  if (st != GCONV_OK) return st;
  if (dw == nullptr || (B > 0 && (x == nullptr || dy == nullptr))) return GCONV_ERR_INVALID_ARG;
  const size_t need = dwconv1d_wgrad_workspace(p);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return GCONV_ERR_WORKSPACE;
  return cuda_status(launch_dwconv1d_wgrad(p, x, dy, dw, workspace, (cudaStream_t)stream));
}

gconv_status dwconv1d_bwd_weight_noalloc(const void* x, const void* dy, void* dw, int B, int T,
                                         int C, int K, int pad_left, int pad_right,
                                         gconv_dtype dtype, void* stream) {
  Conv1d p;
  gconv_status st = make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype);
  if (st != GCONV_OK) return st;
  if (dw == nullptr || (B > 0 && (x == nullptr || dy == nullptr))) return GCONV_ERR_INVALID_ARG;
  if (dwconv1d_wgrad_workspace(p) > dwconv1d_wgrad_noalloc_limit()) return GCONV_ERR_WORKSPACE;
  return cuda_status(launch_dwconv1d_wgrad_noalloc(p, x, dy, dw, (cudaStream_t)stream));
}

size_t dwsep1d_fwd_workspace_size(int B, int T, int C, int K, int pad_left, int pad_right,
                                  int C_out, gconv_dtype dtype, gconv_path path) {
  Conv1d p;
  if (C_out <= 0 || make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype) != GCONV_OK) return 0;
  gconv_status why;
  const int k = dwsep1d_choose(p, C_out, path, nullptr, nullptr, nullptr, nullptr, &why);
  return k < 0 ? 0 : dwsep1d_workspace(p, k);
}

int dwsep1d_select_path(int B, int T, int C, int K, int pad_left, int pad_right, int C_out,
                        gconv_dtype dtype, gconv_path path) {
  Conv1d p;
  if (C_out <= 0) return -(int)GCONV_ERR_INVALID_ARG;
  gconv_status st = make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype);
  if (st != GCONV_OK) return -(int)st;
  const int k = dwsep1d_choose(p, C_out, path, nullptr, nullptr, nullptr, nullptr, &st);
  return k < 0 ? -(int)st : k;
}

gconv_status dwsep1d_fwd(const void* x, const void* w_dw, const void* w_pw, const void* bias,
                         void* z, int B, int T, int C, int K, int pad_left, int pad_right,
                         int C_out, gconv_dtype dtype, gconv_path path, void* workspace,
                         size_t workspace_bytes, void* stream) {
  Conv1d p;
  if (C_out <= 0) return GCONV_ERR_INVALID_ARG;
  gconv_status st = make_conv1d(&p, B, T, C, K, pad_left, pad_right, dtype);
  if (st != GCONV_OK) return st;
  if ((long long)B * p.T_out * C_out > (1LL << 40)) return GCONV_ERR_INVALID_ARG;
  if (B > 0 && (x == nullptr || w_dw == nullptr || w_pw == nullptr || z == nullptr))
    return GCONV_ERR_INVALID_ARG;
  const int kernel = B > 0 ? dwsep1d_choose(p, C_out, path, x, w_dw, w_pw, z, &st)
                           : dwsep1d_choose(p, C_out, path, nullptr, nullptr, nullptr, nullptr,
                                            &st);
  if (kernel < 0) return st;
  const size_t need = dwsep1d_workspace(p, kernel);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return GCONV_ERR_WORKSPACE;
  if (B == 0) return GCONV_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (kernel == GCONV_KERNEL_DWSEP1D_FUSED)
    return cuda_status(launch_dwsep1d_fused(p, C_out, x, w_dw, w_pw, bias, z, s));
  // composition: the depthwise output d [B][T_out][C] in the workspace, then z = the pointwise
  // convolution of d as B images of 1 x T_out pixels (NHWC), weights [C_out][1][1][C]
  const int part = path == GCONV_PATH_GENERIC ? GCONV_PATH_GENERIC : GCONV_PATH_AUTO;
  st = dwconv1d_fwd_path(x, w_dw, workspace, B, T, C, K, pad_left, pad_right, dtype,
                         (gconv_path)part, stream);
  if (st != GCONV_OK) return st;
  Conv2d q;
  st = make_conv2d(&q, B, C, 1, p.T_out, C_out, 1, 1, 1, 0, 1, 1, GCONV_NHWC, dtype);
  if (st != GCONV_OK) return st;
  const int k2 = choose_kernel(q, part, workspace, w_pw, z, &st);
  if (k2 < 0) return st;
  if (k2 == GCONV_KERNEL_IGEMM_TC_NCHW) return GCONV_ERR_UNSUPPORTED;   // NHWC only here
  return launch_forward(k2, q, workspace, w_pw, bias, z, nullptr, 0, s);
}

namespace {
// Depthwise problem p and pointwise problem q of a 2-D block.
gconv_status make_dwsep2d(Conv2d* p, Conv2d* q, int N, int C, int H, int W, int kH, int kW,
                          int stride, int pad, int dilation, int C_out, int layout, int dtype) {
  if (C_out <= 0) return GCONV_ERR_INVALID_ARG;
  gconv_status st = make_conv2d(p, N, C, H, W, C, kH, kW, stride, pad, dilation, C, layout,
                                dtype);
  if (st != GCONV_OK) return st;
  return make_conv2d(q, N, C, p->Ho, p->Wo, C_out, 1, 1, 1, 0, 1, 1, layout, dtype);
}
}  // namespace

size_t dwsep2d_fwd_workspace_size(int N, int C, int H, int W, int kH, int kW, int stride,
                                  int pad, int dilation, int C_out, gconv_layout layout,
                                  gconv_dtype dtype, gconv_path path) {
  Conv2d p, q;
  if (make_dwsep2d(&p, &q, N, C, H, W, kH, kW, stride, pad, dilation, C_out, layout, dtype) !=
      GCONV_OK)
    return 0;
  gconv_status why;
  const int k = dwsep2d_choose(p, C_out, path, nullptr, nullptr, nullptr, nullptr, &why);
  return k == GCONV_KERNEL_DWSEP_UNFUSED ? dwsep2d_ws(p, q, path).total : 0;
}

int dwsep2d_select_path(int N, int C, int H, int W, int kH, int kW, int stride, int pad,
                        int dilation, int C_out, gconv_layout layout, gconv_dtype dtype,
                        gconv_path path) {
  Conv2d p, q;
  gconv_status st =
      make_dwsep2d(&p, &q, N, C, H, W, kH, kW, stride, pad, dilation, C_out, layout, dtype);
  if (st != GCONV_OK) return -(int)st;
  const int k = dwsep2d_choose(p, C_out, path, nullptr, nullptr, nullptr, nullptr, &st);
  return k < 0 ? -(int)st : k;
}

gconv_status dwsep2d_fwd(const void* x, const void* w_dw, const void* w_pw, const void* bias,
                         void* z, int N, int C, int H, int W, int kH, int kW, int stride,
                         int pad, int dilation, int C_out, gconv_layout layout,
                         gconv_dtype dtype, gconv_path path, void* workspace,
                         size_t workspace_bytes, void* stream) {
  Conv2d p, q;
  gconv_status st =
      make_dwsep2d(&p, &q, N, C, H, W, kH, kW, stride, pad, dilation, C_out, layout, dtype);
  if (st != GCONV_OK) return st;
  if (N > 0 && (x == nullptr || w_dw == nullptr || w_pw == nullptr || z == nullptr))
    return GCONV_ERR_INVALID_ARG;
  const int kernel = N > 0 ? dwsep2d_choose(p, C_out, path, x, w_dw, w_pw, z, &st)
                           : dwsep2d_choose(p, C_out, path, nullptr, nullptr, nullptr, nullptr,
                                            &st);
  if (kernel < 0) return st;
  const Dwsep2dWs ws = dwsep2d_ws(p, q, path);
  if (kernel == GCONV_KERNEL_DWSEP_UNFUSED &&
      (workspace == nullptr || workspace_bytes < ws.total || !aligned16(workspace)))
    return GCONV_ERR_WORKSPACE;
  if (N == 0) return GCONV_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (kernel == GCONV_KERNEL_DWSEP2D_FUSED)
    return cuda_status(launch_dwsep2d_fused(p, C_out, x, w_dw, w_pw, bias, z, s));
  const int part = path == GCONV_PATH_GENERIC ? GCONV_PATH_GENERIC : GCONV_PATH_AUTO;
  void* d = workspace;
  void* rest = (char*)workspace + ws.d_bytes;
  const size_t rest_bytes = workspace_bytes - ws.d_bytes;
  st = gconv2d_fwd_path(x, w_dw, nullptr, d, N, C, H, W, C, kH, kW, stride, pad, dilation, C,
                        layout, dtype, (gconv_path)part, rest, rest_bytes, stream);
  if (st != GCONV_OK) return st;
  return gconv2d_fwd_path(d, w_pw, bias, z, N, C, p.Ho, p.Wo, C_out, 1, 1, 1, 0, 1, 1, layout,
                          dtype, (gconv_path)part, rest, rest_bytes, stream);
}

gconv_status gconv_debug_set_tx_surplus(unsigned int bytes) {
  if (bytes % 16u != 0 || bytes > (1u << 16)) return GCONV_ERR_INVALID_ARG;
  g_tx_surplus.store(bytes, std::memory_order_relaxed);
  return GCONV_OK;
}

gconv_status gconv_get_device_error(void* stream, int* code) {
  if (code == nullptr) return GCONV_ERR_INVALID_ARG;
  *code = 0;
  const cudaError_t e = read_and_clear_device_error((cudaStream_t)stream, code);
  if (e != cudaSuccess) return GCONV_ERR_CUDA;
  return *code ? GCONV_ERR_DEVICE_TIMEOUT : GCONV_OK;
}

const char* gconv_status_string(gconv_status s) {
  switch (s) {
    case GCONV_OK: return "GCONV_OK";
    case GCONV_ERR_INVALID_ARG: return "GCONV_ERR_INVALID_ARG";
    case GCONV_ERR_UNSUPPORTED: return "GCONV_ERR_UNSUPPORTED";
    case GCONV_ERR_MISALIGNED: return "GCONV_ERR_MISALIGNED";
    case GCONV_ERR_WORKSPACE: return "GCONV_ERR_WORKSPACE";
    case GCONV_ERR_CUDA: return "GCONV_ERR_CUDA";
    case GCONV_ERR_DEVICE_TIMEOUT: return "GCONV_ERR_DEVICE_TIMEOUT";
    default: return "GCONV_ERR_UNKNOWN";
  }
}

int gconv_version(void) { return 100; }

}  // extern "C"
