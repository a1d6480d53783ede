// Weight gradient of a wide-group conv2d on tcgen05 tensor cores (sm_100a).
//
// For group j and filter tap (kh, kw) the weight gradient is a GEMM whose reduction runs over
// the output positions p = (n, ho, wo):
//   dw[co][kh][kw][ci] = sum_p dy[p][co] * x[n, ho - pad + kh*dil, wo - pad + kw*dil, ci]
// i.e. D[co x ci] = A[co x p] * B[p x ci] with A = dy^T and B = the input shifted by the tap.
// In NHWC both operands have their channels contiguous, so both are read by the MMA as
// MN-major tiles (128-byte swizzle), straight from TMA boxes with no transpose:
//   * A: per block of 128 output pixels of one row, two boxes dy[64 co x 128 px];
//   * B: per block, the input strip of 128 + 8 pixels of the row the tap reads (one box of
//     128 pixels and an 8-pixel halo box per 64 input channels); the kW taps are the same strip
//     read from starting rows kw*dil, so the input is fetched once for all kW taps.
// A CTA owns one (group, 128 filters, block of input channels, kh) and a fixed slice of the
// position blocks; it keeps the kW accumulators D_kw (fp32, TMEM) for its slice and writes
// them as fp32 partials ws[slice][co][kh][kw][ci]; the library's slice-sum kernel adds the
// slices in slice order and rounds once. The slices are a function of the shape only, and
// every accumulation runs in a fixed order, so dw is bitwise reproducible.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer (one thread), warps 2-5
// epilogue (TMEM -> registers -> partials). Every mbarrier wait is bounded (1 s); a wait that
// gives up sets the library's device error word and the CTA drains and exits.
#include <cuda.h>

#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

using namespace ptx;

constexpr int WT_M = 128;              // filters per CTA (MMA M)
constexpr int WT_P = 128;              // output pixels per position block (MMA K per block)
constexpr int WT_HALO = 8;             // extra input pixels per strip: (kW - 1) * dil <= 8
constexpr int WT_THREADS = 192;
constexpr int WT_MAX_STAGES = 4;
constexpr int WT_TARGET_CTAS = 148;    // slices are chosen for about this many CTAs in all
constexpr unsigned int ERR_WT = 1u << 16;

struct WtParams {
  int N, H, W, Ho, Wo, C_in, C_out, kH, kW, pad, dil, cpg_in, cpg_out;
  int NB;                 // input channels per CTA (MMA N): 64 or 128
  int n_cb, n_nb;         // filter blocks (of 128) and input-channel blocks (of NB) per group
  int segs, blocks;       // 128-pixel segments per output row; position blocks in all
  int units, S;           // (group, co block, ci block, kh) units; position slices
  int stages;
  unsigned int x_sub;     // bytes of one 64-channel input strip (1 KB multiple)
  unsigned int a_bytes, stage_bytes, tx_bytes;
  unsigned int idesc, tmem_cols;
  long long E;            // dw entries: C_out * kH * kW * cpg_in
};

// MN-major, 128-byte-swizzle operand: LBO = bytes between 64-element atoms along M / N,
// SBO = bytes between groups of 8 K rows (rows of 128 bytes).
__device__ __forceinline__ unsigned long long desc_mn_sw128(unsigned int saddr,
                                                            unsigned int lbo) {
  unsigned long long d = (unsigned long long)((saddr >> 4) & 0x3FFFu);
  d |= (unsigned long long)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (unsigned long long)(1024u >> 4) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

template <typename T>
__global__ void __launch_bounds__(WT_THREADS, 1)
    wgrad_tc_kernel(const __grid_constant__ CUtensorMap tdy,
                    const __grid_constant__ CUtensorMap tx,
                    const __grid_constant__ CUtensorMap txh, float* __restrict__ part,
                    const WtParams P, unsigned int* err) {
  pdl_launch_dependents();   // the slice sum may be scheduled as this grid's CTAs finish
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem(smem_raw, 1024u);
  unsigned long long* bars =
      reinterpret_cast<unsigned long long*>(smem + (size_t)P.stages * P.stage_bytes);
  unsigned long long* full = bars;
  unsigned long long* empty = full + WT_MAX_STAGES;
  unsigned long long* tfull = empty + WT_MAX_STAGES;
  unsigned long long* done = tfull + 1;
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's unit and slice
  const int unit = blockIdx.x / P.S, slice = blockIdx.x - unit * P.S;
  const int kh = unit % P.kH;
  int r = unit / P.kH;
  const int nb = r % P.n_nb;
  r /= P.n_nb;
  const int cb = r % P.n_cb;
  const int j = r / P.n_cb;
  const int co0 = j * P.cpg_out + cb * WT_M;             // first filter (dy channel)
  const int ci0 = j * P.cpg_in + nb * P.NB;              // first input channel
  const int b_begin = (int)((long long)P.blocks * slice / P.S);
  const int b_end = (int)((long long)P.blocks * (slice + 1) / P.S);

  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tdy);
    prefetch_tmap(&tx);
    prefetch_tmap(&txh);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, P.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned int tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: per position block, dy[128 co x 128 px] and the input
      // strip(s) of the row that tap row kh reads
      int s = 0;
      unsigned int ph = 0;
      long long issued = 0;
      for (int blk = b_begin; blk < b_end; ++blk) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, ERR_WT | 1u)) break;
        const int seg = blk % P.segs;
        const int rr = blk / P.segs;
        const int ho = rr % P.Ho, n = rr / P.Ho;
        const int hi = ho - P.pad + kh * P.dil;
        const int wbase = seg * WT_P - P.pad;
        unsigned char* st = smem + (size_t)s * P.stage_bytes;
        mbar_arrive_expect_tx(&full[s], P.tx_bytes);
        tma_load_4d(st, &tdy, &full[s], co0, seg * WT_P, ho, n);
        tma_load_4d(st + 16384, &tdy, &full[s], co0 + 64, seg * WT_P, ho, n);
        for (int sub = 0; sub < P.NB / 64; ++sub) {
          unsigned char* xs = st + P.a_bytes + sub * P.x_sub;
          tma_load_4d(xs, &tx, &full[s], ci0 + sub * 64, wbase, hi, n);
          tma_load_4d(xs + WT_P * 128, &txh, &full[s], ci0 + sub * 64, wbase + WT_P, hi, n);
        }
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
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: per block, kW taps x 8 K-steps of 16 pixels
      int s = 0;
      unsigned int ph = 0;
      bool ok = true;
      const unsigned long long a_desc0 = desc_mn_sw128(smem_u32(smem), 16384u);
      const unsigned long long b_desc0 = desc_mn_sw128(smem_u32(smem + P.a_bytes), P.x_sub);
      const unsigned long long kw_step = (unsigned long long)P.dil * 8u;   // dil rows of 128 B
      for (int blk = b_begin; blk < b_end; ++blk) {
        if (!mbar_wait(&full[s], ph, abort_flag, err, ERR_WT | 2u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const unsigned long long soff = ((unsigned long long)s * P.stage_bytes) >> 4;
        const unsigned long long ad = a_desc0 + soff;
        const unsigned long long bd = b_desc0 + soff;
        const unsigned int first = blk == b_begin ? 1u : 0u;
        for (int kw = 0; kw < P.kW; ++kw) {
          const unsigned int d = tmem_base + (unsigned int)(kw * P.NB);
          const unsigned long long bk = bd + kw * kw_step;
#pragma unroll
          for (int ks = 0; ks < WT_P / 16; ++ks)
            umma_f16(d, ad + 128u * ks, bk + 128u * ks, P.idesc,
                     (first && ks == 0) ? 0u : 1u);
        }
        umma_commit(&empty[s]);
        if (++s == P.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ok) umma_commit(tfull);
      umma_commit(done);
      mbar_wait_until(done, 0, drain_deadline(), err, ERR_DRAIN);
    }
  } else {
    // ---------------- epilogue: warps 2-5; TMEM lane = filter co0 + row
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const bool got = mbar_wait(tfull, 0, abort_flag, err, ERR_WT | 4u);
    if (__all_sync(0xffffffffu, got)) {
      tc_fence_after();
      const unsigned int taddr = tmem_base + ((unsigned int)(quarter * 32) << 16);
      float* dst0 = part + (long long)slice * P.E +
                    ((long long)(co0 + row) * P.kH + kh) * P.kW * P.cpg_in + nb * P.NB;
      for (int kw = 0; kw < P.kW; ++kw) {
        float* dst = dst0 + (long long)kw * P.cpg_in;
        for (int c = 0; c < P.NB; c += 32) {
          unsigned int v[32];
          tmem_ld32(taddr + (unsigned int)(kw * P.NB + c), v);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<uint4*>(dst + c)[q] =
                make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
}

bool make_wt_params(const Conv2d& p, WtParams* P) {
  if (p.layout != GCONV_NHWC || (p.dtype != GCONV_BF16 && p.dtype != GCONV_F16)) return false;
  if (p.stride != 1 || p.cpg_out % WT_M != 0 || p.cpg_in % 64 != 0) return false;
  if ((p.kW - 1) * p.dil > WT_HALO || p.Wo < 32) return false;
  if (p.N > 65535 || p.H > 65535 || p.W > 65535) return false;
  P->N = p.N; P->H = p.H; P->W = p.W; P->Ho = p.Ho; P->Wo = p.Wo;
  P->C_in = p.C_in; P->C_out = p.C_out; P->kH = p.kH; P->kW = p.kW; P->pad = p.pad;
  P->dil = p.dil; P->cpg_in = p.cpg_in; P->cpg_out = p.cpg_out;
  // kW accumulators of NB columns in 512 TMEM columns
  P->NB = (p.cpg_in % 128 == 0 && p.kW * 128 <= 512) ? 128 : 64;
  if (p.kW * P->NB > 512) return false;
  P->n_cb = p.cpg_out / WT_M;
  P->n_nb = p.cpg_in / P->NB;
  P->segs = (p.Wo + WT_P - 1) / WT_P;
  const long long blocks = (long long)p.N * p.Ho * P->segs;
  const long long units = (long long)p.groups * P->n_cb * P->n_nb * p.kH;
  if (blocks > INT32_MAX || units > INT32_MAX) return false;
  P->blocks = (int)blocks;
  P->units = (int)units;
  // as many slices as fill one wave of 148 CTAs without starting a second (a partial second
  // wave would double the time of the slowest CTA)
  long long S = WT_TARGET_CTAS / units;
  if (S > blocks) S = blocks;
  if (S < 1) S = 1;
  if (units * S > INT32_MAX) return false;
  P->S = (int)S;
  P->a_bytes = 2u * 16384u;
  P->x_sub = ((WT_P + WT_HALO) * 128u + 1023u) & ~1023u;
  P->stage_bytes = P->a_bytes + (unsigned int)(P->NB / 64) * P->x_sub;
  P->tx_bytes = P->a_bytes + (unsigned int)(P->NB / 64) * (WT_P + WT_HALO) * 128u;
  const size_t fixed = 1024 + (2 * WT_MAX_STAGES + 2) * 8 + 16;
  int stages = (int)((227u * 1024u - fixed) / P->stage_bytes);
  if (stages > WT_MAX_STAGES) stages = WT_MAX_STAGES;
  if (stages < 2) return false;
  P->stages = stages;
  const unsigned int fmt = p.dtype == GCONV_BF16 ? 1u : 0u;
  P->idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 15) | (1u << 16) |
             ((unsigned int)(P->NB >> 3) << 17) | ((unsigned int)(WT_M >> 4) << 24);
  unsigned int cols = 32;
  while ((int)cols < p.kW * P->NB) cols <<= 1;
  P->tmem_cols = cols;
  P->E = (long long)p.C_out * p.kH * p.kW * p.cpg_in;
  return true;
}

size_t wt_smem(const WtParams& P) {
  return 1024 + (size_t)P.stages * P.stage_bytes + (2 * WT_MAX_STAGES + 2) * 8 + 16;
}

}  // namespace

bool wgrad_tc_supported(const Conv2d& p) {
  Conv2d q = p;
  q.layout = GCONV_NHWC;   // NCHW runs on NHWC copies staged in the workspace
  WtParams P;
  return make_wt_params(q, &P);
}

int wgrad_tc_slices(const Conv2d& p) {
  Conv2d q = p;
  q.layout = GCONV_NHWC;
  WtParams P;
  return make_wt_params(q, &P) ? P.S : 0;
}

// x, dy NHWC (16-byte aligned); part: S * E fp32 partials in the NHWC weight order.
cudaError_t launch_wgrad_tc(const Conv2d& p, const void* x, const void* dy, float* part,
                            cudaStream_t s) {
  WtParams P;
  if (!make_wt_params(p, &P)) return cudaErrorNotSupported;
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  CUtensorMap tdy, tx, txh;
  const cuuint64_t ddim[4] = {(cuuint64_t)p.C_out, (cuuint64_t)p.Wo, (cuuint64_t)p.Ho,
                              (cuuint64_t)p.N};
  const cuuint64_t dstr[3] = {(cuuint64_t)p.C_out * 2, (cuuint64_t)p.Wo * p.C_out * 2,
                              (cuuint64_t)p.Ho * p.Wo * p.C_out * 2};
  const cuuint32_t dbox[4] = {64, (cuuint32_t)WT_P, 1, 1};
  if (enc(&tdy, dt, 4, const_cast<void*>(dy), ddim, dstr, dbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t xdim[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t xstr[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                              (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t xbox[4] = {64, (cuuint32_t)WT_P, 1, 1};
  const cuuint32_t hbox[4] = {64, (cuuint32_t)WT_HALO, 1, 1};
  if (enc(&tx, dt, 4, const_cast<void*>(x), xdim, xstr, xbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (enc(&txh, dt, 4, const_cast<void*>(x), xdim, xstr, hbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = wt_smem(P);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  // one flag per instantiation: each kernel's shared-memory limit is raised separately
  static std::atomic<unsigned int> configured_bf16{0}, configured_f16{0};
  const bool bf16 = p.dtype == GCONV_BF16;
  const void* fn = bf16 ? (const void*)wgrad_tc_kernel<__nv_bfloat16>
                        : (const void*)wgrad_tc_kernel<__half>;
  cudaError_t e = set_max_dynamic_smem(fn, 227 * 1024, bf16 ? configured_bf16 : configured_f16);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(P.units * P.S);
  if (p.dtype == GCONV_BF16)
    wgrad_tc_kernel<__nv_bfloat16><<<grid, WT_THREADS, smem, s>>>(tdy, tx, txh, part, P,
                                                                   device_error_word());
  else
    wgrad_tc_kernel<__half><<<grid, WT_THREADS, smem, s>>>(tdy, tx, txh, part, P,
                                                            device_error_word());
  return cudaGetLastError();
}

}  // namespace gconv
