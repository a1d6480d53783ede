// Per-group implicit GEMM for grouped conv2d on tcgen05 tensor cores (sm_100a).
//
// For group j the convolution is a GEMM  D[M x N] = A[M x K] * B[K x N]  with
//   M = N_img * Ho * Wo output pixels, N = C_out/g filters of the group,
//   K = kH * kW * (C_in/g): for each filter tap, the group's input channels,
// and A is never materialised (no im2col). Grouped convolutions fall off the fp16
// tensor-core path in the half-precision thread ("F.conv2d runs x15 slower in mixed-precision/
// half-precision mode", second reply); this kernel puts every group on the tensor cores in
// one launch, with the group index taken from the tile index -- the "offset the input and
// output by the group from the grid" idea of "Grouped convolutions" (neon issue #296).
//
// Data path (NHWC activations, weights [C_out][kH][kW][C_in/g]):
//  * a tile is 128 output pixels (BH rows x BW columns of one image) x BN filters of one group;
//  * k-block = (tap (kh, kw), block of BKC <= 64 input channels): TMA loads the 4-D box
//    x[n, ho0-pad+kh*dil .., wo0-pad+kw*dil .., c-block] straight into a K-major,
//    BKC*2-byte-swizzled shared tile -- the tap shift is the box origin and the tensor-map's
//    zero fill outside the image is the padding -- and a 2-D box of the weights;
//  * one thread issues tcgen05.mma (kind::f16, bf16/fp16 in, fp32 accumulate) from the two
//    shared tiles into a TMEM accumulator; tcgen05.commit frees the stage;
//  * four epilogue warps read the accumulator with tcgen05.ld, add the bias, round to the
//    output dtype and store (NHWC vector stores, or NCHW stores coalesced along W).
// Persistent CTAs walk the tile list; TMEM holds two accumulators so the epilogue of one tile
// overlaps the MMAs of the next. Every mbarrier wait is bounded (globaltimer); a wait that
// gives up sets the library's device error word and the CTA winds down cleanly.
//
// NCHW: the activations are first transposed to NHWC and the weights repacked to
// [C_out][kH][kW][C_in/g] in the caller's workspace (two small kernels), and the epilogue
// writes NCHW directly.
#include <cuda.h>

#include "igemm_common.cuh"

namespace gconv {
namespace {

using namespace ptx;

// Kernel parameters of the tile kernel; like every parameter struct of the tcgen05 kernels it
// is kept at 128 bytes or less (fields only the host needs stay in Conv2d): a larger struct
// changed the code generated for the same kernel source and cost the row-strip kernel 25 %.
struct IgemmParams {
  int C_out, Ho, Wo, kW, pad, dil, cpg_in, cpg_out;
  int BW, BH, BN, BKC, cblocks, kblocks, tiles_w, tiles_h, m_tiles, n_tiles, num_tiles;
  int stages;
  unsigned int tx_bytes;       // TMA bytes per stage (A box + B box)
  unsigned int a_stage, b_stage;
  unsigned int idesc;
  unsigned int swz;            // smem-descriptor layout code
  unsigned int sbo;            // bytes between 8-row core-matrix groups
  unsigned int tmem_cols;
  int out_nchw;
  // output variants: out_mode (gconv_out_mode), channels of y, groups merged per tile (1 unless
  // the groups are merged: then a tile covers every group, one accumulator per group)
  int groups, out_mode, out_c, nsub;
};


template <typename T, typename PP>
__device__ __forceinline__ void epilogue_store(const PP& P, T* __restrict__ y,
                                               const T* __restrict__ bias, const unsigned int* r,
                                               int ncols, int n, int ho, int wo, int co) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (bias) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < ncols) v[i] += Elem<T>::to_f32(bias[co + i]);
  }
  if (!P.out_nchw) {
    T* dst = y + (((long long)n * P.Ho + ho) * P.Wo + wo) * P.C_out + co;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (q * 8 < ncols) {
        uint4 u;
        u.x = pack2<T>(make_float2(v[8 * q + 0], v[8 * q + 1]));
        u.y = pack2<T>(make_float2(v[8 * q + 2], v[8 * q + 3]));
        u.z = pack2<T>(make_float2(v[8 * q + 4], v[8 * q + 5]));
        u.w = pack2<T>(make_float2(v[8 * q + 6], v[8 * q + 7]));
        *reinterpret_cast<uint4*>(dst + 8 * q) = u;
      }
    }
  } else {
    const long long plane = (long long)P.Ho * P.Wo;
    T* dst = y + ((long long)n * P.C_out + co) * plane + (long long)ho * P.Wo + wo;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < ncols) dst[i * plane] = Elem<T>::from_f32(v[i]);
  }
}

// Stores `ncols` fp32 values (bias already added) of one output pixel: value i goes to channel
// ch0 + i * chs of y's out_c channels -- chs = 1 for the group-major order and for merged
// groups (16-byte NHWC vectors), chs = groups for the interleaved order (scalar stores).
template <typename T>
__device__ __forceinline__ void epilogue_store_mapped(const IgemmParams& P, T* __restrict__ y,
                                                      const float* v, int ncols, int n, int ho,
                                                      int wo, int ch0, int chs) {
  if (!P.out_nchw) {
    T* dst = y + (((long long)n * P.Ho + ho) * P.Wo + wo) * P.out_c + ch0;
    if (chs == 1) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q * 8 < ncols) {
          uint4 u;
          u.x = pack2<T>(make_float2(v[8 * q + 0], v[8 * q + 1]));
          u.y = pack2<T>(make_float2(v[8 * q + 2], v[8 * q + 3]));
          u.z = pack2<T>(make_float2(v[8 * q + 4], v[8 * q + 5]));
          u.w = pack2<T>(make_float2(v[8 * q + 6], v[8 * q + 7]));
          *reinterpret_cast<uint4*>(dst + 8 * q) = u;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < ncols) dst[(long long)i * chs] = Elem<T>::from_f32(v[i]);
    }
  } else {
    const long long plane = (long long)P.Ho * P.Wo;
    T* dst = y + ((long long)n * P.out_c + ch0) * plane + (long long)ho * P.Wo + wo;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < ncols) dst[(long long)i * chs * plane] = Elem<T>::from_f32(v[i]);
  }
}

template <typename T>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    igemm_tc_kernel(const __grid_constant__ CUtensorMap tma_x,
                    const __grid_constant__ CUtensorMap tma_w, const T* __restrict__ bias,
                    T* __restrict__ y, const IgemmParams P, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 1024u);
  unsigned char* a_base = smem;
  unsigned char* b_base = smem + (size_t)P.stages * P.a_stage;
  unsigned long long* bars =
      reinterpret_cast<unsigned long long*>(b_base + (size_t)P.stages * P.b_stage);
  unsigned long long* full = bars;
  unsigned long long* empty = bars + MAX_STAGES;
  unsigned long long* tfull = bars + 2 * MAX_STAGES;
  unsigned long long* tempty = tfull + 2;
  unsigned long long* done = tempty + 2;
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tma_x);
    prefetch_tmap(&tma_w);
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
      // ---------------- TMA producer
      int s = 0;
      unsigned int ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        const int mt = t % P.m_tiles, rest = t / P.m_tiles;
        const int nt = rest % P.n_tiles, jt = rest / P.n_tiles;
        const int tw = mt % P.tiles_w, r2 = mt / P.tiles_w;
        const int th = r2 % P.tiles_h, n = r2 / P.tiles_h;
        const int hbase = th * P.BH - P.pad, wbase = tw * P.BW - P.pad;
        for (int sub = 0; sub < P.nsub && ok; ++sub) {
          const int j = P.nsub > 1 ? sub : jt;
          const int cbase = j * P.cpg_in, obase = j * P.cpg_out + nt * P.BN;
          for (int kb = 0; kb < P.kblocks; ++kb) {
            if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, ERR_WAIT_PRODUCER)) {
              ok = false;
              break;
            }
            const int tap = kb / P.cblocks, cb = kb - tap * P.cblocks;
            const int kh = tap / P.kW, kw = tap - kh * P.kW;
            mbar_arrive_expect_tx(&full[s], P.tx_bytes);
            tma_load_4d(a_base + (size_t)s * P.a_stage, &tma_x, &full[s], cbase + cb * P.BKC,
                        wbase + kw * P.dil, hbase + kh * P.dil, n);
            tma_load_2d(b_base + (size_t)s * P.b_stage, &tma_w, &full[s],
                        tap * P.cpg_in + cb * P.BKC, obase);
            ++issued;
            if (++s == P.stages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
      }
      // copies in flight must land before the CTA can exit (no-op on the normal path)
      const long long first = issued > P.stages ? issued - P.stages : 0;
      const unsigned long long dl = drain_deadline();
      for (long long i = first; i < issued; ++i)
        mbar_wait_until(&full[i % P.stages], (unsigned int)((i / P.stages) & 1), dl, err,
                        ERR_WAIT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int s = 0, acc = 0;
      unsigned int ph = 0, aph = 0;
      bool ok = true;
      const int ksteps = P.BKC / 16;
      // descriptors are built once; per stage and per K step only their address field moves
      // (a 64-bit add of a 16-byte-unit offset), which keeps the issuing thread's dependent
      // instruction chain short enough for back-to-back MMAs
      const unsigned long long a_desc0 = smem_desc(smem_u32(a_base), P.sbo, P.swz);
      const unsigned long long b_desc0 = smem_desc(smem_u32(b_base), P.sbo, P.swz);
      const int subs = (P.num_tiles > (int)blockIdx.x
                            ? (P.num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0) *
                       P.nsub;
      for (int u = 0; u < subs && ok; ++u) {
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, err, ERR_WAIT_MMA)) break;
        tc_fence_after();
        const unsigned int d_tmem = tmem_base + (unsigned int)(acc * P.BN);
        for (int kb = 0; kb < P.kblocks; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, err, ERR_WAIT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const unsigned long long ad = a_desc0 + (((unsigned long long)s * P.a_stage) >> 4);
          const unsigned long long bd = b_desc0 + (((unsigned long long)s * P.b_stage) >> 4);
          umma_f16(d_tmem, ad, bd, P.idesc, kb != 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < 4; ++kk)
            if (kk < ksteps) umma_f16(d_tmem, ad + 2 * kk, bd + 2 * kk, P.idesc, 1u);
          umma_commit(&empty[s]);
          if (++s == P.stages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      // every issued MMA must complete before TMEM is released
      umma_commit(done);
      mbar_wait_until(done, 0, drain_deadline(), err, ERR_WAIT_DRAIN);
    }
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lane quarter (warp % 4)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int hl = row / P.BW, wl = row - hl * P.BW;
    int acc = 0;
    unsigned int aph = 0;
    const bool merge = P.nsub > 1;
    const bool interleave = P.out_mode == GCONV_OUT_INTERLEAVED;
    bool ok = true;
    for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
      const int mt = t % P.m_tiles, rest = t / P.m_tiles;
      const int nt = rest % P.n_tiles, jt = rest / P.n_tiles;
      const int tw = mt % P.tiles_w, r2 = mt / P.tiles_w;
      const int th = r2 % P.tiles_h, n = r2 / P.tiles_h;
      const int ho = th * P.BH + hl, wo = tw * P.BW + wl;
      const bool valid = hl < P.BH && ho < P.Ho && wo < P.Wo;
      float run[64];   // merged groups: running sum / maximum over the tile's sub-tiles
      for (int sub = 0; sub < P.nsub; ++sub) {
        const bool got = mbar_wait(&tfull[acc], aph, abort_flag, err, ERR_WAIT_EPILOGUE);
        if (!__all_sync(0xffffffffu, got)) {     // warp-uniform: tcgen05.ld is .aligned
          ok = false;
          break;
        }
        tc_fence_after();
        const int j = merge ? sub : jt;
        const int co0 = j * P.cpg_out + nt * P.BN;
        const unsigned int taddr =
            tmem_base + ((unsigned int)(quarter * 32) << 16) + (unsigned int)(acc * P.BN);
        if (!merge) {
          for (int c = 0; c < P.BN; c += 32) {
            unsigned int r[32];
            const int ncols = P.BN - c < 32 ? P.BN - c : 32;
            if (ncols == 32)
              tmem_ld32(taddr + c, r);
            else
              tmem_ld16(taddr + c, r);
            tmem_ld_wait();
            if (!valid) continue;
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] = __uint_as_float(r[i]) +
                     (bias && i < ncols ? Elem<T>::to_f32(bias[co0 + c + i]) : 0.0f);
            if (interleave)
              epilogue_store_mapped<T>(P, y, v, ncols, n, ho, wo,
                                       (nt * P.BN + c) * P.groups + j, P.groups);
            else
              epilogue_store_mapped<T>(P, y, v, ncols, n, ho, wo, co0 + c, 1);
          }
        } else {
          // BN <= 64: both 32-column halves unrolled so that `run` stays in registers
#pragma unroll
          for (int c = 0; c < 64; c += 32) {
            if (c < P.BN) {
              unsigned int r[32];
              const int ncols = P.BN - c < 32 ? P.BN - c : 32;
              if (ncols == 32)
                tmem_ld32(taddr + c, r);
              else
                tmem_ld16(taddr + c, r);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float v = __uint_as_float(r[i]) +
                                (bias && i < ncols ? Elem<T>::to_f32(bias[co0 + c + i]) : 0.0f);
                run[c + i] = sub == 0 ? v
                             : (P.out_mode == GCONV_OUT_MERGE_MAX ? fmaxf(run[c + i], v)
                                                                  : run[c + i] + v);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (ok && merge && valid) {
        const float scale = P.out_mode == GCONV_OUT_MERGE_AVG ? 1.0f / (float)P.groups : 1.0f;
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          if (c < P.BN) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = run[c + i] * scale;
            epilogue_store_mapped<T>(P, y, v, P.BN - c < 32 ? P.BN - c : 32, n, ho, wo,
                                     nt * P.BN + c, 1);
          }
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

// ------------------------------------------------------------------ halo tile kernel
//
// For images narrower than 128 outputs (whole rows per tile: BW = Wo, BH = 128 / Wo rows), a
// stage is one input-channel block and KWS filter columns: per column kw one TMA box of
// BH + (kH-1)*dil input rows x Wo pixels, whose kH taps are the same box read from row offsets
// kh*dil*Wo (whole 8-row swizzle atoms, since Wo % 8 == 0), plus the kH*KWS weight tiles.
// Each stage thus feeds kH*KWS*BKC/16 MMAs to the single issuing thread between barrier waits,
// and the input is fetched once per kw instead of once per tap.
//
// Groups of 16 or 32 input channels are packed gp = 64 / cpg_in to a tile: the box holds their
// 64 channels (one 128-byte row per pixel) and the filter tile is block-diagonal -- filter f of
// packed group g has its cpg_in weights in channel slot g and zeros elsewhere -- so one MMA
// chain computes all gp groups at N = gp*cpg_out. TMA builds the block-diagonal tile: each
// group's filters are read through a [C_out][taps][cpg_in] view with a 64-channel box started
// g*cpg_in channels before the row, so the other slots fall outside the row and are filled
// with zeros.

struct HaloParams {   // at most 128 bytes, as IgemmParams
  int C_out, Ho, Wo, kH, kW, pad, dil, cpg_in, cpg_out;
  int BW, BH, BN, BKC, cblocks, KWS, kw_groups, tiles_h, m_tiles, n_tiles, num_tiles;
  int stages;
  unsigned int a_region, a_stage, b_tile, b_stage, tx_bytes;
  unsigned int idesc, tmem_cols;   // swizzle, SBO and row bytes follow from BKC
  int out_nchw;
  int gp;                      // groups packed per tile (block-diagonal filters)
  int tma_out;                 // NHWC output through shared memory and TMA stores
  unsigned int o_bytes;        // that staging, two buffers of BN/64 blocks of [128 rows][64 ch]
                               // with the 128-byte swizzle
};

// Bytes per box row (BKC 16-bit channels) and the matching swizzle code of the smem
// descriptors (128 / 64 / 32-byte swizzle); the stride between 8-row groups is 8 rows.
__host__ __device__ __forceinline__ unsigned int halo_row_bytes(const HaloParams& P) {
  return (unsigned int)P.BKC * 2u;
}
__host__ __device__ __forceinline__ unsigned int halo_swz(unsigned int row_bytes) {
  return row_bytes == 128 ? 2u : (row_bytes == 64 ? 4u : 6u);
}

__device__ __forceinline__ void halo_decode(const HaloParams& P, int t, int& j, int& nt, int& n,
                                            int& th) {
  const int mt = t % P.m_tiles, rest = t / P.m_tiles;
  nt = rest % P.n_tiles;
  j = rest / P.n_tiles;
  th = mt % P.tiles_h;
  n = mt / P.tiles_h;
}

// One halo stage's MMAs with every descriptor built before the first is issued, so the
// issuing thread sends KWS*KH*KS MMAs back to back (rebuilding descriptors between MMAs costs
// over a hundred cycles each, measured). The dispatchers below return false for shapes without
// an instantiation (more than 18 MMAs per stage), which take the loop in the kernel.
template <int KH, int KWS, int KS>
__device__ __forceinline__ void halo_issue_fixed(unsigned int d, unsigned long long ad0,
                                                 unsigned long long bd0,
                                                 unsigned long long kh_step,
                                                 unsigned long long kw_step,
                                                 unsigned long long bt_step, unsigned int idesc,
                                                 bool first) {
  unsigned long long ad[KWS * KH * KS], bd[KWS * KH * KS];
#pragma unroll
  for (int kwi = 0; kwi < KWS; ++kwi)
#pragma unroll
    for (int kh = 0; kh < KH; ++kh)
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int i = (kwi * KH + kh) * KS + k;
        ad[i] = ad0 + kwi * kw_step + kh * kh_step + 2 * k;
        bd[i] = bd0 + (kwi * KH + kh) * bt_step + 2 * k;
      }
#pragma unroll
  for (int i = 0; i < KWS * KH * KS; ++i)
    umma_f16(d, ad[i], bd[i], idesc, (first && i == 0) ? 0u : 1u);
}

template <int KH, int KS>
__device__ __forceinline__ bool halo_issue_kws(int kws, unsigned int d, unsigned long long ad0,
                                               unsigned long long bd0, unsigned long long kh_step,
                                               unsigned long long kw_step,
                                               unsigned long long bt_step, unsigned int idesc,
                                               bool first) {
  // at most 18 MMAs per stage keep their descriptors in registers
  if constexpr (KH * KS <= 18) {
    if (kws == 1) {
      halo_issue_fixed<KH, 1, KS>(d, ad0, bd0, kh_step, kw_step, bt_step, idesc, first);
      return true;
    }
  }
  if constexpr (KH * KH * KS <= 18) {
    if (kws == KH) {
      halo_issue_fixed<KH, KH, KS>(d, ad0, bd0, kh_step, kw_step, bt_step, idesc, first);
      return true;
    }
  }
  return false;
}

template <int KS>
__device__ __forceinline__ bool halo_issue_kh(int kh, int kws, unsigned int d,
                                              unsigned long long ad0, unsigned long long bd0,
                                              unsigned long long kh_step,
                                              unsigned long long kw_step,
                                              unsigned long long bt_step, unsigned int idesc,
                                              bool first) {
  switch (kh) {
    case 1: return halo_issue_kws<1, KS>(kws, d, ad0, bd0, kh_step, kw_step, bt_step, idesc, first);
    case 3: return halo_issue_kws<3, KS>(kws, d, ad0, bd0, kh_step, kw_step, bt_step, idesc, first);
    case 5: return halo_issue_kws<5, KS>(kws, d, ad0, bd0, kh_step, kw_step, bt_step, idesc, first);
    case 7: return halo_issue_kws<7, KS>(kws, d, ad0, bd0, kh_step, kw_step, bt_step, idesc, first);
    default: return false;
  }
}

template <typename T, bool PACK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    igemm_halo_kernel(const __grid_constant__ CUtensorMap tma_x,
                      const __grid_constant__ CUtensorMap tma_w,
                      const __grid_constant__ CUtensorMap tma_y, const T* __restrict__ bias,
                      T* __restrict__ y, const HaloParams P, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 1024u);
  unsigned char* a_base = smem;
  unsigned char* b_base = smem + (size_t)P.stages * P.a_stage;
  unsigned char* o_base = b_base + (size_t)P.stages * P.b_stage;   // output staging
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(o_base + P.o_bytes);
  unsigned long long* full = bars;
  unsigned long long* empty = bars + MAX_STAGES;
  unsigned long long* tfull = bars + 2 * MAX_STAGES;
  unsigned long long* tempty = tfull + 2;
  unsigned long long* done = tempty + 2;
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tma_x);
    prefetch_tmap(&tma_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, P.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned int tmem_base = *tmem_slot;
  // the setup above may overlap the previous kernel in the stream (launch_pdl)
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int s = 0;
      unsigned int ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        int j, nt, n, th;
        halo_decode(P, t, j, nt, n, th);
        const int hbase = th * P.BH - P.pad;
        const int obase = j * (PACK ? P.gp * P.cpg_out : P.cpg_out) + nt * P.BN;
        for (int cb = 0; cb < P.cblocks && ok; ++cb) {
          const int cin = j * (PACK ? P.gp * P.cpg_in : P.cpg_in) + cb * P.BKC;
          for (int kg = 0; kg < P.kw_groups; ++kg) {
            if (!mbar_try_wait(&empty[s], ph ^ 1u) &&
                !mbar_wait(&empty[s], ph ^ 1u, abort_flag, err, ERR_WAIT_PRODUCER)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], P.tx_bytes);
            unsigned char* a_st = a_base + (size_t)s * P.a_stage;
            unsigned char* b_st = b_base + (size_t)s * P.b_stage;
            for (int kwi = 0; kwi < P.KWS; ++kwi) {
              const int kw = kg * P.KWS + kwi;
              tma_load_4d(a_st + (size_t)kwi * P.a_region, &tma_x, &full[s], cin,
                          kw * P.dil - P.pad, hbase, n);
              for (int kh = 0; kh < P.kH; ++kh) {
                unsigned char* bt = b_st + (size_t)(kwi * P.kH + kh) * P.b_tile;
                if constexpr (!PACK) {
                  tma_load_2d(bt, &tma_w, &full[s], (kh * P.kW + kw) * P.cpg_in + cb * P.BKC,
                              obase);
                } else {
                  for (int g = 0; g < P.gp; ++g)
                    tma_load_3d(bt + (size_t)g * P.cpg_out * halo_row_bytes(P), &tma_w, &full[s],
                                -g * P.cpg_in, kh * P.kW + kw, obase + g * P.cpg_out);
                }
              }
            }
            ++issued;
            if (++s == P.stages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
      }
      const unsigned long long dl = drain_deadline();
      for (long long q = (issued > P.stages ? issued - P.stages : 0); q < issued; ++q)
        mbar_wait_until(&full[q % P.stages], (unsigned int)((q / P.stages) & 1), dl, err,
                        ERR_WAIT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer (descriptors built once, advanced by offsets)
      int s = 0, acc = 0;
      unsigned int ph = 0, aph = 0;
      bool ok = true;
      const int ksteps = P.BKC / 16;
      const unsigned int rb = halo_row_bytes(P);
      const unsigned long long a_desc0 = smem_desc(smem_u32(a_base), 8u * rb, halo_swz(rb));
      const unsigned long long b_desc0 = smem_desc(smem_u32(b_base), 8u * rb, halo_swz(rb));
      const unsigned long long kh_step =
          ((unsigned long long)P.dil * P.BW * rb) >> 4;   // kh rows of the box
      const unsigned long long kw_step = P.a_region >> 4;
      const unsigned long long bt_step = P.b_tile >> 4;
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, err, ERR_WAIT_MMA)) break;
        tc_fence_after();
        const unsigned int d = tmem_base + (unsigned int)(acc * P.BN);
        for (int cb = 0; cb < P.cblocks && ok; ++cb) {
          for (int kg = 0; kg < P.kw_groups; ++kg) {
            if (!mbar_try_wait(&full[s], ph) &&
                !mbar_wait(&full[s], ph, abort_flag, err, ERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            const unsigned long long ad0 = a_desc0 + (((unsigned long long)s * P.a_stage) >> 4);
            const unsigned long long bd0 = b_desc0 + (((unsigned long long)s * P.b_stage) >> 4);
            const bool first = (cb | kg) == 0;
            bool fixed = false;
            if (ksteps == 1)
              fixed = halo_issue_kh<1>(P.kH, P.KWS, d, ad0, bd0, kh_step, kw_step, bt_step,
                                       P.idesc, first);
            else if (ksteps == 2)
              fixed = halo_issue_kh<2>(P.kH, P.KWS, d, ad0, bd0, kh_step, kw_step, bt_step,
                                       P.idesc, first);
            else if (ksteps == 4)
              fixed = halo_issue_kh<4>(P.kH, P.KWS, d, ad0, bd0, kh_step, kw_step, bt_step,
                                       P.idesc, first);
            if (!fixed) {
              for (int kwi = 0; kwi < P.KWS; ++kwi) {
                for (int kh = 0; kh < P.kH; ++kh) {
                  const unsigned long long ad = ad0 + kwi * kw_step + kh * kh_step;
                  const unsigned long long bd = bd0 + (kwi * P.kH + kh) * bt_step;
                  const unsigned int acc0 = (first && (kwi | kh) == 0) ? 0u : 1u;
                  umma_f16(d, ad, bd, P.idesc, acc0);
                  for (int k = 1; k < ksteps; ++k)
                    umma_f16(d, ad + 2 * k, bd + 2 * k, P.idesc, 1u);
                }
              }
            }
            umma_commit(&empty[s]);
            if (++s == P.stages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      umma_commit(done);
      mbar_wait_until(done, 0, drain_deadline(), err, ERR_WAIT_DRAIN);
    }
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lane quarter (warp % 4)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int hl = row / P.BW, wl = row - hl * P.BW;
    const bool store_thread = (warp == 2 && lane == 0);
    int acc = 0, ob = 0;
    unsigned int aph = 0;
    for (int t = blockIdx.x; t < P.num_tiles; t += gridDim.x) {
      int j, nt, n, th;
      halo_decode(P, t, j, nt, n, th);
      const bool got = mbar_wait(&tfull[acc], aph, abort_flag, err, ERR_WAIT_EPILOGUE);
      unsigned char* obuf = o_base + (size_t)ob * (P.o_bytes / 2);
      if (P.tma_out) {
        if (store_thread) bulk_wait_read1();       // the store from two tiles back has read it
        if (!named_all(1, 128, got)) break;        // the four warps leave together
      } else if (!__all_sync(0xffffffffu, got)) {
        break;
      }
      tc_fence_after();
      const int ho = th * P.BH + hl, wo = wl;
      const bool valid = hl < P.BH && ho < P.Ho;
      const int co0 = j * (PACK ? P.gp * P.cpg_out : P.cpg_out) + nt * P.BN;
      const unsigned int taddr =
          tmem_base + ((unsigned int)(quarter * 32) << 16) + (unsigned int)(acc * P.BN);
      for (int c = 0; c < P.BN; c += 32) {
        unsigned int r[32];
        const int ncols = P.BN - c < 32 ? P.BN - c : 32;
        if (ncols == 32)
          tmem_ld32(taddr + c, r);
        else
          tmem_ld16(taddr + c, r);
        tmem_ld_wait();
        if (P.tma_out) {
          // 32 channels -> 4 16-byte chunks of this row's 128-byte line in 64-channel block
          // c / 64; chunk k of row r sits at chunk k ^ (r % 8) (the 128-byte swizzle)
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          if (bias) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += Elem<T>::to_f32(bias[co0 + c + i]);
          }
          unsigned char* line = obuf + (size_t)(c >> 6) * (128 * 128) + (size_t)row * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack2<T>(make_float2(v[8 * q + 0], v[8 * q + 1]));
            u.y = pack2<T>(make_float2(v[8 * q + 2], v[8 * q + 3]));
            u.z = pack2<T>(make_float2(v[8 * q + 4], v[8 * q + 5]));
            u.w = pack2<T>(make_float2(v[8 * q + 6], v[8 * q + 7]));
            const int chunk = ((c & 63) >> 3) + q;
            *reinterpret_cast<uint4*>(line + ((chunk ^ (row & 7)) << 4)) = u;
          }
        } else if (valid) {
          epilogue_store<T>(P, y, bias, r, ncols, n, ho, wo, co0 + c);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (P.tma_out) {
        fence_async_smem();
        named_sync(1, 128);
        if (store_thread) {
          for (int blk = 0; blk < P.BN / 64; ++blk)
            tma_store_4d(&tma_y, obuf + (size_t)blk * (128 * 128), co0 + 64 * blk, 0,
                         th * P.BH, n);
          bulk_commit();
        }
        ob ^= 1;
      }
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
    if (store_thread) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
}

// ------------------------------------------------------------------ row-strip kernel
//
// For rows of at least 128 output pixels (Wo >= 128), a tile is NSUB consecutive 128-pixel
// segments of one output row x BN filters. For each (channel block, kh) the TMA warp loads,
// per segment, one strip of 128 + (kW-1)*dil input pixels; the kW taps of that kh are then
// the same strip read from row offsets kw*dil -- a start-address shift of the K-major,
// 128-byte-swizzled operand. The tensor cores apply the 128-byte swizzle to absolute shared-
// memory address bits, as TMA does when it writes the strip, so a start address moved by whole
// 128-byte rows reads exactly the rows TMA wrote there, with the descriptor's base-offset field
// left at 0 (measured: a non-zero base offset there gives wrong sums) -- and each input strip
// is fetched once per kh instead of once per tap. The NSUB segments share
// every weight tile. Strips and weight tiles have their own stage rings.


struct RowParams {
  int N, H, W, C_in, C_out, Ho, Wo, kH, kW, pad, dil, cpg_in, cpg_out;
  int BN, NSUB, cblocks, segs, n_tiles, num_tiles, strip_rows;
  int a_stages, b_stages;
  unsigned int a_stage, strip_stride, b_stage, a_tx, b_tx;
  unsigned int idesc, tmem_cols;
  int out_nchw;
};

__device__ __forceinline__ void row_decode(const RowParams& P, int t, int& j, int& nt, int& n,
                                           int& ho, int& seg) {
  seg = t % P.segs;
  int r = t / P.segs;
  ho = r % P.Ho;
  r /= P.Ho;
  n = r % P.N;
  r /= P.N;
  nt = r % P.n_tiles;
  j = r / P.n_tiles;
}

template <typename T, int NSUB>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    igemm_row_kernel(const __grid_constant__ CUtensorMap tma_x,
                     const __grid_constant__ CUtensorMap tma_w, const T* __restrict__ bias,
                     T* __restrict__ y, const RowParams P, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 1024u);
  unsigned char* a_base = smem;
  unsigned char* b_base = smem + (size_t)P.a_stages * P.a_stage;
  unsigned long long* bars =
      reinterpret_cast<unsigned long long*>(b_base + (size_t)P.b_stages * P.b_stage);
  unsigned long long* fa = bars;
  unsigned long long* ea = fa + ROW_MAX_A;
  unsigned long long* fb = ea + ROW_MAX_A;
  unsigned long long* eb = fb + ROW_MAX_B;
  unsigned long long* tfull = eb + ROW_MAX_B;
  unsigned long long* tempty = tfull + 2;
  unsigned long long* done = tempty + 2;
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.a_stages; ++s) {
      mbar_init(&fa[s], 1);
      mbar_init(&ea[s], 1);
    }
    for (int s = 0; s < P.b_stages; ++s) {
      mbar_init(&fb[s], 1);
      mbar_init(&eb[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tma_x);
    prefetch_tmap(&tma_w);
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
      // ---------------- TMA producer
      int sa = 0, sb = 0;
      unsigned int pa = 0, pb = 0;
      long long na = 0, nb = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        int j, nt, n, ho, seg;
        row_decode(P, t, j, nt, n, ho, seg);
        const int wbase = seg * NSUB * BM - P.pad;
        const int obase = j * P.cpg_out + nt * P.BN;
        for (int cb = 0; cb < P.cblocks && ok; ++cb) {
          const int cin = j * P.cpg_in + cb * 64;
          for (int kh = 0; kh < P.kH && ok; ++kh) {
            if (!mbar_wait(&ea[sa], pa ^ 1u, abort_flag, err, ERR_WAIT_PRODUCER)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&fa[sa], P.a_tx);
            for (int sub = 0; sub < NSUB; ++sub)
              tma_load_4d(a_base + (size_t)sa * P.a_stage + (size_t)sub * P.strip_stride, &tma_x,
                          &fa[sa], cin, wbase + sub * BM, ho - P.pad + kh * P.dil, n);
            ++na;
            if (++sa == P.a_stages) {
              sa = 0;
              pa ^= 1u;
            }
            for (int kw = 0; kw < P.kW; ++kw) {
              if (!mbar_wait(&eb[sb], pb ^ 1u, abort_flag, err, ERR_WAIT_PRODUCER)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&fb[sb], P.b_tx);
              tma_load_2d(b_base + (size_t)sb * P.b_stage, &tma_w, &fb[sb],
                          (kh * P.kW + kw) * P.cpg_in + cb * 64, obase);
              ++nb;
              if (++sb == P.b_stages) {
                sb = 0;
                pb ^= 1u;
              }
            }
          }
        }
      }
      // copies in flight must land before the CTA exits (no-op on the normal path)
      const unsigned long long dl = drain_deadline();
      for (long long q = (na > P.a_stages ? na - P.a_stages : 0); q < na; ++q)
        mbar_wait_until(&fa[q % P.a_stages], (unsigned int)((q / P.a_stages) & 1), dl, err,
                        ERR_WAIT_DRAIN);
      for (long long q = (nb > P.b_stages ? nb - P.b_stages : 0); q < nb; ++q)
        mbar_wait_until(&fb[q % P.b_stages], (unsigned int)((q / P.b_stages) & 1), dl, err,
                        ERR_WAIT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int sa = 0, sb = 0, acc = 0;
      unsigned int pa = 0, pb = 0, aph = 0;
      bool ok = true;
      // descriptors built once; the loop only adds 16-byte-unit offsets (see the tile kernel)
      const unsigned long long a_desc0 = smem_desc(smem_u32(a_base), 1024u, 2u);
      const unsigned long long b_desc0 = smem_desc(smem_u32(b_base), 1024u, 2u);
      const unsigned long long sub_step = P.strip_stride >> 4;
      const unsigned long long kw_step = (unsigned long long)P.dil * 8u;   // dil rows of 128 B
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, err, ERR_WAIT_MMA)) break;
        tc_fence_after();
        const unsigned int d0 = tmem_base + (unsigned int)(acc * NSUB * P.BN);
        for (int cb = 0; cb < P.cblocks && ok; ++cb) {
          for (int kh = 0; kh < P.kH && ok; ++kh) {
            if (!mbar_wait(&fa[sa], pa, abort_flag, err, ERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const unsigned long long a_st = a_desc0 + (((unsigned long long)sa * P.a_stage) >> 4);
            for (int kw = 0; kw < P.kW; ++kw) {
              if (!mbar_wait(&fb[sb], pb, abort_flag, err, ERR_WAIT_MMA)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const unsigned long long bd = b_desc0 + (((unsigned long long)sb * P.b_stage) >> 4);
              unsigned long long ad[NSUB];
              unsigned int dd[NSUB];
#pragma unroll
              for (int sub = 0; sub < NSUB; ++sub) {
                ad[sub] = a_st + kw * kw_step + sub * sub_step;
                dd[sub] = d0 + (unsigned int)(sub * P.BN);
              }
              const unsigned int acc0 = (cb | kh | kw) == 0 ? 0u : 1u;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int sub = 0; sub < NSUB; ++sub)
                  umma_f16(dd[sub], ad[sub] + 2 * kk, bd + 2 * kk, P.idesc, kk == 0 ? acc0 : 1u);
              umma_commit(&eb[sb]);
              if (++sb == P.b_stages) {
                sb = 0;
                pb ^= 1u;
              }
            }
            if (!ok) break;
            umma_commit(&ea[sa]);
            if (++sa == P.a_stages) {
              sa = 0;
              pa ^= 1u;
            }
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      umma_commit(done);
      mbar_wait_until(done, 0, drain_deadline(), err, ERR_WAIT_DRAIN);
    }
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lane quarter (warp % 4)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int acc = 0;
    unsigned int aph = 0;
    for (int t = blockIdx.x; t < P.num_tiles; t += gridDim.x) {
      int j, nt, n, ho, seg;
      row_decode(P, t, j, nt, n, ho, seg);
      const bool got = mbar_wait(&tfull[acc], aph, abort_flag, err, ERR_WAIT_EPILOGUE);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int co0 = j * P.cpg_out + nt * P.BN;
      for (int sub = 0; sub < NSUB; ++sub) {
        const int wo = (seg * NSUB + sub) * BM + row;
        const bool valid = wo < P.Wo;
        const unsigned int taddr = tmem_base + ((unsigned int)(quarter * 32) << 16) +
                                   (unsigned int)((acc * NSUB + sub) * P.BN);
        for (int c = 0; c < P.BN; c += 32) {
          unsigned int r[32];
          const int ncols = P.BN - c < 32 ? P.BN - c : 32;
          if (ncols == 32)
            tmem_ld32(taddr + c, r);
          else
            tmem_ld16(taddr + c, r);
          tmem_ld_wait();
          if (valid) epilogue_store<T>(P, y, bias, r, ncols, n, ho, wo, co0 + c);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
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


// ------------------------------------------------------------------ NCHW staging kernels

// x[n][c][hw] -> xt[n][hw][c], 64 x 64 tiles through shared memory. When HW and C are
// multiples of 8 both the global loads (8 consecutive hw of one channel) and the global stores
// (8 consecutive channels of one pixel) are 16-byte vectors; the transposition itself is done
// with 2-byte shared-memory accesses (row pitch 66 elements against bank conflicts).
template <typename T, bool VEC>
__device__ __forceinline__ void nchw_to_nhwc_tile(const T* __restrict__ x, T* __restrict__ xt,
                                                  int C, int HW, int n, int c0, int s0,
                                                  unsigned short (*tile)[66]) {
  const unsigned short* xn = reinterpret_cast<const unsigned short*>(x) + (long long)n * C * HW;
  unsigned short* tn = reinterpret_cast<unsigned short*>(xt) + (long long)n * C * HW;
  const int tid = threadIdx.x;
  if (VEC) {
    // 64 channels x 8 vectors of 8 pixels: 512 loads, 2 per thread
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + 256 * r;
      const int cl = i >> 3, v = i & 7;
      const int c = c0 + cl, sp = s0 + v * 8;
      uint4 u = make_uint4(0u, 0u, 0u, 0u);
      if (c < C && sp < HW) u = __ldg(reinterpret_cast<const uint4*>(xn + (long long)c * HW + sp));
      const unsigned short* e = reinterpret_cast<const unsigned short*>(&u);
#pragma unroll
      for (int q = 0; q < 8; ++q) tile[cl][v * 8 + q] = e[q];
    }
    __syncthreads();
    // 64 pixels x 8 vectors of 8 channels
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + 256 * r;
      const int sl = i >> 3, v = i & 7;
      const int sp = s0 + sl, c = c0 + v * 8;
      if (sp < HW && c < C) {
        uint4 u;
        unsigned short* e = reinterpret_cast<unsigned short*>(&u);
#pragma unroll
        for (int q = 0; q < 8; ++q) e[q] = tile[v * 8 + q][sl];
        *reinterpret_cast<uint4*>(tn + (long long)sp * C + c) = u;
      }
    }
  } else {
    const int tx = tid & 31, ty = tid >> 5;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int c = c0 + ty + 8 * r;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int sp = s0 + tx + 32 * h;
        if (c < C && sp < HW) tile[ty + 8 * r][tx + 32 * h] = xn[(long long)c * HW + sp];
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int sp = s0 + ty + 8 * r;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = c0 + tx + 32 * h;
        if (c < C && sp < HW) tn[(long long)sp * C + c] = tile[tx + 32 * h][ty + 8 * r];
      }
    }
  }
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(256) nchw_to_nhwc_kernel(const T* __restrict__ x,
                                                           T* __restrict__ xt, int C, int HW) {
  __shared__ unsigned short tile[64][66];   // [c][hw]
  nchw_to_nhwc_tile<T, VEC>(x, xt, C, HW, blockIdx.z, blockIdx.y * 64, blockIdx.x * 64, tile);
}

// w[co][ci][kh][kw] -> wt[co][kh][kw][ci] for filters of at most 8192 elements: one CTA per
// filter reads it with coalesced loads into shared memory and writes it back tap-major with
// coalesced stores.
template <typename T>
__device__ __forceinline__ void repack_filter(const T* __restrict__ w, T* __restrict__ wt,
                                              int cpg_in, int taps, int f, unsigned short* buf) {
  const int n = cpg_in * taps;
  const unsigned short* src = reinterpret_cast<const unsigned short*>(w) + (long long)f * n;
  unsigned short* dst = reinterpret_cast<unsigned short*>(wt) + (long long)f * n;
  // 8 loads per thread in flight before their stores (one load -> store at a time waited out
  // a DRAM latency per element: ~8 us for the wide-group layer's 1.2 MB, measured)
  for (int base = threadIdx.x; base < n; base += 8 * blockDim.x) {
    unsigned short v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = base + q * blockDim.x;
      v[q] = i < n ? src[i] : (unsigned short)0;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = base + q * blockDim.x;
      if (i < n) buf[i] = v[q];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int tap = i / cpg_in, ci = i - tap * cpg_in;
    dst[i] = buf[ci * taps + tap];
  }
}

template <typename T>
__global__ void __launch_bounds__(256) repack_weight_smem_kernel(const T* __restrict__ w,
                                                                 T* __restrict__ wt, int cpg_in,
                                                                 int taps) {
  __shared__ unsigned short buf[8192];
  repack_filter<T>(w, wt, cpg_in, taps, blockIdx.x, buf);
}

// The NCHW staging in one launch: blocks [0, C_out) repack one filter each (as above), blocks
// from C_out on transpose one 64 x 64 tile of x (tile b -> pixel block b % gx, channel block
// (b / gx) % gy, image b / (gx * gy)). The repack is latency-bound (~8 us on its own for the
// 1.2 MB of the wide-group layer's weights, measured) and now runs beside the transpose.
template <typename T, bool VEC>
__global__ void __launch_bounds__(256) nchw_stage_kernel(const T* __restrict__ x,
                                                         T* __restrict__ xt, int C, int HW,
                                                         unsigned int gx, unsigned int gy,
                                                         const T* __restrict__ w,
                                                         T* __restrict__ wt, int C_out,
                                                         int cpg_in, int taps) {
  __shared__ __align__(16) unsigned short smem[8192];   // a filter, or a [64][66] tile
  const unsigned int b = blockIdx.x;
  if (b < (unsigned int)C_out) {
    repack_filter<T>(w, wt, cpg_in, taps, (int)b, smem);
    return;
  }
  const unsigned int t = b - (unsigned int)C_out;
  const unsigned int bx = t % gx, r = t / gx;
  nchw_to_nhwc_tile<T, VEC>(x, xt, C, HW, (int)(r / gy), (int)(r % gy) * 64, (int)bx * 64,
                            reinterpret_cast<unsigned short (*)[66]>(smem));
}

// w[co][ci][kh][kw] -> wt[co][kh][kw][ci]
template <typename T>
__global__ void repack_weight_kernel(const T* __restrict__ w, T* __restrict__ wt, int C_out,
                                     int cpg_in, int taps) {
  // one filter per grid row: wt[co][tap][ci] = w[co][ci][tap], 32-bit index math
  const int n = cpg_in * taps;
  for (int co = blockIdx.y; co < C_out; co += gridDim.y) {
    const T* src = w + (long long)co * n;
    T* dst = wt + (long long)co * n;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
      const int tap = i / cpg_in, ci = i - tap * cpg_in;
      dst[i] = src[ci * taps + tap];
    }
  }
}

// ------------------------------------------------------------------ host side

int tile_bn(const Conv2d& p) {
  if (p.cpg_out <= 256) return p.cpg_out;
  return p.cpg_out % 128 == 0 ? 128 : 0;
}


bool make_params(const Conv2d& p, IgemmParams* P) {
  P->C_out = p.C_out;
  P->Ho = p.Ho; P->Wo = p.Wo; P->kW = p.kW; P->pad = p.pad; P->dil = p.dil;
  P->cpg_in = p.cpg_in; P->cpg_out = p.cpg_out;
  P->BW = p.Wo < BM ? p.Wo : BM;
  P->BH = BM / P->BW;
  if (P->BH > p.Ho) P->BH = p.Ho;
  P->groups = p.groups;
  P->out_mode = p.out_mode;
  P->out_c = out_channels(p);
  const bool merge = p.out_mode == GCONV_OUT_MERGE_AVG || p.out_mode == GCONV_OUT_MERGE_MAX;
  P->nsub = merge ? p.groups : 1;
  // merged groups keep a running value per accumulator column in the epilogue's registers,
  // so their tiles are at most 64 filters wide
  P->BN = !merge ? tile_bn(p)
                 : (p.cpg_out <= 64 ? p.cpg_out
                                    : (p.cpg_out % 64 == 0 ? 64 : (p.cpg_out % 32 == 0 ? 32 : 16)));
  P->BKC = p.cpg_in % 64 == 0 ? 64 : (p.cpg_in % 32 == 0 ? 32 : 16);
  P->cblocks = p.cpg_in / P->BKC;
  P->kblocks = p.kH * p.kW * P->cblocks;
  P->tiles_w = (p.Wo + P->BW - 1) / P->BW;
  P->tiles_h = (p.Ho + P->BH - 1) / P->BH;
  const long long m_tiles = (long long)p.N * P->tiles_w * P->tiles_h;
  P->n_tiles = p.cpg_out / P->BN;
  const long long tiles = m_tiles * P->n_tiles * (merge ? 1 : p.groups);
  if (m_tiles > INT32_MAX || tiles > INT32_MAX) return false;
  P->m_tiles = (int)m_tiles;
  P->num_tiles = (int)tiles;
  const unsigned int row_bytes = (unsigned int)P->BKC * 2u;
  P->a_stage = (BM * row_bytes + 1023u) & ~1023u;
  P->b_stage = ((unsigned int)P->BN * row_bytes + 1023u) & ~1023u;
  P->tx_bytes = (unsigned int)(P->BW * P->BH) * row_bytes + (unsigned int)P->BN * row_bytes;
  const size_t fixed = 1024 + (2 * MAX_STAGES + 5) * 8 + 16;
  int stages = (int)((SMEM_BUDGET - fixed) / (P->a_stage + P->b_stage));
  if (stages > MAX_STAGES) stages = MAX_STAGES;
  if (stages < 2) return false;
  P->stages = stages;
  P->swz = row_bytes == 128 ? 2u : (row_bytes == 64 ? 4u : 6u);   // 128B / 64B / 32B swizzle
  P->sbo = 8u * row_bytes;
  const unsigned int fmt = p.dtype == GCONV_BF16 ? 1u : 0u;        // A/B: 0 = f16, 1 = bf16
  P->idesc = (1u << 4)                     // D format: f32
             | (fmt << 7) | (fmt << 10)    // A, B formats
             | ((unsigned int)(P->BN >> 3) << 17)   // N / 8
             | ((unsigned int)(BM >> 4) << 24);     // M / 16
  P->tmem_cols = pow2_cols(2 * P->BN);
  P->out_nchw = p.layout == GCONV_NCHW;
  return true;
}

size_t smem_bytes(const IgemmParams& P) {
  return 1024 + (size_t)P.stages * (P.a_stage + P.b_stage) + (2 * MAX_STAGES + 5) * 8 + 16;
}

CUtensorMapSwizzle swizzle_of(int BKC) {
  return BKC == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                   : (BKC == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// Row-strip kernel parameters; false if the problem does not take that kernel (rows shorter
// than 128 outputs, channel blocks narrower than 64, or the stage rings do not fit).
bool make_row_params(const Conv2d& p, RowParams* R) {
  if (p.out_mode != GCONV_OUT_GROUP_MAJOR) return false;
  if (p.Wo < BM || p.cpg_in % 64 != 0) return false;
  const int BN = tile_bn(p);
  if (BN == 0) return false;
  R->N = p.N; R->H = p.H; R->W = p.W; R->C_in = p.C_in; R->C_out = p.C_out;
  R->Ho = p.Ho; R->Wo = p.Wo; R->kH = p.kH; R->kW = p.kW; R->pad = p.pad; R->dil = p.dil;
  R->cpg_in = p.cpg_in; R->cpg_out = p.cpg_out;
  R->BN = BN;
  int nsub = 256 / BN;
  const int row_segs = (p.Wo + BM - 1) / BM;
  if (nsub > row_segs) nsub = row_segs;
  if (nsub >= 4) nsub = 4;
  else if (nsub >= 2) nsub = 2;
  else nsub = 1;
  R->NSUB = nsub;
  R->cblocks = p.cpg_in / 64;
  R->segs = (p.Wo + nsub * BM - 1) / (nsub * BM);
  R->n_tiles = p.cpg_out / BN;
  const long long tiles = (long long)R->segs * p.Ho * p.N * R->n_tiles * p.groups;
  if (tiles > INT32_MAX) return false;
  R->num_tiles = (int)tiles;
  R->strip_rows = BM + (p.kW - 1) * p.dil;
  if (R->strip_rows > 256) return false;
  R->strip_stride = ((unsigned int)R->strip_rows * 128u + 1023u) & ~1023u;
  R->a_stage = (unsigned int)nsub * R->strip_stride;
  R->b_stage = (unsigned int)BN * 128u;
  R->a_tx = (unsigned int)nsub * (unsigned int)R->strip_rows * 128u;
  R->b_tx = (unsigned int)BN * 128u;
  const size_t fixed = 1024 + (2 * (ROW_MAX_A + ROW_MAX_B) + 5) * 8 + 16;
  const size_t budget = SMEM_BUDGET - fixed;
  int a_st = 3;
  if ((size_t)a_st * R->a_stage > budget / 2) a_st = 2;
  if ((size_t)a_st * R->a_stage >= budget) return false;
  int b_st = (int)((budget - (size_t)a_st * R->a_stage) / R->b_stage);
  if (b_st > ROW_MAX_B) b_st = ROW_MAX_B;
  if (b_st < 2) return false;
  R->a_stages = a_st;
  R->b_stages = b_st;
  const unsigned int fmt = p.dtype == GCONV_BF16 ? 1u : 0u;
  R->idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | ((unsigned int)(BN >> 3) << 17) |
             ((unsigned int)(BM >> 4) << 24);
  R->tmem_cols = pow2_cols(2 * nsub * BN);
  if (R->tmem_cols > 512) return false;
  R->out_nchw = p.layout == GCONV_NCHW;
  return true;
}

size_t row_smem_bytes(const RowParams& R) {
  return 1024 + (size_t)R.a_stages * R.a_stage + (size_t)R.b_stages * R.b_stage +
         (2 * (ROW_MAX_A + ROW_MAX_B) + 5) * 8 + 16;
}

template <typename T>
cudaError_t launch_row(const Conv2d& p, const RowParams& R, const void* x, const void* w,
                       const void* bias, void* y, cudaStream_t s) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tx, tw;
  const cuuint64_t xdim[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t xstr[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                              (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t xbox[4] = {64, (cuuint32_t)R.strip_rows, 1, 1};
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  if (enc(&tx, dt, 4, const_cast<void*>(x), xdim, xstr, xbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t ktot = (cuuint64_t)p.kH * p.kW * p.cpg_in;
  const cuuint64_t wdim[2] = {ktot, (cuuint64_t)p.C_out};
  const cuuint64_t wstr[1] = {ktot * 2};
  const cuuint32_t wbox[2] = {64, (cuuint32_t)R.BN};
  if (enc(&tw, dt, 2, const_cast<void*>(w), wdim, wstr, wbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = row_smem_bytes(R);
  if (smem > SMEM_BUDGET) return cudaErrorInvalidValue;
  int grid = sm_count();
  if (grid > R.num_tiles) grid = R.num_tiles;
  static std::atomic<unsigned int> configured[3];
  cudaError_t e;
  switch (R.NSUB) {
    case 1:
      e = set_max_dynamic_smem((const void*)igemm_row_kernel<T, 1>, SMEM_BUDGET, configured[0]);
      if (e != cudaSuccess) return e;
      igemm_row_kernel<T, 1><<<grid, NUM_THREADS, smem, s>>>(tx, tw, (const T*)bias, (T*)y, R,
                                                             device_error_word());
      break;
    case 2:
      e = set_max_dynamic_smem((const void*)igemm_row_kernel<T, 2>, SMEM_BUDGET, configured[1]);
      if (e != cudaSuccess) return e;
      igemm_row_kernel<T, 2><<<grid, NUM_THREADS, smem, s>>>(tx, tw, (const T*)bias, (T*)y, R,
                                                             device_error_word());
      break;
    default:
      e = set_max_dynamic_smem((const void*)igemm_row_kernel<T, 4>, SMEM_BUDGET, configured[2]);
      if (e != cudaSuccess) return e;
      igemm_row_kernel<T, 4><<<grid, NUM_THREADS, smem, s>>>(tx, tw, (const T*)bias, (T*)y, R,
                                                             device_error_word());
      break;
  }
  return cudaGetLastError();
}

// Input rows of a halo tile's TMA box: the tile's output rows plus the kH halo.
int halo_box_rows(const Conv2d& p, const HaloParams& H) { return H.BH + (p.kH - 1) * p.dil; }

// Halo tile kernel parameters; false if the problem does not take it (rows wider than 128,
// a width that is not a multiple of 8, or stages that do not fit).
bool make_halo_params(const Conv2d& p, HaloParams* H) {
  if (p.out_mode != GCONV_OUT_GROUP_MAJOR) return false;
  if (p.Wo > BM || p.Wo % 8 != 0) return false;
  // groups packed per tile: 64 / cpg_in of them when that divides the group count and keeps
  // N = gp * cpg_out within 64. The block-diagonal filter tile makes each MMA as wide as the
  // packed N while the MMA count per group stays the same, and MMA time grows with operand
  // bytes (measured: 128x128x16 ~130 cycles against ~100 for 128x64x16), so packing pays only
  // where it lifts a narrow N (g = 64 of the sweep: 16 -> 64, 504 -> 364 us) -- not for
  // 64-filter groups (ensemble layer: 317 -> 377 us when packed in pairs).
  int gp = 1;
  if ((p.cpg_in == 16 || p.cpg_in == 32) && p.groups % (64 / p.cpg_in) == 0 &&
      (64 / p.cpg_in) * p.cpg_out <= 64 && ((64 / p.cpg_in) * p.cpg_out) % 16 == 0)
    gp = 64 / p.cpg_in;
  H->gp = gp;
  const int gin = gp * p.cpg_in, gout = gp * p.cpg_out;   // channels of a packed tile
  const int BN = gp > 1 ? gout : tile_bn(p);
  if (BN == 0) return false;
  H->C_out = p.C_out; H->Ho = p.Ho; H->Wo = p.Wo; H->kH = p.kH; H->kW = p.kW; H->pad = p.pad; H->dil = p.dil;
  H->cpg_in = p.cpg_in; H->cpg_out = p.cpg_out;
  H->BW = p.Wo;
  H->BH = BM / p.Wo;
  if (H->BH > p.Ho) H->BH = p.Ho;
  H->BN = BN;
  H->BKC = gin % 64 == 0 ? 64 : (gin % 32 == 0 ? 32 : 16);
  H->cblocks = gin / H->BKC;
  H->tiles_h = (p.Ho + H->BH - 1) / H->BH;
  const long long m_tiles = (long long)p.N * H->tiles_h;
  H->n_tiles = gout / BN;
  const long long tiles = m_tiles * H->n_tiles * (p.groups / gp);
  if (tiles > INT32_MAX) return false;
  H->m_tiles = (int)m_tiles;
  H->num_tiles = (int)tiles;
  const int box_rows = halo_box_rows(p, *H);
  if (box_rows > 256) return false;
  const unsigned int row_bytes = halo_row_bytes(*H);
  // rows an MMA may read from a box: up to (kH-1)*dil*BW + 128
  unsigned int rows = (unsigned int)(box_rows * H->BW);
  const unsigned int mma_rows = (unsigned int)((p.kH - 1) * p.dil * H->BW + BM);
  if (mma_rows > rows) rows = mma_rows;
  H->a_region = (rows * row_bytes + 1023u) & ~1023u;
  H->b_tile = (unsigned int)BN * row_bytes;
  H->out_nchw = p.layout == GCONV_NCHW;
  H->tma_out = p.layout == GCONV_NHWC && BN % 64 == 0;
  H->o_bytes = H->tma_out ? 2u * (unsigned int)(BN / 64) * 128u * 128u : 0u;
  const size_t fixed = 1024 + (2 * MAX_STAGES + 5) * 8 + 16 + H->o_bytes;
  const size_t budget = SMEM_BUDGET - fixed;
  // all kw of a channel block per stage (one handshake per kH*kW*BKC/16 MMAs) when enough
  // such stages fit -- two with the TMA-store epilogue, whose stores no longer hold the
  // epilogue up, else three -- otherwise one kw per stage
  const int min_stages = H->tma_out ? 2 : 3;
  int kws = p.kW;
  for (;;) {
    const size_t st = (size_t)kws * H->a_region + ((size_t)kws * p.kH * H->b_tile + 1023) / 1024 * 1024;
    const int n = (int)(budget / st);
    if (n >= min_stages || kws == 1) {
      H->KWS = kws;
      H->a_stage = (unsigned int)((size_t)kws * H->a_region);
      H->b_stage = (unsigned int)(((size_t)kws * p.kH * H->b_tile + 1023) / 1024 * 1024);
      H->stages = n > MAX_STAGES ? MAX_STAGES : n;
      break;
    }
    kws = 1;
  }
  if (H->stages < 2) return false;
  H->kw_groups = p.kW / H->KWS;
  H->tx_bytes = (unsigned int)H->KWS *
                ((unsigned int)(H->BKC * H->BW * box_rows * 2) + (unsigned int)p.kH * H->b_tile);
  const unsigned int fmt = p.dtype == GCONV_BF16 ? 1u : 0u;
  H->idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | ((unsigned int)(BN >> 3) << 17) |
             ((unsigned int)(BM >> 4) << 24);
  H->tmem_cols = pow2_cols(2 * BN);
  return true;
}

size_t halo_smem_bytes(const HaloParams& H) {
  return 1024 + (size_t)H.stages * (H.a_stage + H.b_stage) + H.o_bytes +
         (2 * MAX_STAGES + 5) * 8 + 16;
}

template <typename T>
cudaError_t launch_halo(const Conv2d& p, const HaloParams& H, const void* x, const void* w,
                        const void* bias, void* y, cudaStream_t s) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tx, tw;
  const cuuint64_t xdim[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t xstr[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                              (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t xbox[4] = {(cuuint32_t)H.BKC, (cuuint32_t)H.BW, (cuuint32_t)halo_box_rows(p, H),
                              1};
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  if (enc(&tx, dt, 4, const_cast<void*>(x), xdim, xstr, xbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(H.BKC), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t ktot = (cuuint64_t)p.kH * p.kW * p.cpg_in;
  if (H.gp == 1) {
    const cuuint64_t wdim[2] = {ktot, (cuuint64_t)p.C_out};
    const cuuint64_t wstr[1] = {ktot * 2};
    const cuuint32_t wbox[2] = {(cuuint32_t)H.BKC, (cuuint32_t)H.BN};
    if (enc(&tw, dt, 2, const_cast<void*>(w), wdim, wstr, wbox, ones,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(H.BKC), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    // [C_out][taps][cpg_in] view; a 64-channel box over a cpg_in-channel row reads zeros
    // outside it (block-diagonal filter tiles, see the kernel's comment)
    const cuuint64_t wdim[3] = {(cuuint64_t)p.cpg_in, (cuuint64_t)p.kH * p.kW, (cuuint64_t)p.C_out};
    const cuuint64_t wstr[2] = {(cuuint64_t)p.cpg_in * 2, ktot * 2};
    const cuuint32_t wbox[3] = {(cuuint32_t)H.BKC, 1, (cuuint32_t)p.cpg_out};
    if (enc(&tw, dt, 3, const_cast<void*>(w), wdim, wstr, wbox, ones,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(H.BKC), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  CUtensorMap ty;
  if (H.tma_out) {
    const cuuint64_t ydim[4] = {(cuuint64_t)p.C_out, (cuuint64_t)p.Wo, (cuuint64_t)p.Ho,
                                (cuuint64_t)p.N};
    const cuuint64_t ystr[3] = {(cuuint64_t)p.C_out * 2, (cuuint64_t)p.Wo * p.C_out * 2,
                                (cuuint64_t)p.Ho * p.Wo * p.C_out * 2};
    const cuuint32_t ybox[4] = {64, (cuuint32_t)H.BW, (cuuint32_t)H.BH, 1};
    if (enc(&ty, dt, 4, y, ydim, ystr, ybox, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    ty = tx;                                  // unused by the kernel
  }
  const size_t smem = halo_smem_bytes(H);
  if (smem > SMEM_BUDGET) return cudaErrorInvalidValue;
  // packing is a separate instantiation, so the unpacked kernel carries none of its code
  static std::atomic<unsigned int> configured[2];
  const void* fn = H.gp > 1 ? (const void*)igemm_halo_kernel<T, true>
                            : (const void*)igemm_halo_kernel<T, false>;
  cudaError_t e = set_max_dynamic_smem(fn, SMEM_BUDGET, configured[H.gp > 1 ? 1 : 0]);
  if (e != cudaSuccess) return e;
  int grid = sm_count();
  if (grid > H.num_tiles) grid = H.num_tiles;
  if (H.gp > 1)
    return launch_pdl(igemm_halo_kernel<T, true>, (unsigned)grid, NUM_THREADS, smem, s, tx, tw,
                      ty, (const T*)bias, (T*)y, H, device_error_word());
  return launch_pdl(igemm_halo_kernel<T, false>, (unsigned)grid, NUM_THREADS, smem, s, tx, tw, ty,
                    (const T*)bias, (T*)y, H, device_error_word());
}

// A 1x1, stride-1, unpadded convolution is one GEMM over all pixels. With NHWC pixels (or one
// NCHW image, whose output plane is the same pixel sequence) it is run as an image of
// H' x W' = N*H*W pixels, W' as wide as the kernels take, so that tiles run across image
// rows and images: grouped linear layers (H = W = 1, the per-group GEMMs of a batched-GEMM
// formulation) then fill whole 128 / 256-pixel MMA tiles instead of one pixel each.
// False if the problem is not pointwise, is already one row, or has no such factorisation.
bool flatten_pointwise(const Conv2d& p, Conv2d* q) {
  if (p.kH != 1 || p.kW != 1 || p.stride != 1 || p.pad != 0) return false;
  if (p.layout == GCONV_NCHW && p.N != 1) return false;
  if (p.N == 1 && p.H == 1) return false;
  const long long M = (long long)p.N * p.H * p.W;
  long long Wq = 0;
  if (M <= 65535) {
    Wq = M;
  } else {
    for (long long c = 65535; c >= 128; --c)
      if (M % c == 0 && M / c <= 65535) {
        Wq = c;
        break;
      }
  }
  if (Wq == 0) return false;
  *q = p;
  q->N = 1;
  q->H = q->Ho = (int)(M / Wq);
  q->W = q->Wo = (int)Wq;
  q->dil = 1;
  return true;
}

// x: NHWC activations, w: [C_out][kH][kW][cpg_in] weights (both device pointers).
template <typename T>
cudaError_t launch_tiles(const Conv2d& p, const IgemmParams& P, const void* x, const void* w,
                         const void* bias, void* y, cudaStream_t s) {
  if (igemm_rowt_supported(p)) return launch_igemm_rowt(p, x, w, bias, y, s);
  RowParams R;
  if (make_row_params(p, &R)) return launch_row<T>(p, R, x, w, bias, y, s);
  HaloParams HP;
  if (make_halo_params(p, &HP)) return launch_halo<T>(p, HP, x, w, bias, y, s);
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tx, tw;
  const cuuint64_t xdim[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t xstr[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                              (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t xbox[4] = {(cuuint32_t)P.BKC, (cuuint32_t)P.BW, (cuuint32_t)P.BH, 1};
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  if (enc(&tx, dt, 4, const_cast<void*>(x), xdim, xstr, xbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(P.BKC), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t ktot = (cuuint64_t)p.kH * p.kW * p.cpg_in;
  const cuuint64_t wdim[2] = {ktot, (cuuint64_t)p.C_out};
  const cuuint64_t wstr[1] = {ktot * 2};
  const cuuint32_t wbox[2] = {(cuuint32_t)P.BKC, (cuuint32_t)P.BN};
  if (enc(&tw, dt, 2, const_cast<void*>(w), wdim, wstr, wbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(P.BKC), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = smem_bytes(P);
  if (smem > SMEM_BUDGET) return cudaErrorInvalidValue;
  // the limit is raised once per device to the full budget, so every tile shape fits
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)igemm_tc_kernel<T>, SMEM_BUDGET, configured);
  if (e != cudaSuccess) return e;
  int grid = sm_count();
  if (grid > P.num_tiles) grid = P.num_tiles;
  IgemmParams PL = P;
  PL.tx_bytes += debug_tx_surplus();   // 0 except under the bounded-wait test hook
  igemm_tc_kernel<T><<<grid, NUM_THREADS, smem, s>>>(tx, tw, (const T*)bias, (T*)y, PL,
                                                     device_error_word());
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_core(const Conv2d& p, const IgemmParams& P, const void* x, const void* w,
                        const void* bias, void* y, cudaStream_t s) {
  Conv2d q;
  IgemmParams Q;
  if (flatten_pointwise(p, &q) && make_params(q, &Q))
    return launch_tiles<T>(q, Q, x, w, bias, y, s);
  return launch_tiles<T>(p, P, x, w, bias, y, s);
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

// Eligibility of the tensor-core path: 16-bit data, stride 1, channels per group multiples
// of 16 (UMMA K granularity and 16-byte TMA rows), filters per group 16..256 (UMMA N) or a
// multiple of 128, and tile bookkeeping within int range.
bool igemm_supported(const Conv2d& p) {
  if (p.dtype != GCONV_BF16 && p.dtype != GCONV_F16) return false;
  if (p.stride != 1) return false;
  if (p.cpg_in % 16 != 0 || p.cpg_out % 16 != 0) return false;
  if (tile_bn(p) == 0) return false;
  IgemmParams P;
  Conv2d q;
  if (flatten_pointwise(p, &q)) return make_params(q, &P);   // the shape that is launched
  if (p.N > 65535 || p.H > 65535 || p.W > 65535) return false;
  return make_params(p, &P);
}

size_t igemm_nchw_workspace(const Conv2d& p) {
  return align256((size_t)p.N * p.H * p.W * p.C_in * 2) +
         align256((size_t)p.C_out * p.kH * p.kW * p.cpg_in * 2);
}

cudaError_t launch_igemm_nhwc(const Conv2d& p, const void* x, const void* w, const void* bias,
                              void* y, cudaStream_t s) {
  IgemmParams P;
  if (!make_params(p, &P)) return cudaErrorNotSupported;
  if (p.dtype == GCONV_BF16) return launch_core<__nv_bfloat16>(p, P, x, w, bias, y, s);
  return launch_core<__half>(p, P, x, w, bias, y, s);
}

template <typename T>
cudaError_t launch_nchw_typed(const Conv2d& p, const IgemmParams& P, const void* x, const void* w,
                              const void* bias, void* y, void* workspace, cudaStream_t s) {
  T* xt = (T*)workspace;
  T* wt = (T*)((char*)workspace + align256((size_t)p.N * p.H * p.W * p.C_in * 2));
  const int taps = p.kH * p.kW;
  const int per_filter = p.cpg_in * taps;
  const int HW = p.H * p.W;
  const unsigned int gx = (unsigned int)((HW + 63) / 64), gy = (unsigned int)((p.C_in + 63) / 64);
  const long long stage_blocks = (long long)p.C_out + (long long)gx * gy * p.N;
  if (per_filter <= 8192 && stage_blocks <= INT32_MAX) {
    // weights and activations staged by one launch
    if (HW % 8 == 0 && p.C_in % 8 == 0 && aligned16(x))
      nchw_stage_kernel<T, true><<<(unsigned)stage_blocks, 256, 0, s>>>(
          (const T*)x, xt, p.C_in, HW, gx, gy, (const T*)w, wt, p.C_out, p.cpg_in, taps);
    else
      nchw_stage_kernel<T, false><<<(unsigned)stage_blocks, 256, 0, s>>>(
          (const T*)x, xt, p.C_in, HW, gx, gy, (const T*)w, wt, p.C_out, p.cpg_in, taps);
    const cudaError_t e0 = cudaGetLastError();
    if (e0 != cudaSuccess) return e0;
    return launch_core<T>(p, P, xt, wt, bias, y, s);
  }
  if (per_filter <= 8192) {
    repack_weight_smem_kernel<T><<<(unsigned)p.C_out, 256, 0, s>>>((const T*)w, wt, p.cpg_in,
                                                                   taps);
  } else {
    dim3 wgrid((unsigned)((per_filter + 255) / 256),
               (unsigned)(p.C_out < 65535 ? p.C_out : 65535));
    repack_weight_kernel<T><<<wgrid, 256, 0, s>>>((const T*)w, wt, p.C_out, p.cpg_in, taps);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((HW + 63) / 64, (p.C_in + 63) / 64, p.N);
  if (HW % 8 == 0 && p.C_in % 8 == 0 && aligned16(x))
    nchw_to_nhwc_kernel<T, true><<<grid, 256, 0, s>>>((const T*)x, xt, p.C_in, HW);
  else
    nchw_to_nhwc_kernel<T, false><<<grid, 256, 0, s>>>((const T*)x, xt, p.C_in, HW);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_core<T>(p, P, xt, wt, bias, y, s);
}

namespace {

// y = the maximum over groups of the group-major output g (both 16-bit): with S = cpg_out
// (NHWC) or cpg_out * Ho * Wo (NCHW), output element e has outer index e / S and inner index
// e % S, and reads g[outer * groups * S + j * S + inner] for each group j. VEC: 8 consecutive
// elements per thread as 16-byte vectors (S % 8 == 0, pointers 16-byte aligned).
template <typename T, bool VEC>
__global__ void __launch_bounds__(256) merge_max_groups_kernel(const T* __restrict__ g,
                                                               T* __restrict__ y, long long n_out,
                                                               long long S, int groups) {
  pdl_wait();   // the group-major output of the kernel before (launch_pdl)
  constexpr int V = VEC ? 8 : 1;
  const long long n_items = n_out / V;
  for (long long it = (long long)blockIdx.x * blockDim.x + threadIdx.x; it < n_items;
       it += (long long)gridDim.x * blockDim.x) {
    const long long e = it * V;
    const long long outer = e / S, inner = e - outer * S;
    const T* src = g + outer * groups * S + inner;
    if constexpr (VEC) {
      float m[8];
      uint4 u = *reinterpret_cast<const uint4*>(src);
      const unsigned int* w = &u.x;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack2<T>(w[q]);
        m[2 * q] = f.x;
        m[2 * q + 1] = f.y;
      }
      for (int j = 1; j < groups; ++j) {
        u = *reinterpret_cast<const uint4*>(src + (long long)j * S);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = unpack2<T>(w[q]);
          m[2 * q] = fmaxf(m[2 * q], f.x);
          m[2 * q + 1] = fmaxf(m[2 * q + 1], f.y);
        }
      }
      uint4 o;
      o.x = pack2<T>(make_float2(m[0], m[1]));
      o.y = pack2<T>(make_float2(m[2], m[3]));
      o.z = pack2<T>(make_float2(m[4], m[5]));
      o.w = pack2<T>(make_float2(m[6], m[7]));
      *reinterpret_cast<uint4*>(y + e) = o;
    } else {
      float m = Elem<T>::to_f32(src[0]);
      for (int j = 1; j < groups; ++j) m = fmaxf(m, Elem<T>::to_f32(src[(long long)j * S]));
      y[e] = Elem<T>::from_f32(m);
    }
  }
}

template <typename T>
cudaError_t launch_merge_max_typed(const Conv2d& p, const void* g, void* y, cudaStream_t s) {
  const long long S = p.layout == GCONV_NCHW ? (long long)p.cpg_out * p.Ho * p.Wo
                                             : (long long)p.cpg_out;
  const long long n_out = (long long)p.N * p.cpg_out * p.Ho * p.Wo;
  const bool vec = S % 8 == 0 && aligned16(g) && aligned16(y);
  const long long items = vec ? n_out / 8 : n_out;
  long long blocks = (items + 255) / 256;
  const long long cap = (long long)sm_count() * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (vec)
    return launch_pdl(merge_max_groups_kernel<T, true>, (unsigned)blocks, 256u, 0, s,
                      (const T*)g, (T*)y, n_out, S, p.groups);
  return launch_pdl(merge_max_groups_kernel<T, false>, (unsigned)blocks, 256u, 0, s, (const T*)g,
                    (T*)y, n_out, S, p.groups);
}

}  // namespace

cudaError_t launch_merge_max_groups(const Conv2d& p, const void* g, void* y, cudaStream_t s) {
  if (p.dtype == GCONV_BF16) return launch_merge_max_typed<__nv_bfloat16>(p, g, y, s);
  if (p.dtype == GCONV_F16) return launch_merge_max_typed<__half>(p, g, y, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_nchw_to_nhwc16(const void* x, void* xt, int N, int C, long long HW,
                                  cudaStream_t s) {
  if (HW > INT32_MAX || N > 65535 || (C + 63) / 64 > 65535) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((HW + 63) / 64), (unsigned)((C + 63) / 64), (unsigned)N);
  if (HW % 8 == 0 && C % 8 == 0 && aligned16(x) && aligned16(xt))
    nchw_to_nhwc_kernel<unsigned short, true><<<grid, 256, 0, s>>>(
        (const unsigned short*)x, (unsigned short*)xt, C, (int)HW);
  else
    nchw_to_nhwc_kernel<unsigned short, false><<<grid, 256, 0, s>>>(
        (const unsigned short*)x, (unsigned short*)xt, C, (int)HW);
  return cudaGetLastError();
}

cudaError_t launch_igemm_nchw(const Conv2d& p, const void* x, const void* w, const void* bias,
                              void* y, void* workspace, cudaStream_t s) {
  IgemmParams P;
  if (!make_params(p, &P)) return cudaErrorNotSupported;
  if ((long long)p.H * p.W > INT32_MAX || p.C_in > 65535 * 64) return cudaErrorNotSupported;
  if (p.dtype == GCONV_BF16)
    return launch_nchw_typed<__nv_bfloat16>(p, P, x, w, bias, y, workspace, s);
  return launch_nchw_typed<__half>(p, P, x, w, bias, y, workspace, s);
}

}  // namespace gconv
