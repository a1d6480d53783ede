// Fused depthwise-separable block on (batch, steps, channels): a depthwise conv1d followed by a
// pointwise (1x1) convolution over channels, in one kernel, the intermediate never leaving the
// SM. "Investigate custom Triton kernels for depthwise-separable convolutions in Conformer"
// (speechbrain #2733) names this block (the issue text: the Conformer convolution module; the
// Oct 30 comment: the Fast Conformer downsampler is built the same way):
//   d[b,t,c] = sum_{k<K} w_dw[c,k] * x[b, t+k-pl, c]        (x = 0 outside [0, T))
//   z[b,t,o] = bias[o] + sum_{c<C} w_pw[o,c] * d[b,t,c]
//
// One CTA computes 128 output steps of one batch for all C_out <= 512 outputs:
//   * TMA brings, per block of 64 input channels, the 128 + K - 1 input rows the block needs
//     (128-byte rows, zero fill outside [0, T)) with that block's depthwise taps (bulk copy),
//     and the block's slice w_pw[:, 64 channels] as the MMA's B operand (K-major, 128-byte
//     swizzle);
//   * eight CUDA-core warps compute d for the block (a thread: one channel pair x 16 steps,
//     the K taps of its pair in registers, fp32x2 multiply-adds, each input word read once)
//     and write it, rounded once to the data type, as the MMA's A operand (128 steps x 64
//     channels, K-major, 128-byte swizzle) -- this is the only rounding of the intermediate;
//   * one thread issues tcgen05.mma (M = 128 steps, N = C_out in chunks of <= 256, K = 64 per
//     block, fp32 accumulators in TMEM), so the pointwise GEMM of block j overlaps the
//     depthwise of block j + 1;
//   * after the last block four warps read TMEM, add the bias, round, stage 64-channel slabs
//     in shared memory and write them with per-warp TMA stores (clipped at T_out and C_out).
// All mbarrier waits are bounded (1 s); a wait that gives up sets the library's device error
// word, and the CTA drains its copies and MMAs (bounded too), frees TMEM and exits.
#include <cuda.h>

#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

using namespace ptx;

constexpr int DS_M = 128;            // output steps per CTA (MMA M)
constexpr int DS_CB = 64;            // input channels per block (MMA K per block)
// warp 0 TMA, warp 1 MMA, warps 2-17 depthwise in two groups of 8 that take alternate channel
// blocks (two blocks' depthwise in flight), warps 2-5 also the epilogue
constexpr int DS_THREADS = 576;
constexpr int DS_XS = 2;             // input-block stages
constexpr int DS_AS = 2;             // A-operand stages
constexpr int DS_BS = 2;             // B-operand stages
constexpr int DS_MAX_COUT = 512;     // TMEM columns
constexpr unsigned int ERR_DS = 1u << 12;

struct DsParams {
  int B, T, C, K, pl, T_out, C_out;
  int cblocks, t_tiles;
  int n0, n1;                        // MMA N of the two C_out chunks (n1 = 0 if one chunk)
  unsigned int x_bytes, wdw_bytes, b_bytes;
  unsigned int x_stage, b_stage;     // smem bytes per stage (1 KB multiples)
  unsigned int idesc0, idesc1, tmem_cols;
};

struct DsLayout {
  unsigned int x_off, a_off, b_off, bar_off, total;
};

__host__ __device__ inline DsLayout ds_layout(const DsParams& P) {
  DsLayout L;
  L.x_off = 0;
  L.a_off = L.x_off + DS_XS * P.x_stage;
  L.b_off = L.a_off + DS_AS * (DS_M * 128u);
  L.bar_off = L.b_off + DS_BS * P.b_stage;
  L.total = L.bar_off + 256;
  return L;
}

__device__ __forceinline__ unsigned long long desc_sw128(unsigned int saddr) {
  unsigned long long d = (unsigned long long)((saddr >> 4) & 0x3FFFu);
  d |= 1ull << 16;                                   // LBO (unused for swizzled K-major)
  d |= (unsigned long long)(1024u >> 4) << 32;       // SBO: 8 rows of 128 bytes
  d |= 1ull << 46;                                   // descriptor version
  d |= 2ull << 61;                                   // 128-byte swizzle
  return d;
}

template <typename T, int K>
__global__ void __launch_bounds__(DS_THREADS, 1)
    dwsep1d_tc_kernel(const __grid_constant__ CUtensorMap tmx,
                      const __grid_constant__ CUtensorMap tmw,
                      const __grid_constant__ CUtensorMap tmz, const T* __restrict__ wdw,
                      const T* __restrict__ bias, const DsParams P, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem(smem_raw, 1024u);
  const DsLayout L = ds_layout(P);
  unsigned char* xbuf = smem + L.x_off;
  unsigned char* abuf = smem + L.a_off;
  unsigned char* bbuf = smem + L.b_off;
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(smem + L.bar_off);
  unsigned long long* x_full = bars;                 // producer: x rows + taps (tx bytes)
  unsigned long long* x_empty = x_full + DS_XS;      // 8 depthwise warps
  unsigned long long* a_full = x_empty + DS_XS;      // 256 depthwise threads
  unsigned long long* a_empty = a_full + DS_AS;      // MMA commit
  unsigned long long* b_full = a_empty + DS_AS;      // producer (tx bytes)
  unsigned long long* b_empty = b_full + DS_BS;      // MMA commit
  unsigned long long* t_full = b_empty + DS_BS;      // MMA commit after the last block
  unsigned long long* done = t_full + 1;             // MMA commit before TMEM is released
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / P.t_tiles;
  const int t0 = (blockIdx.x % P.t_tiles) * DS_M;

  if (threadIdx.x == 0) {
    for (int i = 0; i < DS_XS; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 8);
    }
    for (int i = 0; i < DS_AS; ++i) {
      mbar_init(&a_full[i], 256);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < DS_BS; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    mbar_init(t_full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmw);
    prefetch_tmap(&tmz);
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
      // ---------------- producer: per channel block, the input rows with the block's taps,
      // and the block's pointwise weights (one or two 256-row boxes)
      bool ok = true;
      int nx = 0, nb = 0;
      for (int cb = 0; cb < P.cblocks && ok; ++cb) {
        const int xs = cb % DS_XS, bs = cb % DS_BS;
        if (!mbar_wait(&x_empty[xs], ((unsigned int)(cb / DS_XS) & 1u) ^ 1u, abort_flag, err,
                       ERR_DS | 1u)) {
          ok = false;
          break;
        }
        unsigned char* xd = xbuf + (size_t)xs * P.x_stage;
        mbar_arrive_expect_tx(&x_full[xs], P.x_bytes + P.wdw_bytes);
        tma_load_3d(xd, &tmx, &x_full[xs], cb * DS_CB, t0 - P.pl, b);
        bulk_load(xd + P.x_bytes, wdw + (size_t)cb * DS_CB * K, P.wdw_bytes, &x_full[xs]);
        ++nx;
        if (!mbar_wait(&b_empty[bs], ((unsigned int)(cb / DS_BS) & 1u) ^ 1u, abort_flag, err,
                       ERR_DS | 2u)) {
          ok = false;
          break;
        }
        unsigned char* bd = bbuf + (size_t)bs * P.b_stage;
        mbar_arrive_expect_tx(&b_full[bs], P.b_bytes);
        tma_load_2d(bd, &tmw, &b_full[bs], cb * DS_CB, 0);
        if (P.n1 > 0) tma_load_2d(bd + 256 * 128, &tmw, &b_full[bs], cb * DS_CB, 256);
        ++nb;
      }
      // copies in flight land before the CTA exits (instant on the normal path)
      const unsigned long long dl = drain_deadline();
      for (int q = (nx > DS_XS ? nx - DS_XS : 0); q < nx; ++q)
        mbar_wait_until(&x_full[q % DS_XS], (unsigned int)(q / DS_XS) & 1u, dl, err, ERR_DRAIN);
      for (int q = (nb > DS_BS ? nb - DS_BS : 0); q < nb; ++q)
        mbar_wait_until(&b_full[q % DS_BS], (unsigned int)(q / DS_BS) & 1u, dl, err, ERR_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: per block 4 K-steps x (1 or 2) N chunks
      bool ok = true;
      const unsigned long long a0 = desc_sw128(smem_u32(abuf));
      const unsigned long long b0 = desc_sw128(smem_u32(bbuf));
      for (int cb = 0; cb < P.cblocks && ok; ++cb) {
        const int as = cb % DS_AS, bs = cb % DS_BS;
        if (!mbar_wait(&a_full[as], (unsigned int)(cb / DS_AS) & 1u, abort_flag, err,
                       ERR_DS | 4u) ||
            !mbar_wait(&b_full[bs], (unsigned int)(cb / DS_BS) & 1u, abort_flag, err,
                       ERR_DS | 4u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const unsigned long long ad = a0 + ((unsigned long long)(as * DS_M * 128u) >> 4);
        const unsigned long long bd = b0 + ((unsigned long long)(bs * P.b_stage) >> 4);
#pragma unroll
        for (int ks = 0; ks < DS_CB / 16; ++ks) {
          const unsigned int acc = (cb | ks) != 0 ? 1u : 0u;
          umma_f16(tmem_base, ad + 2 * ks, bd + 2 * ks, P.idesc0, acc);
          if (P.n1 > 0)
            umma_f16(tmem_base + 256u, ad + 2 * ks, bd + ((256u * 128u) >> 4) + 2 * ks,
                     P.idesc1, acc);
        }
        umma_commit(&a_empty[as]);
        umma_commit(&b_empty[bs]);
      }
      if (ok) umma_commit(t_full);
      // every issued MMA completes before TMEM is released
      umma_commit(done);
      mbar_wait_until(done, 0, drain_deadline(), err, ERR_DRAIN);
    }
  } else {
    // ---------------- depthwise: group dg takes channel blocks dg, dg + 2, ...; its warp w2
    // owns output steps [16 w2, 16 w2 + 16) of the tile, lane = channel pair (channels
    // 2 lane, 2 lane + 1 of the block)
    const int dg = (warp - 2) >> 3, w2 = (warp - 2) & 7;
    bool ok = true;
    for (int cb = dg; cb < P.cblocks; cb += 2) {
      const int xs = cb % DS_XS, as = cb % DS_AS;
      const bool gx = mbar_wait(&x_full[xs], (unsigned int)(cb / DS_XS) & 1u, abort_flag, err,
                                ERR_DS | 8u);
      const bool ga = gx && mbar_wait(&a_empty[as], ((unsigned int)(cb / DS_AS) & 1u) ^ 1u,
                                      abort_flag, err, ERR_DS | 8u);
      if (!__all_sync(0xffffffffu, gx && ga)) {
        ok = false;
        break;
      }
      const unsigned char* xd = xbuf + (size_t)xs * P.x_stage;
      const T* taps = reinterpret_cast<const T*>(xd + P.x_bytes);
      float2 wk[K];
#pragma unroll
      for (int k = 0; k < K; ++k)
        wk[k] = make_float2(Elem<T>::to_f32(taps[(2 * lane) * K + k]),
                            Elem<T>::to_f32(taps[(2 * lane + 1) * K + k]));
      float2 acc[16];
#pragma unroll
      for (int s = 0; s < 16; ++s) acc[s] = make_float2(0.0f, 0.0f);
      const uint32_t* xr = reinterpret_cast<const uint32_t*>(xd) + (16 * w2) * 32 + lane;
#pragma unroll
      for (int i = 0; i < 16 + K - 1; ++i) {
        const float2 xv = unpack2<T>(xr[i * 32]);
#pragma unroll
        for (int s = 0; s < 16; ++s) {
          const int k = i - s;
          if (k >= 0 && k < K) acc[s] = ffma2(wk[k], xv, acc[s]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&x_empty[xs]);
      // A operand: row t (128 bytes, 64 channels), 16-byte chunk q at (q ^ (t & 7))
      unsigned char* ad = abuf + (size_t)as * DS_M * 128u;
      const int q = lane >> 2;
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const int t = 16 * w2 + s;
        *reinterpret_cast<uint32_t*>(ad + t * 128 + ((q ^ (t & 7)) << 4) + ((lane & 3) << 2)) =
            pack2<T>(acc[s]);
      }
      fence_async_smem();
      mbar_arrive(&a_full[as]);
    }
    // ---------------- epilogue: warps 2-5, TMEM lane quarter warp % 4 = rows of the tile
    if (warp < 6) {
      const int quarter = warp & 3;
      const bool got = ok && mbar_wait(t_full, 0, abort_flag, err, ERR_DS | 16u);
      if (__all_sync(0xffffffffu, got)) {
        tc_fence_after();
        // staging: 2 slabs of 32 rows x 128 bytes per warp, in the (now idle) input ring
        unsigned char* stage = xbuf + (size_t)quarter * 2 * 4096;
        const int row = lane;   // row of this warp's 32-row slab
        const unsigned int taddr = tmem_base + ((unsigned int)(quarter * 32) << 16);
        const int nslab = (P.C_out + 63) / 64;
        for (int sl = 0; sl < nslab; ++sl) {
          unsigned char* st = stage + (sl & 1) * 4096;
          if (sl >= 2) {
            if (lane == 0) bulk_wait_read1();
            __syncwarp();
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c0 = sl * 64 + h * 32;
            unsigned int r[32];
            if (c0 < (int)P.tmem_cols) {
              tmem_ld32(taddr + (unsigned int)c0, r);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = 0u;
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float f[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int o = c0 + 8 * v + i;
                f[i] = __uint_as_float(r[8 * v + i]) +
                       (bias != nullptr && o < P.C_out ? Elem<T>::to_f32(bias[o]) : 0.0f);
              }
              uint4 u;
              u.x = pack2<T>(make_float2(f[0], f[1]));
              u.y = pack2<T>(make_float2(f[2], f[3]));
              u.z = pack2<T>(make_float2(f[4], f[5]));
              u.w = pack2<T>(make_float2(f[6], f[7]));
              const int chunk = h * 4 + v;
              *reinterpret_cast<uint4*>(st + row * 128 + ((chunk ^ (row & 7)) << 4)) = u;
            }
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmz, st, sl * 64, t0 + quarter * 32, b);
            bulk_commit();
          }
        }
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
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

// ------------------------------------------------------------------ 2-D block (NHWC)
//
// The same pipeline for a depthwise conv2d (kernel KS x KS, stride S, zero padding) followed
// by the pointwise convolution: the strided depthwise-separable layers of the Fast Conformer
// downsampler (the Oct 30 comment). A CTA computes a tile of BH output rows x 32 output
// columns (row q of the tile is MMA rows 32q..32q+31, so epilogue warp q stores one output
// row segment with one TMA box); per 64-channel block TMA brings the input box of
// (BH-1)*S + KS rows x 31*S + KS columns (zero fill outside the image). A depthwise warp owns
// 16 consecutive columns of one tile row and reads each input word of its window rows once.

struct Ds2Params {
  int N, H, W, C, pad, Ho, Wo, C_out;
  int BH, box_h, box_w, tiles_w, tiles_h, cblocks;
  int n0, n1;
  unsigned int x_bytes, wdw_bytes, b_bytes;
  unsigned int x_stage, b_stage;
  unsigned int idesc0, idesc1, tmem_cols;
};

__host__ __device__ inline DsLayout ds2_layout(const Ds2Params& P) {
  DsLayout L;
  L.x_off = 0;
  L.a_off = L.x_off + DS_XS * P.x_stage;
  L.b_off = L.a_off + DS_AS * (DS_M * 128u);
  L.bar_off = L.b_off + DS_BS * P.b_stage;
  L.total = L.bar_off + 256;
  return L;
}

template <typename T, int KS, int S>
__global__ void __launch_bounds__(DS_THREADS, 1)
    dwsep2d_tc_kernel(const __grid_constant__ CUtensorMap tmx,
                      const __grid_constant__ CUtensorMap tmw,
                      const __grid_constant__ CUtensorMap tmz, const T* __restrict__ wdw,
                      const T* __restrict__ bias, const Ds2Params P, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem(smem_raw, 1024u);
  const DsLayout L = ds2_layout(P);
  unsigned char* xbuf = smem + L.x_off;
  unsigned char* abuf = smem + L.a_off;
  unsigned char* bbuf = smem + L.b_off;
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(smem + L.bar_off);
  unsigned long long* x_full = bars;
  unsigned long long* x_empty = x_full + DS_XS;
  unsigned long long* a_full = x_empty + DS_XS;
  unsigned long long* a_empty = a_full + DS_AS;
  unsigned long long* b_full = a_empty + DS_AS;
  unsigned long long* b_empty = b_full + DS_BS;
  unsigned long long* t_full = b_empty + DS_BS;
  unsigned long long* done = t_full + 1;
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tw = blockIdx.x % P.tiles_w;
  const int th = (blockIdx.x / P.tiles_w) % P.tiles_h;
  const int n = blockIdx.x / (P.tiles_w * P.tiles_h);
  const int ow0 = tw * 32, oh0 = th * P.BH;

  if (threadIdx.x == 0) {
    for (int i = 0; i < DS_XS; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 8);
    }
    for (int i = 0; i < DS_AS; ++i) {
      mbar_init(&a_full[i], 256);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < DS_BS; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    mbar_init(t_full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmw);
    prefetch_tmap(&tmz);
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
      bool ok = true;
      int nx = 0, nb = 0;
      for (int cb = 0; cb < P.cblocks && ok; ++cb) {
        const int xs = cb % DS_XS, bs = cb % DS_BS;
        if (!mbar_wait(&x_empty[xs], ((unsigned int)(cb / DS_XS) & 1u) ^ 1u, abort_flag, err,
                       ERR_DS | 1u)) {
          ok = false;
          break;
        }
        unsigned char* xd = xbuf + (size_t)xs * P.x_stage;
        mbar_arrive_expect_tx(&x_full[xs], P.x_bytes + P.wdw_bytes);
        tma_load_4d(xd, &tmx, &x_full[xs], cb * DS_CB, ow0 * S - P.pad, oh0 * S - P.pad, n);
        bulk_load(xd + P.x_bytes, wdw + (size_t)cb * DS_CB * KS * KS, P.wdw_bytes, &x_full[xs]);
        ++nx;
        if (!mbar_wait(&b_empty[bs], ((unsigned int)(cb / DS_BS) & 1u) ^ 1u, abort_flag, err,
                       ERR_DS | 2u)) {
          ok = false;
          break;
        }
        unsigned char* bd = bbuf + (size_t)bs * P.b_stage;
        mbar_arrive_expect_tx(&b_full[bs], P.b_bytes);
        tma_load_2d(bd, &tmw, &b_full[bs], cb * DS_CB, 0);
        if (P.n1 > 0) tma_load_2d(bd + 256 * 128, &tmw, &b_full[bs], cb * DS_CB, 256);
        ++nb;
      }
      const unsigned long long dl = drain_deadline();
      for (int q = (nx > DS_XS ? nx - DS_XS : 0); q < nx; ++q)
        mbar_wait_until(&x_full[q % DS_XS], (unsigned int)(q / DS_XS) & 1u, dl, err, ERR_DRAIN);
      for (int q = (nb > DS_BS ? nb - DS_BS : 0); q < nb; ++q)
        mbar_wait_until(&b_full[q % DS_BS], (unsigned int)(q / DS_BS) & 1u, dl, err, ERR_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      const unsigned long long a0 = desc_sw128(smem_u32(abuf));
      const unsigned long long b0 = desc_sw128(smem_u32(bbuf));
      for (int cb = 0; cb < P.cblocks && ok; ++cb) {
        const int as = cb % DS_AS, bs = cb % DS_BS;
        if (!mbar_wait(&a_full[as], (unsigned int)(cb / DS_AS) & 1u, abort_flag, err,
                       ERR_DS | 4u) ||
            !mbar_wait(&b_full[bs], (unsigned int)(cb / DS_BS) & 1u, abort_flag, err,
                       ERR_DS | 4u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const unsigned long long ad = a0 + ((unsigned long long)(as * DS_M * 128u) >> 4);
        const unsigned long long bd = b0 + ((unsigned long long)(bs * P.b_stage) >> 4);
#pragma unroll
        for (int ks = 0; ks < DS_CB / 16; ++ks) {
          const unsigned int acc = (cb | ks) != 0 ? 1u : 0u;
          umma_f16(tmem_base, ad + 2 * ks, bd + 2 * ks, P.idesc0, acc);
          if (P.n1 > 0)
            umma_f16(tmem_base + 256u, ad + 2 * ks, bd + ((256u * 128u) >> 4) + 2 * ks,
                     P.idesc1, acc);
        }
        umma_commit(&a_empty[as]);
        umma_commit(&b_empty[bs]);
      }
      if (ok) umma_commit(t_full);
      umma_commit(done);
      mbar_wait_until(done, 0, drain_deadline(), err, ERR_DRAIN);
    }
  } else {
    // ---------------- depthwise: group dg takes channel blocks dg, dg + 2, ...; its warp w2
    // owns tile pixels 16 w2 .. 16 w2 + 15, i.e. tile row r = w2 / 2, columns
    // 16 (w2 % 2) .. + 15; lane = channel pair
    const int dg = (warp - 2) >> 3, w2 = (warp - 2) & 7;
    const int r = w2 >> 1, c0 = (w2 & 1) * 16;
    const bool row_live = r < P.BH && oh0 + r < P.Ho;
    bool ok = true;
    for (int cb = dg; cb < P.cblocks; cb += 2) {
      const int xs = cb % DS_XS, as = cb % DS_AS;
      const bool gx = mbar_wait(&x_full[xs], (unsigned int)(cb / DS_XS) & 1u, abort_flag, err,
                                ERR_DS | 8u);
      const bool ga = gx && mbar_wait(&a_empty[as], ((unsigned int)(cb / DS_AS) & 1u) ^ 1u,
                                      abort_flag, err, ERR_DS | 8u);
      if (!__all_sync(0xffffffffu, gx && ga)) {
        ok = false;
        break;
      }
      const unsigned char* xd = xbuf + (size_t)xs * P.x_stage;
      const T* taps = reinterpret_cast<const T*>(xd + P.x_bytes);   // [64 ch][KS][KS]
      float2 acc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = make_float2(0.0f, 0.0f);
      if (row_live) {
#pragma unroll
        for (int kh = 0; kh < KS; ++kh) {
          float2 wk[KS];
#pragma unroll
          for (int kw = 0; kw < KS; ++kw)
            wk[kw] = make_float2(Elem<T>::to_f32(taps[((2 * lane) * KS + kh) * KS + kw]),
                                 Elem<T>::to_f32(taps[((2 * lane + 1) * KS + kh) * KS + kw]));
          const uint32_t* xr = reinterpret_cast<const uint32_t*>(xd) +
                               ((r * S + kh) * P.box_w + c0 * S) * 32 + lane;
          // input column i of the window feeds output column j where i = j * S + kw
#pragma unroll
          for (int i = 0; i < 15 * S + KS; ++i) {
            const float2 xv = unpack2<T>(xr[i * 32]);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int kw = i - j * S;
              if (kw >= 0 && kw < KS) acc[j] = ffma2(wk[kw], xv, acc[j]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&x_empty[xs]);
      unsigned char* ad = abuf + (size_t)as * DS_M * 128u;
      const int q = lane >> 2;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int t = 16 * w2 + j;
        *reinterpret_cast<uint32_t*>(ad + t * 128 + ((q ^ (t & 7)) << 4) + ((lane & 3) << 2)) =
            pack2<T>(acc[j]);
      }
      fence_async_smem();
      mbar_arrive(&a_full[as]);
    }
    // ---------------- epilogue: warps 2-5; warp quarter q = tile row q (MMA rows 32q..)
    if (warp < 6) {
      const int quarter = warp & 3;
      const bool got = ok && mbar_wait(t_full, 0, abort_flag, err, ERR_DS | 16u);
      if (__all_sync(0xffffffffu, got) && quarter < P.BH) {
        tc_fence_after();
        unsigned char* stage = xbuf + (size_t)quarter * 2 * 4096;
        const int row = lane;
        const unsigned int taddr = tmem_base + ((unsigned int)(quarter * 32) << 16);
        const int nslab = (P.C_out + 63) / 64;
        for (int sl = 0; sl < nslab; ++sl) {
          unsigned char* st = stage + (sl & 1) * 4096;
          if (sl >= 2) {
            if (lane == 0) bulk_wait_read1();
            __syncwarp();
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c0e = sl * 64 + h * 32;
            unsigned int rr[32];
            if (c0e < (int)P.tmem_cols) {
              tmem_ld32(taddr + (unsigned int)c0e, rr);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) rr[i] = 0u;
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float f[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int o = c0e + 8 * v + i;
                f[i] = __uint_as_float(rr[8 * v + i]) +
                       (bias != nullptr && o < P.C_out ? Elem<T>::to_f32(bias[o]) : 0.0f);
              }
              uint4 u;
              u.x = pack2<T>(make_float2(f[0], f[1]));
              u.y = pack2<T>(make_float2(f[2], f[3]));
              u.z = pack2<T>(make_float2(f[4], f[5]));
              u.w = pack2<T>(make_float2(f[6], f[7]));
              const int chunk = h * 4 + v;
              *reinterpret_cast<uint4*>(st + row * 128 + ((chunk ^ (row & 7)) << 4)) = u;
            }
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_4d(&tmz, st, sl * 64, ow0, oh0 + quarter, n);
            bulk_commit();
          }
        }
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
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

bool make_ds_params(const Conv1d& p, int C_out, DsParams* P) {
  if (p.dtype != GCONV_BF16 && p.dtype != GCONV_F16) return false;
  if (p.C % DS_CB != 0 || C_out % 16 != 0 || C_out > DS_MAX_COUT || C_out < 16) return false;
  if (p.K + DS_M - 1 > 256) return false;                    // one TMA box of input rows
  P->B = p.B; P->T = p.T; P->C = p.C; P->K = p.K; P->pl = p.pad_left; P->T_out = p.T_out;
  P->C_out = C_out;
  P->cblocks = p.C / DS_CB;
  P->t_tiles = (p.T_out + DS_M - 1) / DS_M;
  if ((long long)p.B * P->t_tiles > INT32_MAX) return false;
  P->n0 = C_out < 256 ? C_out : 256;
  P->n1 = C_out - P->n0;
  P->x_bytes = (unsigned int)(DS_M + p.K - 1) * 128u;
  P->wdw_bytes = (unsigned int)DS_CB * p.K * 2u;
  P->x_stage = (P->x_bytes + P->wdw_bytes + 1023u) & ~1023u;
  P->b_bytes = (P->n1 > 0 ? 2u : 1u) * 256u * 128u;
  P->b_stage = P->b_bytes;
  const unsigned int fmt = p.dtype == GCONV_BF16 ? 1u : 0u;
  const unsigned int base = (1u << 4) | (fmt << 7) | (fmt << 10) | ((unsigned int)(DS_M >> 4) << 24);
  P->idesc0 = base | ((unsigned int)(P->n0 >> 3) << 17);
  P->idesc1 = base | ((unsigned int)((P->n1 > 0 ? P->n1 : 16) >> 3) << 17);
  unsigned int cols = 32;
  while ((int)cols < C_out) cols <<= 1;
  P->tmem_cols = cols;
  // the epilogue stages 4 warps x 2 slabs x 4 KB in the input ring
  if (DS_XS * P->x_stage < 4u * 2u * 4096u) return false;
  return 1024 + ds_layout(*P).total <= 227u * 1024u;
}

template <typename T, int K>
cudaError_t launch_ds_typed(const DsParams& P, const CUtensorMap& tx, const CUtensorMap& tw,
                            const CUtensorMap& tz, const void* wdw, const void* bias,
                            cudaStream_t s) {
  static std::atomic<unsigned int> configured{0};
  const size_t smem = 1024 + ds_layout(P).total;
  cudaError_t e = set_max_dynamic_smem((const void*)dwsep1d_tc_kernel<T, K>, 227 * 1024,
                                       configured);
  if (e != cudaSuccess) return e;
  dwsep1d_tc_kernel<T, K><<<P.B * P.t_tiles, DS_THREADS, smem, s>>>(
      tx, tw, tz, (const T*)wdw, (const T*)bias, P, device_error_word());
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ds_k(const DsParams& P, const CUtensorMap& tx, const CUtensorMap& tw,
                        const CUtensorMap& tz, const void* wdw, const void* bias,
                        cudaStream_t s) {
  switch (P.K) {
    case 3: return launch_ds_typed<T, 3>(P, tx, tw, tz, wdw, bias, s);
    case 5: return launch_ds_typed<T, 5>(P, tx, tw, tz, wdw, bias, s);
    case 7: return launch_ds_typed<T, 7>(P, tx, tw, tz, wdw, bias, s);
    case 9: return launch_ds_typed<T, 9>(P, tx, tw, tz, wdw, bias, s);
    case 15: return launch_ds_typed<T, 15>(P, tx, tw, tz, wdw, bias, s);
    case 31: return launch_ds_typed<T, 31>(P, tx, tw, tz, wdw, bias, s);
    default: return cudaErrorNotSupported;
  }
}

bool ds_k_supported(int K) {
  return K == 3 || K == 5 || K == 7 || K == 9 || K == 15 || K == 31;
}

}  // namespace

bool dwsep1d_fused_supported(const Conv1d& p, int C_out) {
  DsParams P;
  return ds_k_supported(p.K) && make_ds_params(p, C_out, &P);
}

cudaError_t launch_dwsep1d_fused(const Conv1d& p, int C_out, const void* x, const void* wdw,
                                 const void* wpw, const void* bias, void* z, cudaStream_t s) {
  DsParams P;
  if (!ds_k_supported(p.K) || !make_ds_params(p, C_out, &P)) return cudaErrorNotSupported;
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint32_t ones[3] = {1, 1, 1};
  CUtensorMap tx, tw, tz;
  const cuuint64_t xdim[3] = {(cuuint64_t)p.C, (cuuint64_t)p.T, (cuuint64_t)p.B};
  const cuuint64_t xstr[2] = {(cuuint64_t)p.C * 2, (cuuint64_t)p.T * p.C * 2};
  const cuuint32_t xbox[3] = {(cuuint32_t)DS_CB, (cuuint32_t)(DS_M + p.K - 1), 1};
  if (enc(&tx, dt, 3, const_cast<void*>(x), xdim, xstr, xbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t wdim[2] = {(cuuint64_t)p.C, (cuuint64_t)C_out};
  const cuuint64_t wstr[1] = {(cuuint64_t)p.C * 2};
  const cuuint32_t wbox[2] = {(cuuint32_t)DS_CB, 256};
  if (enc(&tw, dt, 2, const_cast<void*>(wpw), wdim, wstr, wbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t zdim[3] = {(cuuint64_t)C_out, (cuuint64_t)p.T_out, (cuuint64_t)p.B};
  const cuuint64_t zstr[2] = {(cuuint64_t)C_out * 2, (cuuint64_t)p.T_out * C_out * 2};
  const cuuint32_t zbox[3] = {64, 32, 1};
  if (enc(&tz, dt, 3, z, zdim, zstr, zbox, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (p.dtype == GCONV_BF16) return launch_ds_k<__nv_bfloat16>(P, tx, tw, tz, wdw, bias, s);
  return launch_ds_k<__half>(P, tx, tw, tz, wdw, bias, s);
}

// ------------------------------------------------------------------ 2-D host side
namespace {

bool make_ds2_params(const Conv2d& p, int C_out, Ds2Params* P) {
  if (p.layout != GCONV_NHWC || (p.dtype != GCONV_BF16 && p.dtype != GCONV_F16)) return false;
  if (p.groups != p.C_in || p.C_out != p.C_in || p.kH != p.kW || p.dil != 1) return false;
  if ((p.kH != 3 && p.kH != 5) || (p.stride != 1 && p.stride != 2)) return false;
  if (p.C_in % DS_CB != 0 || C_out % 16 != 0 || C_out > DS_MAX_COUT || C_out < 16) return false;
  if (p.N > 65535 || p.H > 65535 || p.W > 65535) return false;
  // tiles are 32 output columns wide: narrower images would leave most MMA rows and depthwise
  // warps idle (the two-launch composition is faster there)
  if (p.Wo < 32) return false;
  P->N = p.N; P->H = p.H; P->W = p.W; P->C = p.C_in; P->pad = p.pad; P->Ho = p.Ho;
  P->Wo = p.Wo; P->C_out = C_out;
  P->box_w = 31 * p.stride + p.kW;
  // tile rows: as many (up to 4) as let two input stages fit beside the operand rings
  const unsigned int b_stage = (C_out > 256 ? 2u : 1u) * 256u * 128u;
  const unsigned int wdw_bytes = (unsigned int)DS_CB * p.kH * p.kW * 2u;
  const unsigned int x_budget =
      (227u * 1024u - 1024u - 256u - DS_AS * DS_M * 128u - DS_BS * b_stage) / DS_XS;
  int bh = p.Ho < 4 ? p.Ho : 4;
  while (bh > 1 && (((unsigned int)((bh - 1) * p.stride + p.kH) * P->box_w * 128u + wdw_bytes +
                     1023u) & ~1023u) > x_budget)
    --bh;
  P->BH = bh;
  P->box_h = (bh - 1) * p.stride + p.kH;
  if (P->box_w > 256 || P->box_h > 256) return false;
  P->tiles_w = (p.Wo + 31) / 32;
  P->tiles_h = (p.Ho + bh - 1) / bh;
  const long long grid = (long long)p.N * P->tiles_w * P->tiles_h;
  if (grid > INT32_MAX) return false;
  P->cblocks = p.C_in / DS_CB;
  P->n0 = C_out < 256 ? C_out : 256;
  P->n1 = C_out - P->n0;
  P->x_bytes = (unsigned int)P->box_h * P->box_w * 128u;
  P->wdw_bytes = (unsigned int)DS_CB * p.kH * p.kW * 2u;
  P->x_stage = (P->x_bytes + P->wdw_bytes + 1023u) & ~1023u;
  P->b_bytes = (P->n1 > 0 ? 2u : 1u) * 256u * 128u;
  P->b_stage = P->b_bytes;
  const unsigned int fmt = p.dtype == GCONV_BF16 ? 1u : 0u;
  const unsigned int base = (1u << 4) | (fmt << 7) | (fmt << 10) | ((unsigned int)(DS_M >> 4) << 24);
  P->idesc0 = base | ((unsigned int)(P->n0 >> 3) << 17);
  P->idesc1 = base | ((unsigned int)((P->n1 > 0 ? P->n1 : 16) >> 3) << 17);
  unsigned int cols = 32;
  while ((int)cols < C_out) cols <<= 1;
  P->tmem_cols = cols;
  if (DS_XS * P->x_stage < 4u * 2u * 4096u) return false;
  // wdw bulk copy: 16-byte multiple
  if (P->wdw_bytes % 16u != 0) return false;
  return 1024 + ds2_layout(*P).total <= 227u * 1024u;
}

template <typename T, int KS, int S>
cudaError_t launch_ds2_typed(const Ds2Params& P, const CUtensorMap& tx, const CUtensorMap& tw,
                             const CUtensorMap& tz, const void* wdw, const void* bias,
                             cudaStream_t s) {
  static std::atomic<unsigned int> configured{0};
  const size_t smem = 1024 + ds2_layout(P).total;
  cudaError_t e = set_max_dynamic_smem((const void*)dwsep2d_tc_kernel<T, KS, S>, 227 * 1024,
                                       configured);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(P.N * P.tiles_w * P.tiles_h);
  dwsep2d_tc_kernel<T, KS, S><<<grid, DS_THREADS, smem, s>>>(tx, tw, tz, (const T*)wdw,
                                                              (const T*)bias, P,
                                                              device_error_word());
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ds2_k(const Conv2d& p, const Ds2Params& P, const CUtensorMap& tx,
                         const CUtensorMap& tw, const CUtensorMap& tz, const void* wdw,
                         const void* bias, cudaStream_t s) {
  if (p.kH == 3 && p.stride == 1) return launch_ds2_typed<T, 3, 1>(P, tx, tw, tz, wdw, bias, s);
  if (p.kH == 3 && p.stride == 2) return launch_ds2_typed<T, 3, 2>(P, tx, tw, tz, wdw, bias, s);
  if (p.kH == 5 && p.stride == 1) return launch_ds2_typed<T, 5, 1>(P, tx, tw, tz, wdw, bias, s);
  if (p.kH == 5 && p.stride == 2) return launch_ds2_typed<T, 5, 2>(P, tx, tw, tz, wdw, bias, s);
  return cudaErrorNotSupported;
}

}  // namespace

bool dwsep2d_fused_supported(const Conv2d& p, int C_out) {
  Ds2Params P;
  return make_ds2_params(p, C_out, &P);
}

cudaError_t launch_dwsep2d_fused(const Conv2d& p, int C_out, const void* x, const void* wdw,
                                 const void* wpw, const void* bias, void* z, cudaStream_t s) {
  Ds2Params P;
  if (!make_ds2_params(p, C_out, &P)) return cudaErrorNotSupported;
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  CUtensorMap tx, tw, tz;
  const cuuint64_t xdim[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t xstr[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                              (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t xbox[4] = {(cuuint32_t)DS_CB, (cuuint32_t)P.box_w, (cuuint32_t)P.box_h, 1};
  if (enc(&tx, dt, 4, const_cast<void*>(x), xdim, xstr, xbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t wdim[2] = {(cuuint64_t)p.C_in, (cuuint64_t)C_out};
  const cuuint64_t wstr[1] = {(cuuint64_t)p.C_in * 2};
  const cuuint32_t wbox[2] = {(cuuint32_t)DS_CB, 256};
  if (enc(&tw, dt, 2, const_cast<void*>(wpw), wdim, wstr, wbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t zdim[4] = {(cuuint64_t)C_out, (cuuint64_t)p.Wo, (cuuint64_t)p.Ho,
                              (cuuint64_t)p.N};
  const cuuint64_t zstr[3] = {(cuuint64_t)C_out * 2, (cuuint64_t)p.Wo * C_out * 2,
                              (cuuint64_t)p.Ho * p.Wo * C_out * 2};
  const cuuint32_t zbox[4] = {64, 32, 1, 1};
  if (enc(&tz, dt, 4, z, zdim, zstr, zbox, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (p.dtype == GCONV_BF16) return launch_ds2_k<__nv_bfloat16>(p, P, tx, tw, tz, wdw, bias, s);
  return launch_ds2_k<__half>(p, P, tx, tw, tz, wdw, bias, s);
}

}  // namespace gconv
