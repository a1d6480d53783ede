// Transposed row-strip kernel of the per-group implicit GEMM (tcgen05, sm_100a).
//
// For group j the convolution is the GEMM of the tile kernels in igemm_tc.cu (M = output
// pixels, N = the group's filters, K = taps x the group's input channels), computed
// transposed when the filters per group are a multiple of 128 and output rows are at least
// 128 wide: D^T[co x px] = W[co x k] * X^T[k x px] with M = 128 filters and N = 256 (or 128)
// output pixels of one row per MMA. Each tcgen05.mma then carries twice the work of the
// 128 x 128 form, which halves the instructions and barrier waits the single issuing thread
// spends per unit of tensor work. The pixel operand is one input strip per (kh, channel
// block): a TMA box of NPIX rows plus an 8-row box for the halo, read at row offsets kw*dil
// for the kW taps (whole 128-byte rows inside the 128-byte swizzle atoms, descriptor base
// offset 0); the weight operand is one [128 x 64] tile per tap. In the epilogue each thread
// owns one output channel (its TMEM lane): NHWC stores of a warp cover 32 consecutive
// channels of a pixel, NCHW stores of a thread cover 32 consecutive pixels.
//
// Output variants ("Grouped convolutions", neon issue #296, the post on output orderings):
// the plain kernel writes the group-major order or the interleaved one (filter f of group j
// at channel f * groups + j); the average merge across groups has its own kernel, in which one
// tile runs every group's K loop into one accumulator and the epilogue scales by 1/groups.
//
#include <cuda.h>

#include "igemm_common.cuh"

namespace gconv {
namespace {

using namespace ptx;

// Kernel parameters. Keep this struct at 128 bytes or less: with the three merge fields
// appended to a 128-byte version, the same plain-kernel source compiled to code that ran the
// 77-GFLOP wide-group layer in 82 us instead of 65 us (fields only the host needs live in
// Conv2d instead).
struct RowTParams {
  int N, C_out, Ho, Wo, kH, kW, pad, dil, cpg_in, cpg_out;
  int NPIX, cblocks, segs, n_tiles, num_tiles;
  int x_stages, w_stages;
  unsigned int x_stage, w_stage, x_tx, w_tx, box1_bytes;
  unsigned int idesc, tmem_cols;
  int out_nchw, nchw_vec;
  int groups, interleave;   // interleaved output order: filter f of group j -> f * groups + j
  // average merge across groups: every group's K loop accumulates into one tile (jgroups =
  // groups, tiles have no group index), the epilogue scales by 1/groups and writes out_c =
  // C_out/groups channels; otherwise jgroups = 1, out_c = C_out, scale = 1
  int jgroups, out_c;
  float scale;
};

__device__ __forceinline__ void rowt_decode(const RowTParams& P, int t, int& j, int& nt, int& n,
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


template <typename T>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    igemm_rowt_kernel(const __grid_constant__ CUtensorMap tma_x,
                      const __grid_constant__ CUtensorMap tma_xh,
                      const __grid_constant__ CUtensorMap tma_w, const T* __restrict__ bias,
                      T* __restrict__ y, const RowTParams P, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 1024u);
  unsigned char* x_base = smem;
  unsigned char* w_base = smem + (size_t)P.x_stages * P.x_stage;
  unsigned long long* bars =
      reinterpret_cast<unsigned long long*>(w_base + (size_t)P.w_stages * P.w_stage);
  unsigned long long* fx = bars;
  unsigned long long* ex = fx + ROW_MAX_A;
  unsigned long long* fw = ex + ROW_MAX_A;
  unsigned long long* ew = fw + ROW_MAX_B;
  unsigned long long* tfull = ew + ROW_MAX_B;
  unsigned long long* tempty = tfull + 2;
  unsigned long long* done = tempty + 2;
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.x_stages; ++s) {
      mbar_init(&fx[s], 1);
      mbar_init(&ex[s], 1);
    }
    for (int s = 0; s < P.w_stages; ++s) {
      mbar_init(&fw[s], 1);
      mbar_init(&ew[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tma_x);
    prefetch_tmap(&tma_xh);
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
      int sx = 0, sw = 0;
      unsigned int px = 0, pw = 0;
      long long nx = 0, nw = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        int j, nt, n, ho, seg;
        rowt_decode(P, t, j, nt, n, ho, seg);
        const int wbase = seg * P.NPIX - P.pad;
        const int obase = j * P.cpg_out + nt * BM;
        for (int cb = 0; cb < P.cblocks && ok; ++cb) {
          const int cin = j * P.cpg_in + cb * 64;
          for (int kh = 0; kh < P.kH && ok; ++kh) {
            if (!mbar_wait(&ex[sx], px ^ 1u, abort_flag, err, ERR_WAIT_PRODUCER)) {
              ok = false;
              break;
            }
            unsigned char* dst = x_base + (size_t)sx * P.x_stage;
            const int hrow = ho - P.pad + kh * P.dil;
            mbar_arrive_expect_tx(&fx[sx], P.x_tx);
            tma_load_4d(dst, &tma_x, &fx[sx], cin, wbase, hrow, n);
            tma_load_4d(dst + P.box1_bytes, &tma_xh, &fx[sx], cin, wbase + P.NPIX, hrow, n);
            ++nx;
            if (++sx == P.x_stages) {
              sx = 0;
              px ^= 1u;
            }
            for (int kw = 0; kw < P.kW; ++kw) {
              if (!mbar_wait(&ew[sw], pw ^ 1u, abort_flag, err, ERR_WAIT_PRODUCER)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&fw[sw], P.w_tx);
              tma_load_2d(w_base + (size_t)sw * P.w_stage, &tma_w, &fw[sw],
                          (kh * P.kW + kw) * P.cpg_in + cb * 64, obase);
              ++nw;
              if (++sw == P.w_stages) {
                sw = 0;
                pw ^= 1u;
              }
            }
          }
        }
      }
      const unsigned long long dl = drain_deadline();
      for (long long q = (nx > P.x_stages ? nx - P.x_stages : 0); q < nx; ++q)
        mbar_wait_until(&fx[q % P.x_stages], (unsigned int)((q / P.x_stages) & 1), dl, err,
                        ERR_WAIT_DRAIN);
      for (long long q = (nw > P.w_stages ? nw - P.w_stages : 0); q < nw; ++q)
        mbar_wait_until(&fw[q % P.w_stages], (unsigned int)((q / P.w_stages) & 1), dl, err,
                        ERR_WAIT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: descriptors built once, advanced by constant offsets
      int sx = 0, sw = 0, acc = 0;
      unsigned int px = 0, pw = 0, aph = 0;
      bool ok = true;
      const unsigned long long x_desc0 = smem_desc(smem_u32(x_base), 1024u, 2u);
      const unsigned long long w_desc0 = smem_desc(smem_u32(w_base), 1024u, 2u);
      const unsigned long long kw_step = (unsigned long long)P.dil * 8u;   // dil rows of 128 B
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, err, ERR_WAIT_MMA)) break;
        tc_fence_after();
        const unsigned int d = tmem_base + (unsigned int)(acc * P.NPIX);
        for (int cb = 0; cb < P.cblocks && ok; ++cb) {
          for (int kh = 0; kh < P.kH && ok; ++kh) {
            if (!mbar_try_wait(&fx[sx], px) &&
                !mbar_wait(&fx[sx], px, abort_flag, err, ERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            const unsigned long long xs = x_desc0 + (((unsigned long long)sx * P.x_stage) >> 4);
            for (int kw = 0; kw < P.kW; ++kw) {
              if (!mbar_try_wait(&fw[sw], pw) &&
                  !mbar_wait(&fw[sw], pw, abort_flag, err, ERR_WAIT_MMA)) {
                ok = false;
                break;
              }
              const unsigned long long wd = w_desc0 + (((unsigned long long)sw * P.w_stage) >> 4);
              const unsigned long long xd = xs + kw * kw_step;
              const unsigned int acc0 = (cb | kh | kw) == 0 ? 0u : 1u;
              umma_f16(d, wd, xd, P.idesc, acc0);
              umma_f16(d, wd + 2, xd + 2, P.idesc, 1u);
              umma_f16(d, wd + 4, xd + 4, P.idesc, 1u);
              umma_f16(d, wd + 6, xd + 6, P.idesc, 1u);
              umma_commit(&ew[sw]);
              if (++sw == P.w_stages) {
                sw = 0;
                pw ^= 1u;
              }
            }
            if (!ok) break;
            umma_commit(&ex[sx]);
            if (++sx == P.x_stages) {
              sx = 0;
              px ^= 1u;
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
    // ---------------- epilogue: warps 2..5; TMEM lane = output channel of the tile
    const int quarter = warp & 3;
    const int co_l = quarter * 32 + lane;
    int acc = 0;
    unsigned int aph = 0;
    for (int t = blockIdx.x; t < P.num_tiles; t += gridDim.x) {
      int j, nt, n, ho, seg;
      rowt_decode(P, t, j, nt, n, ho, seg);
      const bool got = mbar_wait(&tfull[acc], aph, abort_flag, err, ERR_WAIT_EPILOGUE);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int co_g = j * P.cpg_out + nt * BM + co_l;       // group-major channel
      const int co = P.interleave ? (nt * BM + co_l) * P.groups + j : co_g;   // y's channel
      const float bv = bias ? Elem<T>::to_f32(bias[co_g]) : 0.0f;
      const unsigned int taddr =
          tmem_base + ((unsigned int)(quarter * 32) << 16) + (unsigned int)(acc * P.NPIX);
      for (int c = 0; c < P.NPIX; c += 32) {
        unsigned int r[32];
        tmem_ld32(taddr + c, r);
        tmem_ld_wait();
        const int wo0 = seg * P.NPIX + c;
        if (wo0 >= P.Wo) continue;
        if (!P.out_nchw) {
          T* dst = y + (((long long)n * P.Ho + ho) * P.Wo + wo0) * P.C_out + co;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (wo0 + i < P.Wo)
              dst[(long long)i * P.C_out] = Elem<T>::from_f32(__uint_as_float(r[i]) + bv);
        } else {
          T* dst = y + (((long long)n * P.C_out + co) * P.Ho + ho) * P.Wo + wo0;
          if (P.nchw_vec && wo0 + 32 <= P.Wo) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 u;
              u.x = pack2<T>(make_float2(__uint_as_float(r[8 * q + 0]) + bv,
                                         __uint_as_float(r[8 * q + 1]) + bv));
              u.y = pack2<T>(make_float2(__uint_as_float(r[8 * q + 2]) + bv,
                                         __uint_as_float(r[8 * q + 3]) + bv));
              u.z = pack2<T>(make_float2(__uint_as_float(r[8 * q + 4]) + bv,
                                         __uint_as_float(r[8 * q + 5]) + bv));
              u.w = pack2<T>(make_float2(__uint_as_float(r[8 * q + 6]) + bv,
                                         __uint_as_float(r[8 * q + 7]) + bv));
              reinterpret_cast<uint4*>(dst)[q] = u;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (wo0 + i < P.Wo) dst[i] = Elem<T>::from_f32(__uint_as_float(r[i]) + bv);
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
}

template <typename T>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    igemm_rowt_avg_kernel(const __grid_constant__ CUtensorMap tma_x,
                          const __grid_constant__ CUtensorMap tma_xh,
                          const __grid_constant__ CUtensorMap tma_w, const T* __restrict__ bias,
                          T* __restrict__ y, const RowTParams P, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 1024u);
  unsigned char* x_base = smem;
  unsigned char* w_base = smem + (size_t)P.x_stages * P.x_stage;
  unsigned long long* bars =
      reinterpret_cast<unsigned long long*>(w_base + (size_t)P.w_stages * P.w_stage);
  unsigned long long* fx = bars;
  unsigned long long* ex = fx + ROW_MAX_A;
  unsigned long long* fw = ex + ROW_MAX_A;
  unsigned long long* ew = fw + ROW_MAX_B;
  unsigned long long* tfull = ew + ROW_MAX_B;
  unsigned long long* tempty = tfull + 2;
  unsigned long long* done = tempty + 2;
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.x_stages; ++s) {
      mbar_init(&fx[s], 1);
      mbar_init(&ex[s], 1);
    }
    for (int s = 0; s < P.w_stages; ++s) {
      mbar_init(&fw[s], 1);
      mbar_init(&ew[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tma_x);
    prefetch_tmap(&tma_xh);
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
      int sx = 0, sw = 0;
      unsigned int px = 0, pw = 0;
      long long nx = 0, nw = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        int j, nt, n, ho, seg;
        rowt_decode(P, t, j, nt, n, ho, seg);
        const int wbase = seg * P.NPIX - P.pad;
        // the channel blocks of every group in turn, all into the tile's one accumulator
        const int nblocks = P.jgroups * P.cblocks;
        for (int cbg = 0; cbg < nblocks && ok; ++cbg) {
          const int jx = cbg / P.cblocks;
          const int cb = cbg - jx * P.cblocks;
          const int obase = jx * P.cpg_out + nt * BM;
          const int cin = jx * P.cpg_in + cb * 64;
          for (int kh = 0; kh < P.kH && ok; ++kh) {
            if (!mbar_wait(&ex[sx], px ^ 1u, abort_flag, err, ERR_WAIT_PRODUCER)) {
              ok = false;
              break;
            }
            unsigned char* dst = x_base + (size_t)sx * P.x_stage;
            const int hrow = ho - P.pad + kh * P.dil;
            mbar_arrive_expect_tx(&fx[sx], P.x_tx);
            tma_load_4d(dst, &tma_x, &fx[sx], cin, wbase, hrow, n);
            tma_load_4d(dst + P.box1_bytes, &tma_xh, &fx[sx], cin, wbase + P.NPIX, hrow, n);
            ++nx;
            if (++sx == P.x_stages) {
              sx = 0;
              px ^= 1u;
            }
            for (int kw = 0; kw < P.kW; ++kw) {
              if (!mbar_wait(&ew[sw], pw ^ 1u, abort_flag, err, ERR_WAIT_PRODUCER)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&fw[sw], P.w_tx);
              tma_load_2d(w_base + (size_t)sw * P.w_stage, &tma_w, &fw[sw],
                          (kh * P.kW + kw) * P.cpg_in + cb * 64, obase);
              ++nw;
              if (++sw == P.w_stages) {
                sw = 0;
                pw ^= 1u;
              }
            }
          }
        }
      }
      const unsigned long long dl = drain_deadline();
      for (long long q = (nx > P.x_stages ? nx - P.x_stages : 0); q < nx; ++q)
        mbar_wait_until(&fx[q % P.x_stages], (unsigned int)((q / P.x_stages) & 1), dl, err,
                        ERR_WAIT_DRAIN);
      for (long long q = (nw > P.w_stages ? nw - P.w_stages : 0); q < nw; ++q)
        mbar_wait_until(&fw[q % P.w_stages], (unsigned int)((q / P.w_stages) & 1), dl, err,
                        ERR_WAIT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: descriptors built once, advanced by constant offsets
      int sx = 0, sw = 0, acc = 0;
      unsigned int px = 0, pw = 0, aph = 0;
      bool ok = true;
      const unsigned long long x_desc0 = smem_desc(smem_u32(x_base), 1024u, 2u);
      const unsigned long long w_desc0 = smem_desc(smem_u32(w_base), 1024u, 2u);
      const unsigned long long kw_step = (unsigned long long)P.dil * 8u;   // dil rows of 128 B
      for (int t = blockIdx.x; t < P.num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, err, ERR_WAIT_MMA)) break;
        tc_fence_after();
        const unsigned int d = tmem_base + (unsigned int)(acc * P.NPIX);
        const int nblocks = P.jgroups * P.cblocks;
        for (int cb = 0; cb < nblocks && ok; ++cb) {
          for (int kh = 0; kh < P.kH && ok; ++kh) {
            if (!mbar_try_wait(&fx[sx], px) &&
                !mbar_wait(&fx[sx], px, abort_flag, err, ERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            const unsigned long long xs = x_desc0 + (((unsigned long long)sx * P.x_stage) >> 4);
            for (int kw = 0; kw < P.kW; ++kw) {
              if (!mbar_try_wait(&fw[sw], pw) &&
                  !mbar_wait(&fw[sw], pw, abort_flag, err, ERR_WAIT_MMA)) {
                ok = false;
                break;
              }
              const unsigned long long wd = w_desc0 + (((unsigned long long)sw * P.w_stage) >> 4);
              const unsigned long long xd = xs + kw * kw_step;
              const unsigned int acc0 = (cb | kh | kw) == 0 ? 0u : 1u;
              umma_f16(d, wd, xd, P.idesc, acc0);
              umma_f16(d, wd + 2, xd + 2, P.idesc, 1u);
              umma_f16(d, wd + 4, xd + 4, P.idesc, 1u);
              umma_f16(d, wd + 6, xd + 6, P.idesc, 1u);
              umma_commit(&ew[sw]);
              if (++sw == P.w_stages) {
                sw = 0;
                pw ^= 1u;
              }
            }
            if (!ok) break;
            umma_commit(&ex[sx]);
            if (++sx == P.x_stages) {
              sx = 0;
              px ^= 1u;
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
    // ---------------- epilogue: warps 2..5; TMEM lane = output channel of the tile
    const int quarter = warp & 3;
    const int co_l = quarter * 32 + lane;
    int acc = 0;
    unsigned int aph = 0;
    for (int t = blockIdx.x; t < P.num_tiles; t += gridDim.x) {
      int j, nt, n, ho, seg;
      rowt_decode(P, t, j, nt, n, ho, seg);
      const bool got = mbar_wait(&tfull[acc], aph, abort_flag, err, ERR_WAIT_EPILOGUE);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int co = nt * BM + co_l;   // channel of the merged output
      // bias of the merged channel: the mean of the groups' biases for this filter position
      float bv = 0.0f;
      if (bias) {
        for (int i = 0; i < P.jgroups; ++i)
          bv += Elem<T>::to_f32(bias[i * P.cpg_out + co]);
        bv *= P.scale;
      }
      const float sc = P.scale;   // 1 / groups
      const unsigned int taddr =
          tmem_base + ((unsigned int)(quarter * 32) << 16) + (unsigned int)(acc * P.NPIX);
      for (int c = 0; c < P.NPIX; c += 32) {
        unsigned int r[32];
        tmem_ld32(taddr + c, r);
        tmem_ld_wait();
        const int wo0 = seg * P.NPIX + c;
        if (wo0 >= P.Wo) continue;
        if (!P.out_nchw) {
          T* dst = y + (((long long)n * P.Ho + ho) * P.Wo + wo0) * P.out_c + co;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (wo0 + i < P.Wo)
              dst[(long long)i * P.out_c] =
                  Elem<T>::from_f32(fmaf(__uint_as_float(r[i]), sc, bv));
        } else {
          T* dst = y + (((long long)n * P.out_c + co) * P.Ho + ho) * P.Wo + wo0;
          if (P.nchw_vec && wo0 + 32 <= P.Wo) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 u;
              u.x = pack2<T>(make_float2(fmaf(__uint_as_float(r[8 * q + 0]), sc, bv),
                                         fmaf(__uint_as_float(r[8 * q + 1]), sc, bv)));
              u.y = pack2<T>(make_float2(fmaf(__uint_as_float(r[8 * q + 2]), sc, bv),
                                         fmaf(__uint_as_float(r[8 * q + 3]), sc, bv)));
              u.z = pack2<T>(make_float2(fmaf(__uint_as_float(r[8 * q + 4]), sc, bv),
                                         fmaf(__uint_as_float(r[8 * q + 5]), sc, bv)));
              u.w = pack2<T>(make_float2(fmaf(__uint_as_float(r[8 * q + 6]), sc, bv),
                                         fmaf(__uint_as_float(r[8 * q + 7]), sc, bv)));
              reinterpret_cast<uint4*>(dst)[q] = u;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (wo0 + i < P.Wo)
                dst[i] = Elem<T>::from_f32(fmaf(__uint_as_float(r[i]), sc, bv));
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
}

// Transposed row kernel parameters; false if the problem does not take it.
bool make_rowt_params(const Conv2d& p, RowTParams* R) {
  if (p.out_mode == GCONV_OUT_MERGE_MAX) return false;
  if (p.Wo < BM || p.cpg_in % 64 != 0 || p.cpg_out % BM != 0) return false;
  if ((p.kW - 1) * p.dil > 8) return false;            // halo fits the 8-row second box
  R->N = p.N; R->C_out = p.C_out;
  R->Ho = p.Ho; R->Wo = p.Wo; R->kH = p.kH; R->kW = p.kW; R->pad = p.pad; R->dil = p.dil;
  R->cpg_in = p.cpg_in; R->cpg_out = p.cpg_out;
  R->NPIX = p.Wo > BM ? 256 : 128;
  R->cblocks = p.cpg_in / 64;
  R->segs = (p.Wo + R->NPIX - 1) / R->NPIX;
  R->n_tiles = p.cpg_out / BM;
  const long long tiles = (long long)R->segs * p.Ho * p.N * R->n_tiles * p.groups;
  if (tiles > INT32_MAX) return false;
  R->num_tiles = (int)tiles;
  R->box1_bytes = (unsigned int)R->NPIX * 128u;
  R->x_tx = (unsigned int)(R->NPIX + 8) * 128u;   // strip rows: NPIX + the 8-row halo box
  R->x_stage = (R->x_tx + 1023u) & ~1023u;
  R->w_tx = (unsigned int)BM * 128u;
  R->w_stage = R->w_tx;
  const size_t fixed = 1024 + (2 * (ROW_MAX_A + ROW_MAX_B) + 5) * 8 + 16;
  const size_t budget = SMEM_BUDGET - fixed;
  int xs = 3;
  if ((size_t)xs * R->x_stage > budget / 2) xs = 2;
  int ws = (int)((budget - (size_t)xs * R->x_stage) / R->w_stage);
  if (ws > ROW_MAX_B) ws = ROW_MAX_B;
  if (ws < 2) return false;
  R->x_stages = xs;
  R->w_stages = ws;
  const unsigned int fmt = p.dtype == GCONV_BF16 ? 1u : 0u;
  R->idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | ((unsigned int)(R->NPIX >> 3) << 17) |
             ((unsigned int)(BM >> 4) << 24);
  R->tmem_cols = pow2_cols(2 * R->NPIX);
  if (R->tmem_cols > 512) return false;
  R->out_nchw = p.layout == GCONV_NCHW;
  R->nchw_vec = (p.Wo % 8 == 0) ? 1 : 0;
  R->groups = p.groups;
  R->interleave = p.out_mode == GCONV_OUT_INTERLEAVED;
  const bool avg = p.out_mode == GCONV_OUT_MERGE_AVG;
  R->jgroups = avg ? p.groups : 1;
  R->out_c = out_channels(p);
  R->scale = avg ? 1.0f / (float)p.groups : 1.0f;
  if (avg) R->num_tiles /= p.groups;   // one tile covers every group's K loop
  return true;
}

size_t rowt_smem_bytes(const RowTParams& R) {
  return 1024 + (size_t)R.x_stages * R.x_stage + (size_t)R.w_stages * R.w_stage +
         (2 * (ROW_MAX_A + ROW_MAX_B) + 5) * 8 + 16;
}

template <typename T>
cudaError_t launch_rowt(const Conv2d& p, const RowTParams& R, const void* x, const void* w,
                        const void* bias, void* y, cudaStream_t s) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt =
      p.dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tx, txh, tw;
  const cuuint64_t xdim[4] = {(cuuint64_t)p.C_in, (cuuint64_t)p.W, (cuuint64_t)p.H,
                              (cuuint64_t)p.N};
  const cuuint64_t xstr[3] = {(cuuint64_t)p.C_in * 2, (cuuint64_t)p.W * p.C_in * 2,
                              (cuuint64_t)p.H * p.W * p.C_in * 2};
  const cuuint32_t ones[4] = {1, 1, 1, 1};
  const cuuint32_t xbox[4] = {64, (cuuint32_t)R.NPIX, 1, 1};
  const cuuint32_t hbox[4] = {64, 8, 1, 1};
  if (enc(&tx, dt, 4, const_cast<void*>(x), xdim, xstr, xbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (enc(&txh, dt, 4, const_cast<void*>(x), xdim, xstr, hbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const cuuint64_t ktot = (cuuint64_t)p.kH * p.kW * p.cpg_in;
  const cuuint64_t wdim[2] = {ktot, (cuuint64_t)p.C_out};
  const cuuint64_t wstr[1] = {ktot * 2};
  const cuuint32_t wbox[2] = {64, (cuuint32_t)BM};
  if (enc(&tw, dt, 2, const_cast<void*>(w), wdim, wstr, wbox, ones,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = rowt_smem_bytes(R);
  if (smem > SMEM_BUDGET) return cudaErrorInvalidValue;
  static std::atomic<unsigned int> configured{0}, configured_avg{0};
  const bool avg = R.jgroups > 1;
  cudaError_t e = avg ? set_max_dynamic_smem((const void*)igemm_rowt_avg_kernel<T>, SMEM_BUDGET,
                                             configured_avg)
                      : set_max_dynamic_smem((const void*)igemm_rowt_kernel<T>, SMEM_BUDGET,
                                             configured);
  if (e != cudaSuccess) return e;
  int grid = sm_count();
  if (grid > R.num_tiles) grid = R.num_tiles;
  if (avg)
    return launch_pdl(igemm_rowt_avg_kernel<T>, (unsigned)grid, NUM_THREADS, smem, s, tx, txh,
                      tw, (const T*)bias, (T*)y, R, device_error_word());
  return launch_pdl(igemm_rowt_kernel<T>, (unsigned)grid, NUM_THREADS, smem, s, tx, txh, tw,
                    (const T*)bias, (T*)y, R, device_error_word());
}

}  // namespace

bool igemm_rowt_supported(const Conv2d& p) {
  RowTParams R;
  return make_rowt_params(p, &R);
}

cudaError_t launch_igemm_rowt(const Conv2d& p, const void* x, const void* w, const void* bias,
                              void* y, cudaStream_t s) {
  RowTParams R;
  if (!make_rowt_params(p, &R)) return cudaErrorInvalidValue;
  if (p.dtype == GCONV_BF16) return launch_rowt<__nv_bfloat16>(p, R, x, w, bias, y, s);
  if (p.dtype == GCONV_F16) return launch_rowt<__half>(p, R, x, w, bias, y, s);
  return cudaErrorInvalidValue;
}

}  // namespace gconv
