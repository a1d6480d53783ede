// Depthwise conv1d forward and data gradient on the tensor cores (tcgen05, kind::f16).
//
// The layer is the Conformer convolution module's depthwise convolution on (batch, steps,
// channels) ("Investigate custom Triton kernels for depthwise-separable convolutions in
// Conformer", speechbrain #2733, Oct 27 comment):  y[b,t,c] = sum_k w[c,k] * x[b, t+k-pl, c];
// the data gradient (Oct 30 comment) is the same sum with the filter reversed and the pads
// swapped, so one kernel serves both (FLIP).
//
// Each channel is a banded product. Cut a channel's output steps into blocks of 16 and take
// 128 blocks (2048 steps) as the M = 128 rows of one MMA chain:
//   y_c[16m + 15 - j] = sum_s A_c[m][s] * W_c[j][s]       m < 128, j < 16, s < 16*KS
//   A_c[m][s] = x_c[16m + s - pl]            (block m's input window; zero outside [0, T))
//   W_c[j][s] = w_c[s + j - 15]              (zero outside [0, K))
// so a chain is KS MMAs of M = 128, N = 16, K = 16 (K <= 16*KS - 15). The products are exact
// in fp32 and accumulate in TMEM; the tensor cores do ~1.5x the algorithmic multiply-adds
// (16*KS per output instead of K) at a rate the FP32 pipe cannot approach.
//
// Operand layouts (no swizzle, K-major, 16-byte core-matrix rows):
//  * A: the transposed input of channel c as 16-byte chunks of 8 steps; chunk q = box rows
//    [8q, 8q+8). Even chunks go to E_c, odd ones to O_c. Row m, K-chunk 2j is E_c[m + j] and
//    chunk 2j+1 is O_c[m + j], so the descriptor of K-step j starts at E_c[j] with a 16-byte row
//    stride, LBO = O_c - E_c and SBO = 128: every input chunk is stored once, no window copies.
//  * W: 8 shifted copies of the zero-padded filter, copy r chunk p = wpad[8p + r .. +8). Row
//    j = 8i + r, K-chunk g is copy r chunk g + i, stored at p*128 + 16r: LBO = SBO = 128.
//  The transposes run on shared memory with ldmatrix.trans / stmatrix (8x8 16-bit blocks).
//
// A tile is (16 channels, one batch, 2048 output steps): its input rows are 32 bytes wide (one
// full L2 sector per step), and it is computed as two sub-tiles of 8 channels. Warp roles in a
// persistent CTA:
//   warp 0      TMA producer: the tile's input rows [t0 - pl, t0 - pl + 2032 + 16*KS) x 16 ch
//               and, by a bulk copy, the 16 channels' filter taps
//   warp 1      TMEM owner and MMA issuer (per sub-tile 8 channels x KS MMAs, one commit)
//   warps 2-5   epilogue: TMEM -> registers -> transposed output in the A buffer ->
//               ldmatrix.trans / stmatrix into the tile's buffer as [steps][16 ch] -> TMA store
//   warps 6-9   transpose of the input box into the A layout; filter copies
// Two tile buffers alternate between a CTA's tiles. A tile's buffer first takes its input rows;
// the epilogue then stages the tile's output rows in the same buffer (output half h overwrites
// only the bytes of input half h, which the transpose of half h consumed before the sub-tile's
// MMAs could start), and the buffer goes back to the producer once the tile's TMA store has read
// it. The next tile's input is therefore loaded while this one is computed. Operands and
// accumulators go through a ring of 2 sub-tiles (released once the epilogue has read them).
#include <type_traits>

#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

constexpr int TC_TCH = 16;            // channels per tile (32-byte rows)
constexpr int TC_CH = 8;              // channels per sub-tile (MMA chains per commit)
constexpr int TC_BLOCKS = 128;        // MMA rows: blocks of 16 steps
constexpr int TC_STEPS = 16 * TC_BLOCKS;
constexpr int TC_ASTAGES = 2;         // operand / accumulator stages (sub-tiles)
constexpr int TC_XBUFS = 2;           // tile buffers: input rows, then the tile's output rows
constexpr int TC_THREADS = 320;
constexpr int TC_TMEM_COLS = 256;     // 2 stages x 8 channels x 16 columns
constexpr int TC_MAX_KS = 4;          // K <= 49
constexpr int TC_WS_BYTES = 2048;     // filter taps of a tile: 16 x K x 2 bytes

struct TcLayout {
  int rows;          // input rows a tile needs: 2032 + 16*KS
  int n_boxes;       // TMA boxes per tile
  int box_h;         // rows per box (multiple of 8, at most 256)
  int eoff;          // bytes from E_c to O_c
  int cstride;       // bytes between channels in the A buffer (odd multiple of 16)
  int bstride;       // bytes between channels in the filter copies
  int xs_bytes, as_bytes, bs_bytes;
  int xbuf;          // bytes per tile buffer: the input boxes or the 2048 x 32-byte output rows
  int ws_off, as_off, astage, total;
};

__host__ __device__ constexpr TcLayout tc_layout(int KS) {
  TcLayout L{};
  L.rows = TC_STEPS - 16 + 16 * KS;
  L.n_boxes = (L.rows + 255) / 256;
  L.box_h = ((L.rows + L.n_boxes - 1) / L.n_boxes + 7) / 8 * 8;
  L.eoff = L.rows;                       // rows / 16 chunks of 16 bytes
  L.cstride = 2 * L.rows + 16;
  L.bstride = (2 * KS + 1) * 128;
  L.xs_bytes = L.n_boxes * L.box_h * 32; // rows past `rows` are loaded but not used
  L.as_bytes = ((TC_CH * L.cstride + 1023) / 1024) * 1024;
  L.bs_bytes = ((TC_CH * L.bstride + 1023) / 1024) * 1024;
  L.xbuf = ((L.xs_bytes > TC_STEPS * 32 ? L.xs_bytes : TC_STEPS * 32) + 127) / 128 * 128;
  L.ws_off = TC_XBUFS * L.xbuf;
  L.as_off = ((L.ws_off + TC_XBUFS * TC_WS_BYTES + 1023) / 1024) * 1024;
  L.astage = L.as_bytes + L.bs_bytes;
  L.total = L.as_off + TC_ASTAGES * L.astage;
  return L;
}

constexpr int TC_YSTRIDE = 2 * TC_STEPS + 16;   // transposed output, bytes per channel

struct TcParams {
  int B, T_in, C, K, T_out, pl;
  int n_ct, n_tc, num_tiles;
};

__device__ __forceinline__ unsigned long long desc_plain(unsigned int addr, unsigned int lbo,
                                                         unsigned int sbo) {
  unsigned long long d = (unsigned long long)((addr >> 4) & 0x3FFFu);
  d |= (unsigned long long)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (unsigned long long)((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;                      // descriptor version (sm_100)
  return d;                             // base offset 0, no swizzle
}

struct TileCoord {
  int ct, b, tc;
  __device__ __forceinline__ void set(const TcParams& P, int t) {
    ct = t % P.n_ct;
    const int r = t / P.n_ct;
    b = r % P.B;
    tc = r / P.B;
  }
  // first input step of the tile's box rows
  __device__ __forceinline__ int row0(const TcParams& P) const { return tc * TC_STEPS - P.pl; }
};

// Box i of a tile holds no step of [0, T_in): it is not loaded, its rows are taken as zeros.
__device__ __forceinline__ bool box_outside(const TcParams& P, int r0, int i, int box_h) {
  const int first = r0 + box_h * i;
  return first >= P.T_in || first + box_h - 1 < 0;
}

template <typename T> struct MmaFmt;
template <> struct MmaFmt<__nv_bfloat16> { static constexpr unsigned int v = 1; };
template <> struct MmaFmt<__half> { static constexpr unsigned int v = 0; };

template <typename T, int KS, bool FLIP>
__global__ void __launch_bounds__(TC_THREADS, 1)
    dwconv1d_tc_kernel(const __grid_constant__ CUtensorMap tmx,
                       const __grid_constant__ CUtensorMap tmy, const T* __restrict__ w,
                       const TcParams P, unsigned int* err) {
  using namespace ptx;
  constexpr TcLayout L = tc_layout(KS);
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = ptx::align_smem(smem_raw, 1024u);
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(smem + L.total);
  unsigned long long* xs_full = bars;                          // [2] producer: tx bytes
  unsigned long long* x_free = bars + TC_XBUFS;                // [2] epilogue store thread
  unsigned long long* as_full = bars + 2 * TC_XBUFS;           // 4 transposer warps
  unsigned long long* as_empty = as_full + TC_ASTAGES;         // epilogue store thread
  unsigned long long* tm_full = as_empty + TC_ASTAGES;         // MMA commit
  unsigned int* tmem_slot = reinterpret_cast<unsigned int*>(tm_full + TC_ASTAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = (int)((long long)P.num_tiles * blockIdx.x / gridDim.x);
  const int t_end = (int)((long long)P.num_tiles * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int k = 0; k < TC_XBUFS; ++k) {
      mbar_init(&xs_full[k], 1);
      mbar_init(&x_free[k], 1);
    }
    for (int s = 0; s < TC_ASTAGES; ++s) {
      mbar_init(&as_full[s], 4);
      mbar_init(&as_empty[s], 1);
      mbar_init(&tm_full[s], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmy);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned int tmem_base = *tmem_slot;
  // the setup above may overlap the previous kernel in the stream (launch_pdl)
  pdl_wait();
  pdl_launch_dependents();

  auto xb = [&](int k) { return smem + (size_t)k * L.xbuf; };              // tile buffers
  auto wsb = [&](int k) { return smem + L.ws_off + (size_t)k * TC_WS_BYTES; };
  auto as = [&](int s) { return smem + L.as_off + (size_t)s * L.astage; };
  auto bs = [&](int s) { return as(s) + L.as_bytes; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const unsigned int wbytes = (unsigned int)(TC_TCH * P.K * 2);
      int n = 0;
      for (int t = t_begin; t < t_end; ++t, ++n) {
        const int k = n % TC_XBUFS;
        // buffer k is free again once the TMA store of tile n - 2 has read it
        const unsigned int fph = (unsigned int)(n / TC_XBUFS - 1) & 1u;
        if (n >= TC_XBUFS && !mbar_wait(&x_free[k], fph, abort_flag, err, 256u)) break;
        TileCoord c;
        c.set(P, t);
        const int r0 = c.row0(P);
        unsigned int nbytes = wbytes;
        for (int i = 0; i < L.n_boxes; ++i)
          if (!box_outside(P, r0, i, L.box_h)) nbytes += (unsigned int)L.box_h * 32;
        mbar_arrive_expect_tx(&xs_full[k], nbytes);
        bulk_load(wsb(k), w + (size_t)c.ct * TC_TCH * P.K, wbytes, &xs_full[k]);
        for (int i = 0; i < L.n_boxes; ++i)
          if (!box_outside(P, r0, i, L.box_h))
            tma_load_3d(xb(k) + (size_t)i * L.box_h * 32, &tmx, &xs_full[k], c.ct * TC_TCH,
                        r0 + L.box_h * i, c.b);
      }
      // copies in flight must land before the CTA exits: the last load into each buffer
      const unsigned long long dl = drain_deadline();
      for (int q = (n > TC_XBUFS ? n - TC_XBUFS : 0); q < n; ++q)
        mbar_wait_until(&xs_full[q % TC_XBUFS], (unsigned int)(q / TC_XBUFS) & 1u, dl, err,
                        ERR_DRAIN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr unsigned int idesc = (1u << 4) | (MmaFmt<T>::v << 7) | (MmaFmt<T>::v << 10) |
                                     ((16u >> 3) << 17) | ((128u >> 4) << 24);
      const int n_sub = 2 * (t_end - t_begin);
      int u = 0;
      for (; u < n_sub; ++u) {
        const int s = u % TC_ASTAGES;
        const unsigned int ph = (unsigned int)(u / TC_ASTAGES) & 1u;
        if (!mbar_wait(&as_full[s], ph, abort_flag, err, 512u)) break;
        tc_fence_after();
        const unsigned int a0 = smem_u32(as(s)), b0 = smem_u32(bs(s));
#pragma unroll
        for (int ch = 0; ch < TC_CH; ++ch) {
          const unsigned long long ad = desc_plain(a0 + ch * L.cstride, L.eoff, 128);
          const unsigned long long bd = desc_plain(b0 + ch * L.bstride, 128, 128);
          const unsigned int d = tmem_base + (unsigned int)(s * 128 + ch * 16);
#pragma unroll
          for (int j = 0; j < KS; ++j)
            umma_f16(d, ad + (unsigned long long)j, bd + (unsigned long long)(16 * j), idesc,
                     j > 0 ? 1u : 0u);
        }
        umma_commit(&tm_full[s]);
      }
      // the last chain must finish before TMEM is released (already true on the normal path)
      if (u > 0)
        mbar_wait_until(&tm_full[(u - 1) % TC_ASTAGES], (unsigned int)((u - 1) / TC_ASTAGES) & 1u,
                        drain_deadline(), err, ERR_DRAIN);
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------ transposes + filter copies
    const int tw = warp - 6, tid = threadIdx.x - 192;
    constexpr int NBLK = L.rows / 8;                 // 8x8 blocks per sub-tile
    int n = 0;
    bool ok = true;
    for (int t = t_begin; t < t_end && ok; ++t, ++n) {
      const int k = n % TC_XBUFS;
      const unsigned int xph = (unsigned int)(n / TC_XBUFS) & 1u;
      const unsigned short* wt = reinterpret_cast<const unsigned short*>(wsb(k));
      const unsigned int xsa = smem_u32(xb(k));
      bool got = mbar_try_wait(&xs_full[k], xph);
      if (!got) got = mbar_wait(&xs_full[k], xph, abort_flag, err, 1024u);
      if (!__all_sync(0xffffffffu, got)) break;
      TileCoord c;
      c.set(P, t);
      const int r0 = c.row0(P);
      unsigned int outside = 0;                       // boxes read as zeros, uniform
      for (int i = 0; i < L.n_boxes; ++i)
        if (box_outside(P, r0, i, L.box_h)) outside |= 1u << i;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int u = 2 * n + h, s = u % TC_ASTAGES;
        const unsigned int eph = ((unsigned int)(u / TC_ASTAGES) & 1u) ^ 1u;
        got = mbar_try_wait(&as_empty[s], eph);
        if (!got) got = mbar_wait(&as_empty[s], eph, abort_flag, err, 1024u);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        // filter copies: copy r chunk p holds wpad[8p + r + e], wpad[u] = w'[ch][u - 15]
        constexpr int NP = 2 * KS + 1;
        for (int i = tid; i < TC_CH * NP * 8; i += 128) {
          const int ch = i / (NP * 8), rem = i % (NP * 8), p = rem / 8, r = rem % 8;
          const unsigned short* wc = wt + (8 * h + ch) * P.K;
          unsigned int v[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int k0 = 8 * p + r + 2 * e2 - 15;
            const unsigned int lo =
                (k0 >= 0 && k0 < P.K) ? (unsigned int)wc[FLIP ? P.K - 1 - k0 : k0] : 0u;
            const unsigned int hi =
                (k0 + 1 >= 0 && k0 + 1 < P.K) ? (unsigned int)wc[FLIP ? P.K - 2 - k0 : k0 + 1]
                                              : 0u;
            v[e2] = lo | (hi << 16);
          }
          *reinterpret_cast<uint4*>(bs(s) + ch * L.bstride + p * 128 + 16 * r) =
              make_uint4(v[0], v[1], v[2], v[3]);
        }
        // half h of the input box [rows][16 ch] -> E/O chunks per channel
        const unsigned int asa = smem_u32(as(s));
        const unsigned int src = xsa + (unsigned int)((lane & 7) * 32 + 16 * h);
#pragma unroll 2
        for (int q0 = 4 * tw; q0 < NBLK; q0 += 16) {
          int q = q0 + (lane >> 3);
          if (q > NBLK - 1) q = NBLK - 1;            // spare matrices repeat the last block
          unsigned int r[4];
          ldsm_x4_trans(src + (unsigned int)(q * 256), r);
          if (outside) {
            // register i holds matrix i = block min(q0 + i, NBLK - 1); a block lies in one box
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int qi = q0 + i < NBLK ? q0 + i : NBLK - 1;
              if ((outside >> ((8 * qi) / L.box_h)) & 1u) r[i] = 0u;
            }
          }
          stsm_x4(asa + (unsigned int)((lane & 7) * L.cstride + (q & 1) * L.eoff + (q >> 1) * 16),
                  r);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&as_full[s]);
      }
      // the tile buffer now belongs to the epilogue, which stages the tile's output in it
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int quarter = warp & 3, ew = warp - 2;
    const int m = 32 * quarter + lane;               // MMA row = block of 16 steps
    const bool store_thread = (warp == 2 && lane == 0);
    const int n_sub = 2 * (t_end - t_begin);
    const int hsw = (m >> 2) & 1;                    // store order that avoids bank conflicts
    for (int u = 0; u < n_sub; ++u) {
      const int s = u % TC_ASTAGES, h = u & 1;
      const unsigned int ph = (unsigned int)(u / TC_ASTAGES) & 1u;
      bool got = mbar_try_wait(&tm_full[s], ph);
      if (!got) got = mbar_wait(&tm_full[s], ph, abort_flag, err, 2048u);
      if (!named_all(1, 128, got)) break;          // the four warps leave together
      tc_fence_after();
      unsigned char* ybuf = as(s);                   // A operand is consumed: reuse it
#pragma unroll
      for (int c4 = 0; c4 < TC_CH; c4 += 4) {
        unsigned int v[4][32];
#pragma unroll
        for (int g = 0; g < 4; ++g)
          tmem_ld16(tmem_base + ((unsigned int)(32 * quarter) << 16) +
                        (unsigned int)(s * 128 + (c4 + g) * 16),
                    v[g]);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          // column j holds step 16m + 15 - j
          unsigned int wd[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            wd[e] = pack2<T>(make_float2(__uint_as_float(v[g][15 - 2 * e]),
                                         __uint_as_float(v[g][14 - 2 * e])));
          unsigned char* dst = ybuf + (c4 + g) * TC_YSTRIDE + 32 * m;
          const uint4 lo = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          const uint4 hi = make_uint4(wd[4], wd[5], wd[6], wd[7]);
          *reinterpret_cast<uint4*>(dst + 16 * hsw) = hsw ? hi : lo;
          *reinterpret_cast<uint4*>(dst + 16 * (1 - hsw)) = hsw ? lo : hi;
        }
      }
      tc_fence_before();
      const int n = u >> 1, k = n % TC_XBUFS;
      if (h == 0 && n > 0 && store_thread) {
        bulk_wait_read0();                           // tile n - 1's store has read its buffer
        mbar_arrive(&x_free[(n - 1) % TC_XBUFS]);    // ... which may take tile n + 1's input
      }
      named_sync(1, 128);
      // transposed output -> half h of the [steps][16 ch] rows in the tile's own buffer, whose
      // input half h the transpose consumed before this sub-tile's MMAs
      const unsigned int ya = smem_u32(ybuf) + (unsigned int)((lane & 7) * TC_YSTRIDE);
      const unsigned int oa = smem_u32(xb(k)) + (unsigned int)((lane & 7) * 32 + 16 * h);
#pragma unroll 4
      for (int q0 = 4 * ew; q0 < TC_STEPS / 8; q0 += 16) {
        const int q = q0 + (lane >> 3);
        unsigned int r[4];
        ldsm_x4_trans(ya + (unsigned int)(16 * q), r);
        stsm_x4(oa + (unsigned int)(q * 256), r);
      }
      fence_async_smem();
      named_sync(1, 128);
      if (store_thread) {
        mbar_arrive(&as_empty[s]);                   // operands, accumulator, Y read
        if (h == 1) {
          TileCoord c;
          c.set(P, t_begin + (u >> 1));
          const int t0 = c.tc * TC_STEPS;
          for (int i = 0; i < TC_STEPS / 256; ++i)
            if (t0 + 256 * i < P.T_out)
              tma_store_3d(&tmy, xb(k) + (size_t)i * 256 * 32, c.ct * TC_TCH, t0 + 256 * i,
                           c.b);
          bulk_commit();
        }
      }
    }
    if (store_thread) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TC_TMEM_COLS);
  }
}

bool make_map_rows8(CUtensorMap* m, int dtype, const void* base, int C, int T_len, int B,
                    int rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const CUtensorMapDataType dt =
      dtype == GCONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T_len, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)C * 2, (cuuint64_t)T_len * C * 2};
  const cuuint32_t box[3] = {TC_TCH, (cuuint32_t)rows, 1};
  const cuuint32_t ones[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, ones,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static_assert(tc_layout(TC_MAX_KS).total + 2048 <= 227 * 1024, "shared memory budget");

template <typename T, int KS, bool FLIP>
cudaError_t launch_tc(const Conv1d& p, const void* x, const void* w, void* y, int pl, int T_in,
                      int T_out, cudaStream_t s) {
  constexpr TcLayout L = tc_layout(KS);
  TcParams P;
  P.B = p.B; P.T_in = T_in; P.C = p.C; P.K = p.K; P.T_out = T_out; P.pl = pl;
  P.n_ct = p.C / TC_TCH;
  P.n_tc = (T_out + TC_STEPS - 1) / TC_STEPS;
  const long long tiles = (long long)P.n_ct * p.B * P.n_tc;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  P.num_tiles = (int)tiles;
  CUtensorMap tmx, tmy;
  if (!make_map_rows8(&tmx, p.dtype, x, p.C, T_in, p.B, L.box_h) ||
      !make_map_rows8(&tmy, p.dtype, y, p.C, T_out, p.B, 256))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + (size_t)L.total + 8 * (2 * TC_XBUFS + 3 * TC_ASTAGES) + 16;
  static std::atomic<unsigned int> configured{0};
  cudaError_t e = set_max_dynamic_smem((const void*)dwconv1d_tc_kernel<T, KS, FLIP>, smem,
                                       configured);
  if (e != cudaSuccess) return e;
  long long grid = sm_count();
  if (grid > P.num_tiles) grid = P.num_tiles;
  return launch_pdl(dwconv1d_tc_kernel<T, KS, FLIP>, (unsigned)grid, TC_THREADS, smem, s, tmx,
                    tmy, (const T*)w, P, device_error_word());
}

template <typename T, bool FLIP>
cudaError_t tc_by_ks(const Conv1d& p, const void* x, const void* w, void* y, int pl, int T_in,
                     int T_out, cudaStream_t s) {
  const int ks = (p.K + 15 + 15) / 16;
  switch (ks) {
    case 1: return launch_tc<T, 1, FLIP>(p, x, w, y, pl, T_in, T_out, s);
    case 2: return launch_tc<T, 2, FLIP>(p, x, w, y, pl, T_in, T_out, s);
    case 3: return launch_tc<T, 3, FLIP>(p, x, w, y, pl, T_in, T_out, s);
    default: return launch_tc<T, 4, FLIP>(p, x, w, y, pl, T_in, T_out, s);
  }
}

}  // namespace

bool conv1d_tc_supported(const Conv1d& p) {
  // pads and lengths bounded so that every tile-row coordinate fits in an int
  return p.dtype != GCONV_F32 && p.C % TC_TCH == 0 && p.K >= 1 && p.K <= 16 * TC_MAX_KS - 15 &&
         p.B >= 1 && p.pad_left <= (1 << 24) && p.pad_right <= (1 << 24) && p.T <= (1 << 28) &&
         p.T_out <= (1 << 28);
}

cudaError_t launch_dwconv1d_tc(const Conv1d& p, const void* x, const void* w, void* y, bool flip,
                               int pad_left, int T_in, int T_out, cudaStream_t s) {
  if (p.dtype == GCONV_F16)
    return flip ? tc_by_ks<__half, true>(p, x, w, y, pad_left, T_in, T_out, s)
                : tc_by_ks<__half, false>(p, x, w, y, pad_left, T_in, T_out, s);
  return flip ? tc_by_ks<__nv_bfloat16, true>(p, x, w, y, pad_left, T_in, T_out, s)
              : tc_by_ks<__nv_bfloat16, false>(p, x, w, y, pad_left, T_in, T_out, s);
}

}  // namespace gconv
