// Constants and helpers shared by the implicit-GEMM tile kernels (igemm_tc.cu) and the
// transposed row-strip kernel (igemm_rowt.cu). Everything here has internal linkage: each
// translation unit gets its own copy.
#pragma once

#include "internal.cuh"
#include "sm100_ptx.cuh"

namespace gconv {
namespace {

constexpr int BM = 128;                 // output pixels (or filters) per tile (UMMA M)
constexpr int NUM_THREADS = 192;        // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int MAX_STAGES = 32;
constexpr size_t SMEM_BUDGET = 227 * 1024;
constexpr int ROW_MAX_A = 4;            // row kernels: input-strip stages
constexpr int ROW_MAX_B = 16;           // row kernels: weight-tile stages

enum : unsigned int { ERR_WAIT_PRODUCER = 1u, ERR_WAIT_MMA = 2u, ERR_WAIT_EPILOGUE = 4u,
                      ERR_WAIT_DRAIN = 8u };

// Shared-memory matrix descriptor (tcgen05): start address, leading / stride byte offsets
// (16-byte units), descriptor version 1 at bits 46-47, layout (swizzle) code at bits 61-63.
// The base-offset field (bits 49-51) stays 0: the swizzle is taken from the absolute address.
__device__ __forceinline__ unsigned long long smem_desc(unsigned int saddr, unsigned int sbo,
                                                        unsigned int swz) {
  unsigned long long d = (unsigned long long)((saddr >> 4) & 0x3FFFu);
  d |= (unsigned long long)1u << 16;                          // LBO (unused for swizzled K-major)
  d |= (unsigned long long)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (unsigned long long)1u << 46;
  d |= (unsigned long long)(swz & 7u) << 61;
  return d;
}

// TMEM allocation size: the smallest power of two >= n columns, at least 32.
inline unsigned int pow2_cols(int n) {
  unsigned int c = 32;
  while ((int)c < n) c <<= 1;
  return c;
}

}  // namespace
}  // namespace gconv
