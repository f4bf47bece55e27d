// Warp-level tile helpers shared by the decode step and the importance-mass
// probe (sm_100a): offsets into 128-byte (and 64-byte) XOR-swizzled tiles of
// 64 rows, ldmatrix loads, and m16n8 matrix products with register operands.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "tilemix_ptx.cuh"

namespace tilemix {
namespace dec {

constexpr int kTileRows = 64;  // rows of the tiles these offsets address

// Byte offset of 16-byte chunk c of row r in a tile written by a TMA load
// with 128-byte swizzle (128-byte rows) or 64-byte swizzle (64-byte rows):
// the chunk index is XORed with the row's bits at byte-address bits 7..9
// (respectively 7..8).
__device__ __forceinline__ int sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }
__device__ __forceinline__ int sw64(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

// fp16 row of D channels as boxes of 64: logical 16-byte chunk lc of row r.
template <int D>
__device__ __forceinline__ int k16_off(int r, int lc) {
  return (lc >> 3) * (kTileRows * 128) + sw128(r, lc & 7);
}
// INT8 row of D codes (one box of D bytes): chunk lc of row r.
template <int D>
__device__ __forceinline__ int k8_off(int r, int lc) {
  return D == 128 ? sw128(r, lc) : sw64(r, lc);
}

// 8x8 matrices of 16-bit elements from shared memory: lanes 8m..8m+7 give
// the row addresses of matrix m; thread t receives row t / 4, elements
// 2 (t % 4) and 2 (t % 4) + 1 of each (transposed: those rows of column t / 4).
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(ptx::smem_addr(p)));
}
__device__ __forceinline__ void ldsm4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(ptx::smem_addr(p)));
}
__device__ __forceinline__ void ldsm2_t(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(ptx::smem_addr(p)));
}

// D[16x8] += A[16x16] * B[16x8], fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D[16x8] += A[16x32] * B[32x8], signed INT8 inputs, INT32 accumulate.
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return static_cast<uint32_t>(__half_as_ushort(lo)) |
         (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}

}  // namespace dec
}  // namespace tilemix
