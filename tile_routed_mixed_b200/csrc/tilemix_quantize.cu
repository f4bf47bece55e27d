// Block quantisation of Q and K for the low-precision score path (sm_100a):
// per (head, block of one sequence) symmetric absmax codes, INT8 (/127) or
// FP8 e4m3 (/448).
//
// Method: "TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
// Acceleration" (agihunt.info summary, method paragraphs).
#include <cuda_fp8.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tilemix.h"
#include "tilemix_internal.h"
#include "tilemix_quant.cuh"

namespace tilemix {

// ===================================================================
// Block quantisation ("only Q and K are quantised, Q in 128 x d blocks and K
// in 64 x d blocks, symmetric absmax / 127").  One launch covers every Q block
// and every K block; one CTA per (block, head) stages its block in shared
// memory (at most eight 16-byte chunks per thread at d = 128, four at d = 64),
// so HBM sees each fp16 element read once and each code written once.
// codes = clamp(rne(x / s), +-127) with s = a / 127, both divisions IEEE fp32.
// ===================================================================
constexpr int kQuantThreads = 256;

// One tensor's blocks: tiles tile0 .. tile0 + ntiles - 1 (cu_tiles holds the
// sequences' first tiles, cu_tiles[0] <= tile0), scales [heads][total_tiles].
struct QuantSide {
  const __half* x;
  const int32_t* cu_tiles;
  int8_t* codes;
  float* scales;
  int tile0, ntiles, total_tiles, heads, block_rows;
};

// fmt selects the codes: 0 INT8 (s = a / 127), 2 INT4 (s = a / 7, codes in
// [-7, 7], one per byte; the same rounding, whose no-clamp argument holds with
// 7 for 127: |x / s| < 7.0001), 1 the FP8 low path's e4m3(x / s) with
// s = a / 448 (round to nearest even, saturating; IEEE fp32 division for
// both).
// Thread t takes the 16-byte chunks of rows t / C + j 256 / C (C chunks per
// row), column t mod C, for j < kChunks.
template <int D>
__global__ void __launch_bounds__(kQuantThreads, 5)
    quantize_qk_kernel(QuantSide qs, QuantSide ks, const int32_t* __restrict__ cu_seqlens,
                       int nseq, int* ticket, int fmt) {
  const bool fp8 = fmt == 1;
  constexpr int kCprLog2 = D == 128 ? 4 : 3;                 // 16-byte chunks per row
  constexpr int kRowsPerPass = kQuantThreads >> kCprLog2;    // rows one pass covers
  constexpr int kChunks = TILEMIX_BLOCK_M / kRowsPerPass;    // passes over a Q block
  if (ticket && blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0;
  const int nq = qs.ntiles * qs.heads;
  const bool is_q = static_cast<int>(blockIdx.x) < nq;
  // field-wise selection keeps both parameter structs in the constant bank
  const __half* x = is_q ? qs.x : ks.x;
  const int32_t* cu_tiles = is_q ? qs.cu_tiles : ks.cu_tiles;
  int8_t* codes = is_q ? qs.codes : ks.codes;
  float* scales = is_q ? qs.scales : ks.scales;
  const int total_tiles = is_q ? qs.total_tiles : ks.total_tiles;
  const int heads = is_q ? qs.heads : ks.heads;
  const int block_rows = is_q ? qs.block_rows : ks.block_rows;
  const int b = is_q ? blockIdx.x : blockIdx.x - nq;
  const int rel = b / heads;
  const int h = b - rel * heads;
  const int tile = (is_q ? qs.tile0 : ks.tile0) + rel;
  // owning sequence: last s with cu_tiles[s] <= tile
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu_tiles + mid) <= tile) lo = mid; else hi = mid - 1;
  }
  const int t0 = __ldg(cu_seqlens + lo);
  const int L = __ldg(cu_seqlens + lo + 1) - t0;
  const int r0 = (tile - __ldg(cu_tiles + lo)) * block_rows;
  const int rows = min(block_rows, L - r0);
  const size_t base = (static_cast<size_t>(t0 + r0) * heads + h) * D;
  // offsets inside the block fit 32 bits: rows x heads x d <= 128 x 256 x 128
  const int row_stride = heads * D;
  const int row0 = threadIdx.x >> kCprLog2;
  const int off0 = row0 * row_stride + ((threadIdx.x & ((1 << kCprLog2) - 1)) << 3);
  const int step = kRowsPerPass * row_stride;
  const __half* xb = x + base;
  int8_t* cb = codes + base;

  // The block's chunks go to shared memory with 16-byte asynchronous copies
  // (rows past the block's end are zero-filled): fewer registers per thread
  // than holding them, so five CTAs per SM at d = 128 instead of four, and
  // more bytes in flight.  Each thread reads back only its own chunks, after
  // its own copies have landed.
  __shared__ uint4 stage[kChunks * kQuantThreads];
  const uint32_t st0 = static_cast<uint32_t>(__cvta_generic_to_shared(stage + threadIdx.x));
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const bool valid = row0 + i * kRowsPerPass < rows;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(st0 + i * kQuantThreads * 16),
                 "l"(valid ? xb + off0 + i * step : xb), "r"(valid ? 16 : 0)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  const uint4* u = stage + threadIdx.x;  // chunk i at u[i * kQuantThreads]
  __half2 amax2 = __float2half2_rn(0.f);
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const uint4 c = u[i * kQuantThreads];
    const __half2* hv = reinterpret_cast<const __half2*>(&c);
#pragma unroll
    for (int k = 0; k < 4; ++k) amax2 = __hmax2(amax2, __habs2(hv[k]));
  }
  float amax = fmaxf(__low2float(amax2), __high2float(amax2));
  __shared__ float red[kQuantThreads / 32];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  float a = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) a = fmaxf(a, red[w]);
  const float s = __fdiv_rn(a, fp8 ? 448.0f : fmt == 2 ? 7.0f : 127.0f);
  if (threadIdx.x == 0) scales[static_cast<size_t>(h) * total_tiles + tile] = s;
  const float r = a > 0.f ? __frcp_rn(s) : 0.f;
  if (fp8) {
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      if (row0 + i * kRowsPerPass < rows) {
        uint32_t w[2] = {0u, 0u};
        if (a > 0.f) {
          const uint4 c = u[i * kQuantThreads];
          const __half* hv = reinterpret_cast<const __half*>(&c);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t b8 = __nv_cvt_float_to_fp8(__fdiv_rn(__half2float(hv[e]), s),
                                                      __NV_SATFINITE, __NV_E4M3);
            w[e >> 2] |= b8 << (8 * (e & 3));
          }
        }
        *reinterpret_cast<uint2*>(cb + off0 + i * step) = make_uint2(w[0], w[1]);
      }
    }
    return;
  }

#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    if (row0 + i * kRowsPerPass < rows) {
      const uint2 packed = a > 0.f ? quant_chunk(u[i * kQuantThreads], s, r) : make_uint2(0u, 0u);
      *reinterpret_cast<uint2*>(cb + off0 + i * step) = packed;
    }
  }
}

int launch_quantize_qk(const void* q, const void* k, const int32_t* cu_seqlens,
                       const int32_t* cu_qtiles, const int32_t* cu_ktiles, int nseq,
                       const QuantRange& range, int total_qtiles, int total_ktiles, int hq,
                       int hk, int d, int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                       int* ticket, int fmt, cudaStream_t stream) {
  QuantSide qs{static_cast<const __half*>(q), cu_qtiles, q8, q_scale, range.qtile0,
               q ? range.nqtiles : 0, total_qtiles, hq, TILEMIX_BLOCK_M};
  QuantSide ks{static_cast<const __half*>(k), cu_ktiles, k8, k_scale, range.ktile0,
               k ? range.nktiles : 0, total_ktiles, hk, TILEMIX_BLOCK_N};
  const long long blocks = static_cast<long long>(qs.ntiles) * hq +
                           static_cast<long long>(ks.ntiles) * hk;
  if (blocks == 0)
    return ticket ? static_cast<int>(cudaMemsetAsync(ticket, 0, sizeof(int), stream)) : cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (d == 128)
    quantize_qk_kernel<128><<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
        qs, ks, cu_seqlens, nseq, ticket, fmt);
  else
    quantize_qk_kernel<64><<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
        qs, ks, cu_seqlens, nseq, ticket, fmt);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace tilemix
