// Importance-mass exposure probe (sm_100a): how much of each query row's
// high-importance attention mass falls on INT8-routed key tiles.
//
// "Precision Has a Map: TileMix Routes INT8 Inside Dense Attention"
// (cognaptus.com, last section) and the agihunt.info summary of "TileMix:
// Tile-Centric Mixed-Precision Attention for LLM Inference Acceleration"
// (results paragraph) report that static SpTrans routing at 25% INT8 coverage
// sends only about 8.5% of the selected high-importance attention mass to
// INT8.  The selection is not given; this library's reading: under the
// full-precision probabilities P_ij of row i (fp16 inputs, fp32 scores), the
// high-importance keys are those with P_ij >= 2^-delta max_j P_ij.  Per row the
// probe writes
//   m8 = sum of P_ij over INT8-routed legal keys,
//   h  = sum of P_ij over the high-importance keys,
//   h8 = sum of P_ij over the high-importance INT8-routed keys.
//
// mass_probe_kernel: one CTA (4 warps) per (64-row query block, query head);
// warp w takes rows 16w..16w+15.  Key tiles (64 x d, fp16) stream through a
// two-stage cp.async ring into 128-byte XOR-swizzled shared memory; scores
// are m16n8k16 products (the query rows as A fragments in registers).  Two
// sweeps over the row block's legal key tiles: the row maxima, then the three
// sums against the final maxima.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tilemix.h"
#include "tilemix_internal.h"
#include "tilemix_mma.cuh"

namespace tilemix {
namespace {

constexpr int kMassThreads = 128;
constexpr int kMassRows = 64;  // query rows per CTA (16 per warp)

__device__ __forceinline__ int find_block_seq(const int32_t* cu, int nseq, int x) {
  int lo = 0, hi = nseq - 1;  // the s with cu[s] <= x < cu[s + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_addr(dst)), "l"(src)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(kMassThreads) mass_probe_kernel(MassParams p) {
  constexpr int kKs = D / 16;                 // k-steps of a score product
  constexpr int kTileBytes = 64 * D * 2;      // one fp16 key tile
  __shared__ __align__(1024) uint8_t ring[2][kTileBytes];
  const int blk = blockIdx.x, h = blockIdx.y;
  const int s = find_block_seq(p.cu_ktiles, p.nseq, blk);  // 64-row blocks = key-tile grid
  const int L = __ldg(p.cu_seqlens + s + 1) - __ldg(p.cu_seqlens + s);
  const int start = __ldg(p.cu_seqlens + s);
  const int i0 = (blk - __ldg(p.cu_ktiles + s)) * kMassRows;
  const int kv = p.kv_head_of_q ? __ldg(p.kv_head_of_q + h) : h / (p.hq / p.hk);
  if (kv < 0 || kv >= p.hk) return;  // a head map entry out of range: the head is skipped
  const uint64_t word =
      __ldg(p.masks + static_cast<size_t>(__ldg(p.cu_qtiles + s) + i0 / TILEMIX_BLOCK_M) * p.hk + kv);
  const int gs = __ldg(p.g + s);
  const int last = p.causal ? (min(i0 + kMassRows, L) - 1) / 64 : (L - 1) / 64;
  const int nt = last + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const int r0 = i0 + 16 * warp + g, r1 = r0 + 8;  // this thread's two rows

  // query rows as A fragments (zero past the sequence)
  const __half* q = static_cast<const __half*>(p.q);
  uint32_t qa[kKs][4];
#pragma unroll
  for (int ks = 0; ks < kKs; ++ks) {
    const int c = 16 * ks + 2 * q4;
    const size_t b0 = (static_cast<size_t>(start + r0) * p.hq + h) * D;
    const size_t b1 = (static_cast<size_t>(start + r1) * p.hq + h) * D;
    qa[ks][0] = r0 < L ? __ldg(reinterpret_cast<const uint32_t*>(q + b0 + c)) : 0u;
    qa[ks][1] = r1 < L ? __ldg(reinterpret_cast<const uint32_t*>(q + b1 + c)) : 0u;
    qa[ks][2] = r0 < L ? __ldg(reinterpret_cast<const uint32_t*>(q + b0 + c + 8)) : 0u;
    qa[ks][3] = r1 < L ? __ldg(reinterpret_cast<const uint32_t*>(q + b1 + c + 8)) : 0u;
  }

  // key tile `it` of the sweep (tiles 0..nt-1 twice) into ring slot it % 2
  const __half* kbase = static_cast<const __half*>(p.k);
  auto load_tile = [&](int it) {
    if (it < 2 * nt) {
      const int kt = it % nt;
      const int jn = min(64, L - kt * 64);
      uint8_t* st = ring[it & 1];
      for (int x = tid; x < jn * (D / 8); x += kMassThreads) {
        const int r = x / (D / 8), c = x % (D / 8);
        cp16(st + dec::k16_off<D>(r, c),
             kbase + (static_cast<size_t>(start + kt * 64 + r) * p.hk + kv) * D + c * 8);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float mx0 = -INFINITY, mx1 = -INFINITY;             // row maxima (log2 units)
  float l0 = 0.f, l1 = 0.f, e0 = 0.f, e1 = 0.f;      // all legal / INT8 legal
  float h0 = 0.f, h1 = 0.f, f0 = 0.f, f1 = 0.f;      // high-importance / and INT8
  const int mi = lane >> 3, mr = lane & 7;
  load_tile(0);
  for (int it = 0; it < 2 * nt; ++it) {
    load_tile(it + 1);
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const int kt = it % nt;
    const bool second = it >= nt;
    const bool is_int = (word >> (kt / gs)) & 1ull;
    const uint8_t* K = ring[it & 1];
    if (second && kt == 0) {
      // the maxima are final: reduce them over the four lanes of each row
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    }
#pragma unroll
    for (int n8 = 0; n8 < 8; ++n8) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < kKs / 2; ++q) {
        uint32_t b[4];  // keys 8 n8 .. 8 n8 + 7, channel chunks 4q .. 4q + 3
        dec::ldsm4(b, K + dec::k16_off<D>(8 * n8 + mr, 4 * q + mi));
        dec::mma_f16(acc, qa[2 * q], b[0], b[1]);
        dec::mma_f16(acc, qa[2 * q + 1], b[2], b[3]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = e < 2 ? r0 : r1;
        const int j = kt * 64 + 8 * n8 + 2 * q4 + (e & 1);
        const bool legal = row < L && j < L && (!p.causal || j <= row);
        const float t = legal ? acc[e] * p.scale_log2 : -INFINITY;
        if (!second) {
          if (e < 2) mx0 = fmaxf(mx0, t);
          else mx1 = fmaxf(mx1, t);
        } else if (legal) {
          const float m = e < 2 ? mx0 : mx1;
          const float pe = exp2f(t - m);
          const bool hi = t >= m - p.delta_log2;
          if (e < 2) {
            l0 += pe;
            if (is_int) e0 += pe;
            if (hi) h0 += pe;
            if (hi && is_int) f0 += pe;
          } else {
            l1 += pe;
            if (is_int) e1 += pe;
            if (hi) h1 += pe;
            if (hi && is_int) f1 += pe;
          }
        }
      }
    }
    __syncthreads();  // the slot is free for the copy issued next iteration
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    e0 += __shfl_xor_sync(0xffffffffu, e0, off);
    e1 += __shfl_xor_sync(0xffffffffu, e1, off);
    h0 += __shfl_xor_sync(0xffffffffu, h0, off);
    h1 += __shfl_xor_sync(0xffffffffu, h1, off);
    f0 += __shfl_xor_sync(0xffffffffu, f0, off);
    f1 += __shfl_xor_sync(0xffffffffu, f1, off);
  }
  if (q4 == 0) {
    const size_t T = p.total_tokens;
    if (r0 < L) {
      const size_t o = static_cast<size_t>(h) * T + start + r0;
      p.m8[o] = e0 / l0;
      p.h[o] = h0 / l0;
      p.h8[o] = f0 / l0;
    }
    if (r1 < L) {
      const size_t o = static_cast<size_t>(h) * T + start + r1;
      p.m8[o] = e1 / l1;
      p.h[o] = h1 / l1;
      p.h8[o] = f1 / l1;
    }
  }
}

}  // namespace

int launch_mass_probe(const MassParams& p, cudaStream_t stream) {
  if (p.total_blocks == 0) return static_cast<int>(cudaSuccess);
  const dim3 grid(p.total_blocks, p.hq);
  if (p.d == 128)
    mass_probe_kernel<128><<<grid, kMassThreads, 0, stream>>>(p);
  else
    mass_probe_kernel<64><<<grid, kMassThreads, 0, stream>>>(p);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace tilemix
