// Content-aware (adaptive) routing: words written on the device through the
// same routing-word interface the static templates use (sm_100a).
//
// The pages say the mask interface can take adaptive, content-aware policies
// and evaluate none ("TileMix: Tile-Centric Mixed-Precision Attention for LLM
// Inference Acceleration", agihunt.info summary, limitations paragraph;
// "Precision Has a Map: TileMix Routes INT8 Inside Dense Attention",
// cognaptus.com, "Placement can matter more than the nominal percentage").
// The policy built here is the pooled-score one: for query-tile row r and KV
// head kv, each legal key tile is scored by qbar . kbar (the mean query of the
// row over the KV head's query heads, the mean key of the tile), a group by
// its highest tile, and the row's quota of lowest-scoring groups goes to INT8
// (ties: the lower group).  The quota is the static templates' proportional
// rule.  Both means and the dot are fp32 in a fixed order (8 interleaved
// partial sums added in order; products and sums rounded separately), so the
// words are reproducible bit for bit.
//
//   route_pool_kernel   one CTA per (tile, KV head): 8 x d/8 threads, thread
//                       (j, c8) sums channels 8 c8.. of the items m = j mod 8
//   route_words_kernel  one warp per (query-tile row, KV head)
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tilemix.h"
#include "tilemix_internal.h"

namespace tilemix {
namespace {

constexpr int kRouteLanes = 8;  // interleaved partial sums of a mean

__device__ __forceinline__ int find_seq(const int32_t* cu, int nseq, int x) {
  int lo = 0, hi = nseq - 1;  // the s with cu[s] <= x < cu[s + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// blockIdx.x: tile (query tiles if kQ, else key tiles), blockIdx.y: KV head.
// Thread (j, c8): channels [8 c8, 8 c8 + 8) of the items m = j mod 8, read as
// one 16-byte load per item.
template <int D, bool kQ>
__global__ void __launch_bounds__(kRouteLanes * D / 8) route_pool_kernel(RouteParams p) {
  constexpr int kC8 = D / 8;  // 16-byte channel chunks per row
  __shared__ float part[kRouteLanes][D];
  __shared__ int heads[256];
  __shared__ int nheads;
  const int tile = blockIdx.x, kv = blockIdx.y;
  const int c8 = threadIdx.x % kC8, j = threadIdx.x / kC8;
  const int32_t* cu_tiles = kQ ? p.cu_qtiles : p.cu_ktiles;
  const int s = find_seq(cu_tiles, p.nseq, tile);
  const int L = __ldg(p.cu_seqlens + s + 1) - __ldg(p.cu_seqlens + s);
  const int bm = kQ ? TILEMIX_BLOCK_M : TILEMIX_BLOCK_N;
  const int t0 = (tile - __ldg(cu_tiles + s)) * bm;
  const int R = min(bm, L - t0);  // valid rows of the tile
  const int row0 = __ldg(p.cu_seqlens + s) + t0;
  int H = 1;
  if (kQ) {
    if (threadIdx.x == 0) {
      int n = 0;
      for (int h = 0; h < p.hq; ++h)
        if ((p.kv_head_of_q ? __ldg(p.kv_head_of_q + h) : h / (p.hq / p.hk)) == kv && n < 256)
          heads[n++] = h;
      nheads = n;
    }
    __syncthreads();
    H = nheads;
  }
  // items m = head index * R + row (head-major); this thread takes m = j mod 8,
  // i.e. in head hi the rows i = j - hi R (mod 8), ascending: the order of m
  const __half* x = static_cast<const __half*>(kQ ? p.q : p.k);
  const int nh = kQ ? p.hq : p.hk;
  const size_t step = static_cast<size_t>(kRouteLanes) * nh * D;  // elements between items
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  auto add8 = [&](const uint4& u) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h2[e]);
      acc[2 * e] = __fadd_rn(acc[2 * e], f.x);
      acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], f.y);
    }
  };
  for (int hi = 0; hi < H; ++hi) {
    const int h = kQ ? heads[hi] : kv;
    int i = (j - hi * R) % kRouteLanes;
    if (i < 0) i += kRouteLanes;
    const __half* ptr = x + (static_cast<size_t>(row0 + i) * nh + h) * D + 8 * c8;
    // loads issued four ahead; the adds stay in ascending row order
    for (; i + 3 * kRouteLanes < R; i += 4 * kRouteLanes, ptr += 4 * step) {
      const uint4 u0 = __ldg(reinterpret_cast<const uint4*>(ptr));
      const uint4 u1 = __ldg(reinterpret_cast<const uint4*>(ptr + step));
      const uint4 u2 = __ldg(reinterpret_cast<const uint4*>(ptr + 2 * step));
      const uint4 u3 = __ldg(reinterpret_cast<const uint4*>(ptr + 3 * step));
      add8(u0);
      add8(u1);
      add8(u2);
      add8(u3);
    }
    for (; i < R; i += kRouteLanes, ptr += step) add8(__ldg(reinterpret_cast<const uint4*>(ptr)));
  }
  const int M = H * R;
#pragma unroll
  for (int e = 0; e < 8; ++e) part[j][8 * c8 + e] = acc[e];
  __syncthreads();
  float* out = kQ ? p.qbar : p.kbar;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float tot = part[0][c];
#pragma unroll
    for (int q = 1; q < kRouteLanes; ++q) tot = __fadd_rn(tot, part[q][c]);
    if (M > 0) tot = __fdiv_rn(tot, static_cast<float>(M));
    out[(static_cast<size_t>(tile) * p.hk + kv) * D + c] = tot;
  }
}

__device__ __forceinline__ int last_tile(int qt, int L, int causal) {
  return causal ? min((qt + 1) * TILEMIX_BLOCK_M - 1, L - 1) / TILEMIX_BLOCK_N
                : (L - 1) / TILEMIX_BLOCK_N;
}

template <int D>
__global__ void __launch_bounds__(128) route_words_kernel(RouteParams p) {
  const int warp_global = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (warp_global >= p.total_qtiles * p.hk) return;
  const int r = warp_global / p.hk, kv = warp_global - r * p.hk;
  const int s = find_seq(p.cu_qtiles, p.nseq, r);
  const int L = __ldg(p.cu_seqlens + s + 1) - __ldg(p.cu_seqlens + s);
  const int cq = __ldg(p.cu_qtiles + s), ck = __ldg(p.cu_ktiles + s);
  const int Tm = __ldg(p.cu_qtiles + s + 1) - cq;
  const int qt = r - cq, gs = __ldg(p.g + s), pc = p.int8_percent;
  const int lt = last_tile(qt, L, p.causal);
  const int n = lt / gs + 1;

  // this row's quota: floor(p n / 100) plus one if it is among the rows with
  // the largest remainders (ties to the lower row) that share the leftover
  int sum_n = 0, sum_fl = 0, ahead = 0;
  const int rem_r = pc * n % 100;
  for (int x = lane; x < Tm; x += 32) {
    const int nx = last_tile(x, L, p.causal) / gs + 1;
    const int rem = pc * nx % 100;
    sum_n += nx;
    sum_fl += pc * nx / 100;
    ahead += rem > rem_r || (rem == rem_r && x < qt);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sum_n += __shfl_xor_sync(0xffffffffu, sum_n, off);
    sum_fl += __shfl_xor_sync(0xffffffffu, sum_fl, off);
    ahead += __shfl_xor_sync(0xffffffffu, ahead, off);
  }
  const int left = static_cast<int>((static_cast<long long>(pc) * sum_n + 50) / 100) - sum_fl;
  const int quota = pc * n / 100 + (ahead < left ? 1 : 0);

  // group scores: lane takes groups lane and lane + 32
  const float* qb = p.qbar + (static_cast<size_t>(r) * p.hk + kv) * D;
  float sc[2] = {0.f, 0.f};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int b = lane + 32 * h;
    if (b >= n) continue;
    float best = -INFINITY;
    for (int kt = b * gs; kt < min((b + 1) * gs, lt + 1); ++kt) {
      const float* kb = p.kbar + (static_cast<size_t>(ck + kt) * p.hk + kv) * D;
      float dot = 0.f;
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(qb + c));
        const float4 b4 = __ldg(reinterpret_cast<const float4*>(kb + c));
        dot = __fadd_rn(dot, __fmul_rn(a.x, b4.x));
        dot = __fadd_rn(dot, __fmul_rn(a.y, b4.y));
        dot = __fadd_rn(dot, __fmul_rn(a.z, b4.z));
        dot = __fadd_rn(dot, __fmul_rn(a.w, b4.w));
      }
      best = fmaxf(best, dot);
    }
    sc[h] = best;
  }
  // rank of each of the lane's groups among the row's groups
  int rank[2] = {0, 0};
  for (int b2 = 0; b2 < n; ++b2) {
    const float v = __shfl_sync(0xffffffffu, b2 < 32 ? sc[0] : sc[1], b2 & 31);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int b = lane + 32 * h;
      rank[h] += v < sc[h] || (v == sc[h] && b2 < b);
    }
  }
  const unsigned lo = __ballot_sync(0xffffffffu, lane < n && rank[0] < quota);
  const unsigned hi = __ballot_sync(0xffffffffu, lane + 32 < n && rank[1] < quota);
  if (lane == 0)
    p.masks[static_cast<size_t>(r) * p.hk + kv] =
        static_cast<uint64_t>(lo) | (static_cast<uint64_t>(hi) << 32);
}

template <int D>
cudaError_t launch_route_d(const RouteParams& p, cudaStream_t stream) {
  if (p.total_qtiles > 0)
    route_pool_kernel<D, true>
        <<<dim3(p.total_qtiles, p.hk), kRouteLanes * D / 8, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.total_ktiles > 0)
    route_pool_kernel<D, false>
        <<<dim3(p.total_ktiles, p.hk), kRouteLanes * D / 8, 0, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long warps = static_cast<long long>(p.total_qtiles) * p.hk;
  if (warps > 0)
    route_words_kernel<D><<<static_cast<unsigned>((warps + 3) / 4), 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

int launch_route(const RouteParams& p, cudaStream_t stream) {
  return static_cast<int>(p.d == 128 ? launch_route_d<128>(p, stream)
                                     : launch_route_d<64>(p, stream));
}

}  // namespace tilemix
