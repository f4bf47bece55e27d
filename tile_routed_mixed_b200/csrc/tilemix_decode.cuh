// The decode step with the INT8 K cache (sm_100a): one kernel launch.
//
// Decode is the step after prefill that "TileMix: Tile-Centric Mixed-
// Precision Attention for LLM Inference Acceleration" (agihunt.info summary)
// and "Precision Has a Map: TileMix Routes INT8 Inside Dense Attention"
// (cognaptus.com, last section) name: the INT8 K codes and block scales of the
// quantisation pre-pass become the K cache, and a new token's query reads the
// routing word of its query-tile row.
//
// One CTA (eight warps) per (sequence, KV head, split of the key range):
//   - quantises the KV head's new query rows (one block per row, the same
//     symmetric absmax / 127 as the prefill pre-pass) and keeps them, fp16
//     and INT8, as the A operands of the score products in registers;
//   - streams the split's key tiles through a three-stage shared-memory ring
//     with TMA tile loads (K in the tile's routed precision, V in fp16, both
//     swizzled), so HBM sees only the bytes the routing asks for;
//   - on the sequence's last tile (the one holding the new key), re-quantises
//     the block over its valid rows, writes the codes and scale back to the
//     cache and, if the tile is INT8-routed, scores it with those codes;
//   - per tile, warp w scores keys [8w, 8w + 8) of every query row with one
//     m16n8 product chain (fp16 x fp16 -> fp32, or INT8 x INT8 -> INT32; the
//     16 rows are the group's query heads, zero-padded), the CTA takes the
//     online softmax with P rounded to fp16, and warp w accumulates channels
//     [16w, 16w + 16) (d = 128; [8w, 8w + 8) for d = 64) of O = P.V in fp32
//     registers;
//   - writes its partial softmax state; the CTA that finishes a (sequence, KV
//     head) last merges every split's state into O.
// The step reads every cached key once and is bound by HBM.  Its two products
// per tile are a few hundred multiply-adds per key; as scalar FMAs they left
// the SMs issue-bound below the HBM rate, so they run as warp-level matrix
// products on the tiles already in shared memory.
// Included by tilemix_kernels.cu (one translation unit: the kernels share the
// device status word and the bounded waits).
#pragma once

#include "tilemix_mma.cuh"

namespace tilemix {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeKeys = TILEMIX_BLOCK_N;  // keys per routed tile
constexpr int kMaxGroup = 16;                 // query heads per KV head (the m16 rows)
constexpr int kDecodeStages = 3;
constexpr int kScalePrefetch = 64;            // K block scales staged per CTA

// Shared-memory layout of the decode kernel (offsets from a 1024-byte aligned
// base).  Each ring stage holds a K tile (64 rows: fp16 as blocks of 64
// channels with 128-byte rows, or INT8 codes with rows of d bytes) and a V
// tile (fp16, like K), as the TMA loads write them: 16-byte chunks XOR-
// swizzled by row.  k8 holds the re-quantised last block (INT8 layout); the
// query rows use the same bytes before the first tile.  P is [16][64] fp16
// with 128-byte swizzled rows.
struct DecodeSmem {
  int kbytes, stage, k8, qh, q8, pt, red_m, red_l, small, bars, total;
};

__host__ __device__ inline DecodeSmem decode_smem(int d) {
  DecodeSmem L{};
  L.kbytes = kDecodeKeys * 2 * d;
  L.stage = 2 * L.kbytes;
  int off = kDecodeStages * L.stage;
  L.k8 = off;
  L.qh = off;                      // [16][d] fp16, setup only
  L.q8 = off + kMaxGroup * d * 2;  // [16][d] INT8, setup only
  off += kDecodeKeys * d;          // >= the query rows' 48 d bytes
  L.pt = off;
  off += kMaxGroup * kDecodeKeys * 2;
  L.red_m = off;
  off += kMaxGroup * 8 * 4;
  L.red_l = off;
  off += kMaxGroup * 8 * 4;
  L.small = off;
  off += (kMaxGroup + 8 + kScalePrefetch) * 4 + (kMaxGroup + 4) * 4;
  off = (off + 7) & ~7;
  L.bars = off;
  off += kDecodeStages * 8;
  L.total = ((off + 15) & ~15) + 1024;  // + alignment slack
  return L;
}

namespace dec {

// Device-scope atomic add with acquire-release semantics; returns the old value.
__device__ __forceinline__ int add_acq_rel(int* ptr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ float absmax8(const uint4& u, float a) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
  __half2 m = __habs2(h[0]);
  m = __hmax2(m, __habs2(h[1]));
  m = __hmax2(m, __habs2(h[2]));
  m = __hmax2(m, __habs2(h[3]));
  return fmaxf(a, fmaxf(__low2float(m), __high2float(m)));
}

// Maximum and sum of eight consecutive floats (32-byte aligned), in warp order.
__device__ __forceinline__ float max8(const float* x) {
  const float4 a = *reinterpret_cast<const float4*>(x), b = *reinterpret_cast<const float4*>(x + 4);
  return fmaxf(fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)), fmaxf(fmaxf(b.x, b.y), fmaxf(b.z, b.w)));
}
__device__ __forceinline__ float sum8(const float* x) {
  const float4 a = *reinterpret_cast<const float4*>(x), b = *reinterpret_cast<const float4*>(x + 4);
  return ((((((a.x + a.y) + a.z) + a.w) + b.x) + b.y) + b.z) + b.w;
}


}  // namespace dec

template <int D>
__global__ void __launch_bounds__(kDecodeThreads, 2)
    decode_attn_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int kKs16 = D / 16;  // k-steps of the fp16 score product
  constexpr int kKs8 = D / 32;   // k-steps of the INT8 score product
  constexpr int kNt = D / 64;    // n8 tiles of O per warp
  extern __shared__ __align__(128) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const DecodeSmem L = decode_smem(D);
  uint8_t* k8last = dsm + L.k8;                            // [64][D] re-quantised block
  uint8_t* qh = dsm + L.qh;                                // [16][D] fp16 query rows
  uint8_t* q8s = dsm + L.q8;                               // [16][D] their codes
  uint8_t* pt = dsm + L.pt;                                // [16][64] fp16 P
  float* red_m = reinterpret_cast<float*>(dsm + L.red_m);  // [16][8] per-warp row maxima
  float* red_l = reinterpret_cast<float*>(dsm + L.red_l);  // [16][8] per-warp row sums
  float* qsc = reinterpret_cast<float*>(dsm + L.small);    // [16]
  float* red = qsc + kMaxGroup;                            // [8]
  float* ksc_s = red + 8;                                  // [64] the split's K block scales
  int* heads = reinterpret_cast<int*>(ksc_s + kScalePrefetch);  // [16]
  int* flags = heads + kMaxGroup;  // [0] heads in the group, [1] abort, [2] merger
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + L.bars);

  int bid = blockIdx.x;
  const int split = bid % p.nsplit;
  bid /= p.nsplit;
  const int kv = bid % p.hk;
  const int s = bid / p.hk;
  const int len = __ldg(p.seq_len + s);
  const int t = len - 1;  // position of the new token
  const int ntiles = t / kDecodeKeys + 1;
  const int kt0 = split * p.tiles_per_split;
  if (len < 1 || kt0 >= ntiles) return;  // an empty split: nothing to merge either
  const int n = min(ntiles, kt0 + p.tiles_per_split) - kt0;
  const int nsplit_s = (ntiles + p.tiles_per_split - 1) / p.tiles_per_split;
  const int row0 = __ldg(p.seq_start + s);
  const int gs = __ldg(p.g + s);
  const int ktile0 = __ldg(p.ktile_start + s);
  const uint64_t word =
      __ldg(p.masks + static_cast<size_t>(__ldg(p.qtile_start + s) + t / TILEMIX_BLOCK_M) * p.hk + kv);
  const bool bad = gs < 1 || (ntiles - 1) / gs > 63;  // no division below when bad
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q4 = lane & 3;  // m16n8 fragment: row g (and g + 8), column pair q4

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kDecodeStages; ++i) ptx::mbar_init(&full[i], 1);
    ptx::fence_mbar_init();
    flags[1] = 0;
    ptx::prefetch_tensormap(&p.tm_k);
    ptx::prefetch_tensormap(&p.tm_k8);
    ptx::prefetch_tensormap(&p.tm_v);
  }
  __syncthreads();

  // Tile kt0 + i into ring slot i % stages (one thread).
  auto issue = [&](int i) {
    const int kt = kt0 + i;
    uint8_t* st = dsm + (i % kDecodeStages) * L.stage;
    uint64_t* bar = &full[i % kDecodeStages];
    const bool k8 = kt != ntiles - 1 && ((word >> (kt / gs)) & 1ull);
    const int r = row0 + kt * kDecodeKeys;
    ptx::mbar_expect_tx(bar, static_cast<uint32_t>(kDecodeKeys * (k8 ? D : 2 * D) + L.kbytes));
    if (k8) {
      ptx::tma_load_3d(st, &p.tm_k8, bar, 0, kv, r);
    } else {
#pragma unroll
      for (int b = 0; b < D / 64; ++b)
        ptx::tma_load_3d(st + b * kDecodeKeys * 128, &p.tm_k, bar, 64 * b, kv, r);
    }
#pragma unroll
    for (int b = 0; b < D / 64; ++b)
      ptx::tma_load_3d(st + L.kbytes + b * kDecodeKeys * 128, &p.tm_v, bar, 64 * b, kv, r);
  };
  if (!bad && tid == 0)
    for (int i = 0; i < min(kDecodeStages, n); ++i) issue(i);
  // the split's K block scales, fetched once (a dependent load per tile would
  // put a full memory round trip on every tile's critical path)
  for (int x = tid; x < min(n, kScalePrefetch); x += kDecodeThreads)
    ksc_s[x] = __ldg(p.k_scale + static_cast<size_t>(kv) * p.total_ktiles + ktile0 + kt0 + x);

  if (tid == 0) {
    int cnt = 0;
    for (int h = 0; h < p.hq; ++h)
      if ((p.kv_head_of_q ? __ldg(p.kv_head_of_q + h) : h / p.group) == kv) {
        if (cnt < kMaxGroup) heads[cnt] = h;
        ++cnt;
      }
    // more query heads than the 16 rows of the products (a custom head map):
    // reported, and only the first 16 are computed
    if (cnt > kMaxGroup) atomicOr(&g_status, kStatusBadGroups);
    flags[0] = min(cnt, kMaxGroup);
    if (bad) atomicOr(&g_status, kStatusBadGroups);
  }
  __syncthreads();
  const int G = flags[0];

  // New query rows: warp per row; lane c holds channels [8c, 8c + 8).  Rows
  // G..15 are zero (their scores are zero and never leave the CTA).
  for (int gi = warp; gi < kMaxGroup; gi += kDecodeThreads / 32) {
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (gi < G && lane < D / 8)
      u = *reinterpret_cast<const uint4*>(static_cast<const __half*>(p.q) +
                                          (static_cast<size_t>(s) * p.hq + heads[gi]) * D +
                                          lane * 8);
    float a = dec::absmax8(u, 0.f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    const float sc = __fdiv_rn(a, 127.0f);
    const float rc = a > 0.f ? __frcp_rn(sc) : 0.f;
    if (lane < D / 8) {
      *reinterpret_cast<uint4*>(qh + (gi * D + lane * 8) * 2) = u;
      *reinterpret_cast<uint2*>(q8s + gi * D + lane * 8) =
          a > 0.f ? quant_chunk(u, sc, rc) : make_uint2(0u, 0u);
    }
    if (lane == 0) qsc[gi] = gi < G ? sc : 0.f;
  }
  __syncthreads();
  // A operands of the score products (rows g and g + 8), per k-step
  uint32_t qa[kKs16][4], q8a[kKs8][4];
#pragma unroll
  for (int ks = 0; ks < kKs16; ++ks) {
    const int c = 16 * ks + 2 * q4;
    qa[ks][0] = *reinterpret_cast<const uint32_t*>(qh + (g * D + c) * 2);
    qa[ks][1] = *reinterpret_cast<const uint32_t*>(qh + ((g + 8) * D + c) * 2);
    qa[ks][2] = *reinterpret_cast<const uint32_t*>(qh + (g * D + c + 8) * 2);
    qa[ks][3] = *reinterpret_cast<const uint32_t*>(qh + ((g + 8) * D + c + 8) * 2);
  }
#pragma unroll
  for (int ks = 0; ks < kKs8; ++ks) {
    const int c = 32 * ks + 4 * q4;
    q8a[ks][0] = *reinterpret_cast<const uint32_t*>(q8s + g * D + c);
    q8a[ks][1] = *reinterpret_cast<const uint32_t*>(q8s + (g + 8) * D + c);
    q8a[ks][2] = *reinterpret_cast<const uint32_t*>(q8s + g * D + c + 16);
    q8a[ks][3] = *reinterpret_cast<const uint32_t*>(q8s + (g + 8) * D + c + 16);
  }
  const float qs0 = qsc[g], qs1 = qsc[g + 8];
  __syncthreads();  // the query rows' bytes become the last block's codes

  // softmax state of rows g and g + 8 (the same in every thread)
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[kNt][4];
#pragma unroll
  for (int nt = 0; nt < kNt; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;

  // ldmatrix row addresses: lane gives row mr of matrix mi
  const int mi = lane >> 3, mr = lane & 7;
  const int key_s = 8 * warp + mr;  // score B operand: this warp's keys
  for (int i = 0; i < n && !bad; ++i) {
    const int kt = kt0 + i;
    const int jn = min(kDecodeKeys, len - kt * kDecodeKeys);
    const bool last = kt == ntiles - 1;
    const bool is_int = (word >> (kt / gs)) & 1ull;
    float ksc = 0.f;
    if (is_int && !last)
      ksc = i < kScalePrefetch
                ? ksc_s[i]
                : __ldg(p.k_scale + static_cast<size_t>(kv) * p.total_ktiles + ktile0 + kt);
    const bool ok = wait_bar(&full[i % kDecodeStages], (i / kDecodeStages) & 1, &flags[1],
                             p.timeout_ns);
    if (!__syncthreads_and(ok)) {
      // a copy never landed: leave without writing; wait (bounded) for the
      // copies still in flight into the ring before the CTA exits
      if (tid == 0)
        for (int r = i; r < min(n, i + kDecodeStages); ++r)
          drain_bar(&full[r % kDecodeStages], (r / kDecodeStages) & 1, p.timeout_ns);
      return;
    }
    const uint8_t* K = dsm + (i % kDecodeStages) * L.stage;
    const uint8_t* V = K + L.kbytes;
    const uint8_t* K8 = K;
    if (last) {
      // the block holding the new key: absmax over its valid rows, then its
      // codes into the cache and into k8last
      float a = 0.f;
      for (int c = tid; c < jn * (D / 8); c += kDecodeThreads)
        a = dec::absmax8(
            *reinterpret_cast<const uint4*>(K + dec::k16_off<D>(c / (D / 8), c % (D / 8))), a);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if (lane == 0) red[warp] = a;
      __syncthreads();
      a = fmaxf(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])),
                fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7])));
      ksc = __fdiv_rn(a, 127.0f);
      const float rc = a > 0.f ? __frcp_rn(ksc) : 0.f;
      if (tid == 0) p.k_scale[static_cast<size_t>(kv) * p.total_ktiles + ktile0 + kt] = ksc;
      int8_t* codes = p.k_i8 + (static_cast<size_t>(row0 + kt * kDecodeKeys) * p.hk + kv) * D;
      for (int c = tid; c < kDecodeKeys * (D / 8); c += kDecodeThreads) {
        const int r = c / (D / 8), lc = c % (D / 8);
        uint2 cw = make_uint2(0u, 0u);
        if (r < jn && a > 0.f)
          cw = quant_chunk(*reinterpret_cast<const uint4*>(K + dec::k16_off<D>(r, lc)), ksc, rc);
        if (r < jn)
          *reinterpret_cast<uint2*>(codes + static_cast<size_t>(r) * p.hk * D + lc * 8) = cw;
        *reinterpret_cast<uint2*>(k8last + dec::k8_off<D>(r, lc >> 1) + (lc & 1) * 8) = cw;
      }
      __syncthreads();
      K8 = k8last;
    }
    // scores of rows g / g + 8 at keys 8w + 2 q4 + {0, 1}
    float sv[4];
    if (is_int) {
      int acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < kKs8 / 2; ++q) {
        uint32_t b[4];  // code chunks 4q .. 4q + 3 of keys 8w .. 8w + 7
        dec::ldsm4(b, K8 + dec::k8_off<D>(key_s, 4 * q + mi));
        dec::mma_s8(acc, q8a[2 * q], b[0], b[1]);
        dec::mma_s8(acc, q8a[2 * q + 1], b[2], b[3]);
      }
      const float f0 = qs0 * ksc * p.scale_log2, f1 = qs1 * ksc * p.scale_log2;
      sv[0] = static_cast<float>(acc[0]) * f0;
      sv[1] = static_cast<float>(acc[1]) * f0;
      sv[2] = static_cast<float>(acc[2]) * f1;
      sv[3] = static_cast<float>(acc[3]) * f1;
    } else {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < kKs16 / 2; ++q) {
        uint32_t b[4];  // channel chunks 4q .. 4q + 3 of keys 8w .. 8w + 7
        dec::ldsm4(b, K + dec::k16_off<D>(key_s, 4 * q + mi));
        dec::mma_f16(acc, qa[2 * q], b[0], b[1]);
        dec::mma_f16(acc, qa[2 * q + 1], b[2], b[3]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sv[e] = acc[e] * p.scale_log2;
    }
    const int k0 = 8 * warp + 2 * q4;
    if (k0 >= jn) sv[0] = sv[2] = -INFINITY;
    if (k0 + 1 >= jn) sv[1] = sv[3] = -INFINITY;
    // online softmax: row maxima over the eight warps' keys
    float x0 = fmaxf(sv[0], sv[1]), x1 = fmaxf(sv[2], sv[3]);
    x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 1));
    x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 1));
    x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
    x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
    if (q4 == 0) {
      red_m[g * 8 + warp] = x0;
      red_m[(g + 8) * 8 + warp] = x1;
    }
    __syncthreads();
    const float t0 = dec::max8(red_m + g * 8), t1 = dec::max8(red_m + (g + 8) * 8);
    const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
    // P rounded to fp16, as the P.V of the prefill path takes it
    const __half p00 = __float2half_rn(exp2f(sv[0] - n0));
    const __half p01 = __float2half_rn(exp2f(sv[1] - n0));
    const __half p10 = __float2half_rn(exp2f(sv[2] - n1));
    const __half p11 = __float2half_rn(exp2f(sv[3] - n1));
    // P[row][key], 128-byte rows: keys k0, k0 + 1 sit in chunk w at byte 4 q4
    *reinterpret_cast<uint32_t*>(pt + dec::sw128(g, warp) + q4 * 4) = dec::pack_half2(p00, p01);
    *reinterpret_cast<uint32_t*>(pt + dec::sw128(g + 8, warp) + q4 * 4) = dec::pack_half2(p10, p11);
    float y0 = __half2float(p00) + __half2float(p01), y1 = __half2float(p10) + __half2float(p11);
    y0 += __shfl_xor_sync(0xffffffffu, y0, 1);
    y1 += __shfl_xor_sync(0xffffffffu, y1, 1);
    y0 += __shfl_xor_sync(0xffffffffu, y0, 2);
    y1 += __shfl_xor_sync(0xffffffffu, y1, 2);
    if (q4 == 0) {
      red_l[g * 8 + warp] = y0;
      red_l[(g + 8) * 8 + warp] = y1;
    }
    const float a0 = m0 == -INFINITY ? 0.f : exp2f(m0 - n0);
    const float a1 = m1 == -INFINITY ? 0.f : exp2f(m1 - n1);
    m0 = n0;
    m1 = n1;
    __syncthreads();
    const float z0 = dec::sum8(red_l + g * 8), z1 = dec::sum8(red_l + (g + 8) * 8);
    l0 = l0 * a0 + z0;
    l1 = l1 * a1 + z1;
    // this warp's channels of O = O * alpha + P . V
#pragma unroll
    for (int nt = 0; nt < kNt; ++nt) {
      o[nt][0] *= a0;
      o[nt][1] *= a0;
      o[nt][2] *= a1;
      o[nt][3] *= a1;
    }
#pragma unroll
    for (int ks = 0; ks < kDecodeKeys / 16; ++ks) {
      uint32_t pa[4];  // A: P rows 0-7 / 8-15 at keys 16 ks + {0..7, 8..15}
      dec::ldsm4(pa, pt + dec::sw128(mr + 8 * (mi & 1), 2 * ks + (mi >> 1)));
      const int key = 16 * ks + 8 * (mi & 1) + mr;
      if constexpr (kNt == 2) {
        uint32_t b[4];  // B: keys 16 ks + {0..7, 8..15} of channel chunks 2w, 2w + 1
        dec::ldsm4_t(b, V + dec::k16_off<D>(key, 2 * warp + (mi >> 1)));
        dec::mma_f16(o[0], pa, b[0], b[1]);
        dec::mma_f16(o[1], pa, b[2], b[3]);
      } else {
        uint32_t b[2];  // B: keys 16 ks + {0..7, 8..15} of channel chunk w
        dec::ldsm2_t(b, V + dec::k16_off<D>(key, warp));
        dec::mma_f16(o[0], pa, b[0], b[1]);
      }
    }
    __syncthreads();  // the slot, P and the row reductions are free again
    if (tid == 0 && i + kDecodeStages < n) issue(i + kDecodeStages);
  }

  // Partial state of this split: rows g and g + 8, channels
  // 8 (kNt w + nt) + 2 q4 + {0, 1}.
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = g + 8 * h;
    if (row < G) {
      const size_t pi = (static_cast<size_t>(s) * p.hq + heads[row]) * p.nsplit + split;
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt) {
        const int c = 8 * (kNt * warp + nt) + 2 * q4;
        *reinterpret_cast<float2*>(p.part_acc + pi * D + c) =
            bad ? make_float2(0.f, 0.f) : make_float2(o[nt][2 * h], o[nt][2 * h + 1]);
      }
      if (warp == 0 && q4 == 0) {
        p.part_m[pi] = bad ? -INFINITY : (h ? m1 : m0);
        p.part_l[pi] = bad ? 0.f : (h ? l1 : l0);
      }
    }
  }
  // The last split of this (sequence, KV head) to finish merges them all.
  // The CTA barrier orders every thread's partial writes before thread 0's
  // acquire-release increment; its acquire side, and the barrier after it,
  // order the merging CTA's reads after every other split's writes.
  __syncthreads();
  if (tid == 0) flags[2] = dec::add_acq_rel(p.counters + s * p.hk + kv, 1) == nsplit_s - 1;
  __syncthreads();
  if (!flags[2]) return;
  // merge: per query row the largest split maximum and the weighted sum of
  // the splits' l (warp per row), then O channel by channel
  float* mrow = red_m;  // [16]
  float* lrow = red_l;  // [16]
  for (int gi = warp; gi < G; gi += kDecodeThreads / 32) {
    const size_t pi0 = (static_cast<size_t>(s) * p.hq + heads[gi]) * p.nsplit;
    float m = -INFINITY;
    for (int k = lane; k < nsplit_s; k += 32) m = fmaxf(m, __ldcg(p.part_m + pi0 + k));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int k = lane; k < nsplit_s; k += 32) {
      const float mk = __ldcg(p.part_m + pi0 + k);
      if (mk != -INFINITY) l += exp2f(mk - m) * __ldcg(p.part_l + pi0 + k);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      mrow[gi] = m;
      lrow[gi] = l;
    }
  }
  __syncthreads();
  for (int x = tid; x < G * D; x += kDecodeThreads) {
    const int gi = x / D, c = x - gi * D;
    const size_t pi0 = (static_cast<size_t>(s) * p.hq + heads[gi]) * p.nsplit;
    const float m = mrow[gi], l = lrow[gi];
    float acc = 0.f;
#pragma unroll 4
    for (int k = 0; k < nsplit_s; ++k) {
      const float mk = __ldcg(p.part_m + pi0 + k);
      const float a = __ldcg(p.part_acc + (pi0 + k) * D + c);
      if (mk != -INFINITY) acc += exp2f(mk - m) * a;
    }
    static_cast<__half*>(p.o)[(static_cast<size_t>(s) * p.hq + heads[gi]) * D + c] =
        __float2half_rn(l > 0.f ? acc / l : 0.f);
  }
}

template <int D>
cudaError_t launch_decode_d(const DecodeParams& p, unsigned blocks, cudaStream_t stream) {
  const int smem = decode_smem(D).total;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  decode_attn_kernel<D><<<blocks, kDecodeThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

int launch_decode(const DecodeParams& p, cudaStream_t stream, cudaEvent_t ev_begin,
                  cudaEvent_t ev_end) {
  cudaError_t e = cudaMemsetAsync(p.counters, 0, sizeof(int) * p.nseq * p.hk, stream);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (ev_begin && (e = cudaEventRecord(ev_begin, stream)) != cudaSuccess)
    return static_cast<int>(e);
  const unsigned blocks = static_cast<unsigned>(p.nseq) * p.hk * p.nsplit;
  e = p.d == 128 ? launch_decode_d<128>(p, blocks, stream) : launch_decode_d<64>(p, blocks, stream);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (ev_end && (e = cudaEventRecord(ev_end, stream)) != cudaSuccess)
    return static_cast<int>(e);
  return cudaSuccess;
}

}  // namespace tilemix
