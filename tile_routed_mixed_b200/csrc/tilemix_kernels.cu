// CUDA kernels of the tile-routed FP16/INT8 causal prefill attention (sm_100a).
//
//   quantize_blocks_kernel   per-(head, block) symmetric absmax/127 INT8 codes
//   prefill_fwd_kernel       fused attention: TMA -> tcgen05 kind::f16 or
//                            kind::i8 QK^T per key tile (chosen by the routing
//                            bit) -> shared online softmax -> kind::f16 P.V
//
// Method: "TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
// Acceleration" (agihunt.info summary, method paragraphs) and "Precision Has a
// Map: TileMix Routes INT8 Inside Dense Attention" (cognaptus.com, "The routing
// mechanism is designed to stay inside the hot loop").
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tilemix_internal.h"
#include "tilemix_ptx.cuh"

namespace tilemix {

// Latched device status (see kStatus* bits); read and cleared by
// tilemix_get_error().
__device__ unsigned int g_status;

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 64;   // keys per tile

// ===================================================================
// Block quantisation.  One CTA per (block, head): pass 1 finds the absmax of
// the block's valid rows, pass 2 writes codes = clamp(rne(x / s), +-127) with
// s = a / 127 in IEEE fp32 ("only Q and K are quantised, Q in 128 x d blocks
// and K in 64 x d blocks, symmetric absmax / 127").
// ===================================================================
constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads)
    quantize_blocks_kernel(const __half* __restrict__ x, const int32_t* __restrict__ cu_seqlens,
                           const int32_t* __restrict__ cu_tiles, int nseq, int total_tiles,
                           int heads, int d, int block_rows, int8_t* __restrict__ codes,
                           float* __restrict__ scales) {
  const int tile = blockIdx.x;
  const int h = blockIdx.y;
  // sequence that owns this block (few sequences: linear scan)
  int s = 0;
  while (s + 1 < nseq && cu_tiles[s + 1] <= tile) ++s;
  const int t0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - t0;
  const int r0 = (tile - cu_tiles[s]) * block_rows;
  const int rows = min(block_rows, L - r0);
  const int chunks_per_row = d / 8;  // 16-byte chunks
  const int nchunks = rows * chunks_per_row;

  float amax = 0.f;
  for (int c = threadIdx.x; c < nchunks; c += kQuantThreads) {
    const int r = c / chunks_per_row, cc = c % chunks_per_row;
    const uint4 u = *reinterpret_cast<const uint4*>(
        x + (static_cast<size_t>(t0 + r0 + r) * heads + h) * d + cc * 8);
    const __half2* hv = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(hv[k]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  __shared__ float red[kQuantThreads / 32];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < kQuantThreads / 32 ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float a = red[0];
  const float sc = __fdiv_rn(a, 127.0f);
  if (threadIdx.x == 0) scales[static_cast<size_t>(h) * total_tiles + tile] = sc;

  for (int c = threadIdx.x; c < nchunks; c += kQuantThreads) {
    const int r = c / chunks_per_row, cc = c % chunks_per_row;
    const size_t off = (static_cast<size_t>(t0 + r0 + r) * heads + h) * d + cc * 8;
    const uint4 u = *reinterpret_cast<const uint4*>(x + off);
    const __half2* hv = reinterpret_cast<const __half2*>(&u);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(hv[k]);
      int c0 = 0, c1 = 0;
      if (a > 0.f) {
        c0 = __float2int_rn(__fdiv_rn(f.x, sc));
        c1 = __float2int_rn(__fdiv_rn(f.y, sc));
        c0 = max(-127, min(127, c0));
        c1 = max(-127, min(127, c1));
      }
      const uint32_t b = (static_cast<uint32_t>(c0) & 0xffu) | ((static_cast<uint32_t>(c1) & 0xffu) << 8);
      packed[k >> 1] |= b << ((k & 1) * 16);
    }
    *reinterpret_cast<uint2*>(codes + off) = make_uint2(packed[0], packed[1]);
  }
}

int launch_quantize(const void* x, const int32_t* cu_seqlens, const int32_t* cu_tiles, int nseq,
                    int total_tiles, int heads, int d, int block_rows, int8_t* codes,
                    float* scales, cudaStream_t stream) {
  if (total_tiles == 0 || heads == 0) return cudaSuccess;
  dim3 grid(total_tiles, heads);
  quantize_blocks_kernel<<<grid, kQuantThreads, 0, stream>>>(
      static_cast<const __half*>(x), cu_seqlens, cu_tiles, nseq, total_tiles, heads, d,
      block_rows, codes, scales);
  return static_cast<int>(cudaGetLastError());
}

// ===================================================================
// Fused attention forward.
//
// One CTA per (query-tile row, query head), heaviest rows first.  Warp roles:
//   warp 0     TMA producer: Q (fp16 + int8), then per key tile either the
//              fp16 or the int8 K tile (by the routing bit) and the fp16 V tile
//   warp 1     TMEM owner and MMA issuer: S = Q K^T (kind::f16 -> f32 or
//              kind::i8 -> s32) into one of two TMEM score buffers, then
//              O += P V (kind::f16, P read from TMEM)
//   warps 4-7  softmax: one query row per thread; routed scores -> float
//              score domain, legality mask, online max / normaliser, P in
//              fp16 back to TMEM; final O / l in fp16
// ===================================================================
constexpr int kStages = 3;
constexpr int kPrefillThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P values stay <= 2^8
constexpr uint32_t kTmemCols = 256;

template <int D>
struct Smem {
  static constexpr int kQ = BM * D * 2;       // fp16 Q tile
  static constexpr int kQ8 = BM * D;          // int8 Q tile
  static constexpr int kKSlot = BN * D * 2;   // fp16 K tile (an int8 K tile uses half)
  static constexpr int kV = BN * D * 2;       // fp16 V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffQ8 = kOffQ + kQ;
  static constexpr int kOffK = kOffQ8 + kQ8;
  static constexpr int kOffV = kOffK + kStages * kKSlot;
  static constexpr int kOffBar = kOffV + kStages * kV;
  static constexpr int kBytes = kOffBar + 512 + 1024;  // barriers + alignment slack
  static constexpr int kF16Steps = D / 16;
  static constexpr int kI8Steps = D / 32;
  static constexpr uint32_t kI8Layout = D == 128 ? ptx::kSwizzle128B : ptx::kSwizzle64B;
  static constexpr uint32_t kI8Sbo = 8 * D;  // 8 rows of D bytes
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = D;       // two 64-column score buffers
};

// Every mbarrier below is waited on by parity.  A parity wait is only
// unambiguous when the waiter is at most one phase behind the barrier, so each
// barrier is sized so that this holds: e.g. P(j).V completions alternate
// between two barriers (at tile i the softmax waits for P(i-1).V, and
// P(i-3).V is already known complete because S(i-1) could only be computed
// after it), and the epilogue waits on a barrier of its own.
struct Barriers {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done[2];  // P(j).V of tile j done, one barrier per score buffer
  uint64_t o_final;     // the last P.V of the CTA done
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Bounded wait: gives up after `timeout_ns` (latching kStatusTimeout and the
// CTA's abort flag) or as soon as another role of the CTA has given up.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned long long timeout_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const unsigned long long start = ptx::globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer() - start > timeout_ns) {
        *abort_flag = 1;
        atomicOr(&g_status, kStatusTimeout);
        return false;
      }
    }
  }
}

// Warp-uniform variant for roles whose following instructions are
// warp-collective (.sync.aligned TMEM loads and stores).
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag,
                                              unsigned long long timeout_ns) {
  const bool ok = wait_bar(bar, parity, abort_flag, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

// Drain wait used on the way out: ignores the abort flag, still bounded.
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity,
                                          unsigned long long timeout_ns) {
  const unsigned long long start = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer() - start > timeout_ns) {
      atomicOr(&g_status, kStatusTimeout);
      return;
    }
  }
}

__device__ __forceinline__ bool routed_int8(uint64_t word, int kt, int g) {
  return (word >> (kt / g)) & 1ull;
}

template <int D>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ PrefillParams p) {
  using S = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + S::kOffBar);

  // A wait of an earlier CTA already expired: do not start more work.
  if (*reinterpret_cast<volatile unsigned int*>(&g_status) & kStatusTimeout) return;

  // ---- work item: heaviest query-tile rows first ----
  int b = blockIdx.x;
  const int h = b % p.hq;
  b /= p.hq;
  const int s = b % p.nseq;
  b /= p.nseq;
  const int qt = p.max_qtiles - 1 - b;
  const int t0 = p.cu_seqlens[s];
  const int L = p.cu_seqlens[s + 1] - t0;
  if (qt >= (L + BM - 1) / BM) return;
  const int kv = p.kv_head_of_q ? p.kv_head_of_q[h] : h / p.group;
  const int row0 = qt * BM;
  // causal and boundary legality: independent of the routing word
  const int last_tile = p.causal ? (min(row0 + BM, L) - 1) / BN : (L - 1) / BN;
  const int ntiles = last_tile + 1;
  const int gs = p.g[s];
  if (gs < 1 || last_tile / gs > 63) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusBadGroups);
    return;
  }
  const uint64_t word = p.masks[static_cast<size_t>(p.cu_qtiles[s] + qt) * p.hk + kv];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&bars->k_full[i], 1);
      ptx::mbar_init(&bars->k_empty[i], 1);
      ptx::mbar_init(&bars->v_full[i], 1);
      ptx::mbar_init(&bars->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], 128);
    }
    ptx::mbar_init(&bars->pv_done[0], 1);
    ptx::mbar_init(&bars->pv_done[1], 1);
    ptx::mbar_init(&bars->o_final, 1);
    ptx::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  const unsigned long long tmo = p.timeout_ns;

  uint8_t* sQ = smem + S::kOffQ;
  uint8_t* sQ8 = smem + S::kOffQ8;
  uint8_t* sK = smem + S::kOffK;
  uint8_t* sV = smem + S::kOffV;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      ptx::prefetch_tensormap(&p.tm_q);
      ptx::prefetch_tensormap(&p.tm_k);
      ptx::prefetch_tensormap(&p.tm_v);
      ptx::mbar_expect_tx(&bars->q_full, S::kQ + S::kQ8);
#pragma unroll
      for (int j = 0; j < D / 64; ++j)
        ptx::tma_load_3d(sQ + j * BM * 128, &p.tm_q, &bars->q_full, j * 64, h, t0 + row0);
      ptx::tma_load_3d(sQ8, &p.tm_q8, &bars->q_full, 0, h, t0 + row0);
      int kcnt[kStages] = {}, vcnt[kStages] = {};
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % kStages;
        const uint32_t ph = ((i / kStages) - 1) & 1;
        if (i >= kStages && !wait_bar(&bars->k_empty[st], ph, abort_flag, tmo)) break;
        const int key0 = t0 + i * BN;
        uint8_t* kslot = sK + st * S::kKSlot;
        if (routed_int8(word, i, gs)) {
          ptx::mbar_expect_tx(&bars->k_full[st], BN * D);
          ptx::tma_load_3d(kslot, &p.tm_k8, &bars->k_full[st], 0, kv, key0);
        } else {
          ptx::mbar_expect_tx(&bars->k_full[st], BN * D * 2);
#pragma unroll
          for (int j = 0; j < D / 64; ++j)
            ptx::tma_load_3d(kslot + j * BN * 128, &p.tm_k, &bars->k_full[st], j * 64, kv, key0);
        }
        ++kcnt[st];
        if (i >= kStages && !wait_bar(&bars->v_empty[st], ph, abort_flag, tmo)) break;
        uint8_t* vslot = sV + st * S::kV;
        ptx::mbar_expect_tx(&bars->v_full[st], BN * D * 2);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          ptx::tma_load_3d(vslot + j * BN * 128, &p.tm_v, &bars->v_full[st], j * 64, kv, key0);
        ++vcnt[st];
      }
      // Never leave with copies into this CTA's shared memory in flight.
      drain_bar(&bars->q_full, 0, tmo);
      for (int st = 0; st < kStages; ++st) {
        if (kcnt[st]) drain_bar(&bars->k_full[st], (kcnt[st] - 1) & 1, tmo);
        if (vcnt[st]) drain_bar(&bars->v_full[st], (vcnt[st] - 1) & 1, tmo);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      constexpr uint32_t kIdF16 = ptx::idesc_f16(BM, BN, false);
      constexpr uint32_t kIdI8 = ptx::idesc_s8(BM, BN);
      constexpr uint32_t kIdPV = ptx::idesc_f16(BM, D, true);
      const uint32_t aQ = ptx::smem_addr(sQ), aQ8 = ptx::smem_addr(sQ8);
      const uint32_t aK = ptx::smem_addr(sK), aV = ptx::smem_addr(sV);
      bool ok = wait_bar(&bars->q_full, 0, abort_flag, tmo);
      ptx::tc_fence_after();
      auto issue_pv = [&](int j) -> bool {
        const int st = j % kStages;
        const int sb = j & 1;
        if (!wait_bar(&bars->p_full[sb], (j >> 1) & 1, abort_flag, tmo)) return false;
        if (!wait_bar(&bars->v_full[st], (j / kStages) & 1, abort_flag, tmo)) return false;
        ptx::tc_fence_after();
        const int valid = L - j * BN;
        if (valid < BN) {
          // Keys past the sequence end belong to the next packed sequence:
          // zero their V rows so that 0 * (NaN or Inf) cannot reach O.
          uint8_t* vslot = sV + st * S::kV;
          for (int part = 0; part < D / 64; ++part)
            for (int r = valid; r < BN; ++r) {
              uint4* row = reinterpret_cast<uint4*>(vslot + part * BN * 128 + r * 128);
#pragma unroll
              for (int c = 0; c < 8; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
            }
          ptx::fence_proxy_async_smem();
        }
        const uint32_t vbase = aV + st * S::kV;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = ptx::smem_desc(vbase + kk * 2048, BN * 128, 1024, ptx::kSwizzle128B);
          ptx::mma_f16_ts(tmem + S::kColO, tmem + S::kColS + sb * 64 + kk * 8, bdesc, kIdPV,
                          (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(&bars->pv_done[sb]);
        ptx::mma_commit(&bars->v_empty[st]);
        if (j == ntiles - 1) ptx::mma_commit(&bars->o_final);
        return true;
      };
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i % kStages;
        const int sb = i & 1;
        // score buffer sb is free once P(i-2).V has read P(i-2) from it
        if (i >= 2 && !wait_bar(&bars->pv_done[sb], ((i - 2) >> 1) & 1, abort_flag, tmo)) {
          ok = false;
          break;
        }
        if (!wait_bar(&bars->k_full[st], (i / kStages) & 1, abort_flag, tmo)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t d_s = tmem + S::kColS + sb * 64;
        const uint32_t kbase = aK + st * S::kKSlot;
        if (routed_int8(word, i, gs)) {
#pragma unroll
          for (int k = 0; k < S::kI8Steps; ++k) {
            const uint64_t ad = ptx::smem_desc(aQ8 + k * 32, 16, S::kI8Sbo, S::kI8Layout);
            const uint64_t bd = ptx::smem_desc(kbase + k * 32, 16, S::kI8Sbo, S::kI8Layout);
            ptx::mma_i8_ss(d_s, ad, bd, kIdI8, k > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int k = 0; k < S::kF16Steps; ++k) {
            const uint64_t ad = ptx::smem_desc(aQ + (k >> 2) * (BM * 128) + (k & 3) * 32, 16, 1024,
                                               ptx::kSwizzle128B);
            const uint64_t bd = ptx::smem_desc(kbase + (k >> 2) * (BN * 128) + (k & 3) * 32, 16,
                                               1024, ptx::kSwizzle128B);
            ptx::mma_f16_ss(d_s, ad, bd, kIdF16, k > 0 ? 1u : 0u);
          }
        }
        ptx::mma_commit(&bars->s_full[sb]);
        ptx::mma_commit(&bars->k_empty[st]);
        if (i >= 1 && !issue_pv(i - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(ntiles - 1);
      // all MMAs of this CTA complete before TMEM and shared memory go away
      ptx::mma_commit(&bars->drain);
      drain_bar(&bars->drain, 0, tmo);
    }
  } else if (warp >= kSoftmaxWarp0) {
    // ================= softmax / epilogue =================
    const int tr = threadIdx.x - kSoftmaxWarp0 * 32;  // row within the tile
    const int wq = warp - kSoftmaxWarp0;              // TMEM lane quarter
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const int my_row = row0 + tr;
    const float q_sc =
        p.q_scale[static_cast<size_t>(h) * p.total_qtiles + p.cu_qtiles[s] + qt];
    const float* ks = p.k_scale + static_cast<size_t>(kv) * p.total_ktiles + p.cu_ktiles[s];
    float m = -INFINITY;  // running max, log2 units
    float l = 0.f;        // normaliser (sum of the fp16-rounded P)
    bool ok = true;
    uint32_t r[32], r2[32];
    for (int i = 0; i < ntiles; ++i) {
      const int sb = i & 1;
      if (!wait_bar_warp(&bars->s_full[sb], (i >> 1) & 1, abort_flag, tmo)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t ts = tmem + lane_base + S::kColS + sb * 64;
      ptx::tmem_ld32(ts, r);
      ptx::tmem_ld32(ts + 32, r2);
      ptx::tmem_ld_wait();
      const bool is_int = routed_int8(word, i, gs);
      float x[64];
      if (is_int) {
        const float sc = q_sc * __ldg(ks + i) * p.scale_log2;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          x[j] = static_cast<float>(static_cast<int>(r[j])) * sc;
          x[32 + j] = static_cast<float>(static_cast<int>(r2[j])) * sc;
        }
        if (p.dbg && my_row < L) {
          int32_t* drow = p.dbg + (static_cast<size_t>(h) * p.total_tokens + t0 + my_row) * p.dbg_cols;
          for (int j = 0; j < 64; ++j) {
            const int key = i * BN + j;
            if (key < L) drow[key] = static_cast<int32_t>(j < 32 ? r[j] : r2[j - 32]);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          x[j] = __uint_as_float(r[j]) * p.scale_log2;
          x[32 + j] = __uint_as_float(r2[j]) * p.scale_log2;
        }
      }
      const int key0 = i * BN;
      if (key0 + BN > L || (p.causal && key0 + BN - 1 > row0)) {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int key = key0 + j;
          if (key >= L || (p.causal && key > my_row)) x[j] = -INFINITY;
        }
      }
      float tmax = x[0];
#pragma unroll
      for (int j = 1; j < 64; ++j) tmax = fmaxf(tmax, x[j]);
      const float m_new = fmaxf(m, tmax);
      const bool resc = m_new - m > kRescaleThreshold;
      const float m_use = resc ? m_new : m;
      const float alpha = resc ? ptx::ex2(m - m_new) : 1.0f;
      float lsum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const __half2 hp = __floats2half2_rn(ptx::ex2(x[2 * j] - m_use), ptx::ex2(x[2 * j + 1] - m_use));
        const float2 back = __half22float2(hp);
        lsum += back.x + back.y;
        pk[j] = *reinterpret_cast<const uint32_t*>(&hp);
      }
      l = l * alpha + lsum;
      m = m_use;
      if (__any_sync(0xffffffffu, resc && i > 0)) {
        // O holds P.V of tiles < i: rescale it once P(i-1).V has landed.
        if (!wait_bar_warp(&bars->pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, tmo)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const uint32_t to = tmem + lane_base + S::kColO + c * 32;
          ptx::tmem_ld32(to, r);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
          ptx::tmem_st32(to, r);
        }
      }
      ptx::tmem_st32(ts, pk);
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->p_full[sb]);
    }
    if (ok && wait_bar_warp(&bars->o_final, 0, abort_flag, tmo)) {
      ptx::tc_fence_after();
      const float inv_l = 1.0f / l;
      const bool valid = my_row < L;
      __half* orow = static_cast<__half*>(p.o) +
                     (static_cast<size_t>(t0 + my_row) * p.hq + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        ptx::tmem_ld32(tmem + lane_base + S::kColO + c * 32, r);
        ptx::tmem_ld_wait();
        uint32_t hv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __half2 o2 = __floats2half2_rn(__uint_as_float(r[2 * j]) * inv_l,
                                               __uint_as_float(r[2 * j + 1]) * inv_l);
          hv[j] = *reinterpret_cast<const uint32_t*>(&o2);
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(hv[4 * j], hv[4 * j + 1], hv[4 * j + 2], hv[4 * j + 3]);
        }
      }
      if (p.lse && valid)
        p.lse[static_cast<size_t>(h) * p.total_tokens + t0 + my_row] =
            (m + __log2f(l)) * 0.69314718055994530942f;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
static int launch_prefill_d(const PrefillParams& p, cudaStream_t stream) {
  const int smem = Smem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(prefill_fwd_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return static_cast<int>(e);
  const long long blocks = static_cast<long long>(p.max_qtiles) * p.nseq * p.hq;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  prefill_fwd_kernel<D><<<static_cast<unsigned>(blocks), kPrefillThreads, smem, stream>>>(p);
  return static_cast<int>(cudaGetLastError());
}

int launch_prefill(const PrefillParams& p, int d, cudaStream_t stream) {
  if (d == 128) return launch_prefill_d<128>(p, stream);
  if (d == 64) return launch_prefill_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

int read_and_clear_status(unsigned int* status, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return static_cast<int>(e);
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  if (e != cudaSuccess) return static_cast<int>(e);
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
  *status = v;
  return static_cast<int>(e);
}

}  // namespace tilemix
