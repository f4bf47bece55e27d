// CUDA kernels of the tile-routed FP16/INT8 causal prefill attention (sm_100a).
//
//   prefill_fwd_kernel       fused attention: TMA -> tcgen05 kind::f16 or
//                            kind::i8 QK^T per key tile (chosen by the routing
//                            bit) -> shared online softmax -> kind::f16 P.V
//   decode_attn_kernel       one new query row per sequence against the INT8 K
//                            cache (tilemix_decode.cuh, included at the end)
// The block quantiser that feeds both is in tilemix_quantize.cu.
//
// Method: "TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
// Acceleration" (agihunt.info summary, method paragraphs) and "Precision Has a
// Map: TileMix Routes INT8 Inside Dense Attention" (cognaptus.com, "The routing
// mechanism is designed to stay inside the hot loop").
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "tilemix.h"
#include "tilemix_internal.h"
#include "tilemix_ptx.cuh"
#include "tilemix_quant.cuh"

namespace tilemix {

// Latched device status (see kStatus* bits); read and cleared by
// tilemix_get_error().
__device__ unsigned int g_status;

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 64;   // keys per tile

// ===================================================================
// Fused attention forward.
//
// Persistent CTAs, one per SM, each walking a share of the work items: one
// item per (sequence, query head, pair of query-tile rows 2j and 2j+1),
// heaviest pairs first.  The two 128-row Q tiles of an item share every K/V
// tile load; the K/V ring, the score and P buffers run on across items, so
// one item's last tiles and epilogue overlap the next item's first tiles.
// Warp roles (12 warps, three warpgroups):
//   warp 0      TMA producer: both Q tiles (fp16 and int8), then per key tile
//               the K tile in each precision the two rows' routing bits need,
//               and the fp16 V tile
//   warps 1, 2  MMA issuers of Q tile 0 and Q tile 1 (warp 1 also owns TMEM):
//               S_q = Q_q K^T (kind::f16 -> f32 or kind::i8 -> s32, by row
//               q's routing bit) into one of the two TMEM score buffers of Q
//               tile q, then O_q += P_q V (kind::f16, P read from TMEM)
//   warps 4-7   softmax of Q tile 0, warps 8-11 softmax of Q tile 1: one query
//               row per thread; routed scores -> float score domain, legality
//               mask, online max / normaliser, P in fp16 back to TMEM; when a
//               row's running max moved (rare with lazy rescaling), the warp
//               rescales its rows of O in TMEM after the previous P.V landed,
//               before P is handed to the next P.V; at the end O / l in fp16
// TMEM (512 columns): per Q tile q, O_q [D cols] and two 64-column score
// buffers, at column offset 256 q.
// ===================================================================
constexpr int kStages = 3;
constexpr int kPrefillThreads = 384;
// No register split: every role fits in the registers the launch gives
// each of the 384 threads.
constexpr int kSoftmaxWarp0 = 4;
// Lazy rescaling: the running max used for P is only moved when the tile max
// exceeds it by more than this (log2 units), so P <= 2^15 stays inside fp16
// (65504) and P.V / the normaliser stay exact in their fp32 accumulators.  A
// stale max only shifts fp16 underflow further below the true maximum.
constexpr float kRescaleThreshold = 15.0f;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Smem {
  static constexpr int kQ = BM * D * 2;       // fp16 Q tile
  static constexpr int kQ8 = BM * D;          // int8 Q tile
  static constexpr int kK16 = BN * D * 2;     // fp16 K tile
  static constexpr int kK8 = BN * D;          // int8 K tile
  static constexpr int kV = BN * D * 2;       // fp16 V tile
  static constexpr int kOffQ = 0;                          // + q * kQ
  static constexpr int kOffQ8 = kOffQ + 2 * kQ;            // + q * kQ8
  static constexpr int kOffK16 = kOffQ8 + 2 * kQ8;         // + stage * kK16
  static constexpr int kOffK8 = kOffK16 + kStages * kK16;  // + stage * kK8
  static constexpr int kOffV = kOffK8 + kStages * kK8;     // + stage * kV
  static constexpr int kOffBar = kOffV + kStages * kV;
  static constexpr int kBytes = kOffBar + 512 + 1024;      // + alignment slack
  static constexpr int kF16Steps = D / 16;
  static constexpr int kI8Steps = D / 32;
  static constexpr uint32_t kI8Layout = D == 128 ? ptx::kSwizzle128B : ptx::kSwizzle64B;
  static constexpr uint32_t kI8Sbo = 8 * D;  // 8 rows of D bytes
  // TMEM columns of Q tile q: O [D], S [64], P buffers 0 and 1 [32 each]
  __host__ __device__ static constexpr uint32_t col_o(int q) { return 256u * q; }
  __host__ __device__ static constexpr uint32_t col_s(int q) { return 256u * q + D; }
  __host__ __device__ static constexpr uint32_t col_p(int q, int b) {
    return 256u * q + D + 64u + 32u * b;
  }
};

// Every mbarrier below is waited on by parity.  A parity wait is only
// unambiguous when the waiter is at most one phase behind the barrier; for
// each wait, the barrier's next phase needs an event that cannot happen before
// the waiter has moved on (noted at the waits).  The CTA is persistent, so the
// phases run on across work items: each role keeps running counts.
//   S is single-buffered: S(n+1) needs s_free(n), i.e. the softmax has read
//   S(n).  P is double-buffered; the softmax stores P(n) only after S(n)
//   landed, and the MMA thread issues S(n) after P(n-2).V, so that commit
//   covers P(n-2).V: the MMA thread cannot fall two phases behind p_full.
struct Barriers {
  uint64_t q_full[2];          // Q tile q (fp16 and int8) of the current item landed
  uint64_t q_free[2];          // the last S = Q K^T of Q tile q's item completed
  uint64_t kv_full[kStages];   // K (each precision needed) and V of a key tile landed
  uint64_t kv_empty[kStages];  // both MMA threads are done with that key tile
  uint64_t s_full[2];          // S_q in TMEM
  uint64_t s_free[2];          // S_q read out: the S columns may be refilled
  uint64_t p_full[2][2];       // P_q in TMEM buffer b (and O_q rescaled if needed)
  uint64_t pv_done[2][2];      // the P.V reading P_q buffer b completed
  uint64_t o_final[2];         // the last P.V of Q tile q's item completed
  uint64_t o_free[2];          // the softmax has read O_q of the item out of TMEM
  uint64_t drain[2];
  uint64_t item_full[4];       // a work item index published in ring slot k % 4
  uint64_t item_empty[4];      // every consumer has read ring slot k % 4
  int item_ring[4];            // item indices, -1 = no more work
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Barriers) <= 512, "barrier block exceeds its shared-memory slot");

// The producer thread takes work items from a global ticket (heaviest first,
// so faster SMs simply take more) and publishes them through a small ring;
// both MMA threads and all 256 softmax threads read every slot.
constexpr int kItemSlots = 4;
constexpr int kItemConsumers = 2 + 2 * 128;

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
// A consumer's next work item from ring slot k % 4 (item_full's next phase
// for the slot needs this consumer's item_empty arrival): the index, -1 when
// there is no more work, or kItemAbort if the wait gave up.
constexpr int kItemAbort = -2;
__device__ __forceinline__ int next_item(Barriers* bars, uint32_t k, volatile int* abort_flag,
                                         unsigned long long tmo, bool warp_wide) {
  const int slot = k % kItemSlots;
  const uint32_t parity = (k / kItemSlots) & 1;
  const bool ok = warp_wide ? wait_bar_warp(&bars->item_full[slot], parity, abort_flag, tmo)
                            : wait_bar(&bars->item_full[slot], parity, abort_flag, tmo);
  if (!ok) return kItemAbort;
  const int w = *reinterpret_cast<volatile int*>(&bars->item_ring[slot]);
  ptx::mbar_arrive(&bars->item_empty[slot]);  // release: the read above comes first
  return w;
}

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

// Routing lookup along consecutive key tiles: group = tile / g, tracked
// incrementally (no division in the hot loops); the bit is a shift and a mask.
struct GroupCursor {
  int group = 0, in_group = 0;
  __device__ __forceinline__ bool int8(uint64_t word) const { return (word >> group) & 1ull; }
  __device__ __forceinline__ void next(int g) {
    if (++in_group == g) {
      in_group = 0;
      ++group;
    }
  }
};

__device__ __forceinline__ float max3(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}

// s += low half + high half of a packed f16x2 (each widened exactly).
__device__ __forceinline__ void add_f16x2_to_f32(float& s, uint32_t h2) {
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
      "add.rn.f32.f16 %0, lo, %0;\n\tadd.rn.f32.f16 %0, hi, %0;\n\t}"
      : "+f"(s)
      : "r"(h2));
}

// {a0 * b + c, a1 * b + c} as one packed instruction (sm_100 fp32x2; each
// lane is the IEEE fused multiply-add fmaf gives); b2 and c2 hold b and c in
// both lanes.
__device__ __forceinline__ float2 fma2_bc(float a0, float a1, unsigned long long b2,
                                          unsigned long long c2) {
  unsigned long long a, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b2), "l"(c2));
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}

__device__ __forceinline__ unsigned long long both_lanes(float x) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Shared-memory descriptor from a template holding every field but the start
// address.
__device__ __forceinline__ uint64_t desc_at(uint64_t tmpl, uint32_t addr) {
  return tmpl | static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
}

// S = Q K^T of one 128 x 64 score tile into TMEM column d_s, in the precision
// the routing bit selects.
// kFp8: the low-precision tiles are FP8 e4m3 (kind::f8f6f4, fp32 accumulate;
// the descriptor's e4m3 formats are 0, like f16's) instead of INT8.
template <int D, bool kFp8>
__device__ __forceinline__ void issue_qk(uint32_t d_s, bool is_int, uint32_t aq16, uint32_t aq8,
                                         uint32_t bk16, uint32_t bk8, uint64_t tmpl16,
                                         uint64_t tmpl8) {
  constexpr uint32_t kIdF16 = ptx::idesc_f16(BM, BN, false);
  constexpr uint32_t kIdI8 = ptx::idesc_s8(BM, BN);
  constexpr uint32_t kIdF8 = ptx::idesc_f16(BM, BN, false);
  if (is_int) {
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      if constexpr (kFp8)
        ptx::mma_f8_ss(d_s, desc_at(tmpl8, aq8 + k * 32), desc_at(tmpl8, bk8 + k * 32), kIdF8,
                       k > 0 ? 1u : 0u);
      else
        ptx::mma_i8_ss(d_s, desc_at(tmpl8, aq8 + k * 32), desc_at(tmpl8, bk8 + k * 32), kIdI8,
                       k > 0 ? 1u : 0u);
    }
  } else {
#pragma unroll
    for (int k = 0; k < D / 16; ++k)
      ptx::mma_f16_ss(d_s, desc_at(tmpl16, aq16 + (k >> 2) * (BM * 128) + (k & 3) * 32),
                      desc_at(tmpl16, bk16 + (k >> 2) * (BN * 128) + (k & 3) * 32), kIdF16,
                      k > 0 ? 1u : 0u);
  }
}

// O += P V of one 64-key tile: P (fp16) from TMEM column a_p, V from shared
// memory (MN-major).
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t d_o, uint32_t a_p, uint32_t vbase,
                                         uint64_t tmplv, bool first) {
  constexpr uint32_t kIdPV = ptx::idesc_f16(BM, D, true);
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk)
    ptx::mma_f16_ts(d_o, a_p + kk * 8, desc_at(tmplv, vbase + kk * 2048), kIdPV,
                    (!first || kk > 0) ? 1u : 0u);
}

// One work item: query-tile rows 2 pair and 2 pair + 1 (the second may not
// exist) of sequence s and query head h.  Causal and boundary legality fix
// each row's key-tile count, independently of the routing words.
struct WorkItem {
  int s, h, t0, L, qt0, nt0, nt1, nt, nq, kv, gs, cq, ck;
  uint64_t w0, w1;
};

// Decodes item w.  Items are ordered by (sequence, KV head), then query-tile
// pair heaviest first, then the KV head's query heads, so that the CTAs
// working at any one time share the K/V of a few heads and those stay in L2,
// while each group's lightest items come last.  (With a custom head map the
// order is only a heuristic; every (s, h, pair) is still visited once.)
// False if the sequence has no such pair, if its routing would need a group
// index above 63, or if the head map sends h outside [0, hk) (the last two
// are reported in the status word).
__device__ __forceinline__ bool load_item(const PrefillParams& p, int w, WorkItem& it) {
  const int per_kv = p.max_qpairs * p.group;
  const int kvg = w / per_kv;  // (s, kv) index, sequence-major
  const int rem = w - kvg * per_kv;
  const int pair = p.max_qpairs - 1 - rem / p.group;
  const int h = (kvg % p.hk) * p.group + rem % p.group;
  const int s = kvg / p.hk;
  // independent loads first, so that they overlap
  const int t0 = __ldg(p.cu_seqlens + s);
  const int t1 = __ldg(p.cu_seqlens + s + 1);
  const int gs = __ldg(p.g + s);
  const int cq = __ldg(p.cu_qtiles + s);
  const int ck = __ldg(p.cu_ktiles + s);
  const int kv = p.kv_head_of_q ? __ldg(p.kv_head_of_q + h) : h / p.group;
  const int L = t1 - t0;
  const int tm = (L + BM - 1) / BM;
  const int qt0 = 2 * pair;
  if (qt0 >= tm) return false;
  if (kv < 0 || kv >= p.hk) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusBadHeadMap);
    return false;
  }
  const bool has1 = qt0 + 1 < tm;
  const int nt0 = (p.causal ? min(qt0 * BM + BM, L) - 1 : L - 1) / BN + 1;
  const int nt1 = has1 ? (p.causal ? min(qt0 * BM + 2 * BM, L) - 1 : L - 1) / BN + 1 : 0;
  const int nt = max(nt0, nt1);
  if (gs < 1 || (nt - 1) / gs > 63) {
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusBadGroups);
    return false;
  }
  const uint64_t* wrow = p.masks + static_cast<size_t>(cq + qt0) * p.hk + kv;
  it.s = s;
  it.h = h;
  it.t0 = t0;
  it.L = L;
  it.qt0 = qt0;
  it.nt0 = nt0;
  it.nt1 = nt1;
  it.nt = nt;
  it.nq = has1 ? 2 : 1;
  it.kv = kv;
  it.gs = gs;
  it.cq = cq;
  it.ck = ck;
  it.w0 = __ldg(wrow);
  it.w1 = has1 ? __ldg(wrow + p.hk) : 0ull;
  return true;
}

// What one softmax thread needs about its row and Q tile for the key-tile
// loop, and the row's running state.
struct SoftmaxCtx {
  const PrefillParams* p;
  Barriers* bars;
  volatile int* abort_flag;
  unsigned long long tmo;
  uint32_t ts, to, tp0;           // TMEM addresses of this lane's S, O and P buffer 0
  int q, L, row0, my_row, h, t0, ntq;
  float q_sc;
  const float* ks;                // K block scales of the sequence and KV head
};
struct RowState {
  float m;          // running max, log2 units
  float l;          // normaliser: sum of the fp16-rounded P actually used in P.V
  float k_sc_next;  // K scale of the next key tile (loaded one tile ahead)
  uint32_t n_s;     // S_q read so far
  uint32_t n_p;     // P_q stored so far
};

// One key tile of the shared online softmax for this thread's row: S from
// TMEM, the routed score domain, legality, max / normaliser update, lazy
// rescale of O, P (fp16) to TMEM.  kMask adds the legality mask that only the
// diagonal and sequence-tail tiles need, kDebug the INT32 score dump of debug
// runs; the lean copy runs every other tile, so the hot loop carries no code
// for them.  False if a wait gave up.
template <int D, bool kMask, bool kDebug, bool kFp8>
__device__ __forceinline__ bool softmax_tile(const SoftmaxCtx& cx, RowState& st, int i, bool is_int,
                                             uint32_t (&r)[64]) {
  const int q = cx.q;
  const int sb = st.n_p & 1;
  const float k_sc = st.k_sc_next;
  if (i + 1 < cx.ntq) st.k_sc_next = __ldg(cx.ks + i + 1);
  // s_full's next phase needs s_free from this read
  if (!wait_bar_warp(&cx.bars->s_full[q], st.n_s & 1, cx.abort_flag, cx.tmo)) return false;
  ptx::tc_fence_after();
  ptx::tmem_ld32(cx.ts, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  ptx::tmem_ld32(cx.ts + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  ptx::tmem_ld_wait();
  // S is in registers: the MMA warp may compute the next S now
  ptx::tc_fence_before();
  ptx::mbar_arrive(&cx.bars->s_free[q]);
  ++st.n_s;
  const int key0 = i * BN;
  if (kDebug && !kFp8 && is_int && cx.p->dbg && cx.my_row < cx.L) {
    int32_t* drow = cx.p->dbg +
                    (static_cast<size_t>(cx.h) * cx.p->total_tokens + cx.t0 + cx.my_row) * cx.p->dbg_cols;
    for (int j = 0; j < 64; ++j)
      if (key0 + j < cx.L) drow[key0 + j] = static_cast<int32_t>(r[j]);
  }
  // scores in the float domain, before the log2(e)-scaled softmax:
  // FP16 tile: raw fp32 dot; INT8 tile: exact float of the INT32 dot; FP8
  // tile: the fp32 dot as it is.
  if (!kFp8 && is_int) {
#pragma unroll
    for (int j = 0; j < 64; ++j) r[j] = __float_as_uint(__int2float_rn(static_cast<int>(r[j])));
  }
  const float c = is_int ? cx.q_sc * k_sc * cx.p->scale_log2 : cx.p->scale_log2;
  const bool masked =
      kMask && (key0 + BN > cx.L || (cx.p->causal && key0 + BN - 1 > cx.row0));
  const int lim = cx.p->causal ? min(cx.L, cx.my_row + 1) : cx.L;  // legal keys < lim
  if (masked) {
#pragma unroll
    for (int j = 0; j < 64; ++j)
      if (key0 + j >= lim) r[j] = __float_as_uint(-INFINITY);
  }
  // row max of the tile: eight independent chains, then a short tree
  float g8[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float* x = reinterpret_cast<const float*>(&r[8 * u]);
    g8[u] = fmaxf(max3(max3(x[0], x[1], x[2]), max3(x[3], x[4], x[5]), x[6]), x[7]);
  }
  const float mx = fmaxf(max3(g8[0], g8[1], g8[2]), max3(max3(g8[3], g8[4], g8[5]), g8[6], g8[7]));
  // c >= 0; c == 0 only for an all-zero quantisation block (scores 0)
  const float m_tile = mx == -INFINITY ? -INFINITY : mx * c;
  const float m_new = fmaxf(st.m, m_tile);
  const bool resc = m_new - st.m > kRescaleThreshold;
  const float m_use = resc ? m_new : st.m;
  const float alpha = resc ? ptx::ex2(st.m - m_new) : 1.0f;
  float ls[4] = {0.f, 0.f, 0.f, 0.f};
  // P = 2^(score * c - m), packed in place: pair k lands in r[k]
  const unsigned long long c2 = both_lanes(c), nm2 = both_lanes(-m_use);
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float2 x = fma2_bc(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]), c2, nm2);
    r[k] = pack_f16x2(ptx::ex2(x.x), ptx::ex2(x.y));
    add_f16x2_to_f32(ls[k & 3], r[k]);
  }
  if (masked && c == 0.f) {
    // an all-zero block (c == 0) turns -inf scores into NaN: clear them (for
    // c > 0 the masked keys already gave 2^-inf = 0)
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const uint32_t keep = (key0 + 2 * k < lim ? 0x0000ffffu : 0u) |
                            (key0 + 2 * k + 1 < lim ? 0xffff0000u : 0u);
      r[k] &= keep;
    }
    ls[0] = ls[1] = ls[2] = ls[3] = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) add_f16x2_to_f32(ls[k & 3], r[k]);
  }
  st.l = st.l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
  st.m = m_use;
  if (i > 0 && __any_sync(0xffffffffu, resc)) {
    // O holds P.V of tiles < i: rescale this warp's rows once P(i-1).V has
    // landed (rows without a max move multiply by 1).  The P.V of the previous
    // tile is the (n_p - 1)-th; the next phase of its pv_done barrier needs
    // p_full from this tile.
    if (!wait_bar_warp(&cx.bars->pv_done[q][(st.n_p - 1) & 1], ((st.n_p - 1) >> 1) & 1,
                       cx.abort_flag, cx.tmo))
      return false;
    ptx::tc_fence_after();
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      ptx::tmem_ld32(cx.to + cc * 32, o);
      ptx::tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
      ptx::tmem_st32(cx.to + cc * 32, o);
    }
  }
  // P buffer sb held the P stored two tiles ago.  Its P.V was issued before
  // this tile's S by the same thread, and the commit that signalled S covers
  // every MMA issued before it: no wait needed.
  ptx::tmem_st32(cx.tp0 + 32 * sb, *reinterpret_cast<const uint32_t(*)[32]>(&r[0]));
  ptx::tmem_st_wait();
  ptx::tc_fence_before();
  ptx::mbar_arrive(&cx.bars->p_full[q][sb]);
  ++st.n_p;
  return true;
}

template <int D, bool kFp8>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ PrefillParams p) {
  using S = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + S::kOffBar);

  // A wait of an earlier launch already expired: do not start more work.
  if (*reinterpret_cast<volatile unsigned int*>(&g_status) & kStatusTimeout) return;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Persistent CTA: the first item is blockIdx.x, every later one comes from
  // the ticket (gridDim.x + ticket), in the heaviest-first order.
  const int num_items = p.max_qpairs * p.nseq * p.hq;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&bars->kv_full[i], 1);
      ptx::mbar_init(&bars->kv_empty[i], 2);  // one commit per MMA thread and key tile
    }
    for (int q = 0; q < 2; ++q) {
      ptx::mbar_init(&bars->q_full[q], 1);
      ptx::mbar_init(&bars->q_free[q], 1);
      for (int i = 0; i < 2; ++i) {
        ptx::mbar_init(&bars->p_full[q][i], 128);
        ptx::mbar_init(&bars->pv_done[q][i], 1);
      }
      ptx::mbar_init(&bars->o_final[q], 1);
      ptx::mbar_init(&bars->o_free[q], 128);
      ptx::mbar_init(&bars->s_full[q], 1);
      ptx::mbar_init(&bars->s_free[q], 128);
      ptx::mbar_init(&bars->drain[q], 1);
    }
    for (int i = 0; i < kItemSlots; ++i) {
      ptx::mbar_init(&bars->item_full[i], 1);
      ptx::mbar_init(&bars->item_empty[i], kItemConsumers);
    }
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

  if (warp == 0) {
    // ================= TMA producer =================
    // Per item: each Q tile (fp16 and int8) once its slot is free, then per
    // key tile the K tile in each precision the two rows' routing bits need
    // and the fp16 V tile, into the 3-stage ring, which runs on across items.
    if (lane == 0) {
      ptx::prefetch_tensormap(&p.tm_q);
      ptx::prefetch_tensormap(&p.tm_q8);
      ptx::prefetch_tensormap(&p.tm_k);
      ptx::prefetch_tensormap(&p.tm_k8);
      ptx::prefetch_tensormap(&p.tm_v);
      uint32_t kv_tiles = 0;              // key tiles issued so far (ring position)
      uint32_t q_loads[2] = {0u, 0u};     // loads of each Q slot so far
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        int w = k == 0 ? static_cast<int>(blockIdx.x)
                       : static_cast<int>(gridDim.x) + atomicAdd(p.ticket, 1);
        if (w >= num_items) w = -1;
        // publish it once every consumer has read the slot's previous item
        // (item_empty's next phase needs this publication)
        const int slot = k % kItemSlots;
        if (k >= kItemSlots &&
            !wait_bar(&bars->item_empty[slot], ((k / kItemSlots) - 1) & 1, abort_flag, tmo))
          break;
        *reinterpret_cast<volatile int*>(&bars->item_ring[slot]) = w;
        ptx::mbar_arrive(&bars->item_full[slot]);
        if (w < 0) break;
        WorkItem it;
        if (!load_item(p, w, it)) continue;
        // Q tile q's slot is refilled once the previous item's last S of it
        // completed (q_free's next phase needs this load).  Q tile 1 goes
        // after the item's first key tile, so that the shorter Q tile 0 can
        // start the item while Q tile 1 still finishes the previous one.
        const auto load_q = [&](int q) {
          if (q_loads[q] > 0 &&
              !wait_bar(&bars->q_free[q], (q_loads[q] - 1) & 1, abort_flag, tmo))
            return false;
          const int row = it.t0 + (it.qt0 + q) * BM;
          ptx::mbar_expect_tx(&bars->q_full[q], S::kQ + S::kQ8);
#pragma unroll
          for (int j = 0; j < D / 64; ++j)
            ptx::tma_load_3d(smem + S::kOffQ + q * S::kQ + j * BM * 128, &p.tm_q,
                             &bars->q_full[q], j * 64, it.h, row);
          ptx::tma_load_3d(smem + S::kOffQ8 + q * S::kQ8, &p.tm_q8, &bars->q_full[q], 0, it.h, row);
          ++q_loads[q];
          return true;
        };
        if (!load_q(0)) break;
        GroupCursor gc;
        for (int i = 0; ok && i < it.nt; ++i, gc.next(it.gs)) {
          const int st = kv_tiles % kStages;
          // K precisions the two rows need for this tile (at least one: i < nt)
          const bool b0 = gc.int8(it.w0), b1 = gc.int8(it.w1);
          const bool need8 = (i < it.nt0 && b0) || (i < it.nt1 && b1);
          const bool need16 = (i < it.nt0 && !b0) || (i < it.nt1 && !b1);
          // the stage's previous tile released by both MMA threads
          if (kv_tiles >= kStages &&
              !wait_bar(&bars->kv_empty[st], ((kv_tiles / kStages) - 1) & 1, abort_flag, tmo)) {
            ok = false;
            break;
          }
          const int key0 = it.t0 + i * BN;
          uint64_t* full = &bars->kv_full[st];
          ptx::mbar_expect_tx(full, (need16 ? S::kK16 : 0) + (need8 ? S::kK8 : 0) + S::kV);
          if (need16) {
#pragma unroll
            for (int j = 0; j < D / 64; ++j)
              ptx::tma_load_3d(smem + S::kOffK16 + st * S::kK16 + j * BN * 128, &p.tm_k, full,
                               j * 64, it.kv, key0);
          }
          if (need8)
            ptx::tma_load_3d(smem + S::kOffK8 + st * S::kK8, &p.tm_k8, full, 0, it.kv, key0);
#pragma unroll
          for (int j = 0; j < D / 64; ++j)
            ptx::tma_load_3d(smem + S::kOffV + st * S::kV + j * BN * 128, &p.tm_v, full, j * 64,
                             it.kv, key0);
          ++kv_tiles;
          if (i == 0 && it.nq == 2 && !load_q(1)) ok = false;
        }
      }
      // Never leave with copies into this CTA's shared memory in flight.
      for (int q = 0; q < 2; ++q)
        if (q_loads[q] > 0) drain_bar(&bars->q_full[q], (q_loads[q] - 1) & 1, tmo);
      for (uint32_t st = 0; st < kStages && st < kv_tiles; ++st)
        drain_bar(&bars->kv_full[st], ((kv_tiles - 1 - st) / kStages) & 1, tmo);
    }
  } else if (warp == 1 || warp == 2) {
    // ================= MMA issuers: warp 1 for Q tile 0, warp 2 for Q tile 1 =====
    // Per item, in key-tile order: S_q(0), then per key tile j: S_q(j + 1) as
    // soon as the softmax has read S_q(j) out of TMEM, then P_q(j).V once the
    // softmax has posted P_q(j).  Each thread releases every key tile of every
    // item (count 2 per stage): after its P.V, or once the tile has landed if
    // its Q tile does not use it (so that the arrival cannot count towards
    // the stage's previous tile).
    const int q = warp - 1;
    if (lane == 0) {
      const uint32_t a_smem = ptx::smem_addr(smem);
      const uint64_t t16 = ptx::smem_desc(0, 16, 1024, ptx::kSwizzle128B);
      const uint64_t t8 = ptx::smem_desc(0, 16, S::kI8Sbo, S::kI8Layout);
      const uint64_t tv = ptx::smem_desc(0, BN * 128, 1024, ptx::kSwizzle128B);
      const uint32_t aq16 = a_smem + S::kOffQ + q * S::kQ;
      const uint32_t aq8 = a_smem + S::kOffQ8 + q * S::kQ8;
      const uint32_t d_o = tmem + S::col_o(q);
      const uint32_t d_s = tmem + S::col_s(q);
      uint32_t kv_tiles = 0;  // key tiles of earlier items (ring position)
      uint32_t n_s = 0;       // S_q issued so far
      uint32_t n_p = 0;       // P_q.V issued so far
      uint32_t n_items = 0;   // items that had a Q tile q
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int w = next_item(bars, k, abort_flag, tmo, false);
        if (w == kItemAbort) {
          ok = false;
          break;
        }
        if (w < 0) break;
        WorkItem it;
        if (!load_item(p, w, it)) continue;
        const bool mine = q < it.nq;
        const int ntq = !mine ? 0 : (q ? it.nt1 : it.nt0);
        const uint64_t word = q ? it.w1 : it.w0;
        // q_full's next phase needs this item's last S, issued below
        if (mine && !wait_bar(&bars->q_full[q], n_items & 1, abort_flag, tmo)) {
          ok = false;
          break;
        }
        GroupCursor gc;  // routing group of tile i
        for (int i = 0; i <= it.nt; ++i) {
          if (i < it.nt) {
            const uint32_t t = kv_tiles + i;
            // S(n) overwrites S(n - 1) once the softmax has read it out
            if (i < ntq && n_s > 0 && !wait_bar(&bars->s_free[q], (n_s - 1) & 1, abort_flag, tmo)) {
              ok = false;
              break;
            }
            if (!wait_bar(&bars->kv_full[t % kStages], (t / kStages) & 1, abort_flag, tmo)) {
              ok = false;
              break;
            }
            if (i < ntq) {
              ptx::tc_fence_after();
              const int st = t % kStages;
              issue_qk<D, kFp8>(d_s, gc.int8(word), aq16, aq8, a_smem + S::kOffK16 + st * S::kK16,
                          a_smem + S::kOffK8 + st * S::kK8, t16, t8);
              ptx::mma_commit(&bars->s_full[q]);
              ++n_s;
              if (i == ntq - 1) ptx::mma_commit(&bars->q_free[q]);
            }
            gc.next(it.gs);
          }
          if (i >= 1) {
            const int j = i - 1;
            const int st = (kv_tiles + j) % kStages;
            if (j < ntq) {
              const int valid = it.L - j * BN;
              if (valid < BN) {
                // Keys past the sequence end belong to the next packed
                // sequence: zero their V rows so that 0 * (NaN or Inf) cannot
                // reach O.  Both Q tiles write the same zeros, each before its
                // own P.V.
                uint8_t* vslot = smem + S::kOffV + st * S::kV;
                for (int part = 0; part < D / 64; ++part)
                  for (int r = valid; r < BN; ++r) {
                    uint4* row = reinterpret_cast<uint4*>(vslot + part * BN * 128 + r * 128);
#pragma unroll
                    for (int c = 0; c < 8; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
                  }
                ptx::fence_proxy_async_smem();
              }
              // the first P.V of an item overwrites O_q: the previous item's
              // epilogue must have read it (o_free's next phase needs this
              // item's o_final)
              if (j == 0 && n_items > 0 &&
                  !wait_bar(&bars->o_free[q], (n_items - 1) & 1, abort_flag, tmo)) {
                ok = false;
                break;
              }
              const int pb = n_p & 1;
              if (!wait_bar(&bars->p_full[q][pb], (n_p >> 1) & 1, abort_flag, tmo)) {
                ok = false;
                break;
              }
              ptx::tc_fence_after();
              issue_pv<D>(d_o, tmem + S::col_p(q, pb), a_smem + S::kOffV + st * S::kV, tv, j == 0);
              ptx::mma_commit(&bars->pv_done[q][pb]);
              ++n_p;
              if (j == ntq - 1) ptx::mma_commit(&bars->o_final[q]);
            }
            ptx::mma_commit(&bars->kv_empty[st]);
          }
        }
        kv_tiles += it.nt;
        if (mine) ++n_items;
      }
      // all MMAs of this thread complete before TMEM and shared memory go away
      ptx::mma_commit(&bars->drain[q]);
      drain_bar(&bars->drain[q], 0, tmo);
    }
  } else if (warp >= kSoftmaxWarp0) {
    // ================= softmax / epilogue =================
    const int q = (warp - kSoftmaxWarp0) >> 2;        // Q tile of this warpgroup
    const int tr = threadIdx.x - (kSoftmaxWarp0 + 4 * q) * 32;  // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t n_s = 0;      // S_q read so far
    uint32_t n_p = 0;      // P_q stored so far
    uint32_t n_items = 0;  // items that had a Q tile q
    bool ok = true;
    uint32_t r[64];
    for (uint32_t k = 0; ok; ++k) {
      const int w = next_item(bars, k, abort_flag, tmo, true);
      if (w == kItemAbort) {
        ok = false;
        break;
      }
      if (w < 0) break;
      WorkItem it;
      if (!load_item(p, w, it)) continue;
      if (q >= it.nq) continue;
      const int h = it.h, s = it.s, kv = it.kv, t0 = it.t0, L = it.L, gs = it.gs;
      const int ntq = q ? it.nt1 : it.nt0;
      const uint64_t word = q ? it.w1 : it.w0;
      const int row0 = (it.qt0 + q) * BM;
      const int my_row = row0 + tr;
      const float q_sc = __ldg(p.q_scale + static_cast<size_t>(h) * p.total_qtiles + it.cq + it.qt0 + q);
      const float* ks = p.k_scale + static_cast<size_t>(kv) * p.total_ktiles + it.ck;
      (void)s;
      SoftmaxCtx cx;
      cx.p = &p;
      cx.bars = bars;
      cx.abort_flag = abort_flag;
      cx.tmo = tmo;
      cx.ts = tmem + lane_base + S::col_s(q);
      cx.to = tmem + lane_base + S::col_o(q);
      cx.tp0 = tmem + lane_base + S::col_p(q, 0);
      cx.q = q;
      cx.L = L;
      cx.row0 = row0;
      cx.my_row = my_row;
      cx.h = h;
      cx.t0 = t0;
      cx.ntq = ntq;
      cx.q_sc = q_sc;
      cx.ks = ks;
      RowState st;
      st.m = -INFINITY;
      st.l = 0.f;
      st.k_sc_next = __ldg(ks);
      st.n_s = n_s;
      st.n_p = n_p;
      // Key tiles before the first one that needs the legality mask (the
      // diagonal tiles of a causal row, a sequence's ragged last tile) run the
      // lean body, the rest the masked one; a debug run takes the body with
      // the INT32 dump for every tile.
      int i_hot = ntq;
      if (p.causal) i_hot = min(i_hot, row0 / BN);
      if (L % BN) i_hot = min(i_hot, L / BN);
      GroupCursor gc;
      int i = 0;
      if (p.dbg) {
        for (; i < ntq; ++i, gc.next(gs))
          if (!softmax_tile<D, true, true, kFp8>(cx, st, i, gc.int8(word), r)) {
            ok = false;
            break;
          }
      }
      for (; ok && i < i_hot; ++i, gc.next(gs))
        if (!softmax_tile<D, false, false, kFp8>(cx, st, i, gc.int8(word), r)) {
          ok = false;
          break;
        }
      for (; ok && i < ntq; ++i, gc.next(gs))
        if (!softmax_tile<D, true, false, kFp8>(cx, st, i, gc.int8(word), r)) {
          ok = false;
          break;
        }
      n_s = st.n_s;
      n_p = st.n_p;
      const float m = st.m, l = st.l;
      // o_final's next phase needs o_free from this epilogue
      if (!ok || !wait_bar_warp(&bars->o_final[q], n_items & 1, abort_flag, tmo)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const float inv_l = 1.0f / l;
      const bool valid = my_row < L;
      __half* orow = static_cast<__half*>(p.o) + (static_cast<size_t>(t0 + my_row) * p.hq + h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        ptx::tmem_ld32(tmem + lane_base + S::col_o(q) + cc * 32,
                       *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        ptx::tmem_ld_wait();
        if (cc == D / 32 - 1) {
          // O_q is in registers: the next item's first P.V may overwrite it
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bars->o_free[q]);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j)
          r[32 + j] = pack_f16x2(__uint_as_float(r[2 * j]) * inv_l,
                                 __uint_as_float(r[2 * j + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(r[32 + 4 * j], r[33 + 4 * j], r[34 + 4 * j], r[35 + 4 * j]);
        }
      }
      if (p.lse && valid)
        p.lse[static_cast<size_t>(h) * p.total_tokens + t0 + my_row] =
            (m + __log2f(l)) * 0.69314718055994530942f;
      ++n_items;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kFp8>
static int launch_prefill_d(const PrefillParams& p, cudaStream_t stream) {
  const int smem = Smem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(prefill_fwd_kernel<D, kFp8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return static_cast<int>(e);
  const long long items = static_cast<long long>(p.max_qpairs) * p.nseq * p.hq;
  if (items == 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  // persistent: one CTA per SM (the shared memory admits one), each walking
  // every gridDim.x-th work item
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return static_cast<int>(e);
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return static_cast<int>(e);
  const unsigned blocks = static_cast<unsigned>(items < sms ? items : sms);
  prefill_fwd_kernel<D, kFp8><<<blocks, kPrefillThreads, smem, stream>>>(p);
  return static_cast<int>(cudaGetLastError());
}

int launch_prefill(const PrefillParams& p, int d, cudaStream_t stream) {
  if (d == 128) return p.low_fp8 ? launch_prefill_d<128, true>(p, stream)
                                 : launch_prefill_d<128, false>(p, stream);
  if (d == 64) return p.low_fp8 ? launch_prefill_d<64, true>(p, stream)
                                : launch_prefill_d<64, false>(p, stream);
  return cudaErrorInvalidValue;
}

// Failure-path self test: one warp waits on an mbarrier that nothing ever
// arrives on; the bounded wait must give up and latch kStatusTimeout.
__global__ void selftest_wait_kernel(unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  wait_bar(&bar, 0, &abort_flag, timeout_ns);
}

int launch_selftest_wait(unsigned long long timeout_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(timeout_ns);
  return static_cast<int>(cudaGetLastError());
}

// Scratch of the allocation-free entry point: module-scope device memory,
// present on every GPU that loads this library.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TILEMIX_NOALLOC_SCRATCH_BYTES];

// Identity of the calling thread's current CUDA context (never reused within a
// process, unlike the context handle): false if no context is current or the
// driver calls are unavailable.
static bool current_context_id(unsigned long long* id) {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(f);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

int noalloc_scratch(void** ptr) {
  // The array's device address belongs to the context the library's module
  // was loaded into: it is looked up once per context (each device's primary
  // context, or a context the caller made current), so a context created
  // later -- after cudaDeviceReset, say -- gets its own lookup instead of a
  // stale address.  Host code cannot take the symbol's address directly.
  struct Entry {
    unsigned long long ctx;
    void* addr;
  };
  static std::mutex mu;
  static Entry cache[16];
  static int used = 0, next = 0;
  unsigned long long id = 0;
  bool known = current_context_id(&id);
  std::lock_guard<std::mutex> lock(mu);
  if (known)
    for (int i = 0; i < used; ++i)
      if (cache[i].ctx == id) {
        *ptr = cache[i].addr;
        return cudaSuccess;
      }
  void* p = nullptr;
  // also makes the runtime's context current on this thread if none was
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (!known) known = current_context_id(&id);
  if (known) {
    cache[next] = Entry{id, p};
    next = (next + 1) % 16;
    if (used < 16) ++used;
  }
  *ptr = p;
  return cudaSuccess;
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

#include "tilemix_decode.cuh"
