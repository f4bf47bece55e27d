// Host-side routing-word builder and tile geometry helpers of the C ABI.
//
// Static, data-free precision templates borrowed from sparse attention
// ("TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
// Acceleration", agihunt.info summary, method paragraphs): Band keeps the
// diagonal local, Global keeps designated positions, Row-Random keeps random
// FP16 groups per row, Aligned-Sparse extends right-aligned, BigBird is the
// union of the first three, SpTrans uses a stride plus a tail.  Coverage counts
// legal tile groups, and one template is reused for every KV head.
//
// Each template is built as an FP16 bit set per query-tile row; the word is the
// legal-group set minus that FP16 set.  Row geometry, quota rules and the
// per-row draw streams are the readings written down in the design notes:
//   legal groups n_r   = last legal key tile / g + 1
//   INT8 target        = floor((p * N + 50) / 100) per sequence, N = sum n_r
//   fixed width (Band, Global): widest w with sum min(w, n_r) <= N - K; the
//     remainder adds one group, rows in ascending order, to rows wider than w
//   quota (the other four): k_r = floor(p n_r / 100), remainder units to rows
//     with the largest (p n_r mod 100), ties to the lower row
//   row stream: splitmix64 state = output (row + 1) of the stream at `seed`.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "tilemix.h"
#include "tilemix_internal.h"

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

// splitmix64 (Steele, Lea & Flood 2014), written as the usual stateful
// generator: advance, then finalise.
struct SplitMix {
  uint64_t state;
  uint64_t next() {
    state += kGolden;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

uint64_t row_stream_state(uint64_t seed, int row) {
  SplitMix m{seed};
  uint64_t out = 0;
  for (int i = 0; i <= row; ++i) out = m.next();
  return out;
}

inline uint64_t low_bits(int n) { return n >= 64 ? ~0ull : ((1ull << n) - 1ull); }
inline uint64_t bit_range(int lo, int hi) {  // bits [lo, hi)
  if (hi <= lo) return 0ull;
  return low_bits(hi) & ~low_bits(lo);
}

// Draw `count` distinct entries of `pool` with the partial Fisher-Yates walk
// j = i + r mod (size - i); returns them as a bit set.
uint64_t shuffle_pick(std::vector<int> pool, int count, uint64_t state) {
  SplitMix m{state};
  uint64_t bits = 0;
  const int size = static_cast<int>(pool.size());
  for (int i = 0; i < count; ++i) {
    uint64_t r = m.next();
    int j = i + static_cast<int>(r % static_cast<uint64_t>(size - i));
    std::swap(pool[i], pool[j]);
    bits |= 1ull << pool[i];
  }
  return bits;
}

void fixed_width_counts(const std::vector<int>& n, long long fp16_total, std::vector<int>& out) {
  int widest = 0;
  for (int x : n) widest = std::max(widest, x);
  // sum_r min(w, n_r) is non-decreasing in w: find the widest w that fits.
  auto cost = [&](int w) {
    long long c = 0;
    for (int x : n) c += std::min(w, x);
    return c;
  };
  int w = 0;
  while (w < widest && cost(w + 1) <= fp16_total) ++w;
  long long spare = fp16_total - cost(w);
  out.resize(n.size());
  for (size_t r = 0; r < n.size(); ++r) {
    out[r] = std::min(w, n[r]);
    if (n[r] > w && spare > 0) {
      ++out[r];
      --spare;
    }
  }
}

void quota_counts(const std::vector<int>& n, int pct, long long target, std::vector<int>& k8) {
  const size_t rows = n.size();
  k8.resize(rows);
  std::vector<int> rem(rows);
  long long assigned = 0;
  for (size_t r = 0; r < rows; ++r) {
    k8[r] = pct * n[r] / 100;
    rem[r] = pct * n[r] % 100;
    assigned += k8[r];
  }
  std::vector<int> order(rows);
  for (size_t r = 0; r < rows; ++r) order[r] = static_cast<int>(r);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return rem[a] > rem[b]; });
  for (long long u = 0; u < target - assigned; ++u) ++k8[order[static_cast<size_t>(u)]];
}

// FP16 bit set of one row for the quota templates.
uint64_t quota_row_fp16(int tpl, int n, int f, uint64_t seed, int row) {
  switch (tpl) {
    case TILEMIX_ALIGNED_SPARSE:
      return bit_range(n - f, n);
    case TILEMIX_ROW_RANDOM: {
      std::vector<int> pool(n);
      for (int i = 0; i < n; ++i) pool[i] = i;
      return shuffle_pick(pool, f, row_stream_state(seed, row));
    }
    case TILEMIX_BIGBIRD: {
      const int left = (f + 2) / 3;
      const int right = (f - left + 1) / 2;
      uint64_t bits = bit_range(0, left) | bit_range(n - right, n);
      std::vector<int> middle;
      for (int i = left; i < n - right; ++i) middle.push_back(i);
      return bits | shuffle_pick(middle, f - left - right, row_stream_state(seed, row));
    }
    case TILEMIX_SPTRANS: {
      uint64_t bits = 0;
      int taken = 0;
      auto take = [&](int b) {
        if (taken < f && b >= 0 && !((bits >> b) & 1ull)) {
          bits |= 1ull << b;
          ++taken;
        }
      };
      take(n - 1);  // tail: the two groups nearest the diagonal
      take(n - 2);
      for (int residue = 7; residue >= 0 && taken < f; --residue) {
        // groups b with b % 8 == residue, right to left
        int top = n - 1 - (((n - 1 - residue) % 8) + 8) % 8;
        for (int b = top; b >= 0 && taken < f; b -= 8) take(b);
      }
      return bits;
    }
    default:
      return 0;
  }
}

}  // namespace

extern "C" {

TILEMIX_API int tilemix_auto_g(int seqlen, int* g_out) {
  if (!g_out || seqlen < 0) return TILEMIX_ERR_INVALID_ARG;
  const int tiles = (seqlen + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N;
  int g = (tiles + TILEMIX_MAX_GROUPS - 1) / TILEMIX_MAX_GROUPS;
  *g_out = g < 1 ? 1 : g;
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_host_runs(const int32_t* cu_seqlens_h, int nseq, int chunks,
                                  int32_t* run_start_h, int* nruns) {
  if (!cu_seqlens_h || !run_start_h || !nruns || nseq < 0 || chunks < 1)
    return TILEMIX_ERR_INVALID_ARG;
  if (cu_seqlens_h[0] != 0) return TILEMIX_ERR_INVALID_ARG;
  for (int s = 0; s < nseq; ++s)
    if (cu_seqlens_h[s + 1] < cu_seqlens_h[s]) return TILEMIX_ERR_INVALID_ARG;
  const int n = chunks < nseq ? chunks : nseq;
  int r = 0, s0 = 0;
  run_start_h[0] = 0;
  for (int c = 0; c < n && s0 < nseq; ++c) {
    s0 = tilemix::run_end(cu_seqlens_h, nseq, n, c, s0);
    run_start_h[++r] = s0;
  }
  *nruns = r;
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_tile_offsets(const int32_t* cu_seqlens_h, int nseq, int32_t* cu_qtiles_h,
                                     int32_t* cu_ktiles_h) {
  if (!cu_seqlens_h || !cu_qtiles_h || !cu_ktiles_h || nseq < 0) return TILEMIX_ERR_INVALID_ARG;
  if (cu_seqlens_h[0] != 0) return TILEMIX_ERR_INVALID_ARG;
  long long qsum = 0, ksum = 0;
  cu_qtiles_h[0] = 0;
  cu_ktiles_h[0] = 0;
  for (int s = 0; s < nseq; ++s) {
    const long long L = static_cast<long long>(cu_seqlens_h[s + 1]) - cu_seqlens_h[s];
    if (L < 0) return TILEMIX_ERR_INVALID_ARG;
    qsum += (L + TILEMIX_BLOCK_M - 1) / TILEMIX_BLOCK_M;
    ksum += (L + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N;
    if (ksum > INT32_MAX) return TILEMIX_ERR_INVALID_ARG;
    cu_qtiles_h[s + 1] = static_cast<int32_t>(qsum);
    cu_ktiles_h[s + 1] = static_cast<int32_t>(ksum);
  }
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_build_routing(int tpl, int int8_percent, uint64_t seed,
                                      const int32_t* cu_seqlens_h, int nseq, int n_kv_heads,
                                      const int32_t* g_h, int causal, uint64_t* masks_h,
                                      int64_t* legal_groups_h, int64_t* int8_groups_h) {
  if (tpl < TILEMIX_BAND || tpl > TILEMIX_SPTRANS) return TILEMIX_ERR_INVALID_ARG;
  if (int8_percent < 0 || int8_percent > 100) return TILEMIX_ERR_INVALID_ARG;
  if (!cu_seqlens_h || !g_h || !masks_h || nseq < 0 || n_kv_heads < 1) return TILEMIX_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return TILEMIX_ERR_INVALID_ARG;
  if (cu_seqlens_h[0] != 0) return TILEMIX_ERR_INVALID_ARG;
  size_t out_row = 0;
  std::vector<int> n, widths, k8;
  for (int s = 0; s < nseq; ++s) {
    const int L = cu_seqlens_h[s + 1] - cu_seqlens_h[s];
    const int g = g_h[s];
    if (L < 0 || g < 1) return TILEMIX_ERR_INVALID_ARG;
    const int rows = (L + TILEMIX_BLOCK_M - 1) / TILEMIX_BLOCK_M;
    const int ktiles = (L + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N;
    n.assign(rows, 0);
    long long total = 0;
    for (int r = 0; r < rows; ++r) {
      int last_key = causal ? std::min((r + 1) * TILEMIX_BLOCK_M, L) - 1 : L - 1;
      int last_tile = causal ? last_key / TILEMIX_BLOCK_N : ktiles - 1;
      n[r] = last_tile / g + 1;
      if (n[r] > TILEMIX_MAX_GROUPS) return TILEMIX_ERR_INVALID_ARG;
      total += n[r];
    }
    const long long target = (static_cast<long long>(int8_percent) * total + 50) / 100;
    long long ones = 0;
    const bool fixed = (tpl == TILEMIX_BAND || tpl == TILEMIX_GLOBAL);
    if (fixed) fixed_width_counts(n, total - target, widths);
    else quota_counts(n, int8_percent, target, k8);
    for (int r = 0; r < rows; ++r) {
      uint64_t fp16;
      if (fixed) {
        fp16 = (tpl == TILEMIX_BAND) ? bit_range(n[r] - widths[r], n[r]) : bit_range(0, widths[r]);
      } else {
        fp16 = quota_row_fp16(tpl, n[r], n[r] - k8[r], seed, r);
      }
      const uint64_t word = low_bits(n[r]) & ~fp16;
      ones += __builtin_popcountll(word);
      for (int h = 0; h < n_kv_heads; ++h) masks_h[out_row * n_kv_heads + h] = word;
      ++out_row;
    }
    if (legal_groups_h) legal_groups_h[s] = total;
    if (int8_groups_h) int8_groups_h[s] = ones;
  }
  return TILEMIX_OK;
}

}  // extern "C"
