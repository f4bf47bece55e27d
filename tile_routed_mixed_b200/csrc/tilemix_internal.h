// Internal declarations shared by the host API and the kernel translation unit.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#define TILEMIX_API __attribute__((visibility("default")))

namespace tilemix {

// Bits of the device status word.
enum : unsigned int {
  kStatusTimeout = 1u,       // a bounded mbarrier wait expired
  kStatusBadGroups = 2u,     // a row needed a routing group index above 63
  kStatusBadHeadMap = 4u,    // a head-map entry outside [0, hk)
};


// Everything the fused attention kernel needs, by value (kernel parameter).
struct PrefillParams {
  CUtensorMap tm_q;    // fp16 Q   [T][hq][d], box {64, 1, 128}, 128B swizzle
  CUtensorMap tm_q8;   // int8 Q   [T][hq][d], box {d, 1, 128}
  CUtensorMap tm_k;    // fp16 K   [T][hk][d], box {64, 1, 64}, 128B swizzle
  CUtensorMap tm_k8;   // int8 K   [T][hk][d], box {d, 1, 64}
  CUtensorMap tm_v;    // fp16 V   [T][hk][d], box {64, 1, 64}, 128B swizzle
  void* o;
  float* lse;
  const int32_t* cu_seqlens;
  const int32_t* cu_qtiles;
  const int32_t* cu_ktiles;
  const int32_t* kv_head_of_q;
  const uint64_t* masks;
  const int32_t* g;
  const float* q_scale;   // [hq][total_qtiles]
  const float* k_scale;   // [hk][total_ktiles]
  int32_t* dbg;
  int* ticket;            // work-item ticket, zero at launch (see launch_quantize_qk)
  int dbg_cols;
  int nseq, total_tokens, total_qtiles, total_ktiles, max_qpairs;
  int hq, hk, group;      // group = hq / hk
  int causal;
  float scale_log2;       // softmax scale * log2(e)
  int low_fp8;            // low-precision tiles: 0 integer codes (INT8 or INT4, kind::i8),
                          // 1 FP8 e4m3 (kind::f8f6f4)
  unsigned long long timeout_ns;
};

// Everything the decode kernels need (see tilemix_decode_fwd).
struct DecodeParams {
  CUtensorMap tm_k;          // fp16 K   [cache rows][hk][d], box {64, 1, 64}, 128B swizzle
  CUtensorMap tm_k8;         // int8 K   [cache rows][hk][d], box {d, 1, 64}
  CUtensorMap tm_v;          // fp16 V   [cache rows][hk][d], box {64, 1, 64}, 128B swizzle
  const void* q;             // fp16 [nseq][hq][d]
  const void* k;             // fp16 [cache rows][hk][d]
  const void* v;             // fp16 [cache rows][hk][d]
  int8_t* k_i8;              // int8 [cache rows][hk][d] (last blocks rewritten)
  float* k_scale;            // [hk][total_ktiles] (last blocks rewritten)
  void* o;                   // fp16 [nseq][hq][d]
  const int32_t* seq_start;  // [nseq]
  const int32_t* seq_len;    // [nseq]
  const int32_t* ktile_start;
  const int32_t* qtile_start;
  const uint64_t* masks;
  const int32_t* g;
  const int32_t* kv_head_of_q;
  float* part_m;             // workspace: [nseq][hq][nsplit]
  float* part_l;             // workspace: [nseq][hq][nsplit]
  float* part_acc;           // workspace: [nseq][hq][nsplit][d]
  int* counters;             // workspace: [nseq][hk] finished splits (zeroed per call)
  int nseq, hq, hk, d, group, total_ktiles, nsplit, tiles_per_split;
  float scale_log2;
  unsigned long long timeout_ns;
};

// Pooled-score routing (tilemix_route.cu).
struct RouteParams {
  const void* q;             // fp16 [T][hq][d]
  const void* k;             // fp16 [T][hk][d]
  const int32_t* cu_seqlens;
  const int32_t* cu_qtiles;
  const int32_t* cu_ktiles;
  const int32_t* g;
  const int32_t* kv_head_of_q;
  float* qbar;               // workspace: [total_qtiles][hk][d]
  float* kbar;               // workspace: [total_ktiles][hk][d]
  uint64_t* masks;           // [total_qtiles][hk]
  int nseq, hq, hk, d, causal, int8_percent, total_qtiles, total_ktiles;
};
int launch_route(const RouteParams& p, cudaStream_t stream);

// Importance-mass exposure probe (tilemix_mass.cu).
struct MassParams {
  const void* q;             // fp16 [T][hq][d]
  const void* k;             // fp16 [T][hk][d]
  const int32_t* cu_seqlens;
  const int32_t* cu_qtiles;
  const int32_t* cu_ktiles;  // also the offsets of the 64-row query blocks
  const uint64_t* masks;     // [total_qtiles][hk]
  const int32_t* g;
  const int32_t* kv_head_of_q;
  float* m8;                 // [hq][T]
  float* h;                  // [hq][T]
  float* h8;                 // [hq][T]
  int nseq, hq, hk, d, causal, total_blocks, total_tokens;
  float scale_log2, delta_log2;
};
int launch_mass_probe(const MassParams& p, cudaStream_t stream);

// Launchers implemented in the CUDA translation unit.  Return cudaError_t.
int launch_decode(const DecodeParams& p, cudaStream_t stream, cudaEvent_t ev_begin,
                  cudaEvent_t ev_end);
// One launch quantises Q (128-row blocks) and K (64-row blocks); a null q or
// k skips that side.  A non-null ticket is set to zero by the same launch
// (the fused kernel that follows on the stream hands out work from it).
// Runs of whole sequences for the host-buffer prefill: run c (c < chunks)
// starts at sequence s0 and ends before the returned s1, the first s > s0
// whose token offset cu[s] reaches (c + 1) / chunks of the batch (the last
// run takes every remaining sequence).  Host code; cu has nseq + 1 entries.
inline int run_end(const int32_t* cu, int nseq, int chunks, int c, int s0) {
  const long long target = static_cast<long long>(cu[nseq]) * (c + 1) / chunks;
  int s1 = s0 + 1;
  while (s1 < nseq && (c == chunks - 1 || cu[s1] < target)) ++s1;
  return s1;
}

// Tiles a quantisation launch covers: Q tiles qtile0 .. qtile0 + nqtiles - 1
// and K tiles ktile0 .. ktile0 + nktiles - 1, those of the nseq sequences
// whose offsets cu_seqlens / cu_qtiles / cu_ktiles point at (a whole batch, or
// a run of its sequences with the pointers advanced to the run's first).
struct QuantRange {
  int qtile0, nqtiles, ktile0, nktiles;
};
int launch_quantize_qk(const void* q, const void* k, const int32_t* cu_seqlens,
                       const int32_t* cu_qtiles, const int32_t* cu_ktiles, int nseq,
                       const QuantRange& range, int total_qtiles, int total_ktiles, int hq,
                       int hk, int d, int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                       int* ticket, int fmt, cudaStream_t stream);  // fmt: 0 INT8, 1 FP8, 2 INT4
int launch_prefill(const PrefillParams& p, int d, cudaStream_t stream);
int read_and_clear_status(unsigned int* status, cudaStream_t stream);
// Device address of the allocation-free entry point's scratch array in the
// calling thread's current context (looked up once per context).
int noalloc_scratch(void** ptr);
int launch_selftest_wait(unsigned long long timeout_ns, cudaStream_t stream);

}  // namespace tilemix
