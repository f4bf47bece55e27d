// Host side of the C ABI: argument checks, workspace layout, TMA descriptor
// encoding and the kernel launch sequence.  Allocates no memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "tilemix.h"
#include "tilemix_internal.h"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

unsigned long long wait_timeout_ns() {
  static unsigned long long ns = [] {
    const char* env = std::getenv("TILEMIX_WAIT_TIMEOUT_MS");
    long long ms = env ? std::atoll(env) : 2000;
    if (ms < 1) ms = 1;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return ns;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Packed [rows][heads][d] tensor as a 3-D TMA map {d, heads, rows} with a box
// of {box_inner, 1, box_rows} elements and the given swizzle.
int encode_rows(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                int rows, int heads, int d, int box_inner, int box_rows,
                CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return TILEMIX_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem_bytes,
                                 static_cast<cuuint64_t>(d) * heads * elem_bytes};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 1u,
                             static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TILEMIX_OK : TILEMIX_ERR_CUDA;
}

struct WorkspaceLayout {
  size_t q8, q_scale, k8, k_scale, ticket, total;
};

WorkspaceLayout layout_of(const tilemix_prefill_args* a) {
  WorkspaceLayout w{};
  const size_t T = static_cast<size_t>(a->total_tokens);
  size_t off = 0;
  w.q8 = off;
  off = round_up(off + T * a->hq * a->d, 256);
  w.q_scale = off;
  off = round_up(off + sizeof(float) * a->hq * static_cast<size_t>(a->total_qtiles), 256);
  const bool own_k = a->k_i8 == nullptr;
  w.k8 = off;
  if (own_k) off = round_up(off + T * a->hk * a->d, 256);
  w.k_scale = off;
  if (own_k) off = round_up(off + sizeof(float) * a->hk * static_cast<size_t>(a->total_ktiles), 256);
  w.ticket = off;  // work-item counter of the fused kernel
  off += 256;
  w.total = off;
  return w;
}

int check_args(const tilemix_prefill_args* a) {
  if (!a) return TILEMIX_ERR_INVALID_ARG;
  if (a->d != 64 && a->d != 128) return TILEMIX_ERR_UNSUPPORTED;
  if (a->hq < 1 || a->hk < 1 || a->hq % a->hk != 0) return TILEMIX_ERR_INVALID_ARG;
  if (a->nseq < 0 || a->total_tokens < 0 || a->total_qtiles < 0 || a->total_ktiles < 0 ||
      a->max_seqlen < 0)
    return TILEMIX_ERR_INVALID_ARG;
  if (a->causal != 0 && a->causal != 1) return TILEMIX_ERR_INVALID_ARG;
  if (!(a->softmax_scale >= 0.f) || std::isinf(a->softmax_scale)) return TILEMIX_ERR_INVALID_ARG;
  if ((a->k_i8 == nullptr) != (a->k_scale == nullptr)) return TILEMIX_ERR_INVALID_ARG;
  if (a->low_format < 0 || a->low_format > 2) return TILEMIX_ERR_INVALID_ARG;
  if (a->low_format == 1 && a->debug_int32_scores) return TILEMIX_ERR_UNSUPPORTED;
  if (a->nseq == 0 || a->total_tokens == 0) return TILEMIX_OK;  // nothing to do
  if (!a->q || !a->k || !a->v || !a->o || !a->cu_seqlens || !a->cu_qtiles || !a->cu_ktiles ||
      !a->masks || !a->g)
    return TILEMIX_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o) ||
      (a->k_i8 && !aligned16(a->k_i8)))
    return TILEMIX_ERR_INVALID_ARG;
  if (a->max_seqlen < 1) return TILEMIX_ERR_INVALID_ARG;
  return TILEMIX_OK;
}

// Quantisation of the INT8 operands; a non-null ticket is zeroed by the
// same launch.
int quantize_impl(const void* q_f16, const void* k_f16, const int32_t* cu_seqlens_d,
                  const int32_t* cu_qtiles_d, const int32_t* cu_ktiles_d, int nseq,
                  int total_tokens, const tilemix::QuantRange& range, int total_qtiles,
                  int total_ktiles, int hq, int hk, int d, int8_t* q_i8, float* q_scale,
                  int8_t* k_i8, float* k_scale, int* ticket, int fmt, void* stream) {
  if (d != 64 && d != 128) return TILEMIX_ERR_UNSUPPORTED;
  if (nseq < 0 || total_tokens < 0 || total_qtiles < 0 || total_ktiles < 0)
    return TILEMIX_ERR_INVALID_ARG;
  if (nseq == 0 || total_tokens == 0) return TILEMIX_OK;
  if (!cu_seqlens_d) return TILEMIX_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (q_f16) {
    if (hq < 1 || !cu_qtiles_d || !q_i8 || !q_scale || !aligned16(q_f16) ||
        (reinterpret_cast<uintptr_t>(q_i8) & 7u))
      return TILEMIX_ERR_INVALID_ARG;
  }
  if (k_f16) {
    if (hk < 1 || !cu_ktiles_d || !k_i8 || !k_scale || !aligned16(k_f16) ||
        (reinterpret_cast<uintptr_t>(k_i8) & 7u))
      return TILEMIX_ERR_INVALID_ARG;
  }
  if (tilemix::launch_quantize_qk(q_f16, k_f16, cu_seqlens_d, cu_qtiles_d, cu_ktiles_d, nseq,
                                  range, total_qtiles, total_ktiles, hq, hk, d, q_i8, q_scale,
                                  k_i8, k_scale, ticket, fmt, st) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  return TILEMIX_OK;
}

// What one prefill call shares between the runs of sequences it enqueues:
// the workspace carve-up and the kernel parameters (tensor maps over the
// whole batch's buffers).
struct PrefillPlan {
  tilemix::PrefillParams p;
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  float* k_scale;
  int* ticket;
  bool events;  // record event_kernel_begin / end around the attention launch
};

// Needs check_args(a) == OK and a non-empty batch.
int plan_prefill(const tilemix_prefill_args* a, PrefillPlan* pl) {
  const WorkspaceLayout w = layout_of(a);
  if (!a->workspace || a->workspace_bytes < w.total ||
      (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return TILEMIX_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  pl->q8 = reinterpret_cast<int8_t*>(ws + w.q8);
  pl->q_scale = reinterpret_cast<float*>(ws + w.q_scale);
  pl->k8 = a->k_i8 ? const_cast<int8_t*>(a->k_i8) : reinterpret_cast<int8_t*>(ws + w.k8);
  pl->k_scale = a->k_i8 ? const_cast<float*>(a->k_scale) : reinterpret_cast<float*>(ws + w.k_scale);
  pl->ticket = reinterpret_cast<int*>(ws + w.ticket);
  pl->events = false;

  tilemix::PrefillParams& p = pl->p;
  std::memset(&p, 0, sizeof(p));
  const int T = a->total_tokens, d = a->d;
  int rc;
  const CUtensorMapSwizzle sw8 =
      d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if ((rc = encode_rows(&p.tm_q, a->q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, T, a->hq, d, 64,
                        TILEMIX_BLOCK_M, CU_TENSOR_MAP_SWIZZLE_128B)) != TILEMIX_OK)
    return rc;
  if ((rc = encode_rows(&p.tm_q8, pl->q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, T, a->hq, d, d,
                        TILEMIX_BLOCK_M, sw8)) != TILEMIX_OK)
    return rc;
  if ((rc = encode_rows(&p.tm_k, a->k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, T, a->hk, d, 64,
                        TILEMIX_BLOCK_N, CU_TENSOR_MAP_SWIZZLE_128B)) != TILEMIX_OK)
    return rc;
  if ((rc = encode_rows(&p.tm_k8, pl->k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, T, a->hk, d, d,
                        TILEMIX_BLOCK_N, sw8)) != TILEMIX_OK)
    return rc;
  if ((rc = encode_rows(&p.tm_v, a->v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, T, a->hk, d, 64,
                        TILEMIX_BLOCK_N, CU_TENSOR_MAP_SWIZZLE_128B)) != TILEMIX_OK)
    return rc;
  p.o = a->o;
  p.lse = a->lse;
  p.kv_head_of_q = a->kv_head_of_q;
  p.masks = a->masks;
  p.q_scale = pl->q_scale;
  p.k_scale = pl->k_scale;
  p.dbg = a->debug_int32_scores;
  p.ticket = pl->ticket;
  p.dbg_cols = (a->max_seqlen + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N * TILEMIX_BLOCK_N;
  p.total_tokens = T;
  p.total_qtiles = a->total_qtiles;
  p.total_ktiles = a->total_ktiles;
  p.hq = a->hq;
  p.hk = a->hk;
  p.group = a->hq / a->hk;
  p.causal = a->causal;
  const float scale = a->softmax_scale > 0.f ? a->softmax_scale : 1.0f / std::sqrt(float(d));
  p.scale_log2 = scale * 1.4426950408889634f;
  p.low_fp8 = a->low_format == 1;  // INT4 codes take the INT8 MMA path
  p.timeout_ns = wait_timeout_ns();
  return TILEMIX_OK;
}

// Quantisation and attention of sequences s0 .. s1 - 1 (their tiles `range`,
// their longest sequence max_seqlen) on `st`.  Offsets stay absolute: the
// sequence arrays are read from s0 on, every tensor and workspace array is
// addressed as for the whole batch, so the runs of one call touch disjoint
// rows and the same codes, scales and outputs come out as from one run.
int run_prefill_range(const tilemix_prefill_args* a, PrefillPlan& pl, int s0, int s1,
                      const tilemix::QuantRange& range, int max_seqlen, cudaStream_t st) {
  int rc = quantize_impl(a->q, a->k_i8 ? nullptr : a->k, a->cu_seqlens + s0, a->cu_qtiles + s0,
                         a->cu_ktiles + s0, s1 - s0, a->total_tokens, range, a->total_qtiles,
                         a->total_ktiles, a->hq, a->hk, a->d, pl.q8, pl.q_scale, pl.k8,
                         pl.k_scale, pl.ticket, a->low_format, st);
  if (rc != TILEMIX_OK) return rc;
  tilemix::PrefillParams p = pl.p;
  p.cu_seqlens = a->cu_seqlens + s0;
  p.cu_qtiles = a->cu_qtiles + s0;
  p.cu_ktiles = a->cu_ktiles + s0;
  p.g = a->g + s0;
  p.nseq = s1 - s0;
  p.max_qpairs = ((max_seqlen + TILEMIX_BLOCK_M - 1) / TILEMIX_BLOCK_M + 1) / 2;
  if (pl.events && a->event_kernel_begin &&
      cudaEventRecord(static_cast<cudaEvent_t>(a->event_kernel_begin), st) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  if (tilemix::launch_prefill(p, a->d, st) != cudaSuccess) return TILEMIX_ERR_CUDA;
  if (pl.events && a->event_kernel_end &&
      cudaEventRecord(static_cast<cudaEvent_t>(a->event_kernel_end), st) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  return TILEMIX_OK;
}

}  // namespace

extern "C" {

TILEMIX_API int tilemix_version(void) { return TILEMIX_VERSION; }

TILEMIX_API const char* tilemix_status_string(int status) {
  switch (status) {
    case TILEMIX_OK: return "ok";
    case TILEMIX_ERR_INVALID_ARG: return "invalid argument";
    case TILEMIX_ERR_UNSUPPORTED: return "unsupported configuration";
    case TILEMIX_ERR_CUDA: return "CUDA error";
    case TILEMIX_ERR_TIMEOUT: return "device wait timed out";
    case TILEMIX_ERR_WORKSPACE: return "workspace missing or too small";
    case TILEMIX_ERR_TOO_LARGE:
      return "workspace needed exceeds the 64 MiB scratch of tilemix_prefill_fwd_noalloc";
    default: return "unknown status";
  }
}

TILEMIX_API int tilemix_quantize_qk(const void* q_f16, const void* k_f16,
                                    const int32_t* cu_seqlens_d, const int32_t* cu_qtiles_d,
                                    const int32_t* cu_ktiles_d, int nseq, int total_tokens,
                                    int total_qtiles, int total_ktiles, int hq, int hk, int d,
                                    int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale,
                                    void* stream) {
  return quantize_impl(q_f16, k_f16, cu_seqlens_d, cu_qtiles_d, cu_ktiles_d, nseq, total_tokens,
                       {0, total_qtiles, 0, total_ktiles}, total_qtiles, total_ktiles, hq, hk, d,
                       q_i8, q_scale, k_i8, k_scale, nullptr, 0, stream);
}

TILEMIX_API int tilemix_quantize_qk_fp8(const void* q_f16, const void* k_f16,
                                        const int32_t* cu_seqlens_d, const int32_t* cu_qtiles_d,
                                        const int32_t* cu_ktiles_d, int nseq, int total_tokens,
                                        int total_qtiles, int total_ktiles, int hq, int hk, int d,
                                        int8_t* q_codes, float* q_scale, int8_t* k_codes,
                                        float* k_scale, void* stream) {
  return quantize_impl(q_f16, k_f16, cu_seqlens_d, cu_qtiles_d, cu_ktiles_d, nseq, total_tokens,
                       {0, total_qtiles, 0, total_ktiles}, total_qtiles, total_ktiles, hq, hk, d,
                       q_codes, q_scale, k_codes, k_scale, nullptr, 1, stream);
}

TILEMIX_API int tilemix_quantize_qk_int4(const void* q_f16, const void* k_f16,
                                        const int32_t* cu_seqlens_d, const int32_t* cu_qtiles_d,
                                        const int32_t* cu_ktiles_d, int nseq, int total_tokens,
                                        int total_qtiles, int total_ktiles, int hq, int hk, int d,
                                        int8_t* q_codes, float* q_scale, int8_t* k_codes,
                                        float* k_scale, void* stream) {
  return quantize_impl(q_f16, k_f16, cu_seqlens_d, cu_qtiles_d, cu_ktiles_d, nseq, total_tokens,
                       {0, total_qtiles, 0, total_ktiles}, total_qtiles, total_ktiles, hq, hk, d,
                       q_codes, q_scale, k_codes, k_scale, nullptr, 2, stream);
}

TILEMIX_API int tilemix_workspace_size(const tilemix_prefill_args* args, size_t* bytes) {
  if (!args || !bytes) return TILEMIX_ERR_INVALID_ARG;
  const int rc = check_args(args);
  if (rc != TILEMIX_OK) return rc;
  *bytes = layout_of(args).total;
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_prefill_fwd(const tilemix_prefill_args* a, void* stream) {
  int rc = check_args(a);
  if (rc != TILEMIX_OK) return rc;
  if (a->nseq == 0 || a->total_tokens == 0) return TILEMIX_OK;
  PrefillPlan pl;
  if ((rc = plan_prefill(a, &pl)) != TILEMIX_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a->event_kernel_begin || a->event_kernel_end) pl.events = true;
  return run_prefill_range(a, pl, 0, a->nseq, {0, a->total_qtiles, 0, a->total_ktiles},
                           a->max_seqlen, st);
}

TILEMIX_API int tilemix_prefill_fwd_noalloc(const tilemix_prefill_args* args, void* stream) {
  int rc = check_args(args);
  if (rc != TILEMIX_OK) return rc;
  if (args->nseq == 0 || args->total_tokens == 0) return TILEMIX_OK;
  if (layout_of(args).total > TILEMIX_NOALLOC_SCRATCH_BYTES) return TILEMIX_ERR_TOO_LARGE;
  void* scratch = nullptr;
  if (tilemix::noalloc_scratch(&scratch) != cudaSuccess) return TILEMIX_ERR_CUDA;
  tilemix_prefill_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = TILEMIX_NOALLOC_SCRATCH_BYTES;
  return tilemix_prefill_fwd(&a, stream);
}

TILEMIX_API int tilemix_prefill_host(const tilemix_prefill_host_args* h, void* stream) {
  if (!h) return TILEMIX_ERR_INVALID_ARG;
  const tilemix_prefill_args* a = &h->dev;
  int rc = check_args(a);
  if (rc != TILEMIX_OK) return rc;
  if (a->nseq == 0 || a->total_tokens == 0) return TILEMIX_OK;
  if (!h->cu_seqlens_h || !h->q_h || !h->k_h || !h->v_h || !h->o_h || !h->stream_in ||
      !h->stream_out || !h->events || h->chunks < 1 || h->chunks > (1 << 20) ||
      (h->after_previous != 0 && h->after_previous != 1))
    return TILEMIX_ERR_INVALID_ARG;
  const int32_t* cu = h->cu_seqlens_h;
  const int nseq = a->nseq;
  if (cu[0] != 0 || cu[nseq] != a->total_tokens) return TILEMIX_ERR_INVALID_ARG;
  // the device tile offsets must match the host token offsets
  long long nq = 0, nk = 0;
  for (int s = 0; s < nseq; ++s) {
    const int L = cu[s + 1] - cu[s];
    if (L < 0 || L > a->max_seqlen) return TILEMIX_ERR_INVALID_ARG;
    nq += (L + TILEMIX_BLOCK_M - 1) / TILEMIX_BLOCK_M;
    nk += (L + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N;
  }
  if (nq != a->total_qtiles || nk != a->total_ktiles) return TILEMIX_ERR_INVALID_ARG;
  const int chunks = h->chunks < nseq ? h->chunks : nseq;

  PrefillPlan pl;
  if ((rc = plan_prefill(a, &pl)) != TILEMIX_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t sin = static_cast<cudaStream_t>(h->stream_in);
  cudaStream_t sout = static_cast<cudaStream_t>(h->stream_out);
  cudaEvent_t* ev = static_cast<cudaEvent_t*>(h->events);
  cudaEvent_t join = ev[3 * h->chunks];
  const size_t qrow = static_cast<size_t>(a->hq) * a->d * 2;  // bytes per token
  const size_t krow = static_cast<size_t>(a->hk) * a->d * 2;
  auto at = [](const void* base, size_t off) {
    return static_cast<void*>(static_cast<uint8_t*>(const_cast<void*>(base)) + off);
  };
  // unless the call follows one on the same rows, uploads start once
  // `stream` has finished what precedes this call
  if (!h->after_previous &&
      (cudaEventRecord(join, st) != cudaSuccess || cudaStreamWaitEvent(sin, join, 0) != cudaSuccess))
    return TILEMIX_ERR_CUDA;
  // run c: whole sequences s0 .. s1 - 1, cut where the token count first
  // reaches (c + 1) / chunks of the batch
  int s0 = 0, q0 = 0, k0 = 0;
  for (int c = 0; c < chunks && s0 < nseq; ++c) {
    const int s1 = tilemix::run_end(cu, nseq, chunks, c, s0);
    int nqt = 0, nkt = 0, longest = 0;
    for (int s = s0; s < s1; ++s) {
      const int L = cu[s + 1] - cu[s];
      nqt += (L + TILEMIX_BLOCK_M - 1) / TILEMIX_BLOCK_M;
      nkt += (L + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N;
      longest = std::max(longest, L);
    }
    const size_t t0 = static_cast<size_t>(cu[s0]), n = static_cast<size_t>(cu[s1]) - t0;
    if (n > 0) {
      // events of run c: upload done, kernels done, download done; waiting on
      // the last two first orders this run after the previous call's run c
      cudaEvent_t up = ev[3 * c], kern = ev[3 * c + 1], down = ev[3 * c + 2];
      if (cudaStreamWaitEvent(sin, kern, 0) != cudaSuccess ||
          cudaMemcpyAsync(at(a->q, t0 * qrow), at(h->q_h, t0 * qrow), n * qrow,
                          cudaMemcpyHostToDevice, sin) != cudaSuccess ||
          cudaMemcpyAsync(at(a->k, t0 * krow), at(h->k_h, t0 * krow), n * krow,
                          cudaMemcpyHostToDevice, sin) != cudaSuccess ||
          cudaMemcpyAsync(at(a->v, t0 * krow), at(h->v_h, t0 * krow), n * krow,
                          cudaMemcpyHostToDevice, sin) != cudaSuccess ||
          cudaEventRecord(up, sin) != cudaSuccess ||
          cudaStreamWaitEvent(st, up, 0) != cudaSuccess ||
          cudaStreamWaitEvent(st, down, 0) != cudaSuccess)
        return TILEMIX_ERR_CUDA;
      rc = run_prefill_range(a, pl, s0, s1, {q0, nqt, k0, nkt}, longest, st);
      if (rc != TILEMIX_OK) return rc;
      if (cudaEventRecord(kern, st) != cudaSuccess ||
          cudaStreamWaitEvent(sout, kern, 0) != cudaSuccess ||
          cudaMemcpyAsync(at(h->o_h, t0 * qrow), at(a->o, t0 * qrow), n * qrow,
                          cudaMemcpyDeviceToHost, sout) != cudaSuccess ||
          cudaEventRecord(down, sout) != cudaSuccess)
        return TILEMIX_ERR_CUDA;
    }
    s0 = s1;
    q0 += nqt;
    k0 += nkt;
  }
  // `stream` ends with the last download
  if (cudaEventRecord(join, sout) != cudaSuccess || cudaStreamWaitEvent(st, join, 0) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  return TILEMIX_OK;
}

namespace {

struct DecodeLayout {
  size_t part_m, part_l, part_acc, counters, total;
  int nsplit, tiles_per_split;
};

int check_decode(const tilemix_decode_args* a) {
  if (!a) return TILEMIX_ERR_INVALID_ARG;
  if (a->d != 64 && a->d != 128) return TILEMIX_ERR_UNSUPPORTED;
  if (a->hq < 1 || a->hk < 1 || a->hq % a->hk != 0) return TILEMIX_ERR_INVALID_ARG;
  if (a->kv_head_of_q == nullptr && a->hq / a->hk > 16) return TILEMIX_ERR_UNSUPPORTED;
  if (a->nseq < 0 || a->max_seqlen < 1 || a->total_ktiles < 0 || a->tiles_per_split < 0 ||
      a->cache_rows < 1)
    return TILEMIX_ERR_INVALID_ARG;
  if (!(a->softmax_scale >= 0.f) || std::isinf(a->softmax_scale)) return TILEMIX_ERR_INVALID_ARG;
  if (a->nseq == 0) return TILEMIX_OK;
  if (!a->q || !a->k || !a->v || !a->k_i8 || !a->k_scale || !a->o || !a->seq_start ||
      !a->seq_len || !a->ktile_start || !a->qtile_start || !a->masks || !a->g)
    return TILEMIX_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->k_i8) ||
      !aligned16(a->o))
    return TILEMIX_ERR_INVALID_ARG;
  return TILEMIX_OK;
}

int decode_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return 148;
  return sms;
}

// The key range of every (sequence, KV head) is cut into nsplit splits of
// tiles_per_split key tiles, one CTA each, so that the grid fills the
// resident slots (two CTAs per SM) about once: fewer, longer splits pay the
// per-CTA start (metadata, query rows) and merge less often.
DecodeLayout decode_layout(const tilemix_decode_args* a) {
  DecodeLayout w{};
  const int max_tiles = (a->max_seqlen + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N;
  long long per = a->tiles_per_split;
  if (per <= 0) {
    const long long units = static_cast<long long>(a->nseq) * a->hk;
    long long ns = units > 0 ? 2LL * decode_sms() / units : 1;
    if (ns < 1) ns = 1;
    per = (max_tiles + ns - 1) / ns;
  }
  if (per < 1) per = 1;
  if (per > max_tiles) per = max_tiles;
  w.tiles_per_split = static_cast<int>(per);
  w.nsplit = (max_tiles + w.tiles_per_split - 1) / w.tiles_per_split;
  const size_t rows = static_cast<size_t>(a->nseq) * a->hq;
  size_t off = 0;
  w.part_m = off;
  off = round_up(off + rows * w.nsplit * sizeof(float), 256);
  w.part_l = off;
  off = round_up(off + rows * w.nsplit * sizeof(float), 256);
  w.part_acc = off;
  off = round_up(off + rows * w.nsplit * a->d * sizeof(float), 256);
  w.counters = off;
  off = round_up(off + static_cast<size_t>(a->nseq) * a->hk * sizeof(int), 256);
  w.total = off;
  return w;
}

}  // namespace

TILEMIX_API int tilemix_decode_workspace_size(const tilemix_decode_args* args, size_t* bytes) {
  if (!args || !bytes) return TILEMIX_ERR_INVALID_ARG;
  const int rc = check_decode(args);
  if (rc != TILEMIX_OK) return rc;
  *bytes = args->nseq == 0 ? 0 : decode_layout(args).total;
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_decode_fwd(const tilemix_decode_args* a, void* stream) {
  int rc = check_decode(a);
  if (rc != TILEMIX_OK) return rc;
  if (a->nseq == 0) return TILEMIX_OK;
  const DecodeLayout w = decode_layout(a);
  if (!a->workspace || a->workspace_bytes < w.total ||
      (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return TILEMIX_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  tilemix::DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  const int d = a->d, rows = a->cache_rows;
  if ((rc = encode_rows(&p.tm_k, a->k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, rows, a->hk, d, 64,
                        TILEMIX_BLOCK_N, CU_TENSOR_MAP_SWIZZLE_128B)) != TILEMIX_OK)
    return rc;
  if ((rc = encode_rows(&p.tm_k8, a->k_i8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, a->hk, d, d,
                        TILEMIX_BLOCK_N,
                        d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B)) !=
      TILEMIX_OK)
    return rc;
  if ((rc = encode_rows(&p.tm_v, a->v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, rows, a->hk, d, 64,
                        TILEMIX_BLOCK_N, CU_TENSOR_MAP_SWIZZLE_128B)) != TILEMIX_OK)
    return rc;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.k_i8 = a->k_i8;
  p.k_scale = a->k_scale;
  p.o = a->o;
  p.seq_start = a->seq_start;
  p.seq_len = a->seq_len;
  p.ktile_start = a->ktile_start;
  p.qtile_start = a->qtile_start;
  p.masks = a->masks;
  p.g = a->g;
  p.kv_head_of_q = a->kv_head_of_q;
  p.part_m = reinterpret_cast<float*>(ws + w.part_m);
  p.part_l = reinterpret_cast<float*>(ws + w.part_l);
  p.part_acc = reinterpret_cast<float*>(ws + w.part_acc);
  p.counters = reinterpret_cast<int*>(ws + w.counters);
  p.nseq = a->nseq;
  p.hq = a->hq;
  p.hk = a->hk;
  p.d = a->d;
  p.group = a->hq / a->hk;
  p.total_ktiles = a->total_ktiles;
  p.nsplit = w.nsplit;
  p.tiles_per_split = w.tiles_per_split;
  p.timeout_ns = wait_timeout_ns();
  const float scale = a->softmax_scale > 0.f ? a->softmax_scale : 1.0f / std::sqrt(float(a->d));
  p.scale_log2 = scale * 1.4426950408889634f;
  if (tilemix::launch_decode(p, static_cast<cudaStream_t>(stream),
                             static_cast<cudaEvent_t>(a->event_kernel_begin),
                             static_cast<cudaEvent_t>(a->event_kernel_end)) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  return TILEMIX_OK;
}

namespace {

// Host-side validation of pooled-score routing; fills the tile totals.
int check_route(const tilemix_route_args* a, int* total_qtiles, int* total_ktiles) {
  if (!a) return TILEMIX_ERR_INVALID_ARG;
  if (a->d != 64 && a->d != 128) return TILEMIX_ERR_UNSUPPORTED;
  if (a->nseq < 0 || a->hq < 1 || a->hk < 1 || a->int8_percent < 0 || a->int8_percent > 100 ||
      (a->causal != 0 && a->causal != 1))
    return TILEMIX_ERR_INVALID_ARG;
  if (!a->kv_head_of_q && a->hq % a->hk != 0) return TILEMIX_ERR_INVALID_ARG;
  if (!a->kv_head_of_q && a->hq / a->hk > 256) return TILEMIX_ERR_UNSUPPORTED;
  if (a->kv_head_of_q && a->hq > 256) return TILEMIX_ERR_UNSUPPORTED;
  if (!a->cu_seqlens_h || !a->g_h) return TILEMIX_ERR_INVALID_ARG;
  if (a->cu_seqlens_h[0] != 0) return TILEMIX_ERR_INVALID_ARG;
  long long tq = 0, tk = 0;
  for (int s = 0; s < a->nseq; ++s) {
    const int L = a->cu_seqlens_h[s + 1] - a->cu_seqlens_h[s];
    const int g = a->g_h[s];
    if (L < 0 || g < 1) return TILEMIX_ERR_INVALID_ARG;
    const int rows = (L + TILEMIX_BLOCK_M - 1) / TILEMIX_BLOCK_M;
    const int kt = (L + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N;
    // the row with the most legal groups is the last one
    if (rows > 0 && ((L - 1) / TILEMIX_BLOCK_N) / g + 1 > TILEMIX_MAX_GROUPS)
      return TILEMIX_ERR_INVALID_ARG;
    tq += rows;
    tk += kt;
  }
  if (tq > (1LL << 30) || tk > (1LL << 30)) return TILEMIX_ERR_INVALID_ARG;
  *total_qtiles = static_cast<int>(tq);
  *total_ktiles = static_cast<int>(tk);
  if (a->nseq > 0 && tq > 0) {
    if (!a->q || !a->k || !a->cu_seqlens || !a->cu_qtiles || !a->cu_ktiles || !a->g || !a->masks)
      return TILEMIX_ERR_INVALID_ARG;
    if (!aligned16(a->q) || !aligned16(a->k) || (reinterpret_cast<uintptr_t>(a->masks) & 7u))
      return TILEMIX_ERR_INVALID_ARG;
  }
  return TILEMIX_OK;
}

size_t route_bytes(const tilemix_route_args* a, int tq, int tk, size_t* kbar_off) {
  *kbar_off = round_up(static_cast<size_t>(tq) * a->hk * a->d * sizeof(float), 256);
  return round_up(*kbar_off + static_cast<size_t>(tk) * a->hk * a->d * sizeof(float), 256);
}

}  // namespace

TILEMIX_API int tilemix_route_workspace_size(const tilemix_route_args* a, size_t* bytes) {
  if (!bytes) return TILEMIX_ERR_INVALID_ARG;
  int tq = 0, tk = 0;
  const int rc = check_route(a, &tq, &tk);
  if (rc != TILEMIX_OK) return rc;
  size_t off;
  *bytes = route_bytes(a, tq, tk, &off);
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_route_pooled(const tilemix_route_args* a, void* stream) {
  int tq = 0, tk = 0;
  int rc = check_route(a, &tq, &tk);
  if (rc != TILEMIX_OK) return rc;
  if (a->nseq == 0 || tq == 0) return TILEMIX_OK;
  size_t kbar_off;
  const size_t need = route_bytes(a, tq, tk, &kbar_off);
  if (!a->workspace || a->workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return TILEMIX_ERR_WORKSPACE;
  tilemix::RouteParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = a->q;
  p.k = a->k;
  p.cu_seqlens = a->cu_seqlens;
  p.cu_qtiles = a->cu_qtiles;
  p.cu_ktiles = a->cu_ktiles;
  p.g = a->g;
  p.kv_head_of_q = a->kv_head_of_q;
  p.qbar = static_cast<float*>(a->workspace);
  p.kbar = reinterpret_cast<float*>(static_cast<uint8_t*>(a->workspace) + kbar_off);
  p.masks = a->masks;
  p.nseq = a->nseq;
  p.hq = a->hq;
  p.hk = a->hk;
  p.d = a->d;
  p.causal = a->causal;
  p.int8_percent = a->int8_percent;
  p.total_qtiles = tq;
  p.total_ktiles = tk;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a->event_begin && cudaEventRecord(static_cast<cudaEvent_t>(a->event_begin), st) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  if (tilemix::launch_route(p, st) != cudaSuccess) return TILEMIX_ERR_CUDA;
  if (a->event_end && cudaEventRecord(static_cast<cudaEvent_t>(a->event_end), st) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_mass_probe(const tilemix_mass_args* a, void* stream) {
  if (!a) return TILEMIX_ERR_INVALID_ARG;
  if (a->d != 64 && a->d != 128) return TILEMIX_ERR_UNSUPPORTED;
  if (a->nseq < 0 || a->hq < 1 || a->hk < 1 || (a->causal != 0 && a->causal != 1) ||
      !(a->delta_log2 > 0.f) || std::isinf(a->delta_log2) || !(a->softmax_scale >= 0.f) ||
      std::isinf(a->softmax_scale))
    return TILEMIX_ERR_INVALID_ARG;
  if (!a->kv_head_of_q && a->hq % a->hk != 0) return TILEMIX_ERR_INVALID_ARG;
  if (!a->cu_seqlens_h || !a->g_h || a->cu_seqlens_h[0] != 0) return TILEMIX_ERR_INVALID_ARG;
  long long blocks = 0;
  for (int s = 0; s < a->nseq; ++s) {
    const int L = a->cu_seqlens_h[s + 1] - a->cu_seqlens_h[s];
    if (L < 0 || a->g_h[s] < 1) return TILEMIX_ERR_INVALID_ARG;
    if (L > 0 && ((L - 1) / TILEMIX_BLOCK_N) / a->g_h[s] + 1 > TILEMIX_MAX_GROUPS)
      return TILEMIX_ERR_INVALID_ARG;
    blocks += (L + TILEMIX_BLOCK_N - 1) / TILEMIX_BLOCK_N;
  }
  const long long T = a->nseq > 0 ? a->cu_seqlens_h[a->nseq] : 0;
  if (blocks > (1LL << 30) || T > (1LL << 31) - 1) return TILEMIX_ERR_INVALID_ARG;
  if (blocks == 0) return TILEMIX_OK;
  if (!a->q || !a->k || !a->cu_seqlens || !a->cu_qtiles || !a->cu_ktiles || !a->g ||
      !a->masks || !a->m8 || !a->h || !a->h8)
    return TILEMIX_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k)) return TILEMIX_ERR_INVALID_ARG;
  tilemix::MassParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = a->q;
  p.k = a->k;
  p.cu_seqlens = a->cu_seqlens;
  p.cu_qtiles = a->cu_qtiles;
  p.cu_ktiles = a->cu_ktiles;
  p.masks = a->masks;
  p.g = a->g;
  p.kv_head_of_q = a->kv_head_of_q;
  p.m8 = a->m8;
  p.h = a->h;
  p.h8 = a->h8;
  p.nseq = a->nseq;
  p.hq = a->hq;
  p.hk = a->hk;
  p.d = a->d;
  p.causal = a->causal;
  p.total_blocks = static_cast<int>(blocks);
  p.total_tokens = static_cast<int>(T);
  const float scale = a->softmax_scale > 0.f ? a->softmax_scale : 1.0f / std::sqrt(float(a->d));
  p.scale_log2 = scale * 1.4426950408889634f;
  p.delta_log2 = a->delta_log2;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a->event_begin && cudaEventRecord(static_cast<cudaEvent_t>(a->event_begin), st) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  if (tilemix::launch_mass_probe(p, st) != cudaSuccess) return TILEMIX_ERR_CUDA;
  if (a->event_end && cudaEventRecord(static_cast<cudaEvent_t>(a->event_end), st) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_selftest_wait_timeout(int timeout_ms, void* stream) {
  if (timeout_ms < 1 || timeout_ms > 10000) return TILEMIX_ERR_INVALID_ARG;
  if (tilemix::launch_selftest_wait(static_cast<unsigned long long>(timeout_ms) * 1000000ull,
                                    static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  return TILEMIX_OK;
}

TILEMIX_API int tilemix_get_error(void* stream) {
  unsigned int status = 0;
  if (tilemix::read_and_clear_status(&status, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TILEMIX_ERR_CUDA;
  if (status & tilemix::kStatusTimeout) return TILEMIX_ERR_TIMEOUT;
  if (status & (tilemix::kStatusBadGroups | tilemix::kStatusBadHeadMap))
    return TILEMIX_ERR_INVALID_ARG;
  return TILEMIX_OK;
}

}  // extern "C"
