/* tilemix.h -- C ABI of the B200 (sm_100a) tile-routed FP16/INT8 causal
 * prefill attention library (libtilemix.so).
 *
 * The method ("TileMix: Tile-Centric Mixed-Precision Attention for LLM
 * Inference Acceleration", agihunt.info summary, method paragraphs; also
 * "Precision Has a Map: TileMix Routes INT8 Inside Dense Attention",
 * cognaptus.com, sections "Dense attention does not require uniform precision"
 * and "The routing mechanism is designed to stay inside the hot loop"):
 *   - the score matrix S = Q K^T of each (sequence, query head) is cut into
 *     128 x 64 tiles (BLOCK_M query rows x BLOCK_N keys);
 *   - g adjacent key tiles form one routing group; one bit per group, read by
 *     shift-and-mask from one 64-bit word per (KV head, query-tile row);
 *     bit 1 = INT8 score path, bit 0 = FP16 score path;
 *   - INT8 path: Q quantised in 128 x d blocks and K in 64 x d blocks,
 *     symmetric absmax / 127; INT8 MMA with INT32 accumulation; scores
 *     rescaled by s_q * s_k / sqrt(d) into the float score domain;
 *   - FP16 path: FP16 MMA with fp32 accumulation, scaled by 1 / sqrt(d);
 *   - both paths update one online-softmax state (row max, normaliser,
 *     output accumulator); V and P.V stay FP16;
 *   - causal and boundary legality are applied independently of the routing
 *     words: illegal interactions are never computed;
 *   - GQA query heads read their KV head's word; batches are packed with
 *     cu_seqlens (variable length, no padding).
 *
 * Conventions for every entry point:
 *   - the return value is a tilemix_status; nothing throws or aborts;
 *   - the caller owns every buffer; the library allocates no memory (host or
 *     device) on any path;
 *   - device entry points are asynchronous on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Argument errors are returned synchronously;
 *     faults found on the device (a bounded wait that expired, a routing row
 *     with more than 64 groups) are latched in a device status word and
 *     returned by tilemix_get_error();
 *   - "device" pointers must be CUDA device (or managed) memory of the current
 *     device; "host" pointers are ordinary host memory.
 */
#ifndef TILEMIX_H
#define TILEMIX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TILEMIX_VERSION 1
#define TILEMIX_BLOCK_M 128  /* query rows per tile and per Q quantisation block */
#define TILEMIX_BLOCK_N 64   /* keys per tile and per K quantisation block */
#define TILEMIX_MAX_GROUPS 64

typedef enum {
  TILEMIX_OK = 0,
  TILEMIX_ERR_INVALID_ARG = 1,  /* a pointer, size, layout or alignment is wrong */
  TILEMIX_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. head dim not 64/128) */
  TILEMIX_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  TILEMIX_ERR_TIMEOUT = 4,      /* a bounded device wait expired; outputs undefined */
  TILEMIX_ERR_WORKSPACE = 5,    /* workspace missing or smaller than required */
  TILEMIX_ERR_TOO_LARGE = 6     /* needs more scratch than tilemix_prefill_fwd_noalloc has */
} tilemix_status;

typedef enum {
  TILEMIX_BAND = 0,            /* keeps the diagonal local */
  TILEMIX_GLOBAL = 1,          /* keeps designated (leftmost) positions */
  TILEMIX_ROW_RANDOM = 2,      /* each row keeps random FP16 groups */
  TILEMIX_ALIGNED_SPARSE = 3,  /* right-aligned FP16 extension */
  TILEMIX_BIGBIRD = 4,         /* union of Band, Global and Row-Random */
  TILEMIX_SPTRANS = 5          /* stride plus tail */
} tilemix_template;

/* Library version (TILEMIX_VERSION). */
int tilemix_version(void);

/* Static text for a tilemix_status value; never NULL. */
const char* tilemix_status_string(int status);

/* ---------------------------------------------------------------- host --- */

/* Smallest grouping factor g >= 1 with ceil(ceil(seqlen / 64) / g) <= 64, so
 * that every query-tile row of a sequence of `seqlen` tokens fits one 64-bit
 * word (the grouping factor of the TileMix pages).  seqlen >= 0; g_out host.
 * INVALID_ARG if g_out is NULL or seqlen < 0. */
int tilemix_auto_g(int seqlen, int* g_out);

/* Per-sequence tile offsets of a packed batch.  cu_seqlens_h (host, nseq+1,
 * non-decreasing, starting at 0) -> cu_qtiles_h[s] = sum over s' < s of
 * ceil(L_s' / 128) and cu_ktiles_h[s] = sum of ceil(L_s' / 64) (host, nseq+1
 * each, caller-allocated).  INVALID_ARG on NULL pointers, nseq < 0 or
 * decreasing offsets. */
int tilemix_tile_offsets(const int32_t* cu_seqlens_h, int nseq, int32_t* cu_qtiles_h,
                         int32_t* cu_ktiles_h);

/* The runs of whole sequences tilemix_prefill_host cuts a batch into:
 * run r holds sequences run_start_h[r] .. run_start_h[r + 1] - 1, r < *nruns.
 * Run c ends before the first sequence s whose token offset cu_seqlens_h[s]
 * reaches (c + 1) / min(chunks, nseq) of the batch's tokens; the last run
 * takes every remaining sequence.  run_start_h: host, min(chunks, nseq) + 1
 * entries, caller-allocated (run_start_h[0] = 0, run_start_h[*nruns] = nseq).
 * INVALID_ARG on NULL pointers, nseq < 0, chunks < 1 or offsets that do not
 * start at 0 or decrease. */
int tilemix_host_runs(const int32_t* cu_seqlens_h, int nseq, int chunks, int32_t* run_start_h,
                      int* nruns);

/* Routing words of a static template at a stated INT8 coverage of legal tile
 * groups (TileMix pages: data-free templates borrowed from sparse attention;
 * coverage is the share of legal groups routed INT8, not a FLOP share; the
 * same words are reused for every KV head).
 *   tpl            tilemix_template
 *   int8_percent   0..100; per sequence exactly floor((p * N + 50) / 100) of
 *                  its N legal groups are INT8
 *   seed           seed of the Row-Random / BigBird draws (splitmix64)
 *   cu_seqlens_h   host [nseq+1]
 *   n_kv_heads     >= 1
 *   g_h            host [nseq], grouping factor per sequence (>= 1); a row with
 *                  more than 64 legal groups is INVALID_ARG
 *   causal         0 or 1
 *   masks_h        host [total_qtiles][n_kv_heads] uint64, caller-allocated;
 *                  bit b (LSB first) = group b (key tiles [b*g, (b+1)*g)),
 *                  1 = INT8; bits at and above a row's legal group count are 0
 *   legal_groups_h host [nseq] or NULL: N per sequence
 *   int8_groups_h  host [nseq] or NULL: INT8 groups per sequence
 * The template geometries are stated in the repository's design notes. */
int tilemix_build_routing(int tpl, int int8_percent, uint64_t seed, const int32_t* cu_seqlens_h,
                          int nseq, int n_kv_heads, const int32_t* g_h, int causal,
                          uint64_t* masks_h, int64_t* legal_groups_h, int64_t* int8_groups_h);

/* -------------------------------------------------------------- device --- */

/* Block quantisation of the INT8 score path (TileMix pages: only Q and K are
 * quantised, Q per 128 x d block, K per 64 x d block, symmetric absmax / 127).
 * Per (head, block of one sequence): a = max |x| over the block's valid rows,
 * s = fp32(a / 127) (IEEE division), code = clamp(rne(fp32(x / s)), -127, 127);
 * a == 0 gives s = 0 and codes 0.  Blocks start at each sequence's first token.
 *   q_f16 / k_f16   device fp16 [total_tokens][hq or hk][d], 16-byte aligned;
 *                   either may be NULL to skip that tensor (its outputs too)
 *   cu_seqlens_d, cu_qtiles_d, cu_ktiles_d   device int32 [nseq+1]
 *   q_i8            device int8 [total_tokens][hq][d]
 *   q_scale         device fp32 [hq][total_qtiles]
 *   k_i8            device int8 [total_tokens][hk][d]
 *   k_scale         device fp32 [hk][total_ktiles]
 *   d               64 or 128 (UNSUPPORTED otherwise) */
int tilemix_quantize_qk(const void* q_f16, const void* k_f16, const int32_t* cu_seqlens_d,
                        const int32_t* cu_qtiles_d, const int32_t* cu_ktiles_d, int nseq,
                        int total_tokens, int total_qtiles, int total_ktiles, int hq, int hk,
                        int d, int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale,
                        void* stream);

/* The FP8 low path's operands (an open alternative on the pages: "TileMix:
 * Tile-Centric Mixed-Precision Attention for LLM Inference Acceleration",
 * agihunt.info summary, limitations paragraph).  Same blocks, layouts and
 * arguments as tilemix_quantize_qk; s = fp32(absmax / 448) and code =
 * e4m3(fp32(x / s)) (IEEE division, round to nearest even, saturating to
 * +-448), the e4m3 bytes stored in the int8 arrays; a zero block has s = 0
 * and codes 0.  A tile routed to the low path then scores
 * (sum_c e4m3(q) e4m3(k)) * s_q * s_k / sqrt(d) with fp32 accumulation. */
int tilemix_quantize_qk_fp8(const void* q_f16, const void* k_f16, const int32_t* cu_seqlens_d,
                            const int32_t* cu_qtiles_d, const int32_t* cu_ktiles_d, int nseq,
                            int total_tokens, int total_qtiles, int total_ktiles, int hq, int hk,
                            int d, int8_t* q_codes, float* q_scale, int8_t* k_codes,
                            float* k_scale, void* stream);

/* INT4 low path (the 4-bit integer format the TileMix pages name as an open
 * alternative to INT8: agihunt summary, limitations paragraph; explainer,
 * closing section): the blocks and rounding of tilemix_quantize_qk with 7 in
 * place of 127, s = fp32(a / 7), code = rne(fp32(x / s)) in [-7, 7], one code
 * per int8 element (sm_100a has no 4-bit integer tensor-core kind: the codes
 * take the INT8 MMA, whose int32 dots stay exact).  Arguments, layouts and
 * errors as tilemix_quantize_qk. */
int tilemix_quantize_qk_int4(const void* q_f16, const void* k_f16, const int32_t* cu_seqlens_d,
                             const int32_t* cu_qtiles_d, const int32_t* cu_ktiles_d, int nseq,
                             int total_tokens, int total_qtiles, int total_ktiles, int hq, int hk,
                             int d, int8_t* q_codes, float* q_scale, int8_t* k_codes,
                             float* k_scale, void* stream);

typedef struct tilemix_prefill_args {
  const void* q;          /* device fp16 [total_tokens][hq][d], 16-byte aligned */
  const void* k;          /* device fp16 [total_tokens][hk][d], 16-byte aligned */
  const void* v;          /* device fp16 [total_tokens][hk][d], 16-byte aligned */
  void* o;                /* device fp16 [total_tokens][hq][d], 16-byte aligned (output) */
  float* lse;             /* device fp32 [hq][total_tokens] natural-log LSE, or NULL */
  const int32_t* cu_seqlens; /* device [nseq+1], packed token offsets */
  const int32_t* cu_qtiles;  /* device [nseq+1], see tilemix_tile_offsets */
  const int32_t* cu_ktiles;  /* device [nseq+1] */
  int nseq;
  int total_tokens;       /* cu_seqlens[nseq] */
  int total_qtiles;       /* cu_qtiles[nseq] */
  int total_ktiles;       /* cu_ktiles[nseq] */
  int max_seqlen;         /* max L_s (upper bound accepted) */
  int hq, hk, d;          /* hq % hk == 0; d in {64, 128} */
  const int32_t* kv_head_of_q; /* device [hq], or NULL for h / (hq / hk); a query head
                                  whose entry lies outside [0, hk) is skipped (its
                                  outputs are not written) and tilemix_get_error()
                                  then reports INVALID_ARG */
  const uint64_t* masks;  /* device [total_qtiles][hk] routing words */
  const int32_t* g;       /* device [nseq] grouping factors */
  int causal;             /* 1: key j legal for query i iff j <= i (and j < L_s) */
  float softmax_scale;    /* 0 selects 1 / sqrt(d) */
  const int8_t* k_i8;     /* optional precomputed K codes [total_tokens][hk][d] ... */
  const float* k_scale;   /* ... and scales [hk][total_ktiles]; both or neither */
  void* workspace;        /* device scratch, >= tilemix_workspace_size(), 256-aligned */
  size_t workspace_bytes;
  int32_t* debug_int32_scores; /* NULL, or device int32 [hq][total_tokens][dbg_cols]
                                  with dbg_cols = max_seqlen rounded up to 64: the raw
                                  INT32 score of every INT8-routed key tile computed
                                  (keys < L_s; other entries untouched).  Small
                                  inputs only; slows the kernel. */
  void* event_kernel_begin;    /* NULL, or a cudaEvent_t recorded on `stream` just
                                  before the fused attention kernel ... */
  void* event_kernel_end;      /* ... and one recorded just after it (profiling) */
  int low_format;              /* the low-precision path of bit-1 tiles: 0 = INT8
                                  (the pages' method, default), 1 = FP8 e4m3 (see
                                  tilemix_quantize_qk_fp8; k_i8 / k_scale, when given,
                                  then hold e4m3 codes and their scales; no debug
                                  INT32 dump), 2 = INT4 codes on the INT8 MMA (see
                                  tilemix_quantize_qk_int4; k_i8 / k_scale, when
                                  given, hold INT4 codes and their scales) */
} tilemix_prefill_args;

/* Bytes of device workspace tilemix_prefill_fwd needs for these arguments
 * (it holds the INT8 codes and scales of Q, and of K unless k_i8 is given,
 * and the fused kernel's work-item counter, so calls that may run at the same
 * time on different streams need separate workspaces).
 * INVALID_ARG on a NULL argument. */
int tilemix_workspace_size(const tilemix_prefill_args* args, size_t* bytes);

/* Fused tile-routed mixed-precision causal prefill attention forward:
 * O[t, h] = softmax over legal keys of the routed scores, times V, in fp16
 * (one rounding of the fp32 accumulator divided by the normaliser).
 * Enqueues one quantisation launch (Q, and K unless k_i8 is given) and the
 * fused attention kernel (persistent: one CTA per SM, work items handed out
 * heaviest first through a counter in the workspace) on `stream`. */
int tilemix_prefill_fwd(const tilemix_prefill_args* args, void* stream);

/* Allocation-free variant of tilemix_prefill_fwd.  (The TileMix pages have no
 * counterpart: this is a deployment convenience of this library.)
 *
 * For callers that cannot call cudaMalloc or any allocator at this point: for
 * example code running inside a host application that owns all device memory
 * through its own pool and forbids side allocations, or a latency-critical
 * path where an allocation, which may synchronise the device, is not allowed.
 * The caller still passes q, k, v, o (and the other tensors) as for
 * tilemix_prefill_fwd; args->workspace and args->workspace_bytes are ignored.
 * The INT8 codes and scales (and the work-item counter) that
 * tilemix_prefill_fwd keeps in the caller's workspace live instead in one
 * fixed scratch array of 64 MiB inside the
 * library (TILEMIX_NOALLOC_SCRATCH_BYTES), which every GPU that loads the
 * library holds until the process exits.  A call whose workspace would exceed
 * it (tilemix_workspace_size() > 64 MiB) returns TILEMIX_ERR_TOO_LARGE and
 * launches nothing.  Results equal those of tilemix_prefill_fwd.
 *
 * The first call in a CUDA context (a device's primary context, with that
 * device current, or a context the caller made current) looks up the scratch
 * array's device address in that context; make that first call before any
 * stream capture.  A context created later, for example after
 * cudaDeviceReset, gets a lookup of its own on its first call.  All calls
 * share the one array: calls that overlap on the GPU (on different streams,
 * or from different threads) race on it and must be serialised by the
 * caller.  Nothing in the array needs to start at zero; every call rewrites
 * what it reads. */
#define TILEMIX_NOALLOC_SCRATCH_BYTES (64u << 20)
int tilemix_prefill_fwd_noalloc(const tilemix_prefill_args* args, void* stream);

/* Prefill from host memory, with the copies overlapped with the attention.
 * (The TileMix pages have no counterpart: a deployment convenience of this
 * library for inputs that arrive in host memory.)
 *
 * The batch is cut into at most `chunks` runs of whole sequences, each cut
 * where the token count first reaches a further 1/chunks of the batch.  Per
 * run: its q, k and v rows are copied host -> device on stream_in; once they
 * landed, its quantisation and attention run on `stream` (the kernels of
 * tilemix_prefill_fwd, restricted to the run's sequences); once those
 * finished, its O rows are copied device -> host on stream_out.  So the
 * upload of run c + 1 and the download of run c - 1 overlap the kernels of
 * run c.  Unless after_previous is set, the uploads wait for everything
 * enqueued on `stream` before the call.  `stream` waits for the last
 * download, so work enqueued on `stream` after the call (an event, a
 * synchronisation, the next call) sees o_h complete.  Results equal those
 * of tilemix_prefill_fwd on the same inputs, bit for bit (every block's
 * codes and every output row are computed the same way whichever run holds
 * them).
 *   dev           the device-side arguments, as for tilemix_prefill_fwd:
 *                 dev.q, dev.k, dev.v, dev.o are device buffers of the whole
 *                 batch (this call fills q, k, v and reads o back), the
 *                 metadata arrays are on the device, dev.workspace is sized
 *                 by tilemix_workspace_size(&dev); dev.lse, if given, stays on
 *                 the device; dev.event_kernel_begin / end are not recorded
 *   cu_seqlens_h  host [nseq + 1], the same offsets as dev.cu_seqlens
 *   q_h           host fp16 [total_tokens][hq][d] (as dev.q) ...
 *   k_h, v_h      host fp16 [total_tokens][hk][d] ...
 *   o_h           host fp16 [total_tokens][hq][d] (output); the copies only
 *                 overlap anything when these four are page-locked memory
 *   chunks        1 .. 2^20, the most runs to cut the batch into (at most
 *                 nseq are made)
 *   stream_in, stream_out   two cudaStream_t, each different from `stream`
 *   events        3 * chunks + 1 cudaEvent_t created by the caller (timing
 *                 may be disabled), used by nothing else: per run, its
 *                 upload, kernels and download are recorded in events
 *                 3c, 3c + 1 and 3c + 2 (the last event joins the streams)
 *   after_previous  0, or 1 when this call follows one made with the same
 *                 events array, device buffers, batch and chunks (a stream
 *                 of batches): run c's upload then waits only for that
 *                 call's kernels of run c, and run c's kernels for its
 *                 download of run c, so this batch's uploads start while
 *                 the previous batch finishes; nothing else enqueued on
 *                 `stream` before the call is waited for by the uploads.
 *                 (Run c's waits on events 3c + 1 and 3c + 2 are made in
 *                 both modes; an event never recorded is no wait.)
 * INVALID_ARG also when a host pointer, a stream or `events` is NULL, chunks
 * is outside 1 .. 2^20, after_previous is not 0 or 1, or cu_seqlens_h
 * disagrees with total_tokens, total_qtiles, total_ktiles or max_seqlen (all
 * checked before anything is enqueued); otherwise as tilemix_prefill_fwd.
 * On CUDA, part of the work may already be enqueued. */
typedef struct tilemix_prefill_host_args {
  tilemix_prefill_args dev;
  const int32_t* cu_seqlens_h;
  const void* q_h;
  const void* k_h;
  const void* v_h;
  void* o_h;
  int chunks;
  void* stream_in;
  void* stream_out;
  void* events;               /* cudaEvent_t array [3 * chunks + 1] */
  int after_previous;
} tilemix_prefill_host_args;

int tilemix_prefill_host(const tilemix_prefill_host_args* args, void* stream);

/* ---------------------------------------------------------------------------
 * Decode with the INT8 K cache: one new query token per sequence.
 *
 * The step after prefill named by the pages ("TileMix: Tile-Centric Mixed-
 * Precision Attention for LLM Inference Acceleration", agihunt.info summary;
 * "Precision Has a Map: TileMix Routes INT8 Inside Dense Attention",
 * cognaptus.com, last section): the INT8 K codes and 64-key block scales of
 * the quantisation pre-pass serve as the K cache, and a new token's query
 * reads the routing word of its query-tile row.  The pages give no decode
 * algorithm; this library reads it as the prefill method applied to one row:
 *   - sequence s holds seq_len[s] cached tokens in cache rows
 *     [seq_start[s], seq_start[s] + seq_len[s]); the new token is the last
 *     one, at position t = seq_len[s] - 1, its K and V already written, and it
 *     attends to positions 0..t (causal); a sequence with seq_len[s] = 0 has
 *     no token and is skipped;
 *   - key tile kt (keys 64 kt .. 64 kt + 63) uses the INT8 score path iff bit
 *     (kt / g[s]) of masks[(qtile_start[s] + t / 128) * hk + kv] is set;
 *   - the query is quantised as a block of its own (one row: earlier queries
 *     are not kept), symmetric absmax / 127 with the prefill rounding rules;
 *   - this call re-quantises the K block holding the new key (rows
 *     64 * (t / 64) .. t of the sequence) over its valid rows and writes its
 *     codes and scale into k_i8 / k_scale; every other block must already be
 *     current there (as tilemix_quantize_qk leaves them);
 *   - softmax state in fp32, P rounded to fp16 before P.V, O rounded once to
 *     fp16, as in the prefill path.
 * One kernel launch on `stream` (after a memset of the workspace's split
 * counters; K, V and the INT8 codes are read with TMA tile loads, so rows of
 * a tile past seq_len[s] are read too, and zeros past cache_rows): each CTA
 * takes tiles_per_split key tiles of one (sequence, KV
 * head), quantises the new query rows of that KV head itself, re-quantises
 * the last K block if its range holds it, and the CTA that finishes a
 * (sequence, KV head) last merges the partial softmax states into O.  Bad
 * routing factors, and a head map giving a KV head more than 16 query heads
 * (only the first 16 are computed), are reported by tilemix_get_error() as
 * for prefill. */
typedef struct tilemix_decode_args {
  const void* q;              /* device fp16 [nseq][hq][d]: the new tokens' queries, 16-B aligned */
  const void* k;              /* device fp16 [cache_rows][hk][d], 16-B aligned */
  const void* v;              /* device fp16 [cache_rows][hk][d], 16-B aligned */
  int8_t* k_i8;               /* device int8 [cache_rows][hk][d], 16-B aligned: INT8 K cache */
  float* k_scale;             /* device fp32 [hk][total_ktiles]: K block scales */
  void* o;                    /* device fp16 [nseq][hq][d] */
  const int32_t* seq_start;   /* device [nseq]: first cache row of each sequence */
  const int32_t* seq_len;     /* device [nseq]: tokens in the cache incl. the new one; 0 = an
                                 empty sequence: nothing is computed for it and its O rows
                                 are left as they are */
  const int32_t* ktile_start; /* device [nseq]: k_scale column of each sequence's first K block */
  const int32_t* qtile_start; /* device [nseq]: masks row of each sequence's first query tile */
  const uint64_t* masks;      /* device [total_qtiles][hk] routing words */
  const int32_t* g;           /* device [nseq] routing-group factors */
  const int32_t* kv_head_of_q;/* device [hq] or NULL => h / (hq / hk); a query head whose
                                 entry is outside [0, hk) is not computed */
  int nseq;                   /* >= 0 (0: nothing to do) */
  int max_seqlen;             /* >= every seq_len[s] (sizes the split of the key range) */
  int total_ktiles;           /* columns of k_scale */
  int cache_rows;             /* rows of k, v and k_i8, >= every seq_start[s] + seq_len[s] */
  int hq, hk, d;              /* d in {64, 128}; hq % hk == 0; at most 16 query heads per KV head */
  float softmax_scale;        /* 0 => 1 / sqrt(d) */
  int tiles_per_split;        /* 64-key tiles per CTA, >= 0; 0 => chosen so that the
                                 CTAs fill the resident slots (two per SM) about once */
  void* workspace;            /* device, >= tilemix_decode_workspace_size(), 256-aligned */
  size_t workspace_bytes;
  void* event_kernel_begin;   /* NULL, or a cudaEvent_t recorded on `stream` just before
                                 the attention kernel ... */
  void* event_kernel_end;     /* ... and one recorded just after it (profiling) */
} tilemix_decode_args;

/* Bytes of device workspace tilemix_decode_fwd needs (the splits' partial
 * softmax states and one counter per (sequence, KV head)).  INVALID_ARG / UNSUPPORTED as for
 * tilemix_decode_fwd. */
int tilemix_decode_workspace_size(const tilemix_decode_args* args, size_t* bytes);

/* Decode step as described above.  INVALID_ARG on a NULL required pointer, a
 * misaligned tensor, nseq < 0, max_seqlen < 1, cache_rows < 1, tiles_per_split < 0
 * or hq % hk != 0; UNSUPPORTED for
 * d not in {64, 128} or more than 16 query heads per KV head; WORKSPACE if the
 * workspace is missing, misaligned or too small; CUDA if a launch fails. */
int tilemix_decode_fwd(const tilemix_decode_args* args, void* stream);

/* ---------------------------------------------------------------------------
 * Content-aware (adaptive) routing through the same routing words.
 *
 * The pages say the mask interface can take adaptive policies and evaluate
 * none ("TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
 * Acceleration", agihunt.info summary, limitations paragraph; "Precision Has
 * a Map: TileMix Routes INT8 Inside Dense Attention", cognaptus.com,
 * "Placement can matter more than the nominal percentage").  This library's
 * policy, pooled scores:
 *   - for query-tile row r of sequence s and KV head kv, qbar = the mean of q
 *     over the row's valid query rows and kv's query heads, kbar_kt = the mean
 *     of k over key tile kt's valid keys;
 *   - each legal key tile kt scores qbar . kbar_kt, each legal group the
 *     highest score of its tiles;
 *   - the row's k_r lowest-scoring groups are INT8 (ties: the lower group),
 *     k_r from the proportional quota of the static templates (floor(p n_r /
 *     100), the sequence's leftover to the rows with the largest remainder,
 *     ties to the lower row), so each sequence gets the templates' INT8 count;
 *   - fp32 in a fixed order: a mean sums its items (q head-major, heads
 *     ascending, then rows ascending; k rows ascending) into 8 interleaved
 *     partial sums (item m into sum m mod 8), adds them in order 0..7 and
 *     divides by the count (no items: zero); a dot adds the separately
 *     rounded products over channels ascending.  The words are reproducible
 *     bit for bit.
 * Output: masks[total_qtiles][hk] on the device, the layout
 * tilemix_build_routing writes; bits past a row's legal groups are 0.
 * Three launches on `stream` (query means, key means, words). */
typedef struct tilemix_route_args {
  const void* q;              /* device fp16 [T][hq][d], 16-B aligned */
  const void* k;              /* device fp16 [T][hk][d], 16-B aligned */
  const int32_t* cu_seqlens_h;/* host [nseq + 1]: validation and grid sizes */
  const int32_t* g_h;         /* host [nseq]: routing-group factors */
  const int32_t* cu_seqlens;  /* device copies of the same values ... */
  const int32_t* cu_qtiles;   /* ... and the tile offsets (tilemix_tile_offsets) */
  const int32_t* cu_ktiles;
  const int32_t* g;
  const int32_t* kv_head_of_q;/* device [hq] or NULL => h / (hq / hk); an entry outside
                                 [0, hk) leaves its head out of every mean */
  int nseq, hq, hk, d;        /* d in {64, 128}; at most 256 query heads per KV head */
  int causal;                 /* 0 or 1 */
  int int8_percent;           /* 0..100 */
  uint64_t* masks;            /* device out [total_qtiles][hk] */
  void* workspace;            /* device, >= tilemix_route_workspace_size(), 256-aligned */
  size_t workspace_bytes;
  void* event_begin;          /* NULL, or cudaEvent_t recorded before the launches ... */
  void* event_end;            /* ... and after them (profiling) */
} tilemix_route_args;

/* Bytes of workspace tilemix_route_pooled needs (the fp32 means). */
int tilemix_route_workspace_size(const tilemix_route_args* args, size_t* bytes);

/* Pooled-score routing as described above.  INVALID_ARG on a NULL required
 * pointer, a misaligned tensor, a bad percent, causal flag or g, lengths that
 * do not start at 0 or decrease, a row with more than 64 groups, or hq % hk
 * != 0 without a head map; UNSUPPORTED for d not in {64, 128} or more than 256
 * query heads per KV head; WORKSPACE for a missing or small workspace; CUDA
 * if a launch fails.  All argument errors are returned before any launch. */
int tilemix_route_pooled(const tilemix_route_args* args, void* stream);

/* ---------------------------------------------------------------------------
 * Importance-mass exposure probe.
 *
 * The pages report that static SpTrans routing at 25% INT8 coverage sends only
 * about 8.5% of the selected high-importance attention mass to INT8
 * ("Precision Has a Map: TileMix Routes INT8 Inside Dense Attention",
 * cognaptus.com, last section; agihunt.info summary, results paragraph), and do
 * not say how interactions are selected.  Reading: P_ij is row i's softmax
 * over its legal keys of the full-precision scores (fp16 inputs, fp32
 * scores), and the high-importance keys are those with
 * P_ij >= 2^-delta_log2 * max_j P_ij.  Per (query head, token) the probe
 * writes
 *   m8 = sum of P_ij over INT8-routed legal keys,
 *   h  = sum of P_ij over the high-importance keys,
 *   h8 = sum of P_ij over the high-importance INT8-routed keys,
 * where a key is INT8-routed when the row's routing word (the same words the
 * attention path reads) has its group's bit set.  A batch's exposure is
 * sum h8 / sum h.  One launch; nothing is allocated. */
typedef struct tilemix_mass_args {
  const void* q;              /* device fp16 [T][hq][d], 16-B aligned */
  const void* k;              /* device fp16 [T][hk][d], 16-B aligned */
  const int32_t* cu_seqlens_h;/* host [nseq + 1]: validation and grid size */
  const int32_t* g_h;         /* host [nseq] */
  const int32_t* cu_seqlens;  /* device copies of the same values ... */
  const int32_t* cu_qtiles;   /* ... and the tile offsets (tilemix_tile_offsets) */
  const int32_t* cu_ktiles;
  const int32_t* g;
  const uint64_t* masks;      /* device [total_qtiles][hk] routing words */
  const int32_t* kv_head_of_q;/* device [hq] or NULL => h / (hq / hk); a head whose
                                 entry is outside [0, hk) is skipped (rows not written) */
  int nseq, hq, hk, d;        /* d in {64, 128} */
  int causal;                 /* 0 or 1 */
  float softmax_scale;        /* 0 => 1 / sqrt(d) */
  float delta_log2;           /* > 0; 4 => keys within a factor 16 of the row's largest P */
  float* m8;                  /* device out [hq][T] */
  float* h;                   /* device out [hq][T] */
  float* h8;                  /* device out [hq][T] */
  void* event_begin;          /* NULL, or cudaEvent_t recorded around the launch */
  void* event_end;
} tilemix_mass_args;

/* The probe as described above.  INVALID_ARG on a NULL required pointer, a
 * misaligned tensor, delta_log2 <= 0, a bad causal flag, g or lengths, or
 * hq % hk != 0 without a head map; UNSUPPORTED for d not in {64, 128}; CUDA if
 * the launch fails.  Argument errors return before any launch. */
int tilemix_mass_probe(const tilemix_mass_args* args, void* stream);

/* Self test of the failure path: enqueues one warp that waits on a device
 * barrier nothing ever signals, with the same bounded wait the attention
 * kernel uses, limited to timeout_ms (1..10000).  The wait gives up, latches
 * TILEMIX_ERR_TIMEOUT in the device status word and the kernel returns; the
 * CUDA context stays usable.  INVALID_ARG for an out-of-range timeout. */
int tilemix_selftest_wait_timeout(int timeout_ms, void* stream);

/* Diagnostic (not a step of the method): the tensor-core rate of the MMA
 * forms the fused prefill kernel issues, measured on this GPU.  Launches
 * `ctas` CTAs (1..4096); in each, one thread issues 4 * iters (iters
 * 1..2^20) back-to-back tcgen05.mma of one form with M = 128 and N = n
 * (64, 128 or 256) into TMEM, all accumulating into one tile:
 *   form 0  kind::f16,    A and B in shared memory, K = 16 per MMA
 *   form 1  kind::i8,     A and B in shared memory, K = 32 per MMA
 *   form 2  kind::f16,    A in TMEM, B MN-major in shared memory (the P.V form)
 *   form 3  kind::f8f6f4 (e4m3), A and B in shared memory, K = 32 per MMA
 * cycles_dev (device, caller-owned, [2 * ctas] int64) receives per CTA the SM
 * cycles to issue every MMA and the cycles until all completed (-1 if the
 * completion wait gave up after 2 s).  Operand values are arbitrary small
 * codes.  Asynchronous on `stream`; INVALID_ARG for an argument out of range,
 * CUDA if the launch fails. */
int tilemix_mma_rate(int form, int n, int iters, int ctas, long long* cycles_dev, void* stream);

/* Synchronises `stream`, then returns and clears the device status word:
 * OK, TIMEOUT (a bounded wait expired), INVALID_ARG (a row needed more than 64
 * groups, a bad routing-group factor, or a head-map entry outside [0, hk): the
 * work items concerned are skipped), or CUDA for a sticky CUDA error. */
int tilemix_get_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TILEMIX_H */
