// Kernels of the decode step with the INT8 K cache (sm_100a).
//
//   decode_prep_kernel     re-quantises each sequence's last K block over its
//                          valid rows and quantises each new query row as a
//                          block of its own (symmetric absmax / 127)
//   decode_attn_kernel     one CTA per (sequence, KV head, key-range split):
//                          routed scores of the KV head's query rows against
//                          the split's keys, an online softmax over them, and
//                          the partial P.V with P rounded to fp16
//   decode_combine_kernel  merges the splits' partial softmax states into O
//
// Decode is the step after prefill that "TileMix: Tile-Centric Mixed-
// Precision Attention for LLM Inference Acceleration" (agihunt.info summary)
// and "Precision Has a Map: TileMix Routes INT8 Inside Dense Attention"
// (cognaptus.com, last section) name: the INT8 K codes and block scales of the
// quantisation pre-pass become the K cache, and a new token's query reads the
// routing word of its query-tile row.  It reads every cached key once and is
// bound by HBM, so it runs on the CUDA cores: dp4a for INT8 tiles, fp32 FMA for
// FP16 tiles, a thread per key for the scores and a thread per channel for
// P.V, so that every K and V row is read with full-width loads.
// Included by tilemix_kernels.cu (one translation unit: the kernels share the
// device status word and the routing cursor).
#pragma once

namespace tilemix {

constexpr int kDecodeThreads = 128;
constexpr int kDecodeKeys = TILEMIX_BLOCK_N;  // keys per routed tile
constexpr int kMaxGroup = 16;                 // query heads per KV head

// ---- step 1: last K block of each (sequence, KV head), new query rows ----
// Blocks [0, nseq * hk): K blocks; blocks [nseq * hk, nseq * (hk + hq)): query
// rows.  Each thread holds at most four 16-byte chunks (64 rows x 128 dims).
__global__ void __launch_bounds__(256)
    decode_prep_kernel(DecodeParams p) {
  __shared__ float red[8];
  const int nk = p.nseq * p.hk;
  const bool is_k = static_cast<int>(blockIdx.x) < nk;
  const int b = is_k ? blockIdx.x : blockIdx.x - nk;
  const int cpr_log2 = p.d == 128 ? 4 : 3;  // 16-byte chunks per row
  int s, head, rows;
  size_t base, row_stride;
  if (is_k) {
    s = b / p.hk;
    head = b - s * p.hk;
    const int len = __ldg(p.seq_len + s);
    const int r0 = (len - 1) / TILEMIX_BLOCK_N * TILEMIX_BLOCK_N;  // the new key's block
    rows = len - r0;
    base = (static_cast<size_t>(__ldg(p.seq_start + s) + r0) * p.hk + head) * p.d;
    row_stride = static_cast<size_t>(p.hk) * p.d;
  } else {
    s = b / p.hq;
    head = b - s * p.hq;
    rows = 1;
    base = (static_cast<size_t>(s) * p.hq + head) * p.d;
    row_stride = 0;
  }
  const __half* x = static_cast<const __half*>(is_k ? p.k : p.q);
  const int nchunks = rows << cpr_log2;
  uint4 u[4];
  __half2 amax2 = __float2half2_rn(0.f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = threadIdx.x + i * 256;
    u[i] = make_uint4(0u, 0u, 0u, 0u);
    if (c < nchunks) {
      const size_t off = base + (c >> cpr_log2) * row_stride + ((c & ((1 << cpr_log2) - 1)) << 3);
      u[i] = *reinterpret_cast<const uint4*>(x + off);
    }
    const __half2* hv = reinterpret_cast<const __half2*>(&u[i]);
#pragma unroll
    for (int e = 0; e < 4; ++e) amax2 = __hmax2(amax2, __habs2(hv[e]));
  }
  float a = fmaxf(__low2float(amax2), __high2float(amax2));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  a = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) a = fmaxf(a, red[w]);
  const float sc = __fdiv_rn(a, 127.0f);
  const float rc = a > 0.f ? __frcp_rn(sc) : 0.f;
  int8_t* codes = is_k ? p.k_i8 : p.q8;
  if (threadIdx.x == 0) {
    if (is_k) {
      const int len = __ldg(p.seq_len + s);
      p.k_scale[static_cast<size_t>(head) * p.total_ktiles + __ldg(p.ktile_start + s) +
                (len - 1) / TILEMIX_BLOCK_N] = sc;
    } else {
      p.q_scale[static_cast<size_t>(s) * p.hq + head] = sc;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = threadIdx.x + i * 256;
    if (c < nchunks) {
      const size_t off = base + (c >> cpr_log2) * row_stride + ((c & ((1 << cpr_log2) - 1)) << 3);
      *reinterpret_cast<uint2*>(codes + off) = a > 0.f ? quant_chunk(u[i], sc, rc) : make_uint2(0u, 0u);
    }
  }
}

// ---- step 2: split-key attention -------------------------------------------
template <int D>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_attn_kernel(DecodeParams p) {
  __shared__ int heads[kMaxGroup];
  __shared__ int ngroup;
  __shared__ float qf[kMaxGroup][D];                // query rows as fp32
  __shared__ __align__(16) int8_t q8[kMaxGroup][D];  // and their INT8 codes
  __shared__ float qsc[kMaxGroup];
  __shared__ float score[kMaxGroup][kDecodeKeys];    // log2-domain scores, then P
  __shared__ float m_run[kMaxGroup], l_run[kMaxGroup], alpha[kMaxGroup];

  int bid = blockIdx.x;
  const int split = bid % p.nsplit;
  bid /= p.nsplit;
  const int kv = bid % p.hk;
  const int s = bid / p.hk;
  const int tid = threadIdx.x;
  const int len = __ldg(p.seq_len + s);
  const int t = len - 1;  // position of the new token
  const int row0 = __ldg(p.seq_start + s);
  const int ntiles = t / kDecodeKeys + 1;
  const int kt0 = split * p.tiles_per_split;
  const int kt1 = min(ntiles, kt0 + p.tiles_per_split);
  const int gs = __ldg(p.g + s);
  const uint64_t word =
      __ldg(p.masks + static_cast<size_t>(__ldg(p.qtile_start + s) + t / TILEMIX_BLOCK_M) * p.hk + kv);
  if (tid == 0) {
    int n = 0;
    for (int h = 0; h < p.hq; ++h)
      if ((p.kv_head_of_q ? __ldg(p.kv_head_of_q + h) : h / p.group) == kv) {
        if (n < kMaxGroup) heads[n] = h;
        ++n;
      }
    // more query heads than one CTA holds (a custom head map): reported, and
    // only the first kMaxGroup are computed
    if (n > kMaxGroup) atomicOr(&g_status, kStatusBadGroups);
    ngroup = min(n, kMaxGroup);
    if (ntiles > 0 && (ntiles - 1) / gs > 63) atomicOr(&g_status, kStatusBadGroups);
  }
  __syncthreads();
  const int G = ngroup;
  for (int i = tid; i < G * D; i += kDecodeThreads) {
    const int gi = i / D, c = i - gi * D;
    const size_t qo = (static_cast<size_t>(s) * p.hq + heads[gi]) * D + c;
    qf[gi][c] = __half2float(static_cast<const __half*>(p.q)[qo]);
    q8[gi][c] = p.q8[qo];
  }
  if (tid < G) {
    qsc[tid] = p.q_scale[static_cast<size_t>(s) * p.hq + heads[tid]];
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.f;
  }
  float acc[kMaxGroup];
#pragma unroll
  for (int gi = 0; gi < kMaxGroup; ++gi) acc[gi] = 0.f;
  const bool bad_groups = ntiles > 0 && (ntiles - 1) / gs > 63;
  __syncthreads();

  const __half* kbase = static_cast<const __half*>(p.k);
  const __half* vbase = static_cast<const __half*>(p.v);
  GroupCursor gc;
  gc.group = kt0 / gs;
  gc.in_group = kt0 - gc.group * gs;
  for (int kt = kt0; !bad_groups && kt < kt1; ++kt, gc.next(gs)) {
    const bool is_int = (word >> gc.group) & 1ull;
    const float ksc = p.k_scale[static_cast<size_t>(kv) * p.total_ktiles + __ldg(p.ktile_start + s) + kt];
    // scores: thread j < 64 takes key kt * 64 + j, for every query row of the group
    if (tid < kDecodeKeys) {
      const int j = kt * kDecodeKeys + tid;
      if (j <= t) {
        const size_t ko = (static_cast<size_t>(row0 + j) * p.hk + kv) * D;
        if (is_int) {
          int dot[kMaxGroup];
#pragma unroll
          for (int gi = 0; gi < kMaxGroup; ++gi) dot[gi] = 0;
#pragma unroll
          for (int c = 0; c < D; c += 16) {
            const int4 kw = *reinterpret_cast<const int4*>(p.k_i8 + ko + c);
#pragma unroll
            for (int gi = 0; gi < kMaxGroup; ++gi) {
              if (gi < G) {
                const int4 qw = *reinterpret_cast<const int4*>(&q8[gi][c]);
                dot[gi] = __dp4a(qw.x, kw.x, dot[gi]);
                dot[gi] = __dp4a(qw.y, kw.y, dot[gi]);
                dot[gi] = __dp4a(qw.z, kw.z, dot[gi]);
                dot[gi] = __dp4a(qw.w, kw.w, dot[gi]);
              }
            }
          }
#pragma unroll
          for (int gi = 0; gi < kMaxGroup; ++gi)
            if (gi < G)
              score[gi][tid] = static_cast<float>(dot[gi]) * (qsc[gi] * ksc * p.scale_log2);
        } else {
          float dot[kMaxGroup];
#pragma unroll
          for (int gi = 0; gi < kMaxGroup; ++gi) dot[gi] = 0.f;
#pragma unroll
          for (int c = 0; c < D; c += 8) {
            const uint4 kw = *reinterpret_cast<const uint4*>(kbase + ko + c);
            const __half2* kh = reinterpret_cast<const __half2*>(&kw);
            float kf[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __half22float2(kh[e]);
              kf[2 * e] = f.x;
              kf[2 * e + 1] = f.y;
            }
#pragma unroll
            for (int gi = 0; gi < kMaxGroup; ++gi) {
              if (gi < G) {
#pragma unroll
                for (int e = 0; e < 8; ++e) dot[gi] = fmaf(qf[gi][c + e], kf[e], dot[gi]);
              }
            }
          }
#pragma unroll
          for (int gi = 0; gi < kMaxGroup; ++gi)
            if (gi < G) score[gi][tid] = dot[gi] * p.scale_log2;
        }
      } else {
#pragma unroll
        for (int gi = 0; gi < kMaxGroup; ++gi)
          if (gi < G) score[gi][tid] = -INFINITY;
      }
    }
    __syncthreads();
    // online softmax of the tile: warp w takes query rows w, w + 4, ...
    const int warp = tid >> 5, lane = tid & 31;
    for (int gi = warp; gi < G; gi += kDecodeThreads / 32) {
      const float s0 = score[gi][lane], s1 = score[gi][lane + 32];
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = m_run[gi];
      const float m_new = fmaxf(m_old, mx);
      // P rounded to fp16, as the P.V of the prefill path takes it
      const float p0 = __half2float(__float2half_rn(exp2f(s0 - m_new)));
      const float p1 = __half2float(__float2half_rn(exp2f(s1 - m_new)));
      score[gi][lane] = p0;
      score[gi][lane + 32] = p1;
      float ps = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      if (lane == 0) {
        const float al = m_old == -INFINITY ? 0.f : exp2f(m_old - m_new);
        alpha[gi] = al;
        l_run[gi] = l_run[gi] * al + ps;
        m_run[gi] = m_new;
      }
    }
    __syncthreads();
    // P.V: thread c takes channel c of every query row
    if (tid < D) {
#pragma unroll
      for (int gi = 0; gi < kMaxGroup; ++gi)
        if (gi < G) acc[gi] *= alpha[gi];
      const int jn = min(kDecodeKeys, len - kt * kDecodeKeys);
      for (int jj = 0; jj < jn; ++jj) {
        const float vf = __half2float(
            vbase[(static_cast<size_t>(row0 + kt * kDecodeKeys + jj) * p.hk + kv) * D + tid]);
#pragma unroll
        for (int gi = 0; gi < kMaxGroup; ++gi)
          if (gi < G) acc[gi] = fmaf(score[gi][jj], vf, acc[gi]);
      }
    }
    __syncthreads();
  }
  // partial state of this split: m, l per query row, acc per channel
#pragma unroll
  for (int gi = 0; gi < kMaxGroup; ++gi) {
    if (gi < G) {
      const size_t pi = (static_cast<size_t>(s) * p.hq + heads[gi]) * p.nsplit + split;
      if (tid == 0) {
        p.part_m[pi] = bad_groups ? -INFINITY : m_run[gi];
        p.part_l[pi] = bad_groups ? 0.f : l_run[gi];
      }
      if (tid < D) p.part_acc[pi * D + tid] = bad_groups ? 0.f : acc[gi];
    }
  }
}

// ---- step 3: merge the splits ---------------------------------------------
__global__ void decode_combine_kernel(DecodeParams p) {
  const int s = blockIdx.x / p.hq;
  const int h = blockIdx.x - s * p.hq;
  const size_t pi0 = (static_cast<size_t>(s) * p.hq + h) * p.nsplit;
  float m = -INFINITY;
  for (int k = 0; k < p.nsplit; ++k) m = fmaxf(m, p.part_m[pi0 + k]);
  float l = 0.f, o = 0.f;
  for (int k = 0; k < p.nsplit; ++k) {
    const float mk = p.part_m[pi0 + k];
    if (mk == -INFINITY) continue;
    const float w = exp2f(mk - m);
    l += w * p.part_l[pi0 + k];
    if (static_cast<int>(threadIdx.x) < p.d) o += w * p.part_acc[(pi0 + k) * p.d + threadIdx.x];
  }
  if (static_cast<int>(threadIdx.x) < p.d)
    static_cast<__half*>(p.o)[(static_cast<size_t>(s) * p.hq + h) * p.d + threadIdx.x] =
        __float2half_rn(l > 0.f ? o / l : 0.f);
}

int launch_decode(const DecodeParams& p, cudaStream_t stream, cudaEvent_t ev_begin,
                  cudaEvent_t ev_end) {
  const unsigned prep_blocks = static_cast<unsigned>(p.nseq) * (p.hk + p.hq);
  decode_prep_kernel<<<prep_blocks, 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
  if (ev_begin && (e = cudaEventRecord(ev_begin, stream)) != cudaSuccess)
    return static_cast<int>(e);
  const unsigned attn_blocks = static_cast<unsigned>(p.nseq) * p.hk * p.nsplit;
  if (p.d == 128)
    decode_attn_kernel<128><<<attn_blocks, kDecodeThreads, 0, stream>>>(p);
  else
    decode_attn_kernel<64><<<attn_blocks, kDecodeThreads, 0, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return static_cast<int>(e);
  if (ev_end && (e = cudaEventRecord(ev_end, stream)) != cudaSuccess)
    return static_cast<int>(e);
  decode_combine_kernel<<<static_cast<unsigned>(p.nseq) * p.hq, 128, 0, stream>>>(p);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace tilemix
