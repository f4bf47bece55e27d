// The decode step with the INT8 K cache (sm_100a): one kernel launch.
//
// Decode is the step after prefill that "TileMix: Tile-Centric Mixed-
// Precision Attention for LLM Inference Acceleration" (agihunt.info summary)
// and "Precision Has a Map: TileMix Routes INT8 Inside Dense Attention"
// (cognaptus.com, last section) name: the INT8 K codes and block scales of the
// quantisation pre-pass become the K cache, and a new token's query reads the
// routing word of its query-tile row.
//
// One CTA per (sequence, KV head, split of the key range):
//   - quantises the KV head's new query rows (one block per row, the same
//     symmetric absmax / 127 as the prefill pre-pass) into shared memory;
//   - streams the split's key tiles through a three-stage shared-memory ring
//     with TMA tile loads (K in the tile's routed precision, V in fp16, both
//     swizzled), so HBM sees only the bytes the routing asks for;
//   - on the sequence's last tile (the one holding the new key), re-quantises
//     the block over its valid rows, writes the codes and scale back to the
//     cache and, if the tile is INT8-routed, scores it with those codes;
//   - scores with dp4a (INT8 tiles) or fp32-accumulated fp16 products (FP16
//     tiles), runs the online softmax with P rounded to fp16, and accumulates
//     P.V with fp16 products in fp32;
//   - writes its partial softmax state; the CTA that finishes a (sequence, KV
//     head) last merges every split's state into O.
// The step reads every cached key once and is bound by HBM, so it runs on the
// CUDA cores; no tensor-core tiles.
// Included by tilemix_kernels.cu (one translation unit: the kernels share the
// device status word and the bounded waits).
#pragma once

namespace tilemix {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeKeys = TILEMIX_BLOCK_N;  // keys per routed tile
constexpr int kMaxGroup = 16;                 // query heads per KV head
constexpr int kDecodeStages = 3;

// Shared-memory layout of the decode kernel, from the head dimension and the
// largest number of query heads a KV head may have (gcap <= kMaxGroup).  Each
// ring stage holds a K tile (64 rows, fp16 as 128-byte swizzled boxes of 64
// channels, or INT8 codes as one box swizzled at their row width) and a V
// tile (fp16, like K); offsets are from a 1024-byte aligned base.
struct DecodeSmem {
  int kbytes, stage, qh, q8, spart, pt, gcap4, small, bars, total;
};

__host__ __device__ inline DecodeSmem decode_smem(int d, int gcap) {
  DecodeSmem L{};
  L.kbytes = kDecodeKeys * 2 * d;
  L.stage = 2 * L.kbytes;
  int off = kDecodeStages * L.stage;
  L.qh = off;
  off += gcap * d * 2;
  L.q8 = off;
  off += gcap * d;
  L.spart = off;
  off += 4 * gcap * kDecodeKeys * 4;
  L.gcap4 = (gcap + 3) & ~3;
  L.pt = off;
  off += kDecodeKeys * L.gcap4 * 2;
  L.small = off;
  off += (5 * kMaxGroup + 8) * 4 + (kMaxGroup + 4) * 4;
  off = (off + 7) & ~7;
  L.bars = off;
  off += kDecodeStages * 8;
  L.total = ((off + 15) & ~15) + 1024;  // + alignment slack
  return L;
}

namespace dec {

// Byte offset of 16-byte chunk c of row r in a tile written by a TMA load
// with 128-byte swizzle (128-byte rows) or 64-byte swizzle (64-byte rows):
// the chunk index is XORed with the row's bits at byte-address bits 7..9
// (respectively 7..8).
__device__ __forceinline__ int sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }
__device__ __forceinline__ int sw64(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

// fp16 row of D channels as boxes of 64: logical 16-byte chunk lc of row r.
template <int D>
__device__ __forceinline__ int k16_off(int r, int lc) {
  return (lc >> 3) * (kDecodeKeys * 128) + sw128(r, lc & 7);
}
// INT8 row of D codes (one box of D bytes): chunk lc of row r.
template <int D>
__device__ __forceinline__ int k8_off(int r, int lc) {
  return D == 128 ? sw128(r, lc) : sw64(r, lc);
}

// c += a.lo * b.lo + a.hi * b.hi: fp16 products, exact in fp32, accumulated in
// fp32 one at a time.
__device__ __forceinline__ float dot2(uint32_t a, uint32_t b, float c) {
  asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %0;\n\t"
      "fma.rn.f32.f16 %0, a1, b1, %0;\n\t}"
      : "+f"(c)
      : "r"(a), "r"(b));
  return c;
}

// (c0, c1) += p * (v.lo, v.hi), p the low (kHi false) or high half of pw.
template <bool kHi>
__device__ __forceinline__ void axpy2(float& c0, float& c1, uint32_t pw, uint32_t vw) {
  if (kHi)
    asm("{\n\t.reg .f16 p0, p1, v0, v1;\n\t"
        "mov.b32 {p0, p1}, %2;\n\t"
        "mov.b32 {v0, v1}, %3;\n\t"
        "fma.rn.f32.f16 %0, p1, v0, %0;\n\t"
        "fma.rn.f32.f16 %1, p1, v1, %1;\n\t}"
        : "+f"(c0), "+f"(c1)
        : "r"(pw), "r"(vw));
  else
    asm("{\n\t.reg .f16 p0, p1, v0, v1;\n\t"
        "mov.b32 {p0, p1}, %2;\n\t"
        "mov.b32 {v0, v1}, %3;\n\t"
        "fma.rn.f32.f16 %0, p0, v0, %0;\n\t"
        "fma.rn.f32.f16 %1, p0, v1, %1;\n\t}"
        : "+f"(c0), "+f"(c1)
        : "r"(pw), "r"(vw));
}

__device__ __forceinline__ float absmax8(const uint4& u, float a) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
  __half2 m = __habs2(h[0]);
  m = __hmax2(m, __habs2(h[1]));
  m = __hmax2(m, __habs2(h[2]));
  m = __hmax2(m, __habs2(h[3]));
  return fmaxf(a, fmaxf(__low2float(m), __high2float(m)));
}

}  // namespace dec

// kG: query heads per KV head, exact for kG < kMaxGroup (the plain grouped
// layout); kG == kMaxGroup takes any count up to 16 (a custom head map).
template <int D, int kG>
// (two CTAs per SM; the generic 16-head path gets the registers of one)
__global__ void __launch_bounds__(kDecodeThreads, kG < kMaxGroup ? 2 : 1)
    decode_attn_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int kCpl = D / 32;  // P.V channels per lane
  constexpr bool kExact = kG < kMaxGroup;
  extern __shared__ __align__(128) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int gcap = kG;
  const DecodeSmem L = decode_smem(D, gcap);
  uint8_t* qh = dsm + L.qh;                                  // [gcap][D] fp16 query rows
  int8_t* q8s = reinterpret_cast<int8_t*>(dsm + L.q8);       // [gcap][D] their codes
  float* spart = reinterpret_cast<float*>(dsm + L.spart);    // [4][gcap][64] quarter-row scores
  uint8_t* pt = dsm + L.pt;                                  // [64][gcap4] fp16 P
  float* m_run = reinterpret_cast<float*>(dsm + L.small);
  float* l_run = m_run + kMaxGroup;
  float* alpha = l_run + kMaxGroup;
  float* qsc = alpha + kMaxGroup;
  float* red = qsc + 2 * kMaxGroup;  // [8]
  int* heads = reinterpret_cast<int*>(red + 8);
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
  const bool bad = (ntiles - 1) / gs > 63;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

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

  if (tid == 0) {
    int cnt = 0;
    for (int h = 0; h < p.hq; ++h)
      if ((p.kv_head_of_q ? __ldg(p.kv_head_of_q + h) : h / p.group) == kv) {
        if (cnt < gcap) heads[cnt] = h;
        ++cnt;
      }
    // more query heads than the CTA holds (a custom head map): reported, and
    // only the first gcap are computed
    if (cnt > gcap || (kExact && cnt != kG)) atomicOr(&g_status, kStatusBadGroups);
    flags[0] = min(cnt, gcap);
    if (bad) atomicOr(&g_status, kStatusBadGroups);
  }
  __syncthreads();
  const int G = kExact ? kG : flags[0];

  // New query rows: warp per row; lane c holds channels [8c, 8c + 8).
  for (int gi = warp; gi < G; gi += kDecodeThreads / 32) {
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (lane < D / 8)
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
    if (lane == 0) {
      qsc[gi] = sc;
      m_run[gi] = -INFINITY;
      l_run[gi] = 0.f;
    }
  }

  float acc[kG][kCpl];
#pragma unroll
  for (int gi = 0; gi < kG; ++gi)
#pragma unroll
    for (int e = 0; e < kCpl; ++e) acc[gi][e] = 0.f;

  const int j = tid & (kDecodeKeys - 1);  // score thread: key j, channel quarter hf
  const int hf = tid >> 6;
  constexpr int kQ = D / 4;               // channels of a quarter
  for (int i = 0; i < n && !bad; ++i) {
    const int kt = kt0 + i;
    const int jn = min(kDecodeKeys, len - kt * kDecodeKeys);
    const bool last = kt == ntiles - 1;
    const bool is_int = (word >> (kt / gs)) & 1ull;
    float ksc = 0.f;
    if (is_int && !last)
      ksc = __ldg(p.k_scale + static_cast<size_t>(kv) * p.total_ktiles + ktile0 + kt);
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
    if (last) {
      // the block holding the new key: absmax over its valid rows
      float a = 0.f;
      for (int c = tid; c < jn * (D / 8); c += kDecodeThreads)
        a = dec::absmax8(*reinterpret_cast<const uint4*>(K + dec::k16_off<D>(c / (D / 8), c % (D / 8))),
                         a);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if (lane == 0) red[warp] = a;
      __syncthreads();
      a = fmaxf(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])),
                fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7])));
      ksc = __fdiv_rn(a, 127.0f);
      const float rc = a > 0.f ? __frcp_rn(ksc) : 0.f;
      if (tid == 0) p.k_scale[static_cast<size_t>(kv) * p.total_ktiles + ktile0 + kt] = ksc;
      // scores from the fp16 rows; the codes go back to the cache on the way
      if (j < jn) {
        int8_t* code_out = p.k_i8 +
                           (static_cast<size_t>(row0 + kt * kDecodeKeys + j) * p.hk + kv) * D + hf * kQ;
        float fa[kG], fb[kG];
        int id[kG];
#pragma unroll
        for (int gi = 0; gi < kG; ++gi) {
          fa[gi] = 0.f;
          fb[gi] = 0.f;
          id[gi] = 0;
        }
#pragma unroll
        for (int c = 0; c < kQ / 8; ++c) {
          const uint4 kw = *reinterpret_cast<const uint4*>(K + dec::k16_off<D>(j, hf * (kQ / 8) + c));
          const uint2 cw = a > 0.f ? quant_chunk(kw, ksc, rc) : make_uint2(0u, 0u);
          *reinterpret_cast<uint2*>(code_out + c * 8) = cw;
#pragma unroll
          for (int gi = 0; gi < kG; ++gi) {
            if (gi < G) {
              if (is_int) {
                const uint2 qw = *reinterpret_cast<const uint2*>(q8s + gi * D + hf * kQ + c * 8);
                id[gi] = __dp4a(static_cast<int>(qw.x), static_cast<int>(cw.x), id[gi]);
                id[gi] = __dp4a(static_cast<int>(qw.y), static_cast<int>(cw.y), id[gi]);
              } else {
                const uint4 qw = *reinterpret_cast<const uint4*>(qh + (gi * D + hf * kQ + c * 8) * 2);
                fa[gi] = dec::dot2(qw.x, kw.x, fa[gi]);
                fb[gi] = dec::dot2(qw.y, kw.y, fb[gi]);
                fa[gi] = dec::dot2(qw.z, kw.z, fa[gi]);
                fb[gi] = dec::dot2(qw.w, kw.w, fb[gi]);
              }
            }
          }
        }
#pragma unroll
        for (int gi = 0; gi < kG; ++gi)
          if (gi < G)
            spart[(hf * gcap + gi) * kDecodeKeys + j] =
                is_int ? static_cast<float>(id[gi]) : fa[gi] + fb[gi];
      }
    } else if (j < jn) {
      if (is_int) {
        int ia[kG], ib[kG];
#pragma unroll
        for (int gi = 0; gi < kG; ++gi) {
          ia[gi] = 0;
          ib[gi] = 0;
        }
#pragma unroll
        for (int c = 0; c < kQ / 16; ++c) {
          const int4 kw = *reinterpret_cast<const int4*>(K + dec::k8_off<D>(j, hf * (kQ / 16) + c));
#pragma unroll
          for (int gi = 0; gi < kG; ++gi) {
            if (gi < G) {
              const int4 qw = *reinterpret_cast<const int4*>(q8s + gi * D + hf * kQ + c * 16);
              ia[gi] = __dp4a(qw.x, kw.x, ia[gi]);
              ib[gi] = __dp4a(qw.y, kw.y, ib[gi]);
              ia[gi] = __dp4a(qw.z, kw.z, ia[gi]);
              ib[gi] = __dp4a(qw.w, kw.w, ib[gi]);
            }
          }
        }
#pragma unroll
        for (int gi = 0; gi < kG; ++gi)
          if (gi < G) spart[(hf * gcap + gi) * kDecodeKeys + j] = static_cast<float>(ia[gi] + ib[gi]);
      } else {
        float fa[kG], fb[kG];
#pragma unroll
        for (int gi = 0; gi < kG; ++gi) {
          fa[gi] = 0.f;
          fb[gi] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < kQ / 8; ++c) {
          const uint4 kw = *reinterpret_cast<const uint4*>(K + dec::k16_off<D>(j, hf * (kQ / 8) + c));
#pragma unroll
          for (int gi = 0; gi < kG; ++gi) {
            if (gi < G) {
              const uint4 qw = *reinterpret_cast<const uint4*>(qh + (gi * D + hf * kQ + c * 8) * 2);
              fa[gi] = dec::dot2(qw.x, kw.x, fa[gi]);
              fb[gi] = dec::dot2(qw.y, kw.y, fb[gi]);
              fa[gi] = dec::dot2(qw.z, kw.z, fa[gi]);
              fb[gi] = dec::dot2(qw.w, kw.w, fb[gi]);
            }
          }
        }
#pragma unroll
        for (int gi = 0; gi < kG; ++gi)
          if (gi < G) spart[(hf * gcap + gi) * kDecodeKeys + j] = fa[gi] + fb[gi];
      }
    }
    __syncthreads();
    // online softmax of the tile: warp w takes query rows w, w + 8, ...
    for (int gi = warp; gi < G; gi += kDecodeThreads / 32) {
      const float f = is_int ? qsc[gi] * ksc * p.scale_log2 : p.scale_log2;
      const float* sp = spart + gi * kDecodeKeys;
      const int qs = gcap * kDecodeKeys;  // stride between quarters
      const float s0 = lane < jn ? (((sp[lane] + sp[qs + lane]) + sp[2 * qs + lane]) + sp[3 * qs + lane]) * f
                                 : -INFINITY;
      const float s1 = lane + 32 < jn ? (((sp[lane + 32] + sp[qs + lane + 32]) + sp[2 * qs + lane + 32]) +
                                         sp[3 * qs + lane + 32]) * f
                                      : -INFINITY;
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = m_run[gi];
      const float m_new = fmaxf(m_old, mx);
      // P rounded to fp16, as the P.V of the prefill path takes it
      const __half h0 = __float2half_rn(exp2f(s0 - m_new));
      const __half h1 = __float2half_rn(exp2f(s1 - m_new));
      reinterpret_cast<__half*>(pt)[lane * L.gcap4 + gi] = h0;
      reinterpret_cast<__half*>(pt)[(lane + 32) * L.gcap4 + gi] = h1;
      float ps = __half2float(h0) + __half2float(h1);
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
    // P.V: warp w takes keys [8w, 8w + 8), lane l channels [kCpl l, kCpl l + kCpl)
#pragma unroll
    for (int gi = 0; gi < kG; ++gi)
      if (gi < G) {
        const float al = alpha[gi];
#pragma unroll
        for (int e = 0; e < kCpl; ++e) acc[gi][e] *= al;
      }
    const int jend = min(8 * warp + 8, jn);
    for (int jj = 8 * warp; jj < jend; ++jj) {
      uint32_t vw[kCpl / 2];
      if constexpr (kCpl == 4) {
        const uint2 v2 =
            *reinterpret_cast<const uint2*>(V + dec::k16_off<D>(jj, lane >> 1) + (lane & 1) * 8);
        vw[0] = v2.x;
        vw[1] = v2.y;
      } else {
        vw[0] = *reinterpret_cast<const uint32_t*>(V + dec::k16_off<D>(jj, lane >> 2) + (lane & 3) * 4);
      }
      const uint8_t* prow = pt + jj * L.gcap4 * 2;
#pragma unroll
      for (int g4 = 0; g4 < kG; g4 += 4) {
        if (g4 < G) {
          const uint2 pw = *reinterpret_cast<const uint2*>(prow + g4 * 2);
#pragma unroll
          for (int e = 0; e < kCpl / 2; ++e) {
            if (g4 + 0 < G) dec::axpy2<false>(acc[g4 + 0][2 * e], acc[g4 + 0][2 * e + 1], pw.x, vw[e]);
            if (g4 + 1 < kG && g4 + 1 < G)
              dec::axpy2<true>(acc[g4 + 1][2 * e], acc[g4 + 1][2 * e + 1], pw.x, vw[e]);
            if (g4 + 2 < kG && g4 + 2 < G)
              dec::axpy2<false>(acc[g4 + 2][2 * e], acc[g4 + 2][2 * e + 1], pw.y, vw[e]);
            if (g4 + 3 < kG && g4 + 3 < G)
              dec::axpy2<true>(acc[g4 + 3][2 * e], acc[g4 + 3][2 * e + 1], pw.y, vw[e]);
          }
        }
      }
    }
    __syncthreads();  // the slot is free again
    if (tid == 0 && i + kDecodeStages < n) issue(i + kDecodeStages);
  }

  // Partial state of this split.  Every issued tile was consumed, so the ring
  // holds the eight warps' P.V sums for the reduction.
  float* rbuf = reinterpret_cast<float*>(dsm);  // [8][gcap][D]
#pragma unroll
  for (int gi = 0; gi < kG; ++gi)
    if (gi < G)
#pragma unroll
      for (int e = 0; e < kCpl; ++e) rbuf[(warp * gcap + gi) * D + lane * kCpl + e] = acc[gi][e];
  __syncthreads();
  for (int x = tid; x < G * D; x += kDecodeThreads) {
    const int gi = x / D, c = x - gi * D;
    float sum = rbuf[gi * D + c];
#pragma unroll
    for (int w = 1; w < kDecodeThreads / 32; ++w) sum += rbuf[(w * gcap + gi) * D + c];
    const size_t pi = (static_cast<size_t>(s) * p.hq + heads[gi]) * p.nsplit + split;
    p.part_acc[pi * D + c] = bad ? 0.f : sum;
  }
  if (tid < G) {
    const size_t pi = (static_cast<size_t>(s) * p.hq + heads[tid]) * p.nsplit + split;
    p.part_m[pi] = bad ? -INFINITY : m_run[tid];
    p.part_l[pi] = bad ? 0.f : l_run[tid];
  }
  // the last split of this (sequence, KV head) to finish merges them all
  __threadfence();
  __syncthreads();
  if (tid == 0) flags[2] = atomicAdd(p.counters + s * p.hk + kv, 1) == nsplit_s - 1;
  __syncthreads();
  if (!flags[2]) return;
  __threadfence();
  // merge: per query row the largest split maximum and the weighted sum of
  // the splits' l (warp per row), then O channel by channel
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
      m_run[gi] = m;
      l_run[gi] = l;
    }
  }
  __syncthreads();
  for (int x = tid; x < G * D; x += kDecodeThreads) {
    const int gi = x / D, c = x - gi * D;
    const size_t pi0 = (static_cast<size_t>(s) * p.hq + heads[gi]) * p.nsplit;
    const float m = m_run[gi], l = l_run[gi];
    float o = 0.f;
#pragma unroll 8
    for (int k = 0; k < nsplit_s; ++k) {
      const float mk = __ldcg(p.part_m + pi0 + k);
      const float a = __ldcg(p.part_acc + (pi0 + k) * D + c);
      if (mk != -INFINITY) o += exp2f(mk - m) * a;
    }
    static_cast<__half*>(p.o)[(static_cast<size_t>(s) * p.hq + heads[gi]) * D + c] =
        __float2half_rn(l > 0.f ? o / l : 0.f);
  }
}

template <int D, int kG>
cudaError_t launch_decode_kernel(const DecodeParams& p, unsigned blocks, cudaStream_t stream) {
  const int smem = decode_smem(D, kG).total;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<D, kG>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  decode_attn_kernel<D, kG><<<blocks, kDecodeThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_d(const DecodeParams& p, unsigned blocks, cudaStream_t stream) {
  switch (p.gcap) {
    case 1: return launch_decode_kernel<D, 1>(p, blocks, stream);
    case 2: return launch_decode_kernel<D, 2>(p, blocks, stream);
    case 3: return launch_decode_kernel<D, 3>(p, blocks, stream);
    case 4: return launch_decode_kernel<D, 4>(p, blocks, stream);
    case 5: return launch_decode_kernel<D, 5>(p, blocks, stream);
    case 6: return launch_decode_kernel<D, 6>(p, blocks, stream);
    case 7: return launch_decode_kernel<D, 7>(p, blocks, stream);
    case 8: return launch_decode_kernel<D, 8>(p, blocks, stream);
    default: return launch_decode_kernel<D, kMaxGroup>(p, blocks, stream);
  }
}

// p.gcap: the exact group size (1..8) of the plain grouped layout, else 16.
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
