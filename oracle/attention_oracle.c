/* CPU oracle for tile-routed FP16/INT8 causal prefill attention (TileMix).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  It shares no
 * code with the CUDA path.
 *
 * One output row at a time, element by element, in fp64 / int64:
 *
 *  - score of a legal pair (i, j) of sequence s, query head h:
 *      key tile kt = j / 64, routing group b = kt / g_s, routing word
 *      w = masks[(first q-tile row of s + i / 128) * hk + kv(h)]
 *      ("TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
 *      Acceleration", agihunt.info summary, method paragraphs: one bit per
 *      group of g adjacent key tiles, one 64-bit word per KV head and
 *      query-tile row, 1 = INT8, 0 = FP16, shift-and-mask lookup).
 *      bit 1:  A = sum_c q8[i][c] * k8[j][c] as an exact int64, then
 *              score = A * s_q * s_k * scale     (INT8 MMA, INT32 accumulate,
 *              rescale by the block scales and 1/sqrt(d): same paragraph).
 *      bit 0:  score = (sum_c q[i][c] * k[j][c]) * scale in fp64 (FP16 path).
 *  - legality: j < L_s, and j <= i when causal.  Illegal pairs are skipped
 *    whatever the routing bits say (same paragraph: causal and boundary
 *    legality are independent of the routing map).
 *  - two-pass softmax over the legal scores (max, then exp and sum), output
 *    O[i] = sum_j p_j v_j / sum_j p_j with V in its fp16 values, and
 *    LSE = max + log(sum).
 *
 * Layouts: q [T, hq, d], k and v [T, hk, d] as IEEE half bit patterns; q8 and
 * k8 the int8 codes in the same layouts; q_scale [hq, total_qtiles],
 * k_scale [hk, total_ktiles] fp32; masks [total_qtiles, hk] uint64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#define BLOCK_M 128
#define BLOCK_N 64

static double g_half[65536];
static int g_half_ready = 0;

/* IEEE binary16 bit pattern -> double (exact). */
static double half_bits_to_double(uint16_t h) {
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

static void init_half_table(void) {
    if (g_half_ready) return;
    for (int i = 0; i < 65536; ++i) g_half[i] = half_bits_to_double((uint16_t)i);
    g_half_ready = 1;
}

double oracle_half_to_double(uint16_t h) { return half_bits_to_double(h); }

/* rows: nrows triples (sequence, query head, row index inside the sequence).
 * Returns 0, or -1 if a routing group index would exceed 63, or -2 on a bad
 * row triple, or -3 if memory runs out. */
/* An e4m3 code as a double: sign, 4 exponent bits (bias 7), 3 mantissa bits;
 * exponent 0 is subnormal (m / 8 * 2^-6); exponent 15 with mantissa 7 is NaN. */
static double e4m3_to_double(uint8_t c) {
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return sgn ? -v : v;
}

int oracle_attention_rows_fmt(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                              const int8_t* q8, const float* q_scale, const int8_t* k8,
                              const float* k_scale, const uint64_t* masks, const int32_t* g,
                              const int32_t* cu_seqlens, const int32_t* cu_qtiles,
                              const int32_t* cu_ktiles, int nseq, int total_qtiles,
                              int total_ktiles, int hq, int hk, int d, int causal,
                              const int32_t* kv_map, double scale, const int64_t* rows,
                              int64_t nrows, double* out, double* lse, int low_fp8);

int oracle_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const int8_t* q8, const float* q_scale, const int8_t* k8,
                          const float* k_scale, const uint64_t* masks, const int32_t* g,
                          const int32_t* cu_seqlens, const int32_t* cu_qtiles,
                          const int32_t* cu_ktiles, int nseq, int total_qtiles,
                          int total_ktiles, int hq, int hk, int d, int causal,
                          const int32_t* kv_map, double scale, const int64_t* rows,
                          int64_t nrows, double* out, double* lse) {
    return oracle_attention_rows_fmt(q, k, v, q8, q_scale, k8, k_scale, masks, g, cu_seqlens,
                                     cu_qtiles, cu_ktiles, nseq, total_qtiles, total_ktiles, hq,
                                     hk, d, causal, kv_map, scale, rows, nrows, out, lse, 0);
}

/* As oracle_attention_rows; low_fp8 != 0 reads the codes as e4m3 values:
 * a low-precision tile scores (sum_c e4m3(q8) * e4m3(k8)) * s_q * s_k * scale,
 * exact in fp64 (products of two 4-significant-bit values, 128 of them). */
int oracle_attention_rows_fmt(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                              const int8_t* q8, const float* q_scale, const int8_t* k8,
                              const float* k_scale, const uint64_t* masks, const int32_t* g,
                              const int32_t* cu_seqlens, const int32_t* cu_qtiles,
                              const int32_t* cu_ktiles, int nseq, int total_qtiles,
                              int total_ktiles, int hq, int hk, int d, int causal,
                              const int32_t* kv_map, double scale, const int64_t* rows,
                              int64_t nrows, double* out, double* lse, int low_fp8) {
    init_half_table();
    int max_len = 0;
    for (int s = 0; s < nseq; ++s) {
        int L = cu_seqlens[s + 1] - cu_seqlens[s];
        if (L > max_len) max_len = L;
    }
    int status = 0;
#pragma omp parallel
    {
        double* sc = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
        if (!sc) {
#pragma omp atomic write
            status = -3;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!sc) continue;
            int s = (int)rows[3 * r], h = (int)rows[3 * r + 1], i = (int)rows[3 * r + 2];
            if (s < 0 || s >= nseq || h < 0 || h >= hq) {
#pragma omp atomic write
                status = -2;
                continue;
            }
            int t0 = cu_seqlens[s];
            int L = cu_seqlens[s + 1] - t0;
            if (i < 0 || i >= L) {
#pragma omp atomic write
                status = -2;
                continue;
            }
            int kv = kv_map[h];
            int qt = i / BLOCK_M;
            uint64_t w = masks[(int64_t)(cu_qtiles[s] + qt) * hk + kv];
            int gs = g[s];
            int jend = causal ? i + 1 : L;
            const uint16_t* qi = q + ((int64_t)(t0 + i) * hq + h) * d;
            const int8_t* q8i = q8 + ((int64_t)(t0 + i) * hq + h) * d;
            double sq = (double)q_scale[(int64_t)h * total_qtiles + cu_qtiles[s] + qt];
            double m = -INFINITY;
            for (int j = 0; j < jend; ++j) {
                int kt = j / BLOCK_N;
                int b = kt / gs;
                if (b > 63) {
#pragma omp atomic write
                    status = -1;
                    jend = j;
                    break;
                }
                double score;
                if ((w >> b) & 1ULL) {
                    const int8_t* k8j = k8 + ((int64_t)(t0 + j) * hk + kv) * d;
                    double sk = (double)k_scale[(int64_t)kv * total_ktiles + cu_ktiles[s] + kt];
                    if (low_fp8) {
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c)
                            acc += e4m3_to_double((uint8_t)q8i[c]) * e4m3_to_double((uint8_t)k8j[c]);
                        score = acc * sq * sk * scale;
                    } else {
                        int64_t acc = 0;
                        for (int c = 0; c < d; ++c) acc += (int64_t)q8i[c] * (int64_t)k8j[c];
                        score = (double)acc * sq * sk * scale;
                    }
                } else {
                    const uint16_t* kj = k + ((int64_t)(t0 + j) * hk + kv) * d;
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c) acc += g_half[qi[c]] * g_half[kj[c]];
                    score = acc * scale;
                }
                sc[j] = score;
                if (score > m) m = score;
            }
            double l = 0.0;
            for (int j = 0; j < jend; ++j) {
                double p = exp(sc[j] - m);
                sc[j] = p;
                l += p;
            }
            double* o = out + r * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int j = 0; j < jend; ++j) {
                const uint16_t* vj = v + ((int64_t)(t0 + j) * hk + kv) * d;
                double p = sc[j];
                for (int c = 0; c < d; ++c) o[c] += p * g_half[vj[c]];
            }
            for (int c = 0; c < d; ++c) o[c] /= l;
            lse[r] = m + log(l);
        }
        free(sc);
    }
    return status;
}

/* Exact int64 score matrix A[i][j] = q8[i] . k8[j] of one (sequence, head)
 * for every legal pair (i, j) of INT8-routed tiles; other entries untouched.
 * a_out is [L_s, L_s] row-major.  Small inputs only. */
int oracle_int_scores(const int8_t* q8, const int8_t* k8, const uint64_t* masks,
                      const int32_t* g, const int32_t* cu_seqlens, const int32_t* cu_qtiles,
                      int s, int h, int hq, int hk, int d, int causal,
                      const int32_t* kv_map, int64_t* a_out) {
    int t0 = cu_seqlens[s];
    int L = cu_seqlens[s + 1] - t0;
    int kv = kv_map[h];
    for (int i = 0; i < L; ++i) {
        uint64_t w = masks[(int64_t)(cu_qtiles[s] + i / BLOCK_M) * hk + kv];
        int jend = causal ? i + 1 : L;
        for (int j = 0; j < jend; ++j) {
            int b = (j / BLOCK_N) / g[s];
            if (b > 63) return -1;
            if (!((w >> b) & 1ULL)) continue;
            int64_t acc = 0;
            const int8_t* a = q8 + ((int64_t)(t0 + i) * hq + h) * d;
            const int8_t* c = k8 + ((int64_t)(t0 + j) * hk + kv) * d;
            for (int x = 0; x < d; ++x) acc += (int64_t)a[x] * (int64_t)c[x];
            a_out[(int64_t)i * L + j] = acc;
        }
    }
    return 0;
}
