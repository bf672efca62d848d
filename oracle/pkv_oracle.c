/*
 * Paged GQA decode attention and paged KV-cache write: float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, plainly written statement
 * of what the CUDA library computes. Only the test suite, the smoke check of
 * the package entry and the CPU-baseline leg of the benchmark may load it. It
 * shares no code, header, table or helper with the CUDA library, and the
 * CUDA library never calls it.
 *
 * Sources (cited by page title and section):
 *  - "rvLLM 소개" (discuss.pytorch.kr), §PagedAttention과 FlashAttention-3:
 *    the KV cache is managed by PagedAttention through block tables; attention
 *    is grouped-query (Qwen2.5: 12 query heads share 2 KV heads); the KV cache
 *    is f16 by default, FP8 E4M3 optionally.
 *  - "rvLLM 소개", §CUDA 그래프 리플레이: block tables and context lengths are
 *    per-step metadata uploaded before the attention kernels run.
 *  - vLLM talk summary (aitrends.kr), §용어 해설 (KV Cache, PagedAttention):
 *    keys and values of earlier tokens are kept; the cache is split into
 *    fixed-size pages mapped like OS virtual memory.
 *  The pages give no formulas, layouts or interfaces. The readings this file
 *  takes where they are silent are listed next to each function:
 *   R1 query head h uses KV head g = floor(h / (Hq/Hkv));
 *   R2 cache layout [num_blocks, block_size, Hkv, D], K and V separate,
 *      token t of sequence b is in block block_tables[b][t / block_size],
 *      row t % block_size; q and out are [B, Hq, D];
 *   R3 context_lens[b] counts every token attended to, this step's included;
 *   R4 context length 0 gives an all-zero output row (log-sum-exp = -inf);
 *   R5 FP8 is OCP E4M3 "FN" (bias 7, no infinities, S.1111.111 = NaN);
 *      quantisation divides by a per-tensor fp32 scale in fp32, then rounds
 *      to nearest even and saturates to +-448; dequantisation multiplies the
 *      decoded value by the scale;
 *   R6 split-KV partitions are aligned to multiples of partition_tokens in
 *      logical token order and are merged with the log-sum-exp rule;
 *   R7 a negative slot in the cache write means "skip this token";
 *   R8 (FP8 variants) a scale may also be given per KV head, scale[h]
 *      replacing the per-tensor scale for every element of head h; a scale
 *      computed from data is fp32(amax) / 448 divided in fp32, amax being
 *      the largest |x| over the non-NaN elements (per head, or over the
 *      whole tensor), and 1 when that maximum is 0 (or no element counts).
 *  Fused Add+RMSNorm+QKV ("rvLLM 소개", §퓨즈드 CUDA 커널: each layer runs
 *  the residual add, the RMSNorm and the QKV projection as one fused kernel
 *  whose outputs feed attention and the cache write); the page gives no
 *  formula, so:
 *   R9  the add is s = x + residual, rounded once to binary16 (nearest
 *       even); s is the new residual stream and is returned;
 *   R10 RMSNorm is y_k = s_k / sqrt(mean_k(s_k^2) + eps) * gamma_k over the
 *       hidden size H, from the binary16 s, in float64;
 *   R11 the projection is qkv_n = sum_k W[n][k] * y_k (+ bias_n when a bias
 *       is given) with W [N, H] row-major and N = (Hq + 2 Hkv) * D; rows
 *       [0, Hq D) are the query heads, the next Hkv D the key heads, the
 *       last Hkv D the value heads, each head's D rows consecutive; no
 *       rotary embedding is applied (the pages name none).
 *  Paged (chunked) prefill: the pages name prefill only as work the engine
 *  does besides decode ("rvLLM 소개", §H100 SXM 80GB 직접 엔진 벤치마크:
 *  the wall times include it), so:
 *   R12 sequence b brings n_b = query_start[b+1] - query_start[b] query
 *       tokens, the last n_b of its context_lens[b] = L_b tokens, whose K/V
 *       are already in the cache; query i of b sits at position
 *       p = L_b - n_b + i and attends causally to tokens [0, p] of b through
 *       its block table, with R1's head map. q and out are [sum n_b, Hq, D]
 *       with query_start [B+1] the prefix sums of n_b. n_b = 1 is decode;
 *       n_b = L_b is a prefill from an empty cache.
 *
 * Build: gcc -O2 -fopenmp -fPIC -shared -ffp-contract=off (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- formats */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);      /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* OCP E4M3 (R5): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * e == 0 is subnormal (m/8 * 2^-6); e == 15 with m == 7 is NaN; no infinity. */
double oracle_e4m3_to_f64(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                   /* m/8 * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10);         /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Round an fp32 value to E4M3 (R5): nearest representable value, ties to the
 * even mantissa, magnitudes above 448 saturate to 448, NaN gives 0x7F, the
 * sign is kept (a negative value that rounds to zero gives 0x80).
 * Written from the definition: for |x| in the binade [2^E, 2^(E+1)) with
 * E >= -6 the spacing of E4M3 values is 2^(E-3); below 2^-6 (subnormals) it
 * is 2^-9. rint() rounds half to even in the default rounding mode. */
uint8_t oracle_e4m3_from_f32(float x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;             /* saturate (covers inf) */
    int E;
    double fr = frexp(a, &E);                       /* a = fr * 2^E, fr in [0.5,1) */
    (void)fr;
    int binade = E - 1;                             /* a in [2^binade, 2^(binade+1)) */
    if (a == 0.0 || binade < -6) binade = -6;
    double quantum = ldexp(1.0, binade - 3);
    double r = rint(a / quantum) * quantum;         /* exact: a/quantum is exact */
    if (r > 448.0) r = 448.0;                       /* cannot happen below 448, kept for clarity */
    if (r == 0.0) return sign;
    /* encode r */
    int rE;
    frexp(r, &rE);
    int rb = rE - 1;
    int code;
    if (rb < -6) {                                  /* subnormal: r = m * 2^-9 */
        code = (int)(r / ldexp(1.0, -9));
    } else {
        int m = (int)(r / ldexp(1.0, rb - 3)) - 8;  /* r = (8+m) * 2^(rb-3) */
        code = ((rb + 7) << 3) | m;
    }
    return sign | (uint8_t)code;
}

/* One binary16 value quantised with a per-tensor scale (R5):
 * byte = e4m3(fp32(x) / scale), the division done in fp32. */
static uint8_t quantize_one(uint16_t x, float scale) {
    float xf = (float)oracle_f16_to_f64(x);         /* exact: f16 is a subset of fp32 */
    float qf = xf / scale;                          /* IEEE fp32 division */
    return oracle_e4m3_from_f32(qf);
}

void oracle_quantize_e4m3(const uint16_t* x, int64_t n, float scale, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = quantize_one(x[i], scale);
}

/* ------------------------------------------------------------ cache write */

/* reshape_and_cache: token i of this step goes to slot s = slot_mapping[i],
 * i.e. block s / block_size, row s % block_size (R2); for every KV head h
 * and channel d:  k_cache[blk][row][h][d] = k_new[i][h][d], same for V.
 * FP8 caches store e4m3(k_new / k_scales[h]) (R5, R8: one scale per KV head).
 * Negative slots are skipped (R7). Returns 0, or -1 if a slot lies outside
 * the pool. */
int oracle_paged_kv_cache_write_scaled(const uint16_t* k_new, const uint16_t* v_new,
                                       void* k_cache, void* v_cache,
                                       const int64_t* slot_mapping, int T, int Hkv, int D,
                                       int num_blocks, int block_size, int kv_fp8,
                                       const float* k_scales, const float* v_scales) {
    for (int i = 0; i < T; ++i) {
        int64_t s = slot_mapping[i];
        if (s < 0) continue;
        int64_t blk = s / block_size, row = s % block_size;
        if (blk >= num_blocks) return -1;
        for (int h = 0; h < Hkv; ++h) {
            for (int d = 0; d < D; ++d) {
                int64_t src = ((int64_t)i * Hkv + h) * D + d;
                int64_t dst = ((blk * block_size + row) * Hkv + h) * D + d;
                if (kv_fp8) {
                    ((uint8_t*)k_cache)[dst] = quantize_one(k_new[src], k_scales[h]);
                    ((uint8_t*)v_cache)[dst] = quantize_one(v_new[src], v_scales[h]);
                } else {
                    ((uint16_t*)k_cache)[dst] = k_new[src];
                    ((uint16_t*)v_cache)[dst] = v_new[src];
                }
            }
        }
    }
    return 0;
}

/* The same write with one per-tensor scale: every KV head uses it (R5). */
int oracle_paged_kv_cache_write(const uint16_t* k_new, const uint16_t* v_new,
                                void* k_cache, void* v_cache,
                                const int64_t* slot_mapping, int T, int Hkv, int D,
                                int num_blocks, int block_size, int kv_fp8,
                                float k_scale, float v_scale) {
    float* ks = (float*)malloc(sizeof(float) * (size_t)(Hkv > 0 ? Hkv : 1));
    float* vs = (float*)malloc(sizeof(float) * (size_t)(Hkv > 0 ? Hkv : 1));
    for (int h = 0; h < Hkv; ++h) { ks[h] = k_scale; vs[h] = v_scale; }
    int rc = oracle_paged_kv_cache_write_scaled(k_new, v_new, k_cache, v_cache, slot_mapping, T, Hkv,
                                                D, num_blocks, block_size, kv_fp8, ks, vs);
    free(ks);
    free(vs);
    return rc;
}

/* ------------------------------------------------------------- FP8 scales */

/* Largest |x| of the non-NaN elements of x[rows][Hkv][D] (binary16), per KV
 * head (per_head != 0: amax[h], h < Hkv) or over the whole tensor (amax[0]);
 * 0 when nothing counts (R8). */
void oracle_absmax_f16(const uint16_t* x, int64_t rows, int Hkv, int D, int per_head, float* amax) {
    int n_out = per_head ? Hkv : 1;
    for (int h = 0; h < n_out; ++h) amax[h] = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int h = 0; h < Hkv; ++h)
            for (int d = 0; d < D; ++d) {
                double v = fabs(oracle_f16_to_f64(x[(r * Hkv + h) * D + d]));
                if (isnan(v)) continue;
                float* a = &amax[per_head ? h : 0];
                if (v > (double)*a) *a = (float)v;      /* exact: a binary16 magnitude is an fp32 */
            }
}

/* Scale of an E4M3 cache for a given amax (R8): fp32 division by 448, so the
 * largest magnitude maps onto the largest finite code; 1 for amax 0. */
float oracle_fp8_scale_from_amax(float amax) {
    if (!(amax > 0.0f)) return 1.0f;
    return amax / 448.0f;                           /* IEEE fp32 division */
}

/* --------------------------------------------------------- decode attention */

/* Cache element (token row `slot` of the pool, KV head g, channel d) as f64:
 * f16 directly, FP8 as decoded value times the scale of KV head g (R5, R8). */
static double cache_elem(const void* cache, int kv_fp8, double scale,
                         int64_t slot, int Hkv, int D, int g, int d) {
    int64_t idx = (slot * Hkv + g) * D + d;
    if (kv_fp8) return oracle_e4m3_to_f64(((const uint8_t*)cache)[idx]) * scale;
    return oracle_f16_to_f64(((const uint16_t*)cache)[idx]);
}

/* Attention of one query head (b, h) over tokens [t0, t1) of its sequence.
 * Writes the running statistics of that range: m = max logit, l = sum of
 * exp(s_t - m), o[d] = sum_t exp(s_t - m) v_t[d] / l.  Returns -1 if a block
 * table entry lies outside the pool. */
static int attend_range(double* m_out, double* l_out, double* o, double* s,
                        const uint16_t* q, const void* k_cache, const void* v_cache,
                        const int32_t* bt_row, int b, int h, int Hq, int Hkv, int D,
                        int block_size, int num_blocks, double scale, int kv_fp8,
                        const float* k_scales, const float* v_scales, int t0, int t1) {
    int G = Hq / Hkv;
    int g = h / G;                                  /* R1 */
    double k_scale = kv_fp8 ? (double)k_scales[g] : 1.0, v_scale = kv_fp8 ? (double)v_scales[g] : 1.0;
    const uint16_t* qh = q + ((int64_t)b * Hq + h) * D;
    /* logits s_t = scale * sum_d q[d] k_t[d], gathering k_t through the table */
    double m = -INFINITY;
    for (int t = t0; t < t1; ++t) {
        int32_t phys = bt_row[t / block_size];
        if (phys < 0 || phys >= num_blocks) return -1;
        int64_t slot = (int64_t)phys * block_size + t % block_size;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += oracle_f16_to_f64(qh[d]) * cache_elem(k_cache, kv_fp8, k_scale, slot, Hkv, D, g, d);
        s[t - t0] = scale * dot;
        if (s[t - t0] > m) m = s[t - t0];
    }
    /* softmax weights and the weighted sum of values */
    double l = 0.0;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int t = t0; t < t1; ++t) {
        double p = exp(s[t - t0] - m);
        l += p;
        int64_t slot = (int64_t)bt_row[t / block_size] * block_size + t % block_size;
        for (int d = 0; d < D; ++d)
            o[d] += p * cache_elem(v_cache, kv_fp8, v_scale, slot, Hkv, D, g, d);
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    *m_out = m;
    *l_out = l;
    return 0;
}

/* out[b][h][:] = sum_t softmax_t(scale * q[b][h] . K_t) V_t over t < context_lens[b],
 * K_t, V_t read through block_tables (R1-R5). With partition_tokens > 0 the
 * tokens are cut into partitions [p*P, min((p+1)*P, L)) (R6), each partition
 * gives (m_p, l_p, o_p) as above, and they are merged with
 *   M = max_p m_p,  w_p = l_p * exp(m_p - M),  out = sum_p w_p o_p / sum_p w_p.
 * lse (optional, [B][Hq]) receives the log-sum-exp of the logits: m + ln l,
 * or M + ln(sum_p w_p) when split; -inf for an empty context (R4).
 * Returns 0, -1 for a table entry outside the pool, -2 for a bad length. */
int oracle_paged_gqa_decode_scaled(double* out, double* lse, const uint16_t* q,
                                   const void* k_cache, const void* v_cache,
                                   const int32_t* block_tables, const int32_t* context_lens,
                                   int B, int Hq, int Hkv, int D, int block_size,
                                   int max_blocks_per_seq, int num_blocks, float softmax_scale,
                                   int kv_fp8, const float* k_scales, const float* v_scales,
                                   int partition_tokens) {
    if (Hkv <= 0 || Hq % Hkv != 0) return -2;
    int status = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            int L = context_lens[b];
            double* ob = out + ((int64_t)b * Hq + h) * D;
            if (L < 0 || L > max_blocks_per_seq * block_size) {
#pragma omp atomic write
                status = -2;
                continue;
            }
            for (int d = 0; d < D; ++d) ob[d] = 0.0;
            if (lse) lse[(int64_t)b * Hq + h] = -INFINITY;
            if (L == 0) continue;                   /* R4 */
            const int32_t* bt_row = block_tables + (int64_t)b * max_blocks_per_seq;
            double* s = (double*)malloc(sizeof(double) * (size_t)L);
            int P = partition_tokens > 0 ? partition_tokens : L;
            int nparts = (L + P - 1) / P;
            double* mp = (double*)malloc(sizeof(double) * (size_t)nparts);
            double* lp = (double*)malloc(sizeof(double) * (size_t)nparts);
            double* op = (double*)malloc(sizeof(double) * (size_t)nparts * D);
            int bad = 0;
            for (int p = 0; p < nparts && !bad; ++p) {
                int t0 = p * P, t1 = (p + 1) * P < L ? (p + 1) * P : L;
                if (attend_range(&mp[p], &lp[p], &op[(int64_t)p * D], s, q, k_cache, v_cache,
                                 bt_row, b, h, Hq, Hkv, D, block_size, num_blocks,
                                 (double)softmax_scale, kv_fp8, k_scales, v_scales, t0, t1))
                    bad = 1;
            }
            if (bad) {
#pragma omp atomic write
                status = -1;
            } else if (nparts == 1) {              /* single pass: the definition itself */
                for (int d = 0; d < D; ++d) ob[d] = op[d];
                if (lse) lse[(int64_t)b * Hq + h] = mp[0] + log(lp[0]);
            } else {
                double M = -INFINITY;
                for (int p = 0; p < nparts; ++p) if (mp[p] > M) M = mp[p];
                double wsum = 0.0;
                for (int p = 0; p < nparts; ++p) {
                    double w = lp[p] * exp(mp[p] - M);
                    wsum += w;
                    for (int d = 0; d < D; ++d) ob[d] += w * op[(int64_t)p * D + d];
                }
                for (int d = 0; d < D; ++d) ob[d] /= wsum;
                if (lse) lse[(int64_t)b * Hq + h] = M + log(wsum);
            }
            free(s); free(mp); free(lp); free(op);
        }
    }
    return status;
}

/* The same attention with one per-tensor scale for K and one for V (R5). */
int oracle_paged_gqa_decode(double* out, double* lse, const uint16_t* q,
                            const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            int B, int Hq, int Hkv, int D, int block_size,
                            int max_blocks_per_seq, int num_blocks, float softmax_scale,
                            int kv_fp8, float k_scale, float v_scale, int partition_tokens) {
    if (Hkv <= 0) return -2;
    float* ks = (float*)malloc(sizeof(float) * (size_t)Hkv);
    float* vs = (float*)malloc(sizeof(float) * (size_t)Hkv);
    for (int h = 0; h < Hkv; ++h) { ks[h] = k_scale; vs[h] = v_scale; }
    int rc = oracle_paged_gqa_decode_scaled(out, lse, q, k_cache, v_cache, block_tables, context_lens,
                                            B, Hq, Hkv, D, block_size, max_blocks_per_seq, num_blocks,
                                            softmax_scale, kv_fp8, ks, vs, partition_tokens);
    free(ks);
    free(vs);
    return rc;
}

/* ------------------------------------------------------ paged prefill */

/* Chunked prefill attention through the block tables (R12, R1-R5). out[i]
 * (and lse[i], optional, [total, Hq]) for every query row i; per-tensor FP8
 * scales as in decode. Returns 0, -1 for a table entry outside the pool, -2
 * for bad lengths (n_b < 0, n_b > L_b, L_b beyond the table) or head counts. */
int oracle_paged_prefill(double* out, double* lse, const uint16_t* q, const void* k_cache,
                         const void* v_cache, const int32_t* block_tables,
                         const int32_t* context_lens, const int32_t* query_start, int B, int Hq,
                         int Hkv, int D, int block_size, int max_blocks_per_seq, int num_blocks,
                         float softmax_scale, int kv_fp8, float k_scale, float v_scale) {
    if (Hkv <= 0 || Hq % Hkv != 0 || B < 0 || query_start[0] != 0) return -2;
    for (int b = 0; b < B; ++b) {
        int n = query_start[b + 1] - query_start[b], L = context_lens[b];
        if (n < 0 || L < n || L > max_blocks_per_seq * block_size) return -2;
    }
    float* ks = (float*)malloc(sizeof(float) * (size_t)Hkv);
    float* vs = (float*)malloc(sizeof(float) * (size_t)Hkv);
    for (int g = 0; g < Hkv; ++g) { ks[g] = k_scale; vs[g] = v_scale; }
    int status = 0;
    int max_L = 1;
    for (int b = 0; b < B; ++b) max_L = context_lens[b] > max_L ? context_lens[b] : max_L;
    const int64_t total = B > 0 ? query_start[B] : 0;
    /* query rows are independent: one row per iteration, any thread (the arithmetic of a row does
     * not depend on which thread computes it) */
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)max_L);
#pragma omp for schedule(dynamic, 4)
        for (int64_t row = 0; row < total; ++row) {
            /* the row's sequence: the last b with query_start[b] <= row (sequences without
             * queries share their start with the next one) */
            int lo = 0, hi = B;                     /* query_start[lo] <= row < query_start[hi] */
            while (hi - lo > 1) {
                int mid = (lo + hi) / 2;
                if (query_start[mid] <= row) lo = mid; else hi = mid;
            }
            const int b = lo;
            const int n = query_start[b + 1] - query_start[b], L = context_lens[b];
            const int32_t* bt_row = block_tables + (int64_t)b * max_blocks_per_seq;
            const int i = (int)(row - query_start[b]);
            int pos = L - n + i;                    /* R12: this query's position */
            const uint16_t* q_row = q + row * Hq * D;
            for (int h = 0; h < Hq; ++h) {
                double m, l;
                double* o = out + (row * Hq + h) * D;
                /* query row `row` is passed as sequence 0 of a one-row q */
                if (attend_range(&m, &l, o, s, q_row, k_cache, v_cache, bt_row, 0, h, Hq, Hkv, D,
                                 block_size, num_blocks, (double)softmax_scale, kv_fp8, ks, vs,
                                 0, pos + 1)) {
#pragma omp atomic write
                    status = -1;
                    continue;
                }
                if (lse) lse[row * Hq + h] = m + log(l);
            }
        }
        free(s);
    }
    free(ks);
    free(vs);
    return status;
}

/* ------------------------------------------------ fused Add+RMSNorm+QKV */

/* Round a float64 value to binary16 (R9): nearest representable value, ties
 * to the even significand; magnitudes from 65520 (halfway between 65504 and
 * 2^16) up become infinity; NaN gives 0x7E00. Written from the definition:
 * in the binade [2^E, 2^(E+1)) with E >= -14 the spacing is 2^(E-10); below
 * 2^-14 (subnormals) it is 2^-24. */
uint16_t oracle_f16_from_f64(double x) {
    if (isnan(x)) return 0x7E00;
    uint16_t sign = signbit(x) ? 0x8000 : 0x0000;
    double a = fabs(x);
    if (a >= 65520.0) return sign | 0x7C00;
    int E;
    frexp(a, &E);
    int binade = E - 1;
    if (a == 0.0 || binade < -14) binade = -14;
    double quantum = ldexp(1.0, binade - 10);
    double r = quantum * rint(a / quantum);         /* a / quantum is exact */
    if (r == 0.0) return sign;
    int rE;
    frexp(r, &rE);                                  /* r may have reached the next binade */
    int rb = rE - 1;
    int code;
    if (rb < -14)
        code = (int)(r / ldexp(1.0, -24));          /* subnormal: r = f * 2^-24 */
    else
        code = ((rb + 15) << 10) | ((int)(r / ldexp(1.0, rb - 10)) - 1024);
    return sign | (uint16_t)code;
}

/* One decode step's residual add, RMSNorm and QKV projection (R9-R11).
 * x, residual: [T, H] binary16; gamma: [H]; w: [N, H]; bias: [N] or NULL.
 * Writes residual_out [T, H] (binary16 codes of s) and qkv [T, N] in
 * float64. eps must be >= 0; returns -1 on bad sizes. */
int oracle_add_rmsnorm_qkv(const uint16_t* x, const uint16_t* residual, const uint16_t* gamma,
                           const uint16_t* w, const uint16_t* bias, int T, int H, int N,
                           double eps, uint16_t* residual_out, double* qkv) {
    if (T < 0 || H <= 0 || N <= 0 || !(eps >= 0.0)) return -1;
#pragma omp parallel for schedule(dynamic)
    for (int t = 0; t < T; ++t) {
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        double sumsq = 0.0;
        for (int k = 0; k < H; ++k) {               /* R9: s = f16(x + residual) */
            int64_t i = (int64_t)t * H + k;
            double sum = oracle_f16_to_f64(x[i]) + oracle_f16_to_f64(residual[i]);   /* exact */
            uint16_t s16 = oracle_f16_from_f64(sum);
            residual_out[i] = s16;
            y[k] = oracle_f16_to_f64(s16);
            sumsq += y[k] * y[k];
        }
        double inv_rms = 1.0 / sqrt(sumsq / H + eps);                              /* R10 */
        for (int k = 0; k < H; ++k) y[k] = y[k] * inv_rms * oracle_f16_to_f64(gamma[k]);
        for (int n = 0; n < N; ++n) {               /* R11 */
            const uint16_t* wr = w + (int64_t)n * H;
            double acc = 0.0;
            for (int k = 0; k < H; ++k) acc += oracle_f16_to_f64(wr[k]) * y[k];
            if (bias) acc += oracle_f16_to_f64(bias[n]);
            qkv[(int64_t)t * N + n] = acc;
        }
        free(y);
    }
    return 0;
}

/* Number of threads the OpenMP runtime would use for a parallel region. */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
