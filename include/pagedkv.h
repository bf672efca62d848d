/*
 * pagedkv.h -- C ABI of the B200 (sm_100a) paged-KV decode library.
 *
 * The operations of one decode step of a vLLM-style serving engine:
 *
 *  1. paged_kv_cache_write ("reshape_and_cache"): scatter this step's new K/V
 *     vectors into their physical slots of the paged KV cache.
 *  2. paged_gqa_decode_attention: grouped-query attention of one new query
 *     token per sequence over that sequence's cached keys and values, read
 *     through a PagedAttention block table, with an optional split-KV
 *     (flash-decoding) mode whose partial softmaxes are merged by the
 *     log-sum-exp rule inside the same launch.
 *  3. paged_gqa_decode_step: 1 and 2 in one launch.
 * and around them: fused_add_rmsnorm_qkv, the residual add, RMSNorm and QKV
 * projection that produce the step's q and new K/V; paged_kv_fp8_scales and
 * the *_fp8_scaled variants, FP8 caches with scales on the device; and
 * paged_gqa_prefill_attention, many query tokens per sequence over the same
 * paged cache (chunked prefill), load-balanced over the SMs when given the
 * workspace paged_gqa_prefill_workspace_size names.
 *
 * Sources, cited by page title and section:
 *  - "rvLLM 소개" (discuss.pytorch.kr), §PagedAttention과 FlashAttention-3:
 *    the KV cache is managed by PagedAttention through block tables; attention
 *    is grouped-query, Qwen2.5's 12 query heads sharing 2 KV heads, and
 *    serving every query head of a KV head from one read of that head's K/V
 *    is what cuts KV bandwidth 6x; the cache is f16, FP8 E4M3 optionally.
 *  - same page, §CUDA 그래프 리플레이: decode steps are replayed from CUDA
 *    graphs on the caller's stream, after the per-step upload of block tables
 *    and context lengths. Hence every call here takes a stream, reads no
 *    device data on the host, allocates nothing and never synchronises, so
 *    it can be captured into a graph.
 *  - vLLM talk summary (aitrends.kr), §용어 해설 (KV Cache, PagedAttention):
 *    the cache keeps the keys and values of earlier tokens in fixed-size
 *    pages mapped like OS virtual memory.
 * The pages state no layout, argument list or numerical convention; the
 * ones below are this library's readings, listed with each function.
 *
 * Common conventions
 *  - All pointers are DEVICE pointers (cudaMalloc'd or equivalent) unless a
 *    comment says otherwise. The caller owns every buffer, the workspace
 *    included. The library allocates no device memory.
 *  - Layouts are dense row-major (C order), innermost dimension last:
 *      q, out        [B, Hq, D]                   float16
 *      k/v cache     [num_blocks, block_size, Hkv, D]  float16, or uint8 E4M3
 *      k/v new       [T, Hkv, D]                  float16
 *      block_tables  [B, max_blocks_per_seq]      int32 (physical block ids)
 *      context_lens  [B]                          int32
 *      slot_mapping  [T]                          int64
 *    Query head h reads KV head h / (Hq / Hkv) (contiguous groups).
 *    Token t of sequence b lives in physical block block_tables[b][t / bs],
 *    row t % bs. context_lens[b] counts every token attended to, this step's
 *    token included. Rows past context_lens[b] and table entries past
 *    ceil(context_lens[b] / bs) are never read and may hold anything.
 *  - FP8 caches use OCP E4M3 ("FN": bias 7, max 448, no infinities) with one
 *    fp32 scale per tensor: stored = RNE_satfinite(x / scale) (division in
 *    fp32), value = decoded * scale.
 *  - v1 supports D == 128, block_size == 16, 1 <= Hq/Hkv <= 8, and pointers
 *    aligned to 16 bytes; other shapes return PKV_ERR_UNSUPPORTED.
 *  - Argument errors are detected on the host, before any launch, and
 *    returned synchronously. A failed launch returns PKV_ERR_CUDA (the CUDA
 *    error is left set, readable with cudaGetLastError). Device data (table
 *    entries, lengths, slots) is not read on the host; kernels clamp or skip
 *    values outside the pool and record them in a device error word that
 *    pkv_device_error() returns.
 *  - Every call is asynchronous with respect to the host and ordered on
 *    `stream` (a cudaStream_t; NULL = legacy default stream).
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer */
    PKV_ERR_UNSUPPORTED = 2,   /* valid but not implemented in this version */
    PKV_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    PKV_ERR_CUDA = 4           /* a CUDA runtime call or launch failed */
} pkv_status;

typedef enum {
    PKV_KV_F16 = 0,            /* float16 cache */
    PKV_KV_FP8_E4M3 = 1        /* uint8 OCP E4M3 cache, per-tensor or per-KV-head scales */
} pkv_kv_dtype;

/* partition_tokens value that lets the library plan the split-KV work: the
 * load-balanced streaming kernel (every warp of a persistent grid takes an
 * equal share of the batch's pages, whatever the length mix). */
#define PKV_PARTITION_AUTO (-1)

/* flags of paged_gqa_decode_step */
#define PKV_STEP_OVERLAP_PREVIOUS 0x1u
/* Failure-detection self-test of paged_gqa_decode_step (never needed in
 * service): worker warp 0 of the persistent grid issues none of its page
 * loads, so its first barrier wait can never complete, and every barrier
 * wait of the launch gives up after 2 ms instead of one second. The launch
 * ends normally with PKV_DEVERR_WAIT_TIMEOUT set; that worker's share of the
 * output is left unwritten, no copy is left in flight, and the workspace
 * must be zero-filled again before its next use (see below). */
#define PKV_STEP_SELFTEST_WAIT_TIMEOUT 0x100u

/* Bits of the device error word (pkv_device_error). */
#define PKV_DEVERR_CONTEXT_LEN   0x1u  /* a context length exceeded max_context_len or the
                                          table capacity; it was clamped */
#define PKV_DEVERR_BLOCK_ID      0x2u  /* a table entry lay outside [0, num_blocks); its
                                          block read as zeros */
#define PKV_DEVERR_SLOT          0x4u  /* a slot lay outside the pool; the token was skipped */
#define PKV_DEVERR_WAIT_TIMEOUT  0x8u  /* an on-chip barrier wait ran out of its time limit */
#define PKV_DEVERR_SCALE         0x10u /* a device-side FP8 scale was not positive and finite;
                                          the results that used it are undefined */

/*
 * paged_kv_cache_write -- reshape_and_cache.
 *
 * For each token i < num_tokens with s = slot_mapping[i] >= 0, writes
 *   k_cache[s / block_size][s % block_size][h][:] = k_new[i][h][:]   for all h < Hkv
 * and the same for V. An FP8 cache stores E4M3 codes of k_new / k_scale
 * (v_new / v_scale), rounded to nearest even and saturated to +-448; the
 * scales are ignored for an f16 cache. Negative slots are skipped (padding).
 * Slots at or beyond num_blocks * block_size are skipped and flagged
 * (PKV_DEVERR_SLOT). Two tokens with the same slot: the result is one of
 * them, unspecified which. f16 writes are bit-exact copies.
 *
 * Arguments: k_new, v_new [T, Hkv, D] f16; k_cache, v_cache as above;
 * slot_mapping [T] int64; scales > 0 and finite when kv_dtype is FP8.
 * num_tokens == 0 is a no-op returning PKV_OK.
 */
pkv_status paged_kv_cache_write(const void* k_new, const void* v_new,
                                void* k_cache, void* v_cache,
                                const int64_t* slot_mapping,
                                int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                int32_t num_blocks, int32_t block_size,
                                int32_t kv_dtype, float k_scale, float v_scale,
                                void* stream);

/*
 * Bytes of workspace paged_gqa_decode_attention needs for these sizes:
 * 0 when partition_tokens == 0 (single pass); for partition_tokens > 0 the
 * partial results of n = ceil(max_context_len / partition_tokens) partitions
 * per (sequence, query head) plus the counters of their merge tree (fan-in 8:
 * one per partition per level, ceil(log8 n) levels, per (sequence, KV head)); for
 * PKV_PARTITION_AUTO two partial results per worker warp of the persistent
 * grid on the CURRENT device plus the counters. Returns 0 for invalid sizes.
 */
size_t paged_gqa_decode_workspace_size(int32_t batch, int32_t num_q_heads,
                                       int32_t num_kv_heads, int32_t head_dim,
                                       int32_t max_context_len, int32_t partition_tokens);

/*
 * A partition size for split-KV that gives the GPU enough independent work:
 * a multiple of block_size chosen from the batch, KV heads, the longest
 * context and the SM count (sm_count <= 0: query the current device).
 * Returns 0 (single pass) when splitting would not add parallelism.
 */
int32_t paged_gqa_decode_suggest_partition(int32_t batch, int32_t num_kv_heads,
                                           int32_t max_context_len, int32_t block_size,
                                           int32_t sm_count);

/*
 * paged_gqa_decode_attention -- one decode step of grouped-query attention.
 *
 * For every sequence b < batch and query head h < Hq, with g = h / (Hq/Hkv)
 * and L = context_lens[b]:
 *   s_t    = softmax_scale * dot(q[b][h], K_t)                     t < L
 *   out[b][h] = sum_t softmax(s)_t * V_t                           (f16, RNE)
 * where K_t = k_cache[block_tables[b][t / bs]][t % bs][g] (times k_scale for
 * FP8) and likewise V_t. L == 0 gives an all-zero row. Accumulation is fp32.
 *
 * partition_tokens == PKV_PARTITION_AUTO: the library's plan, normally the
 *   load-balanced streaming kernel: a persistent grid whose worker warps each
 *   take an equal contiguous share of all (sequence, KV head, page) units;
 *   pieces of a (sequence, KV head) split between workers are merged by the
 *   log-sum-exp rule below by the last piece to finish. Batches above 8192
 *   sequences fall back to fixed partitions of
 *   paged_gqa_decode_suggest_partition(...) tokens.
 * partition_tokens == 0: one pass per (sequence, KV head).
 * partition_tokens  > 0: a multiple of block_size; tokens [p*P, (p+1)*P) form
 *   partition p, each partition computes its own (max, sum, output) and the
 *   last partition of a (sequence, KV head) to finish merges them:
 *   M = max m_p, w_p = l_p * exp(m_p - M), out = sum w_p o_p / sum w_p.
 *   `workspace` must then hold paged_gqa_decode_workspace_size(...) bytes,
 *   256-byte aligned, and must be ZERO-FILLED before its first use; every
 *   call that completes without a device error leaves it ready for the next
 *   one (its counters back at zero), so a workspace is allocated and cleared
 *   once and reused. A call that ended with a barrier-wait timeout
 *   (PKV_DEVERR_WAIT_TIMEOUT) can leave counters set: zero-fill the
 *   workspace again before reusing it. Calls that share a workspace must not
 *   run concurrently on different streams.
 *
 * max_context_len must be >= every context_lens[b] (larger lengths are
 * clamped and flagged) and <= max_blocks_per_seq * block_size.
 * num_blocks is the pool size; table entries outside it read zeros and are
 * flagged. The value of softmax_scale is used as given (e.g. 1/sqrt(D)).
 */
pkv_status paged_gqa_decode_attention(void* out, const void* q,
                                      const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, const int32_t* context_lens,
                                      int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t block_size,
                                      int32_t max_blocks_per_seq, int32_t num_blocks,
                                      int32_t max_context_len, float softmax_scale,
                                      int32_t kv_dtype, float k_scale, float v_scale,
                                      int32_t partition_tokens,
                                      void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * paged_gqa_decode_step -- one decode step in one launch: this step's token
 * of every sequence is written into the cache and attended to.
 *
 * For each b with L = context_lens[b] > 0, the token at position L - 1 (the
 * context length counts it) is the new one: its K/V, k_new[b] and v_new[b]
 * ([B, Hkv, D] f16), are stored at slot block_tables[b][(L-1)/bs]*bs + (L-1)%bs
 * exactly as paged_kv_cache_write stores them (FP8: the same E4M3 codes),
 * and out is what paged_gqa_decode_attention computes on the updated cache.
 * The pages motivate the fusion: the engine's fused kernels and graph replay
 * exist to cut per-step launches ("rvLLM 소개", §CUDA 그래프 리플레이 and
 * §퓨즈드 CUDA 커널); the kernel that reads the new token's page patches the
 * row in shared memory and writes it to the cache, so no second launch is
 * needed. Always the load-balanced plan: `workspace` as for
 * paged_gqa_decode_attention with PKV_PARTITION_AUTO (zero-filled before its
 * first use). Batches whose tables do not fit the kernel's shared memory
 * (above 8192 sequences) return PKV_ERR_UNSUPPORTED.
 *
 * flags: 0, or PKV_STEP_OVERLAP_PREVIOUS (PKV_STEP_SELFTEST_WAIT_TIMEOUT may
 * be added for the self-test above). The kernel is launched with
 * programmatic dependent launch, so it may start while the previous launch
 * in `stream` finishes. By default it waits for that launch before reading
 * any input. With PKV_STEP_OVERLAP_PREVIOUS it first reads context_lens,
 * block_tables and the cache pages and only then waits (before q, k_new,
 * v_new, the workspace and out): the caller promises that the launch
 * immediately before this one in `stream` writes none of context_lens,
 * block_tables and the cache pages. In a layer loop, where the step follows
 * the QKV projection and the pages were written by earlier steps, this lets
 * the first page loads overlap the previous kernel. A prefill or a separate
 * cache write launched just before the step breaks the promise.
 */
pkv_status paged_gqa_decode_step(void* out, const void* q, const void* k_new, const void* v_new,
                                 void* k_cache, void* v_cache,
                                 const int32_t* block_tables, const int32_t* context_lens,
                                 int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t block_size,
                                 int32_t max_blocks_per_seq, int32_t num_blocks,
                                 int32_t max_context_len, float softmax_scale,
                                 int32_t kv_dtype, float k_scale, float v_scale,
                                 void* workspace, size_t workspace_bytes, uint32_t flags,
                                 void* stream);

/*
 * fused_add_rmsnorm_qkv -- the step before attention, fused: residual add,
 * RMSNorm and the QKV projection of num_tokens decode tokens in one launch
 * (tcgen05 tensor cores, split-K over a thread-block cluster),
 * writing q in the layout paged_gqa_decode_attention / _step take and k_new,
 * v_new in the layout the cache write and the fused step take.
 *
 * "rvLLM 소개" (discuss.pytorch.kr), §퓨즈드 CUDA 커널: every layer runs the
 * residual add, the RMSNorm and the QKV projection as one kernel (Add+RMSNorm
 * +QKV GEMV), so the normalised activations are never written out. The page
 * gives no formula; this library's reading, with T = num_tokens, H = hidden,
 * D = head_dim and N = (num_q_heads + 2 num_kv_heads) * D:
 *   residual_out[t] = f16(x[t] + residual[t])      (one rounding, nearest even)
 *   y[t]            = s / sqrt(mean_k(s_k^2) + eps) * gamma,  s = residual_out[t]
 *   qkv[t][n]       = sum_k w_qkv[n][k] * y[t][k] + bias[n]   (bias may be NULL)
 * where rows [0, Hq D) of w_qkv give q[t] ([T, Hq, D]), the next Hkv D rows
 * k_new[t] and the last Hkv D rows v_new[t] ([T, Hkv, D]), each head's D rows
 * consecutive, as in a fused qkv_proj weight. No rotary embedding is applied
 * (the pages name none).
 *
 * Arguments (device pointers, float16, row-major, 16-byte aligned):
 *   x, residual     [T, H]       the sublayer output and the residual stream
 *   gamma           [H]          RMSNorm weight
 *   w_qkv           [N, H]       projection weight; bias [N] or NULL
 *   residual_out    [T, H]       s, the new residual stream
 *   q, k_new, v_new [T, Hq, D], [T, Hkv, D], [T, Hkv, D]
 * No output may overlap x, residual or another output (residual_out cannot
 * update `residual` in place: other CTAs still read it).
 *
 * Precision: residual_out is exact (bit-for-bit the rounded sum). q, k_new,
 * v_new are f16 (nearest even) of an fp32-accumulated dot product of s (exact
 * in f16) with the weight row scaled by gamma and rounded once to f16,
 * f16(w[n][k] * gamma[k]); the 1/RMS factor is applied in fp32 after the sum.
 * The error is within 2^-10 * sum_k |w[n][k] y[t][k]| plus the output
 * rounding, provided no |w[n][k] * gamma[k]| exceeds 65504.
 *
 * Supported: H a multiple of 64 and at most 8192, D a multiple of 8,
 * N <= 2^24, T <= 4194240; others return PKV_ERR_UNSUPPORTED. eps must be
 * finite and >= 0. T == 0 is a no-op (the per-token pointers may then be
 * NULL; gamma and w_qkv may not).
 *
 * flags: 0, or PKV_STEP_OVERLAP_PREVIOUS. The kernel is launched with
 * programmatic dependent launch. With the flag it requests its first weight
 * tiles before waiting for the previous launch in `stream`: the caller
 * promises that launch does not write w_qkv.
 */
pkv_status fused_add_rmsnorm_qkv(const void* x, const void* residual, const void* gamma,
                                 const void* w_qkv, const void* bias, void* residual_out,
                                 void* q, void* k_new, void* v_new,
                                 int32_t num_tokens, int32_t hidden, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, float eps,
                                 uint32_t flags, void* stream);

/*
 * paged_gqa_prefill_attention -- chunked prefill: many query tokens per
 * sequence, each attending causally to the sequence's cached tokens through
 * its block table.
 *
 * The pages name prefill as the engine's other attention work besides decode
 * ("rvLLM 소개" (discuss.pytorch.kr), §H100 SXM 80GB 직접 엔진 벤치마크: the
 * wall times include it), over the same paged cache (§PagedAttention과
 * FlashAttention-3). This library's reading: sequence b brings
 * n_b = query_start[b+1] - query_start[b] query tokens, the last n_b of its
 * context_lens[b] = L_b tokens, whose K/V the cache write has already stored.
 * Query i of b sits at position p = L_b - n_b + i and attends to positions
 * [0, p]; query head h reads KV head h / (Hq / Hkv). With one query per
 * sequence this is paged_gqa_decode_attention.
 *
 * Arguments (device pointers unless noted):
 *   out, q          [total_queries, Hq, D] float16, rows in sequence order
 *   k/v cache, block_tables, context_lens, block_size, num_blocks, FP8
 *                   scales: as for paged_gqa_decode_attention (per-tensor scales)
 *   query_start     [batch + 1] int32, query_start[0] = 0, non-decreasing,
 *                   query_start[batch] = total_queries
 *   max_query_len   host bound on n_b (sizes the grid); <= max_context_len
 *   max_context_len host bound on L_b
 * A sequence whose lengths are inconsistent on the device (n_b > L_b,
 * L_b > max_context_len, n_b > max_query_len, rows outside [0,
 * total_queries)) is flagged (PKV_DEVERR_CONTEXT_LEN) and its rows are left
 * unwritten. Supported shapes as for decode.
 *
 * workspace (optional, f16 cache): NULL runs whole work items (two query
 *   tiles of one KV head of one sequence over all their KV tiles) on a
 *   persistent grid, costliest first. With a workspace of
 *   paged_gqa_prefill_workspace_size(...) bytes, 256-byte aligned and
 *   ZERO-FILLED before its first use, every CTA takes an equal share of all
 *   KV tiles of all items; an item cut at a CTA boundary is computed in
 *   pieces whose partial (max, sum, output) rows the piece that finishes last
 *   merges by the log-sum-exp rule of paged_gqa_decode_attention. A call
 *   that completes without a device error leaves the workspace ready for the
 *   next one; after PKV_DEVERR_WAIT_TIMEOUT zero-fill it again. Calls that
 *   share a workspace must not run concurrently. A workspace that is too
 *   small or misaligned returns PKV_ERR_WORKSPACE. FP8 caches ignore it.
 */
pkv_status paged_gqa_prefill_attention(void* out, const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       const int32_t* query_start, int32_t batch, int32_t total_queries,
                                       int32_t max_query_len, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                                       int32_t num_blocks, int32_t max_context_len, float softmax_scale,
                                       int32_t kv_dtype, float k_scale, float v_scale, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * Bytes of workspace paged_gqa_prefill_attention's load-balanced schedule
 * needs on the CURRENT device: two partial results (both 128-row query
 * tiles, fp32 output rows plus max and sum) per SM, then the merge tickets.
 * 0 for an FP8 cache (its kernel takes none) and for invalid sizes.
 */
size_t paged_gqa_prefill_workspace_size(int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                        int32_t kv_dtype);

/*
 * fused_add_rmsnorm_qkv_plan -- the launch plan fused_add_rmsnorm_qkv uses on
 * the current device for these sizes, for reports and tuning. Writes five
 * int32 to plan (host memory): weight-tile rows (128), slices of the hidden
 * size per cluster (split-K), tokens per token tile (64, 128 or 256), CTAs,
 * token tiles. Host-only (queries the device's cluster occupancy);
 * PKV_ERR_UNSUPPORTED as the projection.
 */
pkv_status fused_add_rmsnorm_qkv_plan(int32_t num_tokens, int32_t hidden, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t* plan);

/* Static text for a status code. Never NULL. */
const char* pkv_status_string(pkv_status status);

/*
 * Reads and clears the device error word of the current device (PKV_DEVERR_*
 * bits) into *flags. Synchronous: waits for all prior work on the device.
 * Must not be called while a stream is being captured.
 */
pkv_status pkv_device_error(uint32_t* flags);

/*
 * Size of the library-owned split-KV scratch used by
 * paged_gqa_decode_attention_static_workspace (16 MiB per GPU).
 */
#define PKV_STATIC_WORKSPACE_BYTES (16u << 20)

/*
 * paged_gqa_decode_attention_static_workspace -- the same attention as
 * paged_gqa_decode_attention, for callers that cannot allocate device memory.
 * The pages have no counterpart of this entry point; it exists for callers
 * such as a serving engine that hands (nearly) all free GPU memory to its KV
 * cache pool at start-up (the `--gpu-memory-utilization 0.90` setting the
 * rvLLM page shows) and owns no allocator for per-call scratch, a step being
 * recorded into a CUDA graph where cudaMalloc must not be called, or a
 * foreign-language caller with no access to the process's allocator.
 *
 * Arguments are those of paged_gqa_decode_attention without the workspace,
 * and every plan is served: PKV_PARTITION_AUTO (the balanced kernel, or the
 * fixed partitions it falls back to for very large batches), fixed
 * partitions, and the single pass. The scratch is a fixed
 * PKV_STATIC_WORKSPACE_BYTES array inside the library (a file-scope
 * __device__ array: every GPU that loads the library holds it until the
 * process exits). Nothing is allocated and no allocating library routine is
 * called.
 *  - A plan whose scratch exceeds PKV_STATIC_WORKSPACE_BYTES is rejected
 *    with PKV_ERR_WORKSPACE before any launch. The balanced plan needs two
 *    partial results per worker warp of the persistent grid (about 10 MiB on
 *    a 148-SM B200 with an FP8 cache); fixed partitions need
 *    paged_gqa_decode_workspace_size(...) bytes; a single pass needs none.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture on the device.
 *  - Every call on a device shares the one array, which keeps the previous
 *    call's contents; each call clears the part that must start at zero (its
 *    merge counters) on `stream` before launching, so a call that ended with
 *    a device error (PKV_DEVERR_*) does not affect the next one. Calls whose
 *    execution overlaps on the GPU (other streams, other threads) race on
 *    the array and give undefined results: serialise them.
 */
pkv_status paged_gqa_decode_attention_static_workspace(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
    int32_t max_context_len, float softmax_scale, int32_t kv_dtype,
    float k_scale, float v_scale, int32_t partition_tokens, void* stream);

/*
 * FP8 E4M3 caches with device-side scales (per tensor or per KV head).
 *
 * The pages name an FP8 E4M3 KV cache and no more ("rvLLM 소개"
 * (discuss.pytorch.kr), §PagedAttention과 FlashAttention-3). These entry points
 * take the reading, stated beside each one, that a scale may be given per KV
 * head and computed from data on the device, so that a step can be
 * calibrated and captured in a CUDA graph without reading anything back to
 * the host. Scale arrays are device pointers to float: one element when
 * scales_per_head is 0 (per tensor), num_kv_heads elements (head h uses
 * element h) when it is 1. They must hold positive finite values by the time
 * the kernels run; a violation is flagged (PKV_DEVERR_SCALE), not checked on
 * the host. Everything else is as for the per-tensor entry points above.
 */

/*
 * paged_kv_fp8_scales -- E4M3 scales from data.
 *
 * x: [rows, num_kv_heads, head_dim] f16, contiguous (for example this step's
 * new K, or the live rows of a cache being calibrated). Writes, on `stream`,
 *   scales[h] = amax_h / 448   (fp32 IEEE division), or 1 when amax_h is 0,
 * where amax_h is the largest |x| over the non-NaN elements of head h
 * (scales_per_head == 1, scales[num_kv_heads]) or of the whole tensor
 * (scales_per_head == 0, scales[1]); 448 is the largest finite E4M3 value,
 * so the largest magnitude maps onto the largest code. Infinite elements give
 * an infinite scale, which the FP8 kernels then flag. rows == 0 writes 1.
 * scales_per_head == 1 needs num_kv_heads <= 1024. head_dim must be a
 * multiple of 8 and x 16-byte aligned.
 */
pkv_status paged_kv_fp8_scales(const void* x, int64_t rows, int32_t num_kv_heads, int32_t head_dim,
                               int32_t scales_per_head, float* scales, void* stream);

/*
 * paged_kv_cache_write_fp8_scaled -- paged_kv_cache_write for an FP8 cache
 * with device-side scales: head h of a token is stored as E4M3 codes of
 * k_new / k_scales[h or 0] (v_new / v_scales[h or 0]), rounded to nearest
 * even and saturated to +-448.
 */
pkv_status paged_kv_cache_write_fp8_scaled(const void* k_new, const void* v_new,
                                           void* k_cache, void* v_cache,
                                           const int64_t* slot_mapping,
                                           int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                           int32_t num_blocks, int32_t block_size,
                                           const float* k_scales, const float* v_scales,
                                           int32_t scales_per_head, void* stream);

/*
 * paged_gqa_decode_attention_fp8_scaled -- paged_gqa_decode_attention on an
 * FP8 cache whose element of KV head g dequantises as decode(byte) times
 * k_scales[g or 0] (V: v_scales[g or 0]). All plans (single pass, fixed
 * partitions, PKV_PARTITION_AUTO) and the same workspace rules apply.
 */
pkv_status paged_gqa_decode_attention_fp8_scaled(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
    int32_t max_context_len, float softmax_scale,
    const float* k_scales, const float* v_scales, int32_t scales_per_head,
    int32_t partition_tokens, void* workspace, size_t workspace_bytes, void* stream);

/*
 * paged_gqa_decode_step_fp8_scaled -- paged_gqa_decode_step on an FP8 cache
 * with device-side scales: the new token is quantised with, and every element
 * dequantised with, the scales of its KV head as above.
 */
pkv_status paged_gqa_decode_step_fp8_scaled(
    void* out, const void* q, const void* k_new, const void* v_new,
    void* k_cache, void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
    int32_t max_context_len, float softmax_scale,
    const float* k_scales, const float* v_scales, int32_t scales_per_head,
    void* workspace, size_t workspace_bytes, uint32_t flags, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
