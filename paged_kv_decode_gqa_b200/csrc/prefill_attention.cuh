// Paged (chunked) prefill attention for sm_100a: many query tokens per
// sequence, each attending causally to the sequence's cached tokens.
//
// What it computes: the pages name prefill as the engine's other attention
// work besides decode ("rvLLM 소개" (discuss.pytorch.kr), §H100 SXM 80GB 직접
// 엔진 벤치마크: the wall times include it) and its KV cache is paged
// (§PagedAttention과 FlashAttention-3). The library's reading: sequence b
// brings n_b query tokens, the last n_b of its context_lens[b] = L tokens,
// whose K/V the cache write has already stored; query i sits at position
// p = L - n_b + i and attends to positions [0, p] through the block table,
// query head h reading KV head h / G. One query per sequence is decode.
//
// Work unit: one CTA per (chunk of kConsumers query tokens, KV head g,
// sequence b). The CTA streams pages 0 .. page(last position of the chunk)
// of (b, g) once and serves every query of the chunk and all G heads of g
// from that read.
//  * Producer (last warp): block-table windows of 32 entries, one page (K
//    and V, 16 rows x 128 channels, 128-byte swizzled TMA tiles) per stage of
//    a kStages-deep ring, completion by transaction bytes.
//  * Consumer warp w owns query token chunk * kConsumers + w: the per-page
//    online-softmax update of the decode kernels (tokens on M, the G <= 8
//    heads on N = 8 of mma.sync m16n8k16), for the pages up to its position;
//    the causal cut is a prefix of valid rows of its last page. Every
//    consumer releases every stage, so the ring stays in step.
//  * Each warp owns its query outright: it writes out[row, heads of g]
//    itself, with no merge.
#pragma once

#include "decode_page.cuh"

namespace pkv {

struct PrefillParams {
    __half* out;                  // [total, Hq, D]
    const __half* q;              // [total, Hq, D]
    const int32_t* block_tables;  // [B, max_blocks_per_seq]
    const int32_t* context_lens;  // [B]
    const int32_t* query_start;   // [B + 1]
    int32_t total;                // rows of q and out
    int32_t Hq, Hkv, G;
    int32_t max_blocks_per_seq, num_blocks, max_context_len, max_query_len;
    float logit_scale_log2;       // softmax_scale * log2(e) (* k_scale for FP8)
    float out_scale;              // 1 (v_scale for FP8)
};

// 3-D tiled TMA load of one box into shared memory, completing on `bar`,
// with the default L2 policy (every chunk of a sequence re-reads its pages).
__device__ __forceinline__ void tma_load_3d_reused(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                   int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

template <bool kFp8, int kConsumers, int kStages>
struct PrefillShape {
    static constexpr int kTileBytes = kFp8 ? 2048 : 4096;     // 16 rows x 128 ch, one of K/V
    static constexpr int kStageBytes = 2 * kTileBytes;        // one page: K tile, then V tile
    static constexpr int kThreads = 32 * (kConsumers + 1);
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kSmemBytes = 1024 + kRingBytes + 2 * kStages * 8;
};

template <bool kFp8, int kConsumers, int kStages>
__global__ void __launch_bounds__(32 * (kConsumers + 1))
prefill_attention_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const PrefillParams p) {
    using S = PrefillShape<kFp8, kConsumers, kStages>;
    extern __shared__ uint8_t smem_raw[];
    const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G;

    grid_dependency_wait();                      // inputs may come from the previous launch
    grid_dependents_launch();
    // ---- this sequence's queries and context (uniform across the CTA) ----
    const int qs0 = __ldg(p.query_start + b), qs1 = __ldg(p.query_start + b + 1);
    const int L = __ldg(p.context_lens + b);
    const int n = qs1 - qs0;
    const int cap = min(p.max_context_len, p.max_blocks_per_seq * kPageRows);
    if (qs0 < 0 || n < 0 || qs1 > p.total || n > p.max_query_len || L < n || L > cap) {
        // inconsistent lengths: flagged, and the sequence's rows are left alone
        if (threadIdx.x == 0 && chunk == 0 && g == 0) flag_error(PKV_DEVERR_CONTEXT_LEN);
        return;
    }
    const int qa = chunk * kConsumers;           // first query of the chunk
    if (qa >= n) return;
    const int nq = min(kConsumers, n - qa);
    const int last_pos = L - n + qa + nq - 1;
    const int npages = last_pos / kPageRows + 1;

    // ---- shared memory: 1024-aligned ring (128B swizzle atoms) + barriers ----
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t ring = (raw + 1023u) & ~1023u;
    const uint32_t bars = ring + S::kRingBytes;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
    auto k_tile = [&](int s) { return ring + s * S::kStageBytes; };
    auto v_tile = [&](int s) { return ring + s * S::kStageBytes + S::kTileBytes; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), kConsumers);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == kConsumers) {
        // =============================== producer ===============================
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
        }
        const int32_t* bt = p.block_tables + (int64_t)b * p.max_blocks_per_seq;
        for (int wbase = 0; wbase < npages; wbase += 32) {
            const int wn = min(32, npages - wbase);
            const int mine = lane < wn ? __ldg(bt + wbase + lane) : -1;
            for (int k = 0; k < wn; ++k) {
                const int it = wbase + k;
                int pb = __shfl_sync(0xffffffffu, mine, k);
                const int s = it % kStages;
                int ok = 1;
                if (lane == 0) {
                    ok = mbar_wait(empty_bar(s), ((it / kStages) & 1) ^ 1);
                    if (ok) {
                        if (pb < 0 || pb >= p.num_blocks) {   // reads as zeros (out of box)
                            flag_error(PKV_DEVERR_BLOCK_ID);
                            pb = -1;
                        }
                        const int row = pb * kPageRows;
                        mbar_arrive_expect_tx(full_bar(s), 2 * S::kTileBytes);
                        if constexpr (kFp8) {
                            tma_load_3d_reused(k_tile(s), &tm_k, full_bar(s), 0, g, row);
                            tma_load_3d_reused(v_tile(s), &tm_v, full_bar(s), 0, g, row);
                        } else {
                            tma_load_3d_reused(k_tile(s), &tm_k, full_bar(s), 0, g, row);
                            tma_load_3d_reused(k_tile(s) + 2048, &tm_k, full_bar(s), 64, g, row);
                            tma_load_3d_reused(v_tile(s), &tm_v, full_bar(s), 0, g, row);
                            tma_load_3d_reused(v_tile(s) + 2048, &tm_v, full_bar(s), 64, g, row);
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) return;
            }
        }
        return;
    }

    // ================================ consumers ================================
    const int r = lane >> 2, c = lane & 3;      // fragment row group / column pair
    const int qi = qa + warp;                    // this warp's query within the sequence
    const bool active = warp < nq;
    const int pos = L - n + qi;                  // its position
    const int64_t row = (int64_t)qs0 + qi;      // its row of q and out
    QOperand<kFp8> qf;
    load_q_fragments(qf, active && r < G ? p.q + (row * p.Hq + (int64_t)g * G + r) * kHeadDim : nullptr, lane);
    WarpState st;
    st.reset();

    bool done = true;
    for (int it = 0; it < npages; ++it) {
        const int s = it % kStages;
        const int ok = mbar_wait(full_bar(s), (it / kStages) & 1);
        // a timed-out wait (flagged) ends this warp's loop and leaves its row unwritten
        if (!__all_sync(0xffffffffu, ok)) {
            done = false;
            break;
        }
        const int first = it * kPageRows;
        if (active && first <= pos)
            attend_page<kFp8>(st, k_tile(s), v_tile(s), min(kPageRows, pos - first + 1), qf, p.logit_scale_log2,
                              lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
    }
    if (!active || !done) return;

    // ---- out[row, heads of g] = O / l ----
    st.reduce_l();
    __half* out_g = p.out + (row * p.Hq + (int64_t)g * G) * kHeadDim;
    const float s0 = p.out_scale / st.l0, s1 = p.out_scale / st.l1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int d_lo = out_channel_lo<kFp8>(r, i), d_hi = out_channel_hi<kFp8>(r, i);
        if (2 * c < G) {
            out_g[(2 * c) * kHeadDim + d_lo] = __float2half_rn(st.o[i][0] * s0);
            out_g[(2 * c) * kHeadDim + d_hi] = __float2half_rn(st.o[i][2] * s0);
        }
        if (2 * c + 1 < G) {
            out_g[(2 * c + 1) * kHeadDim + d_lo] = __float2half_rn(st.o[i][1] * s1);
            out_g[(2 * c + 1) * kHeadDim + d_hi] = __float2half_rn(st.o[i][3] * s1);
        }
    }
}

}  // namespace pkv
