// Paged grouped-query decode attention for sm_100a.
//
// What it computes (rvLLM 소개 (discuss.pytorch.kr), §PagedAttention과
// FlashAttention-3): for each sequence b and query head h, attention of the one
// new query over the sequence's cached keys/values, read through the
// PagedAttention block table; query heads sharing a KV head (Qwen2.5: 12 over
// 2) are served from one read of that head's K/V, which is where the page's
// "6x less KV bandwidth" comes from. The cache is f16 or FP8 E4M3.
//
// Work unit: one CTA per (partition p, KV head g, sequence b). A partition is
// `partition_tokens` consecutive logical tokens (the whole sequence when not
// splitting). The CTA streams its blocks' K and V once and serves all G query
// heads of g from them.
//
// CTA layout: kConsumers consumer warps + 1 producer warp.
//  * Producer (last warp): reads the block-table window with one coalesced
//    warp load per 32 blocks, and for each stage issues TMA tile loads of
//    kConsumers physical blocks (K and V, 16 rows x 128 channels each,
//    128-byte swizzled) into a kStages-deep shared-memory ring, signalling a
//    per-stage "full" mbarrier by transaction bytes.
//  * Consumer warp w takes block w of every stage: S^T = K Q^T and
//    O^T += V^T P^T on the tensor cores (mma.sync m16n8k16, f16 in, f32
//    accumulate) with the KV tokens on the M side and the G <= 8 query heads
//    on N = 8, an online softmax in registers (exp2 domain), and frees the
//    stage with an arrive on its "empty" mbarrier.
//  * The consumer warps' (m, l, O) are merged through shared memory. With one
//    partition the CTA writes out[b, heads of g]; otherwise it writes the
//    partition's (m, l, O/l) to the workspace and the CTA that finishes the
//    last partition of (b, g) -- found by a release-acquire ticket, no
//    waiting -- merges all partitions by the log-sum-exp rule and writes the
//    output, with 16 partitions' loads in flight per (head, 4 channels).
//
// FP8 E4M3 blocks are expanded to f16 in registers (exact), with k_scale
// folded into the logit scale and v_scale into the output.
#pragma once

#include "decode_page.cuh"

namespace pkv {

struct DecodeParams {
    __half* out;                  // [B, Hq, D]
    const __half* q;              // [B, Hq, D]
    const int32_t* block_tables;  // [B, max_blocks_per_seq]
    const int32_t* context_lens;  // [B]
    float* ws_o;                  // [B*Hq, nparts, D]   partition outputs O/l
    float* ws_m;                  // [B*Hq, nparts]      partition max (exp2 domain)
    float* ws_l;                  // [B*Hq, nparts]      partition sum
    unsigned int* ws_count;       // [B*Hkv]             finished partitions (ticket)
    int32_t Hq, Hkv, G;
    int32_t max_blocks_per_seq, num_blocks, max_context_len;
    int32_t partition_tokens;     // multiple of kPageRows
    int32_t nparts;               // partitions per sequence covered by the grid
    float logit_scale_log2;       // softmax_scale * log2(e) (* k_scale for FP8 with per-tensor scales)
    float out_scale;              // 1 (v_scale for FP8 with per-tensor scales)
    const float* k_scales;        // FP8 device scales [1] or [Hkv], or null: then for KV head g the
    const float* v_scales;        // logit scale is logit_scale_log2 * k_scales[g], the output v_scales[g]
    int32_t scales_per_head;
};

template <bool kFp8, int kConsumers, int kStages>
struct DecodeShape {
    static constexpr int kTileBytes = kFp8 ? 2048 : 4096;            // 16 rows x 128 ch, one of K/V
    static constexpr int kStageBytes = 2 * kConsumers * kTileBytes;  // K tiles then V tiles
    static constexpr int kThreads = 32 * (kConsumers + 1);
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kMergeBytes = kConsumers * kGroupPad * (kHeadDim + 2) * 4;
    static constexpr int kSmemBytes = 1024 + kRingBytes + 2 * kStages * 8 + 16;
    static_assert(kMergeBytes <= kRingBytes, "merge scratch must fit in the ring");
    static_assert((32 * kConsumers) % kHeadDim == 0, "merge maps one thread per channel");
    static_assert(32 % kConsumers == 0, "table window must hold whole stages");
};

__device__ __forceinline__ void consumer_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" :: "r"(nthreads) : "memory");
}

template <bool kFp8, int kConsumers, int kStages>
__global__ void __launch_bounds__(32 * (kConsumers + 1))
decode_attention_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
    using S = DecodeShape<kFp8, kConsumers, kStages>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_is_last;

    const int part = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G;

    grid_dependency_wait();                      // inputs may come from the previous launch
    grid_dependents_launch();
    // ---- this CTA's token range (uniform across the CTA) ----
    int L = __ldg(p.context_lens + b);
    const int cap = min(p.max_context_len, p.max_blocks_per_seq * kPageRows);
    if (L < 0 || L > cap) {
        if (threadIdx.x == 0 && part == 0 && g == 0) flag_error(PKV_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : cap;
    }
    const int P = p.partition_tokens;
    __half* out_g = p.out + ((int64_t)b * p.Hq + (int64_t)g * G) * kHeadDim;
    if (L == 0) {                                  // empty context: zero rows
        if (part == 0)
            for (int i = threadIdx.x; i < G * kHeadDim; i += blockDim.x) out_g[i] = __float2half_rn(0.f);
        return;
    }
    const int t_begin = part * P;
    if (t_begin >= L) return;
    const int t_end = min(t_begin + P, L);
    const int nparts_b = (L + P - 1) / P;
    const int blk0 = t_begin / kPageRows;
    const int nblk = (t_end - t_begin + kPageRows - 1) / kPageRows;
    const int n_iters = (nblk + kConsumers - 1) / kConsumers;
    // t_begin is page aligned, so only the partition's last block can be partial
    const int last_valid = t_end - (blk0 + nblk - 1) * kPageRows;

    // ---- shared memory: 1024-aligned ring (128B swizzle atoms) + barriers ----
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t ring = (raw + 1023u) & ~1023u;
    uint8_t* ring_ptr = smem_raw + (ring - raw);
    const uint32_t bars = ring + S::kRingBytes;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
    auto k_tile = [&](int s, int w) { return ring + s * S::kStageBytes + w * S::kTileBytes; };
    auto v_tile = [&](int s, int w) {
        return ring + s * S::kStageBytes + (kConsumers + w) * S::kTileBytes;
    };

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
        const uint64_t policy = l2_evict_first_policy();
        const int32_t* bt = p.block_tables + (int64_t)b * p.max_blocks_per_seq + blk0;
        int it = 0;
        for (int wbase = 0; wbase < nblk; wbase += 32) {
            const int wn = min(32, nblk - wbase);
            const int mine = lane < wn ? __ldg(bt + wbase + lane) : -1;
            for (int k = 0; k < wn; k += kConsumers, ++it) {
                int phys[kConsumers];
#pragma unroll
                for (int q = 0; q < kConsumers; ++q) phys[q] = __shfl_sync(0xffffffffu, mine, (k + q) & 31);
                const int s = it % kStages;
                int ok = 1;
                if (lane == 0) {
                    ok = mbar_wait(empty_bar(s), ((it / kStages) & 1) ^ 1);
                    if (ok) {
                        const int nb = min(kConsumers, wn - k);
                        mbar_arrive_expect_tx(full_bar(s), nb * 2 * S::kTileBytes);
                        for (int q = 0; q < nb; ++q) {
                            int pb = phys[q];
                            if (pb < 0 || pb >= p.num_blocks) {   // reads as zeros (out of box)
                                flag_error(PKV_DEVERR_BLOCK_ID);
                                pb = -1;
                            }
                            const int row = pb * kPageRows;
                            if constexpr (kFp8) {
                                tma_load_3d(k_tile(s, q), &tm_k, full_bar(s), 0, g, row, policy);
                                tma_load_3d(v_tile(s, q), &tm_v, full_bar(s), 0, g, row, policy);
                            } else {
                                tma_load_3d(k_tile(s, q), &tm_k, full_bar(s), 0, g, row, policy);
                                tma_load_3d(k_tile(s, q) + 2048, &tm_k, full_bar(s), 64, g, row, policy);
                                tma_load_3d(v_tile(s, q), &tm_v, full_bar(s), 0, g, row, policy);
                                tma_load_3d(v_tile(s, q) + 2048, &tm_v, full_bar(s), 64, g, row, policy);
                            }
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
    // logit and output scales of KV head g
    const float sl = p.k_scales ? p.logit_scale_log2 * head_scale(p.k_scales, p.scales_per_head, g)
                                : p.logit_scale_log2;
    const float out_scale = p.v_scales ? head_scale(p.v_scales, p.scales_per_head, g) : p.out_scale;
    if (p.k_scales && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0)
        check_scales(p.k_scales, p.v_scales, p.scales_per_head ? p.Hkv : 1, 0, 1);
    QOperand<kFp8> qf;
    load_q_fragments(qf, r < G ? p.q + ((int64_t)b * p.Hq + (int64_t)g * G + r) * kHeadDim : nullptr, lane);
    WarpState st;
    st.reset();

    for (int it = 0; it < n_iters; ++it) {
        const int s = it % kStages;
        const int ok = mbar_wait(full_bar(s), (it / kStages) & 1);
        // A timed-out wait (flagged) ends this warp's loop; the warp still
        // joins the merge barriers below so that no other warp waits for it.
        if (!__all_sync(0xffffffffu, ok)) break;
        const int blk = it * kConsumers + warp;
        if (blk < nblk) {
            const int valid = blk == nblk - 1 ? last_valid : kPageRows;
            attend_page<kFp8>(st, k_tile(s, warp), v_tile(s, warp), valid, qf, sl, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
    }

    // ---- merge the consumer warps through shared memory (ring reused) ----
    st.reduce_l();
    constexpr int kCT = 32 * kConsumers;
    consumer_sync(kCT);                           // every warp is done with the ring
    float* red_o = reinterpret_cast<float*>(ring_ptr);                 // [warp][head][D]
    float* red_m = red_o + kConsumers * kGroupPad * kHeadDim;          // [warp][head]
    float* red_l = red_m + kConsumers * kGroupPad;
    {
        float* ow = red_o + warp * kGroupPad * kHeadDim;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int d_lo = out_channel_lo<kFp8>(r, i), d_hi = out_channel_hi<kFp8>(r, i);
            ow[(2 * c) * kHeadDim + d_lo] = st.o[i][0];
            ow[(2 * c + 1) * kHeadDim + d_lo] = st.o[i][1];
            ow[(2 * c) * kHeadDim + d_hi] = st.o[i][2];
            ow[(2 * c + 1) * kHeadDim + d_hi] = st.o[i][3];
        }
        if (r == 0) {
            red_m[warp * kGroupPad + 2 * c] = st.m0;
            red_m[warp * kGroupPad + 2 * c + 1] = st.m1;
            red_l[warp * kGroupPad + 2 * c] = st.l0;
            red_l[warp * kGroupPad + 2 * c + 1] = st.l1;
        }
    }
    consumer_sync(kCT);

    const int d = threadIdx.x % kHeadDim;
    const int h_first = threadIdx.x / kHeadDim, h_step = kCT / kHeadDim;
    const int64_t row0 = (int64_t)b * p.Hq + (int64_t)g * G;   // first query head of g
    for (int h = h_first; h < G; h += h_step) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, red_m[w * kGroupPad + h]);
        float lsum = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
            const float sc = fast_exp2(red_m[w * kGroupPad + h] - M);
            lsum += red_l[w * kGroupPad + h] * sc;
            acc += red_o[(w * kGroupPad + h) * kHeadDim + d] * sc;
        }
        if (nparts_b == 1) {
            out_g[h * kHeadDim + d] = __float2half_rn(acc / lsum * out_scale);
        } else {
            const int64_t pr = (row0 + h) * p.nparts + part;
            p.ws_o[pr * kHeadDim + d] = acc / lsum;
            if (d == 0) {
                p.ws_m[pr] = M;
                p.ws_l[pr] = lsum;
            }
        }
    }
    if (nparts_b == 1) return;

    // ---- split-KV: the last partition of (b, g) to finish merges them all ----
    // The barrier orders every thread's workspace stores before thread 0's
    // release-acquire ticket; the merger's loads follow its acquire and the
    // barrier after it.
    consumer_sync(kCT);
    if (threadIdx.x == 0) {
        const unsigned int prev = atomic_add_acq_rel_gpu(p.ws_count + (int64_t)b * p.Hkv + g, 1u);
        s_is_last = prev == (unsigned int)(nparts_b - 1);
    }
    consumer_sync(kCT);
    if (!s_is_last) return;
    // weights w_q = l_q * exp2(m_q - M) of every partition and head, staged in
    // shared memory (the ring is free), then one pass over the outputs
    float* wts = reinterpret_cast<float*>(ring_ptr);             // [G][nparts_b]
    const bool staged = (size_t)G * nparts_b * sizeof(float) <= (size_t)S::kRingBytes;
    if (staged) {
        for (int i = threadIdx.x; i < G * nparts_b; i += kCT) {
            const int h = i / nparts_b, q = i - h * nparts_b;
            wts[i] = __ldcg(p.ws_m + (row0 + h) * p.nparts + q);
        }
        consumer_sync(kCT);
        // one warp per head: max, weights, normaliser
        for (int h = warp; h < G; h += kConsumers) {
            float* wh = wts + h * nparts_b;
            float M = -INFINITY;
            for (int q = lane; q < nparts_b; q += 32) M = fmaxf(M, wh[q]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
            float sum = 0.f;
            for (int q = lane; q < nparts_b; q += 32) {
                const float w = __ldcg(p.ws_l + (row0 + h) * p.nparts + q) * fast_exp2(wh[q] - M);
                wh[q] = w;
                sum += w;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            __syncwarp();
            for (int q = lane; q < nparts_b; q += 32) wh[q] *= out_scale / sum;
        }
        consumer_sync(kCT);
        // one (head, 4 channels) item per thread, 16 partitions' float4 loads in flight at a time
        constexpr int kBatch = 16;
        for (int it = threadIdx.x; it < G * (kHeadDim / 4); it += kCT) {
            const int h = it / (kHeadDim / 4), cq = it % (kHeadDim / 4);
            const float* wh = wts + h * nparts_b;
            const float4* src = reinterpret_cast<const float4*>(p.ws_o + (row0 + h) * p.nparts * kHeadDim) + cq;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int q0 = 0; q0 < nparts_b; q0 += kBatch) {
                float4 v[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u)
                    if (q0 + u < nparts_b) v[u] = __ldcg(src + (int64_t)(q0 + u) * (kHeadDim / 4));
#pragma unroll
                for (int u = 0; u < kBatch; ++u)
                    if (q0 + u < nparts_b) {                        // partition order
                        const float w = wh[q0 + u];
                        acc.x += w * v[u].x;
                        acc.y += w * v[u].y;
                        acc.z += w * v[u].z;
                        acc.w += w * v[u].w;
                    }
            }
            uint2 o;
            o.x = pack_half2(acc.x, acc.y);
            o.y = pack_half2(acc.z, acc.w);
            *reinterpret_cast<uint2*>(out_g + h * kHeadDim + 4 * cq) = o;
        }
    } else {
        for (int h = h_first; h < G; h += h_step) {
            const int64_t pr0 = (row0 + h) * p.nparts;
            float M = -INFINITY;
            for (int q = 0; q < nparts_b; ++q) M = fmaxf(M, __ldcg(p.ws_m + pr0 + q));
            float wsum = 0.f, acc = 0.f;
            for (int q = 0; q < nparts_b; ++q) {
                const float w = __ldcg(p.ws_l + pr0 + q) * fast_exp2(__ldcg(p.ws_m + pr0 + q) - M);
                wsum += w;
                acc += w * __ldcg(p.ws_o + (pr0 + q) * kHeadDim + d);
            }
            out_g[h * kHeadDim + d] = __float2half_rn(acc / wsum * out_scale);
        }
    }
    if (threadIdx.x == 0) p.ws_count[(int64_t)b * p.Hkv + g] = 0u;   // ready for the next call
}

}  // namespace pkv
