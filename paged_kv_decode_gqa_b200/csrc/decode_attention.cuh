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
//    partition's (m, l, O/l) to the workspace, and the partitions of (b, g)
//    merge by the log-sum-exp rule in a tree of fan-in 8: the CTA that
//    finishes a group last (a release-acquire ticket, no waiting) merges its
//    entries, every load in flight at once, into the group's first entry;
//    the merge that leaves one entry writes the output.
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
    unsigned int* ws_count;       // [levels][B*Hkv][nparts] merge-tree tickets, zero between calls
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

// Fan-in of the split-KV merge tree over fixed partitions: a merge reads at
// most this many partition entries, all of them in flight at once.
constexpr int kPartFan = 8;

// Levels of that tree for n partitions (1 for n <= kPartFan).
__host__ __device__ constexpr int part_merge_levels(int n) {
    int l = 1;
    for (int64_t c = kPartFan; c < n; c *= kPartFan) ++l;
    return l;
}

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

    // ---- split-KV: a merge tree of fan-in kPartFan over the partitions ----
    // Level 0 items are the partitions. At each level the last item of a group
    // of kPartFan to finish (a release-acquire ticket, no waiting) merges the
    // group by the log-sum-exp rule into the entry of the group's first item;
    // the merge that leaves one item writes the output.
    const int64_t BH = (int64_t)gridDim.z * p.Hkv;
    int item = part, n_items = nparts_b, span = 1;
    for (int lvl = 0;; ++lvl) {
        const int first = item - item % kPartFan, last = min(first + kPartFan, n_items) - 1;
        unsigned int* cnt = p.ws_count + ((int64_t)lvl * BH + (int64_t)b * p.Hkv + g) * p.nparts + first * span;
        // The barrier orders every thread's workspace stores before thread 0's
        // ticket; the merger's loads follow its acquire and the barrier after it.
        consumer_sync(kCT);
        if (threadIdx.x == 0) {
            const unsigned int prev = atomic_add_acq_rel_gpu(cnt, 1u);
            s_is_last = prev == (unsigned int)(last - first);
        }
        consumer_sync(kCT);
        if (!s_is_last) return;
        const int n_it = last - first + 1;
        const int n_next = (n_items + kPartFan - 1) / kPartFan;
        // one (head, 4 channels) item per thread; the items' (m, l) and O are requested together,
        // one round trip, and weighted after they land (a warp serves one head)
        for (int it = threadIdx.x; it < G * (kHeadDim / 4); it += kCT) {
            const int h = it / (kHeadDim / 4), cq = it % (kHeadDim / 4);
            const int64_t e0 = (row0 + h) * p.nparts + (int64_t)first * span;
            float4* base = reinterpret_cast<float4*>(p.ws_o + e0 * kHeadDim) + cq;
            float4 v[kPartFan];
            float mj[kPartFan], lj[kPartFan];
#pragma unroll
            for (int j = 0; j < kPartFan; ++j)
                if (j < n_it) {
                    const int64_t off = (int64_t)j * span;
                    v[j] = __ldcg(base + off * (kHeadDim / 4));
                    mj[j] = __ldcg(p.ws_m + e0 + off);
                    lj[j] = __ldcg(p.ws_l + e0 + off);
                }
            float M = -INFINITY;
#pragma unroll
            for (int j = 0; j < kPartFan; ++j)
                if (j < n_it) M = fmaxf(M, mj[j]);
            float L = 0.f;
#pragma unroll
            for (int j = 0; j < kPartFan; ++j)
                if (j < n_it) {
                    mj[j] = lj[j] * fast_exp2(mj[j] - M);          // the item's weight
                    L += mj[j];
                }
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < kPartFan; ++j)
                if (j < n_it) {                                    // item order
                    const float w = mj[j] / L;
                    acc.x += w * v[j].x;
                    acc.y += w * v[j].y;
                    acc.z += w * v[j].z;
                    acc.w += w * v[j].w;
                }
            if (n_next == 1) {
                uint2 o;
                o.x = pack_half2(acc.x * out_scale, acc.y * out_scale);
                o.y = pack_half2(acc.z * out_scale, acc.w * out_scale);
                *reinterpret_cast<uint2*>(out_g + h * kHeadDim + 4 * cq) = o;
            } else {
                base[0] = acc;                                     // the group is one item of the next level
                if (cq == 0) {
                    p.ws_m[e0] = M;
                    p.ws_l[e0] = L;
                }
            }
        }
        if (threadIdx.x == 0) *cnt = 0u;                         // ready for the next call
        if (n_next == 1) return;
        item = first / kPartFan;
        n_items = n_next;
        span *= kPartFan;
    }
}

}  // namespace pkv
