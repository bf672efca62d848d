// Paged GQA decode attention, load-balanced streaming form (the library's
// default plan, partition_tokens = PKV_PARTITION_AUTO).
//
// What it computes is the decode attention of "rvLLM 소개" (discuss.pytorch.kr),
// §PagedAttention과 FlashAttention-3 (see decode_page.cuh). How the work is cut:
//
//  * A unit is one page (16 tokens) of one KV head of one sequence; the batch
//    has U = sum_b Hkv * ceil(L_b / 16) units, ordered (sequence, KV head,
//    page). Every CTA computes that order from context_lens (a scan in shared
//    memory), so nothing is planned on the host and the launch is graph-safe.
//  * Every consumer warp of the persistent grid is a worker that owns an equal
//    contiguous range of units (+-1), so all SMs stream the same number of
//    KV bytes whatever the length mix. A worker drives its own TMA pipeline: a
//    ring of kStages page slots with one transaction barrier each, refilled
//    by the warp's lane 0 right after the slot is consumed; physical block ids
//    come from a 32-entry window of the block table loaded one window ahead.
//  * A worker's range cuts (sequence, KV head) segments into pieces. A piece
//    that is a whole segment writes the output directly. Otherwise the piece
//    writes (m, l, O/l) to the workspace in the warp's fragment order
//    (fragment i of all 32 lanes in one 512-byte run, so every store and load
//    of an item is fully coalesced) and joins a merge tree of fan-in 32: the last
//    of each group of 32 items to finish (an atomic ticket) merges the group
//    by the log-sum-exp rule into the slot of the group's first piece, which
//    is an item of the next level; the merge that leaves one item writes the
//    output. A segment split over hundreds of workers (one very long
//    sequence) thus merges in two or three short levels. No warp ever waits
//    for another CTA.
#pragma once

#include "decode_page.cuh"

namespace pkv {

struct BalancedParams {
    __half* out;                  // [B, Hq, D]
    const __half* q;              // [B, Hq, D]
    const int32_t* block_tables;  // [B, max_blocks_per_seq]
    const int32_t* context_lens;  // [B]
    float4* ws_o;                 // [2 * workers][8][32 lanes] float4   piece outputs O/l
    float4* ws_ml;                // [2 * workers][4] (m, l) pairs of heads 2c, 2c+1
    unsigned int* ws_count;       // [kMergeLevels][2 * workers] tickets of the merge tree
    // fused decode step only: this step's token of every sequence, written to
    // position context_lens[b] - 1 of the cache and attended to in the same launch
    const __half* k_new;          // [B, Hkv, D] f16
    const __half* v_new;
    void* k_cache;                // the pool the tensor maps view (f16 or E4M3 bytes)
    void* v_cache;
    float k_scale, v_scale;       // FP8 quantisation scales of the write
    int32_t B, Hq, Hkv, G;
    int32_t max_blocks_per_seq, num_blocks, max_context_len;
    int32_t min_units_per_worker;
    int32_t overlap_previous;     // read pages/tables/lengths before waiting on the previous launch
    float logit_scale_log2;       // softmax_scale * log2(e) (* k_scale for FP8)
    float out_scale;              // 1 (v_scale for FP8)
    const float* k_scales;        // FP8 device scales [1] or [Hkv], or null: then for KV head g the
    const float* v_scales;        // logit scale is logit_scale_log2 * k_scales[g], the output scale
    int32_t scales_per_head;      // v_scales[g], and the new token is quantised with them
    // failure-detection self-test: this worker (-1: none) issues none of its page loads, so its
    // first barrier wait never completes; every wait of the launch gives up after wait_limit_ns
    int32_t stall_worker;
    uint64_t wait_limit_ns;
};

// Fan-in of the merge tree (at most 32, one item per lane when merging);
// kMergeLevels levels cover every worker of the largest grid.
#ifndef PKV_MERGE_FAN
#define PKV_MERGE_FAN 32
#endif
constexpr int kMergeFan = PKV_MERGE_FAN;
static_assert(kMergeFan >= 2 && kMergeFan <= 32, "merge fan-in");
constexpr int kMergeFloats = 32 * 8 + 16;     // per warp: weights of up to 32 items x 8 heads, M, L
constexpr int merge_levels(int fan) { int l = 1, n = fan; while (n < 4096) { n *= fan; ++l; } return l; }
constexpr int kMergeLevels = merge_levels(kMergeFan);   // fan^levels >= 4096 pieces per segment

template <bool kFp8, int kWarps, int kStages>
struct BalancedShape {
    static constexpr int kTileBytes = kFp8 ? 2048 : 4096;      // one page of K (or V), one head
    static constexpr int kSlotBytes = 2 * kTileBytes;           // K then V
    static constexpr int kRingBytes = kWarps * kStages * kSlotBytes;
    static constexpr int kThreads = 32 * kWarps;
    static size_t smem_bytes(int B) {
        const size_t tables = ((size_t)(2 * B + 1) * 4 + 15) / 16 * 16;
        return 1024 + kRingBytes + tables + (size_t)kWarps * kMergeFloats * 4 + (size_t)kWarps * kStages * 8;
    }
};

// Worker that owns unit u: the largest k with floor(k * U / W) <= u.
__device__ __forceinline__ int worker_of(int64_t u, int64_t U, int W) {
    return (int)(((u + 1) * W - 1) / U);
}

__device__ __forceinline__ int64_t range_start(int k, int64_t U, int W) { return (int64_t)k * U / W; }

// Sequence holding unit u: the last b with prefix[b] <= u (prefix has B + 1 entries).
__device__ __forceinline__ int seq_of_unit(const int* prefix, int B, int u) {
    int lo = 0, hi = B;                         // prefix[lo] <= u < prefix[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= u) lo = mid; else hi = mid;
    }
    return lo;
}

// Four f16 channels divided by `scale` in fp32 (IEEE division), rounded to
// nearest even E4M3 with saturation to +-448, as 4 bytes in channel order.
__device__ __forceinline__ uint32_t quantize4_e4m3(uint2 x, float scale) {
    const __half2* h = reinterpret_cast<const __half2*>(&x);
    uint32_t out = 0;
#pragma unroll
    for (int p2 = 0; p2 < 2; ++p2) {
        const float2 f = __half22float2(h[p2]);
        const float lo = f.x / scale, hi = f.y / scale;
        uint16_t two;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(hi), "f"(lo));
        out |= static_cast<uint32_t>(two) << (16 * p2);
    }
    return out;
}

// Merges at the end of a worker's range stage the items' values in the
// worker's free ring by cp.async (1) or load them into registers like merges
// mid-range (0); a tuning switch.
#ifndef PKV_MERGE_STAGED
#define PKV_MERGE_STAGED 0
#endif

// Two consecutive pages of one segment per online-softmax step (when the
// segment has them in the worker's range): two independent logit chains and
// one max / rescale / shuffle round per 32 tokens. Measured faster for both
// cache types (FP8 0.69 -> 0.78, Qwen2.5-7B f16 0.84 -> 0.91 of the copy peak).
#ifndef PKV_PAGE_PAIRS_FP8
#define PKV_PAGE_PAIRS_FP8 1
#endif
#ifndef PKV_PAGE_PAIRS_F16
#define PKV_PAGE_PAIRS_F16 1
#endif

template <bool kFp8, int kWarps, int kStages, bool kFuseWrite>
__global__ void __launch_bounds__(32 * kWarps)
decode_balanced_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const BalancedParams p) {
    using S = BalancedShape<kFp8, kWarps, kStages>;
    constexpr bool kPagePairs = (kFp8 ? PKV_PAGE_PAIRS_FP8 : PKV_PAGE_PAIRS_F16) && kStages >= 2;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_warp_sum[kWarps];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = p.B, Hkv = p.Hkv, G = p.G;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t ring = (raw + 1023u) & ~1023u;
    int* prefix = reinterpret_cast<int*>(smem_raw + (ring - raw) + S::kRingBytes);   // [B + 1]
    int* lens = prefix + (B + 1);                                                      // [B]
    float* merge_scratch = reinterpret_cast<float*>(
        smem_raw + (ring - raw) + S::kRingBytes + (((2 * B + 1) * 4 + 15) / 16 * 16));  // [warps][kMergeFloats]
    const uint32_t bars = ring + S::kRingBytes + (uint32_t)(((2 * B + 1) * 4 + 15) / 16 * 16) +
                          (uint32_t)(kWarps * kMergeFloats * 4);

    // Everything above touched only shared memory. Inputs may come from the
    // previous launch in the stream: wait for it here, unless the caller
    // declared that it writes none of the KV pages, tables and lengths read
    // before the second wait point below (overlap_previous).
    if (!p.overlap_previous) grid_dependency_wait();
    grid_dependents_launch();

    // ---- unit order: units of sequence b start at prefix[b] ----
    {
        const int cap = min(p.max_context_len, p.max_blocks_per_seq * kPageRows);
        const int per = (B + S::kThreads - 1) / S::kThreads;
        const int b_lo = min(B, (int)threadIdx.x * per), b_hi = min(B, b_lo + per);
        int local = 0;
        for (int b = b_lo; b < b_hi; ++b) {
            int L = __ldg(p.context_lens + b);
            if (L < 0 || L > cap) {
                if (blockIdx.x == 0) flag_error(PKV_DEVERR_CONTEXT_LEN);
                L = L < 0 ? 0 : cap;
            }
            lens[b] = L;
            local += Hkv * ((L + kPageRows - 1) / kPageRows);
        }
        int incl = local;                                   // inclusive scan over the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) s_warp_sum[warp] = incl;
        __syncthreads();
        int run = incl - local;
        for (int w = 0; w < warp; ++w) run += s_warp_sum[w];
        for (int b = b_lo; b < b_hi; ++b) {
            prefix[b] = run;
            run += Hkv * ((lens[b] + kPageRows - 1) / kPageRows);
        }
        if (b_hi == B && b_lo < B) prefix[B] = run;
        if (B == 0 && threadIdx.x == 0) prefix[0] = 0;
        if (lane == 0)
            for (int s = 0; s < kStages; ++s) mbar_init(bars + 8u * (warp * kStages + s), 1);
        mbar_init_fence();
        __syncthreads();
    }
    // ---- this warp's range of units ----
    const int U = prefix[B];
    const int W_total = gridDim.x * kWarps;
    const int worker = blockIdx.x * kWarps + warp;
    // empty contexts get zero rows, spread over all warps (after the wait)
    auto zero_rows = [&]() {
        for (int bb = worker; bb < B; bb += W_total) {
            if (lens[bb] != 0) continue;
            uint4* ob = reinterpret_cast<uint4*>(p.out + (int64_t)bb * p.Hq * kHeadDim);
            for (int i = lane; i < p.Hq * kHeadDim / 8; i += 32) ob[i] = make_uint4(0, 0, 0, 0);
        }
    };
    const int want = (U + p.min_units_per_worker - 1) / p.min_units_per_worker;
    const int W = min(W_total, max(1, want));
    const int u0 = U == 0 ? 0 : (int)range_start(worker, U, W);
    const int n = (U == 0 || worker >= W) ? 0 : (int)range_start(worker + 1, U, W) - u0;
    if (n <= 0) {
        if (p.overlap_previous) grid_dependency_wait();
        zero_rows();
        return;
    }
    if (lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }

    auto full_bar = [&](int s) { return bars + 8u * (warp * kStages + s); };
    auto k_tile = [&](int s) { return ring + (warp * kStages + s) * S::kSlotBytes; };
    auto v_tile = [&](int s) { return k_tile(s) + S::kTileBytes; };
    auto units_of = [&](int b) { return (prefix[b + 1] - prefix[b]) / Hkv; };   // pages per head

    // Block-table window: lane k holds (physical block, KV head) of unit 32w + k.
    auto load_window = [&](int w, int& phys, int& head) {
        const int t = 32 * w + lane;
        phys = -1;
        head = 0;
        if (t < n) {
            const int u = u0 + t;
            const int b = seq_of_unit(prefix, B, u);
            const int nb = units_of(b);
            const int rr = u - prefix[b];
            head = rr / nb;
            phys = __ldg(p.block_tables + (int64_t)b * p.max_blocks_per_seq + (rr - head * nb));
        }
    };
    int win_phys, win_head, nxt_phys, nxt_head, cur_win = 0;
    load_window(0, win_phys, win_head);
    load_window(1, nxt_phys, nxt_head);
    const uint64_t policy = l2_evict_first_policy();
    const bool stalled = worker == p.stall_worker;   // self-test: this worker loads nothing
    int issued = 0;                                  // units [0, issued) have their loads in flight or landed

    // Issues the TMA loads of unit t (t < n) into slot t % kStages; whole warp.
    auto issue = [&](int t) {
        const int w = t >> 5;
        if (w != cur_win) {                     // windows are consumed in order
            win_phys = nxt_phys;
            win_head = nxt_head;
            cur_win = w;
            load_window(w + 1, nxt_phys, nxt_head);
        }
        int pb = __shfl_sync(0xffffffffu, win_phys, t & 31);
        const int hg = __shfl_sync(0xffffffffu, win_head, t & 31);
        if (stalled) return;
        issued = t + 1;
        if (lane == 0) {
            if (pb < 0 || pb >= p.num_blocks) {     // outside the pool: reads as zeros
                flag_error(PKV_DEVERR_BLOCK_ID);
                pb = -1;
            }
            const int s = t % kStages;
            const int row = pb * kPageRows;
            fence_proxy_async_shared();         // earlier generic reads of the slot come first
            mbar_arrive_expect_tx(full_bar(s), S::kSlotBytes);
            if constexpr (kFp8) {
                tma_load_3d(k_tile(s), &tm_k, full_bar(s), 0, hg, row, policy);
                tma_load_3d(v_tile(s), &tm_v, full_bar(s), 0, hg, row, policy);
            } else {
                tma_load_3d(k_tile(s), &tm_k, full_bar(s), 0, hg, row, policy);
                tma_load_3d(k_tile(s) + 2048, &tm_k, full_bar(s), 64, hg, row, policy);
                tma_load_3d(v_tile(s), &tm_v, full_bar(s), 0, hg, row, policy);
                tma_load_3d(v_tile(s) + 2048, &tm_v, full_bar(s), 64, hg, row, policy);
            }
        }
    };
    const int prologue = min(n, kStages);
    for (int t = 0; t < prologue; ++t) issue(t);
    // From here on: q, this step's new tokens, the workspace and out, which
    // the previous launch may produce or still use.
    if (p.overlap_previous) grid_dependency_wait();

    // ---- stream the range ----
    const int r = lane >> 2, c = lane & 3;
    int b = seq_of_unit(prefix, B, u0);
    int nb = units_of(b);
    int g = (u0 - prefix[b]) / nb;
    int j = (u0 - prefix[b]) - g * nb;
    int piece_j0 = j;                          // first page of the current piece
    bool first_piece = true;
    auto q_row = [&](int bb, int gg) -> const __half* {
        return r < G ? p.q + ((int64_t)bb * p.Hq + (int64_t)gg * G + r) * kHeadDim : nullptr;
    };
    QOperand<kFp8> qf;
    load_q_fragments(qf, q_row(b, g), lane);
    // scales of the current segment's KV head (device scales are read after the wait)
    float sl = p.logit_scale_log2, out_scale = p.out_scale, k_quant = p.k_scale, v_quant = p.v_scale;
    auto set_head_scales = [&](int gg) {
        if (p.k_scales) {
            k_quant = head_scale(p.k_scales, p.scales_per_head, gg);
            v_quant = head_scale(p.v_scales, p.scales_per_head, gg);
            sl = p.logit_scale_log2 * k_quant;
            out_scale = v_quant;
        }
    };
    set_head_scales(g);
    if (p.k_scales && blockIdx.x == 0 && warp == 0)
        check_scales(p.k_scales, p.v_scales, p.scales_per_head ? Hkv : 1, lane, 32);
    WarpState st;
    st.reset();

    // Writes out[b, heads of g] from fragment-order values (heads 2c, 2c+1).
    auto write_out = [&](const float (&v)[8][4], float s0, float s1) {
        __half* out_g = p.out + ((int64_t)b * p.Hq + (int64_t)g * G) * kHeadDim;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int dl = out_channel_lo<kFp8>(r, i), dh = out_channel_hi<kFp8>(r, i);
            if (2 * c < G) {
                out_g[(2 * c) * kHeadDim + dl] = __float2half_rn(v[i][0] * s0);
                out_g[(2 * c) * kHeadDim + dh] = __float2half_rn(v[i][2] * s0);
            }
            if (2 * c + 1 < G) {
                out_g[(2 * c + 1) * kHeadDim + dl] = __float2half_rn(v[i][1] * s1);
                out_g[(2 * c + 1) * kHeadDim + dh] = __float2half_rn(v[i][3] * s1);
            }
        }
    };
    // (m, l, O/l) of one partial result, in fragment order, at workspace slot sl.
    auto store_item = [&](int sl, const float (&v)[8][4], float m0, float l0, float m1, float l1) {
        float4* dst = p.ws_o + (int64_t)sl * 256 + lane;
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[32 * i] = make_float4(v[i][0], v[i][1], v[i][2], v[i][3]);
        if (r == 0) p.ws_ml[(int64_t)sl * 4 + c] = make_float4(m0, l0, m1, l1);
    };
    float* wts = merge_scratch + warp * kMergeFloats;     // [32 items][8 heads] + M[8] + L[8]

    // Finishes the piece of segment (b, g) whose last page is j_last. `at_end`:
    // the worker's range ends here, so its ring is free to stage merge loads.
    auto finish_piece = [&](int j_last, bool at_end) {
        st.reduce_l();
        if (piece_j0 == 0 && j_last == nb - 1) {          // the whole segment: write it
            write_out(st.o, out_scale / st.l0, out_scale / st.l1);
            return;
        }
        // The segment's pieces belong to workers k_first..k_last, one each. They
        // are merged by a tree of fan-in 32: at each level the last item of a
        // group of 32 to finish merges the group (ticket, no waiting) into the
        // slot of the group's first piece; one item left means done.
        const int seg_first = prefix[b] + g * nb;
        const int k_first = worker_of(seg_first, U, W);
        const int k_last = worker_of(seg_first + nb - 1, U, W);
        auto slot_of_piece = [&](int q) {
            const int k = k_first + q;
            return 2 * k + (range_start(k, U, W) >= seg_first ? 0 : 1);
        };
        float v[8][4];
        float m0 = st.m0, m1 = st.m1, l0 = st.l0, l1 = st.l1;
        {
            const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[i][0] = st.o[i][0] * i0; v[i][1] = st.o[i][1] * i1;
                v[i][2] = st.o[i][2] * i0; v[i][3] = st.o[i][3] * i1;
            }
        }
        int item = worker - k_first, n_items = k_last - k_first + 1, span = 1;
        store_item(slot_of_piece(item), v, m0, l0, m1, l1);
        for (int lvl = 0;; ++lvl) {
            const int first = item - item % kMergeFan, last = min(first + kMergeFan, n_items) - 1;
            const int cslot = slot_of_piece(first * span);
            unsigned int* cnt = p.ws_count + (int64_t)lvl * 2 * W_total + cslot;
            // The warp barrier orders every lane's stores before lane 0's
            // release-acquire ticket; the merger's loads follow its acquire.
            __syncwarp();
            unsigned int prev = 0;
            if (lane == 0) prev = atomic_add_acq_rel_gpu(cnt, 1u);
            prev = __shfl_sync(0xffffffffu, prev, 0);
            if (prev != (unsigned int)(last - first)) return;   // another item merges the group
            // ---- merge items first..last ----
            // (m, l) are loaded lane-parallel. The items' values come either
            // staged in the worker's free ring (at the end of its range: up to
            // the ring's size in 4 KiB items per round trip, by cp.async) or,
            // mid-range (rare), through registers two items at a time.
            const int n_it = last - first + 1;
            const int my_slot = lane < n_it ? slot_of_piece((first + lane) * span) : 0;
            constexpr int kBatch = kStages * S::kSlotBytes / 4096;        // items per staged round trip
            const uint32_t stage = k_tile(0);
            auto fetch = [&](int b0) {
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    if (b0 + u < n_it) {
                        const int sl = __shfl_sync(0xffffffffu, my_slot, b0 + u);
                        const float4* src = p.ws_o + (int64_t)sl * 256 + lane;
#pragma unroll
                        for (int i = 0; i < 8; ++i) cp_async16(stage + u * 4096 + lane * 128 + 16 * i, src + 32 * i);
                    }
                }
                cp_async_commit();
            };
            auto load_vals = [&](float4 (&dst)[2][8], int t) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    if (t + u < n_it) {
                        const int sl = __shfl_sync(0xffffffffu, my_slot, t + u);
                        const float4* src = p.ws_o + (int64_t)sl * 256 + lane;
#pragma unroll
                        for (int i = 0; i < 8; ++i) dst[u][i] = __ldcg(src + 32 * i);
                    }
                }
            };
            constexpr int kPairs = kFp8 ? 1 : 2;       // register buffers of two items (FP8: register-bound)
            float4 va[kPairs][2][8];
            const bool staged = PKV_MERGE_STAGED && at_end;
            if (staged) fetch(0);
            else load_vals(va[0], 0);
            float mm[8], ll[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float4 a = make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
                if (lane < n_it) a = __ldcg(p.ws_ml + (int64_t)my_slot * 4 + k);
                mm[2 * k] = a.x; ll[2 * k] = a.y; mm[2 * k + 1] = a.z; ll[2 * k + 1] = a.w;
            }
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                float M = mm[h];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
                const float w = lane < n_it ? ll[h] * fast_exp2(mm[h] - M) : 0.f;
                float L = w;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
                wts[lane * 8 + h] = w / L;
                if (lane == 0) {
                    wts[256 + h] = M;
                    wts[264 + h] = L;
                }
            }
            __syncwarp();
            float acc[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
            auto add_item = [&](const float4 (&v)[8], int t) {
                const float w0 = wts[t * 8 + 2 * c], w1 = wts[t * 8 + 2 * c + 1];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    acc[i][0] += w0 * v[i].x; acc[i][1] += w1 * v[i].y;
                    acc[i][2] += w0 * v[i].z; acc[i][3] += w1 * v[i].w;
                }
            };
            if (staged) {
                for (int b0 = 0; b0 < n_it; b0 += kBatch) {
                    cp_async_wait_all();
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        if (b0 + u < n_it) {
                            float4 v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const uint4 raw = lds128(stage + u * 4096 + lane * 128 + 16 * i);
                                v[i] = make_float4(__uint_as_float(raw.x), __uint_as_float(raw.y),
                                                   __uint_as_float(raw.z), __uint_as_float(raw.w));
                            }
                            add_item(v, b0 + u);
                        }
                    }
                    __syncwarp();
                    if (b0 + kBatch < n_it) fetch(b0 + kBatch);
                }
            } else {
                // kPairs buffers: the loads of the next pairs are in flight while one is added
#pragma unroll 1
                for (int t0 = 0; t0 < n_it; t0 += 2 * kPairs) {
#pragma unroll
                    for (int k = 1; k < kPairs; ++k)
                        if (t0 + 2 * k < n_it) load_vals(va[k], t0 + 2 * k);
#pragma unroll
                    for (int k = 0; k < kPairs; ++k) {
#pragma unroll
                        for (int u = 0; u < 2; ++u)
                            if (t0 + 2 * k + u < n_it) add_item(va[k][u], t0 + 2 * k + u);
                        if (k == 0 && t0 + 2 * kPairs < n_it) load_vals(va[0], t0 + 2 * kPairs);
                    }
                }
            }
            m0 = wts[256 + 2 * c]; m1 = wts[256 + 2 * c + 1];
            l0 = wts[264 + 2 * c]; l1 = wts[264 + 2 * c + 1];
            __syncwarp();
            if (lane == 0) *cnt = 0u;                          // ready for the next call
            const int n_next = (n_items + kMergeFan - 1) / kMergeFan;
            if (n_next == 1) {
                write_out(acc, out_scale, out_scale);
                return;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[i][0] = acc[i][0]; v[i][1] = acc[i][1]; v[i][2] = acc[i][2]; v[i][3] = acc[i][3];
            }
            store_item(cslot, v, m0, l0, m1, l1);              // the group is one item of level + 1
            item = first / kMergeFan;
            n_items = n_next;
            span *= kMergeFan;
        }
    };

    // Fused decode step: writes this step's K/V of segment (b, g) into row
    // (L - 1) % 16 of the page in slot s -- in shared memory for this launch,
    // in the cache for later ones. Lane l holds channels 4l..4l+3. The page's
    // TMA copy may hold the row's old contents; the shared row is overwritten
    // after the copy landed, so attention sees the new token either way.
    auto write_new_token = [&](int s, int jl) {          // jl = nb - 1, the segment's last page
        const int row = (lens[b] - 1) & (kPageRows - 1);
        const int64_t src = ((int64_t)b * Hkv + g) * kHeadDim + 4 * lane;
        const uint2 kh = __ldg(reinterpret_cast<const uint2*>(p.k_new + src));
        const uint2 vh = __ldg(reinterpret_cast<const uint2*>(p.v_new + src));
        const int pb = __ldg(p.block_tables + (int64_t)b * p.max_blocks_per_seq + jl);
        const bool in_pool = pb >= 0 && pb < p.num_blocks;
        const int64_t dst = (((int64_t)pb * kPageRows + row) * Hkv + g) * kHeadDim + 4 * lane;
        if constexpr (kFp8) {
            const uint32_t kq = quantize4_e4m3(kh, k_quant), vq = quantize4_e4m3(vh, v_quant);
            const uint32_t off = row * 128 + ((((lane >> 2) ^ (row & 7))) << 4) + (lane & 3) * 4;
            asm volatile("st.shared.u32 [%0], %1;" :: "r"(k_tile(s) + off), "r"(kq) : "memory");
            asm volatile("st.shared.u32 [%0], %1;" :: "r"(v_tile(s) + off), "r"(vq) : "memory");
            if (in_pool) {
                reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.k_cache) + dst)[0] = kq;
                reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.v_cache) + dst)[0] = vq;
            }
        } else {
            const uint32_t off = (lane >> 4) * 2048 + row * 128 +
                                 ((((lane & 15) >> 1) ^ (row & 7)) << 4) + (lane & 1) * 8;
            asm volatile("st.shared.v2.u32 [%0], {%1, %2};" :: "r"(k_tile(s) + off), "r"(kh.x), "r"(kh.y)
                         : "memory");
            asm volatile("st.shared.v2.u32 [%0], {%1, %2};" :: "r"(v_tile(s) + off), "r"(vh.x), "r"(vh.y)
                         : "memory");
            if (in_pool) {
                *reinterpret_cast<uint2*>(static_cast<__half*>(p.k_cache) + dst) = kh;
                *reinterpret_cast<uint2*>(static_cast<__half*>(p.v_cache) + dst) = vh;
            }
        }
        __syncwarp();
    };

    // A wait that ran out (flagged by mbar_wait) ends this worker: first it
    // waits, again with the limit, for the loads it issued after unit `lost`,
    // so that no copy into its ring is in flight when it returns. Its piece
    // is neither written nor merged; the caller learns of it from the
    // device error word, and the workspace's tickets must be cleared.
    auto drain_after = [&](int lost) {
        for (int u = lost + 1; u < issued; ++u)
            mbar_wait(full_bar(u % kStages), (u / kStages) & 1, p.wait_limit_ns);
    };
    for (int t = 0; t < n; ++t) {
        const int s = t % kStages;
        if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), (t / kStages) & 1, p.wait_limit_ns))) {
            drain_after(t);
            return;
        }
        if (kPagePairs && j + 1 < nb && t + 1 < n) {
            // pages t and t + 1 are consecutive pages of one segment: one softmax step
            const int s2 = (t + 1) % kStages;
            if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s2), ((t + 1) / kStages) & 1, p.wait_limit_ns))) {
                drain_after(t + 1);
                return;
            }
            const int valid_b = j + 1 == nb - 1 ? lens[b] - (j + 1) * kPageRows : kPageRows;
            if constexpr (kFuseWrite) {
                if (j + 1 == nb - 1) write_new_token(s2, j + 1);   // page B holds position L - 1
            }
            attend_page_pair<kFp8>(st, k_tile(s), v_tile(s), k_tile(s2), v_tile(s2), valid_b, qf, sl, lane);
            __syncwarp();
            if (t + kStages < n) issue(t + kStages);
            if (t + 1 + kStages < n) issue(t + 1 + kStages);
            ++t;                                   // the cursor moves to page B
            ++j;
        } else {
            const int valid = j == nb - 1 ? lens[b] - j * kPageRows : kPageRows;
            if constexpr (kFuseWrite) {
                if (j == nb - 1) write_new_token(s, j);    // this page holds position L - 1
            }
            attend_page<kFp8>(st, k_tile(s), v_tile(s), valid, qf, sl, lane);
            __syncwarp();
            if (t + kStages < n) issue(t + kStages);
        }
        // advance the cursor; a segment boundary (or the range end) closes the piece
        const bool seg_end = j == nb - 1;
        if (seg_end || t == n - 1) {
            finish_piece(j, t == n - 1);
            if (t == n - 1) break;
            first_piece = false;
            st.reset();
            if (seg_end) {
                j = 0;
                if (++g == Hkv) {
                    g = 0;
                    do { ++b; } while (units_of(b) == 0);
                    nb = units_of(b);
                }
                load_q_fragments(qf, q_row(b, g), lane);
                set_head_scales(g);
            }
            piece_j0 = j;
        } else {
            ++j;
        }
    }
    zero_rows();
}

}  // namespace pkv
