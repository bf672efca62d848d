// Paged (chunked) prefill attention on the fifth-generation tensor cores
// (tcgen05, TMEM accumulators), f16 cache.
//
// What it computes is the chunked prefill of prefill_attention.cuh (same
// reading: query i of sequence b sits at position L_b - n_b + i and attends
// causally to positions [0, p] of the sequence's paged cache, query head h
// reading KV head h / G); pages: "rvLLM 소개" (discuss.pytorch.kr),
// §PagedAttention과 FlashAttention-3 (paged cache, GQA) and §H100 SXM 80GB 직접
// 엔진 벤치마크 (prefill as the engine's other attention work).
//
// Unlike decode, prefill is a dense contraction, so each CTA runs it as two
// GEMMs per KV tile on tcgen05:
//  * Work unit: one CTA per (tile of T = floor(128 / G) query tokens, KV head
//    g, sequence b). The tile's M = T * G <= 128 rows are its queries x the G
//    query heads of g, row r = token r / G, head r % G, so every K/V byte a
//    CTA stages serves all G heads of every query in it.
//  * A KV tile is 128 tokens (8 pages). K and V pages come by TMA into
//    three-stage rings, K and V with their own barriers and their own TMA
//    warp: a K stage is refilled as soon as S of its tile is done, a V stage
//    once O += P V of its tile is. Each refill takes over a microsecond to
//    land from L2, so the rings hold as many tiles as shared memory allows:
//    the probabilities stay in TMEM, which frees the room. Q (the CTA's rows)
//    comes once.
//  * The KV tiles are split by parity into two independent online softmaxes,
//    each with its own running maximum, row sum and accumulator, merged by
//    the log-sum-exp rule at the end (split-KV inside the CTA). Softmax warps
//    0-3 serve the even tiles and warps 4-7 the odd ones; warps w and w + 4
//    share a scheduler and a TMEM lane quarter (rows 32 (w % 4) .. +31), and
//    as they work on different tiles one's exp2 runs while the other loads or
//    takes maxima. A thread owns a whole row of its tiles, so no maximum
//    crosses warps.
//  * One thread issues S = Q K^T (M = 128, N = 128, K = 128; K-major A and
//    B) into the TMEM columns of the tile's parity, [0, 128) or [128, 256),
//    and after the softmax O_par += P V into [256, 384) or [384, 512), with P
//    read from TMEM (the A operand of `tcgen05.mma` may live there: row r in
//    lane r, two f16 per column) and V MN-major from shared memory. S of tile
//    j + 1 is issued before O += P V of tile j; S of tile j + 2 waits until
//    O += P V of tile j has read P out of the same columns.
//  * Softmax of a tile, per thread (row r): pass 1 reads the row's 128
//    logits from TMEM in four 32-column loads and takes their maximum (the
//    causal mask only on tiles that reach past the tile's first position);
//    the running maximum (exp2 domain) is raised only when a tile's maximum
//    exceeds it by more than 8 (a factor 256), and only then are the row's
//    accumulator and sum rescaled. Pass 2 reads the logits again and forms
//    exp2(s * scale - m) with one fused multiply-add and the fp32 exp2,
//    rounds to f16, adds exactly those f16 values to the row sum in fp32
//    (mixed-precision add), and stores the f16 pairs over the logits already
//    read. The output is (O_even a_e + O_odd a_o) / (l_e a_e + l_o a_o) in
//    f16, a = exp2(m - max(m_e, m_o)); warps 0-3 write channels 0-63, 4-7
//    the rest.
//  * Rows past the context in the sequence's last page (free slots, any
//    content) are zeroed in shared memory before their V is used; pages past
//    the tile's last position are loaded from outside the pool, which TMA
//    fills with zeros.
// Every barrier wait has a time limit; one that runs out flags
// PKV_DEVERR_WAIT_TIMEOUT and makes every role stop, wait for what it has in
// flight, and leave; TMEM is always freed.
#pragma once

#include "decode_page.cuh"
#include "prefill_attention.cuh"
#include "umma.cuh"

namespace pkv {

struct PrefillTcShape {
    static constexpr int kRows = 128;                  // M: query tokens x heads
    static constexpr int kKvTok = 128;                 // N of S, K of P V: tokens per KV tile
    static constexpr int kStages = 2;
    static constexpr int kQTiles = 2;                  // query tiles per CTA, sharing every K/V stage
    static constexpr int kChunk = 128 * 128;           // one 64-channel (or 64-token) half of a tile: 16 KiB
    static constexpr int kQBytes = 2 * kChunk;         // Q: 128 rows x 128 channels
    static constexpr int kKvBytes = 2 * kChunk;        // K or V of one tile: 128 tokens x 128 channels
    static constexpr int kBarBytes = 256;
    static constexpr int kSmemBytes = 1024 + kQTiles * kQBytes + 2 * kStages * kKvBytes + kBarBytes;
    static constexpr int kSoftmaxWarps = 8;
    static constexpr int kThreads = 32 * (kSoftmaxWarps + 3);   // warps 0-7 softmax, 8 TMA K (and Q), 9 TMA V, 10 MMA
    static constexpr int kTmaKWarp = kSoftmaxWarps, kTmaVWarp = kSoftmaxWarps + 1, kMmaWarp = kSoftmaxWarps + 2;
    static constexpr uint32_t kTmemCols = 512;         // S_A, S_B (P over them), O_A, O_B: 128 columns each
    static constexpr float kRescaleThreshold = 8.f;    // log2 of the largest unnormalised probability
};

// acc += the f16 value in the low (hi = false) or high half of w, exactly (mixed-precision add).
__device__ __forceinline__ float add_f16_lo(float acc, uint32_t w) {
    asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; add.rn.f32.f16 %0, lo, %0; }" : "+f"(acc) : "r"(w));
    return acc;
}
__device__ __forceinline__ float add_f16_hi(float acc, uint32_t w) {
    asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; add.rn.f32.f16 %0, hi, %0; }" : "+f"(acc) : "r"(w));
    return acc;
}

// One work item of the persistent grid (every thread computes the same).
struct PrefillItem {
    int b, g, qs0, i0, nq, pos0, ntiles, npages, L;
};

template <int kDummy = 0>
__global__ void __launch_bounds__(PrefillTcShape::kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const PrefillParams p, const int tok_per_tile,
                  const int q_groups, const int batch) {
    using S = PrefillTcShape;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G, T = tok_per_tile;

    grid_dependency_wait();                      // inputs may come from the previous launch
    grid_dependents_launch();
    // ---- work items: (group of two query tiles, KV head, sequence), costliest groups first ----
    const int per_q = p.Hkv * batch;
    const int n_items = q_groups * per_q;
    const int C = gridDim.x;
    // the r-th item of this CTA in the snake order (CTA c takes c, 2C - 1 - c, 2C + c, ...), or -1
    auto item_index = [&](int r) -> int {
        const int i = r * C + ((r & 1) ? C - 1 - (int)blockIdx.x : (int)blockIdx.x);
        return i < n_items ? i : -1;
    };
    const int cap = min(p.max_context_len, p.max_blocks_per_seq * kPageRows);
    // false: the item has no queries (or its sequence is inconsistent: flagged once, rows left alone)
    auto item_info = [&](int i, PrefillItem& it) -> bool {
        const int qg = q_groups - 1 - i / per_q, rem = i % per_q;
        it.g = rem % p.Hkv;
        it.b = rem / p.Hkv;
        it.qs0 = __ldg(p.query_start + it.b);
        const int qs1 = __ldg(p.query_start + it.b + 1);
        it.L = __ldg(p.context_lens + it.b);
        const int n = qs1 - it.qs0;
        if (it.qs0 < 0 || n < 0 || qs1 > p.total || n > p.max_query_len || it.L < n || it.L > cap) {
            if (threadIdx.x == 0 && qg == 0 && it.g == 0) flag_error(PKV_DEVERR_CONTEXT_LEN);
            return false;
        }
        it.i0 = qg * S::kQTiles * T;             // first query of the item's two tiles
        if (it.i0 >= n) return false;
        it.nq = min(S::kQTiles * T, n - it.i0);  // queries of the two tiles
        it.pos0 = it.L - n + it.i0;              // position of the first query
        const int p_max = it.pos0 + it.nq - 1;   // and of the last
        it.ntiles = p_max / S::kKvTok + 1;
        it.npages = p_max / kPageRows + 1;       // pages 0 .. npages-1 are read
        return true;
    };

    // ---- shared memory ----
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    auto q_s = [&](int t) { return base + t * S::kQBytes; };
    const uint32_t kv_base = base + S::kQTiles * S::kQBytes;
    auto k_s = [&](int s) { return kv_base + s * S::kKvBytes; };
    auto v_s = [&](int s) { return kv_base + (S::kStages + s) * S::kKvBytes; };
    const uint32_t bars = kv_base + 2 * S::kStages * S::kKvBytes;
    const uint32_t q_full = bars, drain = bars + 8;
    // per query tile t: S ready (MMA commit), P stored over it in TMEM (its 128 threads),
    // O += P V done (MMA commit), O read out for the item (its 128 threads)
    auto s_full = [&](int t) { return bars + 16 + 8u * t; };
    auto p_full = [&](int t) { return bars + 32 + 8u * t; };
    auto o_done = [&](int t) { return bars + 48 + 8u * t; };
    auto o_free = [&](int t) { return bars + 64 + 8u * t; };
    // K and V stages: full (TMA landed) and empty (the MMAs that read it are done)
    auto k_full = [&](int s) { return bars + 80 + 8u * s; };
    auto k_empty = [&](int s) { return bars + 96 + 8u * s; };
    auto v_full = [&](int s) { return bars + 112 + 8u * s; };
    auto v_empty = [&](int s) { return bars + 128 + 8u * s; };
    const uint32_t q_empty = bars + 144;         // the item's last S has read Q (MMA commit)
    const uint32_t tmem_slot = bars + 248;

    const int rows = G * tok_per_tile;           // rows of Q the TMA fills; the rest stay zero
    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        mbar_init(drain, 1);
        for (int t = 0; t < S::kQTiles; ++t) {
            mbar_init(s_full(t), 1);
            mbar_init(p_full(t), 128);
            mbar_init(o_done(t), 1);
            mbar_init(o_free(t), 128);
        }
        for (int s = 0; s < S::kStages; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        mbar_init_fence();
    }
    for (int i = threadIdx.x; i < S::kQTiles * (S::kRows - rows) * 16; i += S::kThreads) {
        const int t = i / ((S::kRows - rows) * 16), k = i % ((S::kRows - rows) * 16);
        const int r = rows + k / 16, part = k % 16;          // 2 chunks x 8 pieces of 16 bytes
        const uint32_t a = q_s(t) + (part >> 3) * S::kChunk + r * 128 + (part & 7) * 16;
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" :: "r"(a), "r"(0u) : "memory");
    }
    fence_proxy_async_shared();
    if (warp == S::kMmaWarp) {
        tmem_alloc(tmem_slot, S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t tmem;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(tmem_slot) : "memory");
    auto tmem_s = [&](int t) { return tmem + 128u * t; };
    auto tmem_o = [&](int t) { return tmem + 256u + 128u * t; };

    // Bounded wait that also gives up once another role has given up.
    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        if (mbar_try_wait(bar, parity)) return true;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t it = 0;; ++it) {
            if (mbar_try_wait(bar, parity)) return true;
            if ((it & 63u) == 63u) {
                if (*reinterpret_cast<volatile int*>(&s_abort)) return false;
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    flag_error(PKV_DEVERR_WAIT_TIMEOUT);
                    *reinterpret_cast<volatile int*>(&s_abort) = 1;
                    return false;
                }
            }
        }
    };

    if (warp == S::kTmaKWarp || warp == S::kTmaVWarp) {
        // ============================ TMA: K or V ============================
        // KV tiles are numbered across the CTA's items (gj); the K warp also loads each item's Q
        // once the previous item's last S has read the buffers.
        const bool is_k = warp == S::kTmaKWarp;
        if (lane == 0) {
            prefetch_tensormap(is_k ? &tm_k : &tm_v);
            if (is_k) prefetch_tensormap(&tm_q);
        }
        const CUtensorMap* map = is_k ? &tm_k : &tm_v;
        int gj = 0, k = 0;
        bool ok = true;
        for (int ri = 0; ok; ++ri) {
            const int item = item_index(ri);
            if (item < 0) break;
            PrefillItem it;
            if (!item_info(item, it)) continue;
            if (is_k) {
                if (k >= 1 && !(ok = __all_sync(0xffffffffu, wait(q_empty, (k - 1) & 1)))) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(q_full, S::kQTiles * 2 * 128 * rows);
                    for (int t = 0; t < S::kQTiles; ++t) {
                        tma_load_3d_reused(q_s(t), &tm_q, q_full, 0, it.g * G, it.qs0 + it.i0 + t * T);
                        tma_load_3d_reused(q_s(t) + S::kChunk, &tm_q, q_full, 64, it.g * G, it.qs0 + it.i0 + t * T);
                    }
                }
            }
            ++k;
            const int32_t* bt = p.block_tables + (int64_t)it.b * p.max_blocks_per_seq;
            for (int j = 0; j < it.ntiles; ++j, ++gj) {
                const int s = gj % S::kStages;
                const uint32_t full = is_k ? k_full(s) : v_full(s), dst = is_k ? k_s(s) : v_s(s);
                if (gj >= S::kStages &&
                    !(ok = __all_sync(0xffffffffu, wait(is_k ? k_empty(s) : v_empty(s), ((gj / S::kStages) - 1) & 1))))
                    break;
                // physical blocks of the tile's 8 pages, one per lane
                const int jj = 8 * j + lane;
                int pb = -1;
                if (lane < 8 && jj < it.npages) {
                    pb = __ldg(bt + jj);
                    if (pb < 0 || pb >= p.num_blocks) {      // outside the pool: reads as zeros
                        if (is_k) flag_error(PKV_DEVERR_BLOCK_ID);
                        pb = -1;
                    }
                }
                if (lane == 0) mbar_arrive_expect_tx(full, 2 * S::kChunk);
                for (int pg = 0; pg < 8; ++pg) {
                    const int blk = __shfl_sync(0xffffffffu, pb, pg);
                    if (lane == 0) {
                        const int row = blk * kPageRows;         // -16: a box wholly outside the pool
                        tma_load_3d_reused(dst + pg * 2048, map, full, 0, it.g, row);
                        tma_load_3d_reused(dst + S::kChunk + pg * 2048, map, full, 64, it.g, row);
                    }
                }
            }
        }
        // nothing of ours may be in flight when the CTA leaves
        for (int j = max(0, gj - S::kStages); j < gj; ++j)
            mbar_wait(is_k ? k_full(j % S::kStages) : v_full(j % S::kStages), (j / S::kStages) & 1);
        if (is_k && k >= 1) mbar_wait(q_full, (k - 1) & 1);
    } else if (warp == S::kMmaWarp) {
        // ================================ MMA ================================
        constexpr uint32_t kIdescS = umma_idesc_f16(128, 128, 0);    // Q K^T: both K-major
        constexpr uint32_t kIdescPV = umma_idesc_f16(128, 128, 1);   // P V: V is MN-major
        // S_t = Q_t K^T of global KV tile gg, once O_t += P_t V of tile gg - 1 has read P_t out
        // of S_t; `last`: the item's last tile, after which Q may be reloaded
        auto issue_s = [&](int t, int gg, bool last) -> bool {
            if (gg >= 1 && !__all_sync(0xffffffffu, wait(o_done(t), (gg - 1) & 1))) return false;
            tc_fence_after();
            if (lane == 0) {
                const int s = gg % S::kStages;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = (kk >> 2) * S::kChunk + (kk & 3) * 32;
                    umma_f16_ss(tmem_s(t), umma_desc_sw128(q_s(t) + koff, 16, 1024),
                                umma_desc_sw128(k_s(s) + koff, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
                }
                umma_commit(s_full(t));
                if (t == S::kQTiles - 1) {
                    umma_commit(k_empty(s));                       // both tiles have read K
                    if (last) umma_commit(q_empty);                // and Q, for the last time
                }
            }
            __syncwarp();
            return true;
        };
        // O_t += P_t V of global KV tile gg, P_t read from TMEM; `first`: the item's first tile,
        // whose product overwrites O_t
        auto issue_pv = [&](int t, int gg, bool first) -> bool {
            const int s = gg % S::kStages;
            if (!__all_sync(0xffffffffu, wait(p_full(t), gg & 1))) return false;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bdesc = umma_desc_sw128(v_s(s) + kk * 2048, S::kChunk, 1024);
                    umma_f16_ts(tmem_o(t), tmem_s(t) + 8 * kk, bdesc, kIdescPV, (!first || kk > 0) ? 1u : 0u);
                }
                umma_commit(o_done(t));
                if (t == S::kQTiles - 1) umma_commit(v_empty(s));      // both tiles have read V
            }
            __syncwarp();
            return true;
        };
        int gj = 0, k = 0;
        bool ok = true;
        for (int ri = 0; ok; ++ri) {
            const int item = item_index(ri);
            if (item < 0) break;
            PrefillItem it;
            if (!item_info(item, it)) continue;
            const int last_page = (it.L - 1) / kPageRows;
            const int valid_last = it.L - last_page * kPageRows;     // live rows of that page
            if (!(ok = __all_sync(0xffffffffu, wait(q_full, k & 1)))) break;
            if (!(ok = __all_sync(0xffffffffu, wait(k_full(gj % S::kStages), (gj / S::kStages) & 1)))) break;
            for (int t = 0; ok && t < S::kQTiles; ++t) ok = issue_s(t, gj, it.ntiles == 1);
            // per KV tile j: O_A += P_A V(j), S_A(j + 1), O_B += P_B V(j), S_B(j + 1) -- the tensor
            // core works on one query tile while the other tile's softmax runs
            for (int j = 0; ok && j < it.ntiles; ++j) {
                const int gg = gj + j, s = gg % S::kStages;
                if (!(ok = __all_sync(0xffffffffu, wait(v_full(s), (gg / S::kStages) & 1)))) break;
                // rows past the context in the sequence's last page may hold anything (NaN in free
                // slots): zero their V before it meets a zero probability
                if (last_page >= 8 * j && last_page < 8 * j + 8 && last_page < it.npages && valid_last < kPageRows) {
                    const int pg = last_page - 8 * j;
                    const int nz = (kPageRows - valid_last) * 8;      // 16-byte pieces per chunk
                    for (int i = lane; i < 2 * nz; i += 32) {
                        const int c = i / nz, q = i % nz;
                        const uint32_t a = v_s(s) + c * S::kChunk + (pg * kPageRows + valid_last + q / 8) * 128 + (q % 8) * 16;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" :: "r"(a), "r"(0u) : "memory");
                    }
                    fence_proxy_async_shared();
                }
                __syncwarp();
                const bool more = j + 1 < it.ntiles;
                for (int t = 0; ok && t < S::kQTiles; ++t) {
                    // an item's first product overwrites O_t: the previous item's O_t has been read out
                    if (j == 0 && k >= 1 && !(ok = __all_sync(0xffffffffu, wait(o_free(t), (k - 1) & 1)))) break;
                    ok = issue_pv(t, gg, j == 0);
                    if (ok && more && t == 0)
                        ok = __all_sync(0xffffffffu, wait(k_full((gg + 1) % S::kStages), ((gg + 1) / S::kStages) & 1));
                    if (ok && more) ok = issue_s(t, gg + 1, j + 2 == it.ntiles);
                }
            }
            gj += it.ntiles;
            ++k;
        }
        // every MMA issued has completed before TMEM is freed
        if (lane == 0) umma_commit(drain);
        __syncwarp();
        mbar_wait(drain, 0);
    } else {
        // ============================== softmax ==============================
        const int quarter = warp & 3, t = warp >> 2;             // rows, and the query tile served
        const int r = 32 * quarter + lane;                       // row = TMEM lane
        const int ti = r / G, hh = r - ti * G;                  // token within the tile, head within g
        const int qi = t * T + ti;                               // query within the item's two tiles
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const uint32_t s_row = tmem_s(t) + lane_base, o_row = tmem_o(t) + lane_base;
        const float sl = p.logit_scale_log2;
        int gj = 0;
        bool ok = true;
        for (int ri = 0; ok; ++ri) {
            const int item = item_index(ri);
            if (item < 0) break;
            PrefillItem it;
            if (!item_info(item, it)) continue;
            const bool valid = r < rows && qi < it.nq;
            const int prow = it.pos0 + min(qi, it.nq - 1);       // causal limit of the row
            float m_run = -INFINITY, l_run = 0.f;                // running maximum (exp2 domain) and sum
            for (int j = 0; j < it.ntiles; ++j, ++gj) {
                if (!(ok = __all_sync(0xffffffffu, wait(s_full(t), gj & 1)))) break;
                tc_fence_after();
                // pass 1: causal mask and maximum of the row's raw logits (four independent chains);
                // the scale sl > 0 is applied to the maximum and inside the exponent's multiply-add
                const int t0 = j * S::kKvTok;
                const bool edge = t0 + S::kKvTok - 1 > it.pos0 + t * T;   // some entries past a row's position
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {                    // two 32-column loads in flight at a time
                    float x[2][32];
                    tmem_ld32x2(s_row + 64 * h, x[0], s_row + 64 * h + 32, x[1]);
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const int c = 2 * h + c2;
                        if (edge) {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                mx[i & 3] = fmaxf(mx[i & 3], t0 + 32 * c + i <= prow ? x[c2][i] : -INFINITY);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) mx[i & 3] = fmaxf(mx[i & 3], x[c2][i]);
                        }
                    }
                }
                float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                mt = mt > -INFINITY ? mt * sl : -INFINITY;       // (a zero scale must not make -inf * 0)
                // running maximum, raised only by more than the threshold
                const bool raise = mt > m_run + S::kRescaleThreshold;
                const float m_new = raise ? mt : m_run;
                // O_t += P V of the previous KV tile completed before S_t of this one was issued, so
                // O_t is final for it and may be rescaled; the item's first product overwrites O_t
                if (j > 0 && __any_sync(0xffffffffu, raise)) {
                    if (!(ok = __all_sync(0xffffffffu, wait(o_done(t), (gj - 1) & 1)))) break;
                    tc_fence_after();
                    const float alpha = raise ? fast_exp2(m_run - m_new) : 1.f;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        float o[32];
                        tmem_ld32(o_row + 32 * c, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= alpha;
                        tmem_st32(o_row + 32 * c, o);
                    }
                    l_run *= alpha;
                }
                m_run = m_new;
                // pass 2: probabilities exp2(s * sl - m_new) as f16 pairs (tokens 2 i, 2 i + 1 of a 64-token
                // half), one fused multiply-add and the fp32 exp2, masked entries 0; the row sum adds
                // exactly those f16 values, in four independent partial sums. P overwrites the logits it
                // came from: the pairs of tokens 64 h .. 64 h + 63 go to columns 32 h .. 32 h + 31 of
                // S_t, which pass 2 has read.
                float lt[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    float w[32];
                    float xx[2][32];
                    tmem_ld32x2(s_row + 64 * h, xx[0], s_row + 64 * h + 32, xx[1]);
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const int c = 2 * h + c2;
                        const float (&x)[32] = xx[c2];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float e0 = fmaf(x[2 * i], sl, -m_new), e1 = fmaf(x[2 * i + 1], sl, -m_new);
                            if (edge) {
                                e0 = t0 + 32 * c + 2 * i <= prow ? e0 : -INFINITY;
                                e1 = t0 + 32 * c + 2 * i + 1 <= prow ? e1 : -INFINITY;
                            }
                            const uint32_t pw = pack_half2(fast_exp2(e0), fast_exp2(e1));
                            lt[i & 3] = add_f16_hi(add_f16_lo(lt[i & 3], pw), pw);
                            w[16 * c2 + i] = __uint_as_float(pw);
                        }
                    }
                    tmem_st32(s_row + 32 * h, w);
                }
                l_run += (lt[0] + lt[1]) + (lt[2] + lt[3]);
                tmem_wait_st();                                  // P and any rescaled O are in TMEM
                tc_fence_before();
                mbar_arrive(p_full(t));
            }
            if (!ok) break;
            // ---- out = O_t / l ----
            if (!(ok = __all_sync(0xffffffffu, wait(o_done(t), (gj - 1) & 1)))) break;
            tc_fence_after();
            const float inv = p.out_scale / l_run;
            __half* dst = p.out + ((int64_t)(it.qs0 + it.i0 + qi) * p.Hq + (int64_t)it.g * G + hh) * kHeadDim;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float o[32];
                tmem_ld32(o_row + 32 * c, o);
                if (valid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 u;
                        u.x = pack_half2(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
                        u.y = pack_half2(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
                        u.z = pack_half2(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
                        u.w = pack_half2(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
                        *reinterpret_cast<uint4*>(dst + 32 * c + 8 * q) = u;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(o_free(t));                              // O_t may be overwritten
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == S::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, S::kTmemCols);
    }
}

}  // namespace pkv
