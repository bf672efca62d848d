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
//  * Query tile: T = floor(128 / G) query tokens of one sequence x the G
//    query heads of one KV head g, M = T * G <= 128 rows, row r = (token
//    r / G, head r % G), so every K/V byte a CTA stages serves all G heads of
//    every query in it. A work item is two such tiles (A and B, 2 T
//    consecutive queries) of one (sequence, KV head), over the KV tiles
//    their positions reach.
//  * Persistent grid, one CTA per SM, TMEM, barriers and rings set up once;
//    barrier phases run on across a CTA's work through global KV-tile and
//    item counters. Without a workspace a CTA takes whole items, costliest
//    first, in snake order. With one, every CTA takes an equal run of all
//    items' KV tiles (stream-K); an item cut at a CTA boundary is computed
//    in pieces, each piece stores its rows' (max, sum, unnormalised output),
//    and the piece that takes the last ticket merges them by the log-sum-exp
//    rule. Nobody waits on another CTA.
//  * A KV tile is 128 tokens (8 pages). K and V have their own two-stage
//    rings, barriers and TMA warp (warp 8: Q and K, warp 9: V). Pages past
//    the item's last position are loaded from block -1, a box wholly outside
//    the pool, which TMA fills with zeros; rows past the context in the
//    sequence's last page are zeroed in shared memory before their V is used.
//  * TMEM: S_A, S_B, O_A, O_B, 128 columns each. One thread (warp 10) issues
//    S_t = Q_t K^T (M = N = K = 128, both K-major) and O_t += P_t V with P_t
//    read from TMEM (the A operand of `tcgen05.mma` may live there: row r in
//    lane r, two f16 per column) and V MN-major from shared memory. Per KV
//    tile j: O_A += P_A V(j), S_A(j + 1), O_B += P_B V(j), S_B(j + 1), so the
//    tensor core works on one tile while the other tile's softmax runs.
//  * Softmax: warps 0-3 serve tile A, warps 4-7 tile B, one row (TMEM lane)
//    per thread. Pass 1 takes the row's maximum (the causal mask only on KV
//    tiles that reach past the query tile's first position); the running
//    maximum (exp2 domain) is raised only when a tile's maximum exceeds it by
//    more than 8 (a factor 256), and only then are the row's O and sum
//    rescaled. Pass 2 forms exp2(s * scale - m) with one fused multiply-add
//    and the fp32 exp2, rounds to f16, adds exactly those f16 values to the
//    row sum in fp32 (mixed-precision add), and stores the f16 pairs over
//    the logits already read. The output is O / sum in f16.
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
    // stream-K schedule: one piece's partial result for one query tile, O as [32 float4 of
    // channels][128 rows] and (m, l) per row; two slots per CTA (its first and its last piece)
    static constexpr int kPartBytes = 128 * 128 * 4 + 128 * 8;
    static constexpr int kMinTiles = 4;                // fewest KV tiles a CTA is given
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

// The KV tiles [j0, j1) of an item that one CTA processes: the whole item, or a piece of it
// when the stream-K schedule cuts the item at a CTA boundary. u: the item's first unit.
struct PrefillPiece {
    PrefillItem it;
    int j0, j1;
    int64_t u;
};

template <bool kStream>
__global__ void __launch_bounds__(PrefillTcShape::kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const PrefillParams p, const int tok_per_tile,
                  const int q_groups, const int batch, uint8_t* const ws, unsigned int* const ws_count) {
    using S = PrefillTcShape;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort;
    __shared__ long long s_red[S::kThreads / 32];
    __shared__ long long s_first[2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G, T = tok_per_tile;

    grid_dependency_wait();                      // inputs may come from the previous launch
    grid_dependents_launch();
    // ---- work items: (group of two query tiles, KV head, sequence) ----
    const int cap = min(p.max_context_len, p.max_blocks_per_seq * kPageRows);
    // item (query group qg, KV head g, sequence b): 1, or 0 when the group is past the
    // sequence's queries, -1 when the sequence's lengths are inconsistent
    auto make_item = [&](int b, int g, int qg, PrefillItem& it) -> int {
        it.b = b;
        it.g = g;
        it.qs0 = __ldg(p.query_start + b);
        const int qs1 = __ldg(p.query_start + b + 1);
        it.L = __ldg(p.context_lens + b);
        const int n = qs1 - it.qs0;
        if (it.qs0 < 0 || n < 0 || qs1 > p.total || n > p.max_query_len || it.L < n || it.L > cap) return -1;
        it.i0 = qg * S::kQTiles * T;             // first query of the item's two tiles
        if (it.i0 >= n) return 0;
        it.nq = min(S::kQTiles * T, n - it.i0);  // queries of the two tiles
        it.pos0 = it.L - n + it.i0;              // position of the first query
        const int p_max = it.pos0 + it.nq - 1;   // and of the last
        it.ntiles = p_max / S::kKvTok + 1;
        it.npages = p_max / kPageRows + 1;       // pages 0 .. npages-1 are read
        return 1;
    };
    // Without a workspace every CTA takes whole items, costliest first (the last query groups
    // see the longest contexts), dealt out in snake order: CTA c takes items c, 2C - 1 - c,
    // 2C + c, ... of the C CTAs. With one (stream-K), the items in (sequence, KV head, query
    // group) order form a row of U KV tiles ("units"); CTA c < C' takes units
    // [c U / C', (c + 1) U / C'), C' <= C being the most CTAs that get kMinTiles or more, and
    // an item cut at a CTA boundary becomes pieces whose partial softmaxes the piece that
    // finishes last merges by the log-sum-exp rule.
    constexpr bool stream = kStream;             // the launch passes a workspace exactly then
    const int C = gridDim.x;
    int64_t U = 0, u_lo = 0, u_hi = 0;
    int ctas = 1;
    // KV tiles of all items of sequence b under one KV head (0: no queries, or inconsistent)
    auto seq_tiles = [&](int b) -> int64_t {
        const int qs0 = __ldg(p.query_start + b), qs1 = __ldg(p.query_start + b + 1);
        const int L = __ldg(p.context_lens + b), n = qs1 - qs0;
        if (qs0 < 0 || n < 0 || qs1 > p.total || n > p.max_query_len || L < n || L > cap) return 0;
        int64_t s = 0;
        for (int i0 = 0; i0 < n; i0 += S::kQTiles * T) s += (L - n + min(i0 + S::kQTiles * T, n) - 1) / S::kKvTok + 1;
        return s;
    };
    // inclusive scan of x over the block; total: the block's sum (uses s_red, ends synchronised)
    auto block_scan = [&](int64_t x, int64_t& total) -> int64_t {
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) s_red[warp] = x;
        __syncthreads();
        int64_t before = 0;
        total = 0;
        for (int i = 0; i < S::kThreads / 32; ++i) {
            before += i < warp ? s_red[i] : 0;
            total += s_red[i];
        }
        __syncthreads();
        return before + x;
    };
    if (stream) {
        // units of every sequence (all KV heads), scanned; the first chunk of sequences is kept
        int64_t my_w = 0, my_incl = 0, first_total = 0;
        for (int b0 = 0; b0 < batch; b0 += S::kThreads) {
            const int b = b0 + (int)threadIdx.x;
            int64_t w = 0;
            if (b < batch) {
                w = seq_tiles(b) * p.Hkv;
                PrefillItem it;
                if (blockIdx.x == 0 && make_item(b, 0, 0, it) < 0) flag_error(PKV_DEVERR_CONTEXT_LEN);
            }
            int64_t total;
            const int64_t incl = U + block_scan(w, total);
            if (b0 == 0) {
                my_w = w;
                my_incl = incl;
                first_total = total;
            }
            U += total;
        }
        ctas = (int)max((int64_t)1, min((int64_t)C, U / S::kMinTiles));
        u_lo = blockIdx.x < ctas ? (int64_t)blockIdx.x * U / ctas : U;
        u_hi = blockIdx.x < ctas ? ((int64_t)blockIdx.x + 1) * U / ctas : U;
        // the sequence that holds unit u_lo, and the units before it: in the first chunk from the
        // values kept, past it (more sequences than threads) by scanning again
        if (u_lo < u_hi) {
            if (my_w > 0 && my_incl - my_w <= u_lo && u_lo < my_incl) {
                s_first[0] = threadIdx.x;
                s_first[1] = my_incl - my_w;
            }
            int64_t base = first_total;
            for (int b0 = S::kThreads; b0 < batch && base <= u_lo; b0 += S::kThreads) {
                const int b = b0 + (int)threadIdx.x;
                const int64_t w = b < batch ? seq_tiles(b) * p.Hkv : 0;
                int64_t total;
                const int64_t incl = base + block_scan(w, total);
                if (w > 0 && incl - w <= u_lo && u_lo < incl) {
                    s_first[0] = b;
                    s_first[1] = incl - w;
                }
                base += total;
            }
        }
        __syncthreads();
    }
    // first unit of CTA c's range, and the CTA whose range holds unit u
    auto range_lo = [&](int c) -> int64_t { return (int64_t)c * U / ctas; };
    auto cta_of = [&](int64_t u) -> int {
        int c = (int)min((int64_t)ctas - 1, u * ctas / U);
        while (c > 0 && range_lo(c) > u) --c;
        while (c + 1 < ctas && range_lo(c + 1) <= u) ++c;
        return c;
    };
    // cursor: snake rank, or the stream-K item (qg of KV head cg of sequence cb, first unit cu)
    int ri = 0, cb = batch, cg = 0, cq = 0;
    int64_t cu = U;
    if (stream && u_lo < u_hi) {
        cb = (int)s_first[0];
        const int64_t per_g = seq_tiles(cb);
        cg = (int)((u_lo - s_first[1]) / per_g);
        cu = s_first[1] + cg * per_g;
        // the query group holding u_lo: its sequence's lengths once, then arithmetic
        const int L = __ldg(p.context_lens + cb);
        const int n = __ldg(p.query_start + cb + 1) - __ldg(p.query_start + cb);
        for (int i0 = 0; i0 < n; i0 += S::kQTiles * T) {
            const int ntiles = (L - n + min(i0 + S::kQTiles * T, n) - 1) / S::kKvTok + 1;
            if (cu + ntiles > u_lo) break;
            cu += ntiles;
            ++cq;
        }
    }
    const int per_q = p.Hkv * batch;
    const int n_items = q_groups * per_q;
    // the CTA's next piece; false when it has none left
    auto next_piece = [&](PrefillPiece& pc) -> bool {
        if (!stream) {
            for (;;) {
                const int i = ri * C + ((ri & 1) ? C - 1 - (int)blockIdx.x : (int)blockIdx.x);
                ++ri;
                if (i >= n_items) return false;
                const int qg = q_groups - 1 - i / per_q, rem = i % per_q;
                const int r = make_item(rem / p.Hkv, rem % p.Hkv, qg, pc.it);
                if (r < 0 && threadIdx.x == 0 && qg == 0 && rem % p.Hkv == 0) flag_error(PKV_DEVERR_CONTEXT_LEN);
                if (r > 0) {
                    pc.j0 = 0;
                    pc.j1 = pc.it.ntiles;
                    pc.u = 0;
                    return true;
                }
            }
        }
        while (cu < u_hi && cb < batch) {
            const int r = make_item(cb, cg, cq, pc.it);
            if (r <= 0) {                        // next KV head, or next sequence
                cq = 0;
                if (r < 0 || ++cg == p.Hkv) {
                    cg = 0;
                    ++cb;
                }
                continue;
            }
            pc.u = cu;
            pc.j0 = (int)(max(cu, u_lo) - cu);
            pc.j1 = (int)(min(cu + pc.it.ntiles, u_hi) - cu);
            cu += pc.it.ntiles;
            ++cq;
            return true;
        }
        return false;
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
        // KV tiles are numbered across the CTA's pieces (gj); the K warp also loads each piece's Q
        // once the previous piece's last S has read the buffers.
        const bool is_k = warp == S::kTmaKWarp;
        if (lane == 0) {
            prefetch_tensormap(is_k ? &tm_k : &tm_v);
            if (is_k) prefetch_tensormap(&tm_q);
        }
        const CUtensorMap* map = is_k ? &tm_k : &tm_v;
        int gj = 0, k = 0;
        bool ok = true;
        PrefillPiece pc;
        while (ok && next_piece(pc)) {
            const PrefillItem& it = pc.it;
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
            for (int j = pc.j0; j < pc.j1; ++j, ++gj) {
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
        // of S_t; `last`: the piece's last tile, after which Q may be reloaded
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
        // O_t += P_t V of global KV tile gg, P_t read from TMEM; `first`: the piece's first tile,
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
        PrefillPiece pc;
        while (ok && next_piece(pc)) {
            // the piece's bounds and page limits, held in registers for the issue loop (the empty
            // asm keeps the compiler from re-deriving them from the loads they came from in every
            // iteration, which slowed each KV tile by about a tenth)
            int pj0 = pc.j0, pj1 = pc.j1, npages = pc.it.npages;
            int last_page = (pc.it.L - 1) / kPageRows;
            int valid_last = pc.it.L - last_page * kPageRows;        // live rows of that page
            asm volatile("" : "+r"(pj0), "+r"(pj1), "+r"(npages), "+r"(last_page), "+r"(valid_last));
            if (!(ok = __all_sync(0xffffffffu, wait(q_full, k & 1)))) break;
            if (!(ok = __all_sync(0xffffffffu, wait(k_full(gj % S::kStages), (gj / S::kStages) & 1)))) break;
            for (int t = 0; ok && t < S::kQTiles; ++t) ok = issue_s(t, gj, pj1 - pj0 == 1);
            // per KV tile j: O_A += P_A V(j), S_A(j + 1), O_B += P_B V(j), S_B(j + 1) -- the tensor
            // core works on one query tile while the other tile's softmax runs
            for (int j = pj0; ok && j < pj1; ++j) {
                const int gg = gj + (j - pj0), s = gg % S::kStages;
                if (!(ok = __all_sync(0xffffffffu, wait(v_full(s), (gg / S::kStages) & 1)))) break;
                // rows past the context in the sequence's last page may hold anything (NaN in free
                // slots): zero their V before it meets a zero probability
                if (last_page >= 8 * j && last_page < 8 * j + 8 && last_page < npages && valid_last < kPageRows) {
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
                const bool more = j + 1 < pj1;
                for (int t = 0; ok && t < S::kQTiles; ++t) {
                    // a piece's first product overwrites O_t: the previous piece's O_t has been read out
                    if (j == pj0 && k >= 1 && !(ok = __all_sync(0xffffffffu, wait(o_free(t), (k - 1) & 1)))) break;
                    ok = issue_pv(t, gg, j == pj0);
                    if (ok && more && t == 0)
                        ok = __all_sync(0xffffffffu, wait(k_full((gg + 1) % S::kStages), ((gg + 1) / S::kStages) & 1));
                    if (ok && more) ok = issue_s(t, gg + 1, j + 2 == pj1);
                }
            }
            gj += pj1 - pj0;
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
        PrefillPiece pc;
        while (ok && next_piece(pc)) {
            const PrefillItem& it = pc.it;
            const bool valid = r < rows && qi < it.nq;
            const int prow = it.pos0 + min(qi, it.nq - 1);       // causal limit of the row
            float m_run = -INFINITY, l_run = 0.f;                // running maximum (exp2 domain) and sum
            for (int j = pc.j0; j < pc.j1; ++j, ++gj) {
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
                // O_t is final for it and may be rescaled; the piece's first product overwrites O_t
                if (j > pc.j0 && __any_sync(0xffffffffu, raise)) {
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
            if (!(ok = __all_sync(0xffffffffu, wait(o_done(t), (gj - 1) & 1)))) break;
            tc_fence_after();
            __half* dst = p.out + ((int64_t)(it.qs0 + it.i0 + qi) * p.Hq + (int64_t)it.g * G + hh) * kHeadDim;
            auto store_out = [&](int c, const float (&o)[32], float inv) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 u;
                    u.x = pack_half2(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
                    u.y = pack_half2(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
                    u.z = pack_half2(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
                    u.w = pack_half2(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
                    *reinterpret_cast<uint4*>(dst + 32 * c + 8 * q) = u;
                }
            };
            if (!kStream || (pc.j0 == 0 && pc.j1 == it.ntiles)) {
                // ---- a whole item: out = O_t / l ----
                const float inv = p.out_scale / l_run;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float o[32];
                    tmem_ld32(o_row + 32 * c, o);
                    if (valid) store_out(c, o, inv);
                }
                tc_fence_before();
                mbar_arrive(o_free(t));                          // O_t may be overwritten
                continue;
            }
            // ---- a piece of an item cut at a CTA boundary ----
            // Every piece stores its (m, l, O) rows; a warp's ticket then counts its 32 rows, and the
            // warp that takes the last ticket merges the pieces of those rows:
            // M = max m_k, out = sum_k 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k. The merger's own O
            // is still in TMEM (O_t is released after the ticket); the others' come from L2.
            const int c_first = cta_of(pc.u), c_last = cta_of(pc.u + it.ntiles - 1);
            // a piece's slot: 0 if it starts the range of CTA c, else 1 (the CTA's last piece)
            auto part_of = [&](int c) -> uint8_t* {
                const int slot = 2 * c + (max(pc.u, range_lo(c)) == range_lo(c) ? 0 : 1);
                return ws + ((int64_t)slot * S::kQTiles + t) * S::kPartBytes;
            };
            auto ml_of = [&](int c) { return reinterpret_cast<const float2*>(part_of(c) + 128 * 128 * 4) + r; };
            {
                uint8_t* part = part_of((int)blockIdx.x);
                float4* po = reinterpret_cast<float4*>(part);
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    float o[2][32];
                    tmem_ld32x2(o_row + 64 * h, o[0], o_row + 64 * h + 32, o[1]);
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            __stcg(po + (16 * h + 8 * c2 + q) * 128 + r,
                                   make_float4(o[c2][4 * q], o[c2][4 * q + 1], o[c2][4 * q + 2], o[c2][4 * q + 3]));
                }
                __stcg(reinterpret_cast<float2*>(part + 128 * 128 * 4) + r, make_float2(m_run, l_run));
            }
            // the warp barrier orders every lane's stores before lane 0's release-acquire ticket;
            // the merger's loads follow its acquire
            __syncwarp();
            unsigned int* cnt = ws_count + ((int64_t)c_last * S::kQTiles + t) * 4 + quarter;
            unsigned int prev = 0;
            if (lane == 0) prev = atomic_add_acq_rel_gpu(cnt, 1u);
            prev = __shfl_sync(0xffffffffu, prev, 0);
            __syncwarp();
            const int n_oth = c_last - c_first;                  // pieces besides this one
            if (prev == (unsigned int)n_oth) {
                if (lane == 0) *cnt = 0u;                        // ready for the next call
                const int me = (int)blockIdx.x;
                auto oth = [&](int k) { return c_first + k + (c_first + k >= me ? 1 : 0); };
                // online log-sum-exp over the pieces, 64 channels at a time: each other piece's
                // (m, l) comes with its 64 values in one round trip
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    float o[2][32];
                    tmem_ld32x2(o_row + 64 * h, o[0], o_row + 64 * h + 32, o[1]);
                    float M = m_run, den = l_run;
                    if (valid) {
#pragma unroll 1
                        for (int k = 0; k < n_oth; ++k) {
                            const uint8_t* part = part_of(oth(k));
                            const float4* src = reinterpret_cast<const float4*>(part) + 16 * h * 128 + r;
                            float4 v[16];
#pragma unroll
                            for (int q = 0; q < 16; ++q) v[q] = __ldcg(src + q * 128);
                            const float2 ml = __ldcg(reinterpret_cast<const float2*>(part + 128 * 128 * 4) + r);
                            // a piece that saw no position has m = -inf, l = 0 and O = 0
                            const float m_new = fmaxf(M, ml.x);
                            const float a = M == m_new ? 1.f : fast_exp2(M - m_new);
                            const float w = ml.x == m_new ? 1.f : fast_exp2(ml.x - m_new);
                            den = fmaf(den, a, w * ml.y);
#pragma unroll
                            for (int q = 0; q < 16; ++q) {
                                float* d = &o[q >> 3][4 * (q & 7)];
                                d[0] = fmaf(d[0], a, w * v[q].x);
                                d[1] = fmaf(d[1], a, w * v[q].y);
                                d[2] = fmaf(d[2], a, w * v[q].z);
                                d[3] = fmaf(d[3], a, w * v[q].w);
                            }
                            M = m_new;
                        }
                        const float inv = p.out_scale / den;
                        store_out(2 * h, o[0], inv);
                        store_out(2 * h + 1, o[1], inv);
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
