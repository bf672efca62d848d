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
//  * A KV tile is 128 tokens (8 pages). K and V pages come by TMA into a
//    two-stage ring, K and V with their own barriers and their own TMA warp:
//    a K stage is refilled as soon as S of its tile is done, a V stage once
//    O += P V of its tile is, so each load has about two tile periods to land
//    (the cache is mostly L2-resident; its latency, not HBM, is what the ring
//    hides). Q (the CTA's rows) comes once.
//  * One thread issues S = Q K^T (M = 128, N = 128, K = 128; K-major A and
//    B) into TMEM columns [0, 128), and after the softmax O += P V (K = 128
//    tokens; P K-major from shared memory, V MN-major) into columns
//    [128, 256) and l += P 1 (N = 16 against a tile of ones) into [256, 272),
//    so the row sum is the sum of exactly the f16 probabilities the product
//    used, accumulated in fp32 by the tensor core. S of tile j + 1 is issued
//    before O += P V of tile j, so the tensor core works on one while the
//    softmax warps work on the other.
//  * Softmax: 8 warps, two per row quarter. Warp w serves rows (TMEM lanes)
//    32 (w % 4) .. +31 and the half w / 4 of the columns: 64 tokens of S, 64
//    channels of O, one 64-token chunk of P. Per tile a thread loads its
//    half row of S, masks the causal edge (only on tiles that reach past the
//    tile's first position), and takes the half row's maximum; the two halves
//    of a row exchange maxima through shared memory (a barrier per pair of
//    warps). The running maximum (exp2 domain) is raised only when a tile's
//    maximum exceeds it by more than 8 (a factor 256); then, and only then,
//    the row of O and its l are rescaled in TMEM. A probability is
//    exp2(s * scale - m): one fused multiply-add and the fp32 exp2, rounded to
//    f16. (The two-wide f16 exp2 would halve the multi-function unit's work,
//    but its f16 argument, 2^-9 apart near -8, moved outputs of magnitude
//    about 4 past the 2e-3 bound.) Probabilities are computed into
//    registers first; once O += P V of the previous tile has completed (its
//    P buffer is then free, and O may be rescaled) they are written to shared
//    memory as f16 in the operand layout. The output is O / l in f16.
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
    static constexpr int kChunk = 128 * 128;           // one 64-channel (or 64-token) half of a tile: 16 KiB
    static constexpr int kQBytes = 2 * kChunk;         // Q: 128 rows x 128 channels
    static constexpr int kKvBytes = 4 * kChunk;        // K then V, 128 tokens x 128 channels each
    static constexpr int kPBytes = 2 * kChunk;         // P: 128 rows x 128 tokens (one buffer)
    static constexpr int kBarBytes = 256;
    static constexpr int kXchgBytes = 2 * 2 * 128 * 4;  // per-half row values, two buffers
    static constexpr int kOnesBytes = 2 * 16 * 128;    // 16 rows x 128 tokens of f16 ones (K-major, N = 16)
    static constexpr int kSmemBytes = 1024 + kQBytes + kStages * kKvBytes + kPBytes + kOnesBytes + kBarBytes + kXchgBytes;
    static constexpr int kSoftmaxWarps = 8;
    static constexpr int kThreads = 32 * (kSoftmaxWarps + 3);   // warps 0-7 softmax, 8 TMA K (and Q), 9 TMA V, 10 MMA
    static constexpr int kTmaKWarp = kSoftmaxWarps, kTmaVWarp = kSoftmaxWarps + 1, kMmaWarp = kSoftmaxWarps + 2;
    static constexpr uint32_t kTmemCols = 512;         // S [0, 128), O [128, 256), l [256, 272)
    static constexpr float kRescaleThreshold = 8.f;    // log2 of the largest unnormalised probability
};

template <int kDummy = 0>
__global__ void __launch_bounds__(PrefillTcShape::kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const PrefillParams p, const int tok_per_tile) {
    using S = PrefillTcShape;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort;
    const int qt = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
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
        if (threadIdx.x == 0 && qt == 0 && g == 0) flag_error(PKV_DEVERR_CONTEXT_LEN);
        return;
    }
    const int i0 = qt * tok_per_tile;            // first query of the tile
    if (i0 >= n) return;
    const int nq = min(tok_per_tile, n - i0);
    const int pos0 = L - n + i0;                 // position of the tile's first query
    const int p_max = pos0 + nq - 1;             // and of its last
    const int ntiles = p_max / S::kKvTok + 1;
    const int npages = p_max / kPageRows + 1;    // pages 0 .. npages-1 are read

    // ---- shared memory ----
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t q_s = base;
    auto k_s = [&](int s) { return base + S::kQBytes + s * S::kKvBytes; };
    auto v_s = [&](int s) { return k_s(s) + 2 * S::kChunk; };
    const uint32_t p_s = base + S::kQBytes + S::kStages * S::kKvBytes;
    const uint32_t ones_s = p_s + S::kPBytes;                        // [2 token halves][16 rows][128 B]
    const uint32_t bars = ones_s + S::kOnesBytes;
    const uint32_t q_full = bars, s_full = bars + 8, s_free = bars + 16, o_done = bars + 24, drain = bars + 32;
    // K and V stages: full (TMA landed) and empty (the MMA that read it is done)
    auto k_full = [&](int s) { return bars + 40 + 8u * s; };
    auto k_empty = [&](int s) { return bars + 56 + 8u * s; };
    auto v_full = [&](int s) { return bars + 184 + 8u * s; };
    auto v_empty = [&](int s) { return bars + 200 + 8u * s; };
    const uint32_t p_full = bars + 72;
    // pair barriers: the two warps of row quarter q meet at xchg(q, j & 1) every tile
    auto xchg = [&](int q, int i) { return bars + 88 + 8u * (2 * q + i); };
    const uint32_t tmem_slot = bars + 248;
    float* red = reinterpret_cast<float*>(smem_raw + (bars + S::kBarBytes - raw));   // [2][2 halves][128 rows]

    const int rows = G * tok_per_tile;           // rows of Q the TMA fills; the rest stay zero
    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(q_full, 1);
        mbar_init(s_full, 1);
        mbar_init(s_free, 32 * S::kSoftmaxWarps);
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        for (int s = 0; s < S::kStages; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        mbar_init(p_full, 32 * S::kSoftmaxWarps);
        for (int q = 0; q < 4; ++q) {
            mbar_init(xchg(q, 0), 64);
            mbar_init(xchg(q, 1), 64);
        }
        mbar_init_fence();
    }
    for (int i = threadIdx.x; i < (S::kRows - rows) * 16; i += S::kThreads) {
        const int r = rows + i / 16, part = i % 16;          // 2 chunks x 8 pieces of 16 bytes
        const uint32_t a = q_s + (part >> 3) * S::kChunk + r * 128 + (part & 7) * 16;
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" :: "r"(a), "r"(0u) : "memory");
    }
    for (int i = threadIdx.x; i < S::kOnesBytes / 16; i += S::kThreads)     // f16 1.0 pairs
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" :: "r"(ones_s + 16 * i), "r"(0x3C003C00u) : "memory");
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
    const uint32_t tmem_s = tmem, tmem_o = tmem + 128, tmem_l = tmem + 256;

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
        const bool is_k = warp == S::kTmaKWarp;
        if (lane == 0) {
            prefetch_tensormap(is_k ? &tm_k : &tm_v);
            if (is_k) {
                prefetch_tensormap(&tm_q);
                mbar_arrive_expect_tx(q_full, 2 * 128 * rows);
                tma_load_3d_reused(q_s, &tm_q, q_full, 0, g * G, qs0 + i0);
                tma_load_3d_reused(q_s + S::kChunk, &tm_q, q_full, 64, g * G, qs0 + i0);
            }
        }
        const CUtensorMap* map = is_k ? &tm_k : &tm_v;
        const int32_t* bt = p.block_tables + (int64_t)b * p.max_blocks_per_seq;
        int issued = 0;
        for (int j = 0; j < ntiles; ++j) {
            const int s = j & 1;
            const uint32_t full = is_k ? k_full(s) : v_full(s), dst = is_k ? k_s(s) : v_s(s);
            if (j >= 2 && !__all_sync(0xffffffffu, wait(is_k ? k_empty(s) : v_empty(s), ((j - 2) >> 1) & 1))) break;
            // physical blocks of the tile's 8 pages, one per lane
            const int jj = 8 * j + lane;
            int pb = -1;
            if (lane < 8 && jj < npages) {
                pb = __ldg(bt + jj);
                if (pb < 0 || pb >= p.num_blocks) {          // outside the pool: reads as zeros
                    if (is_k) flag_error(PKV_DEVERR_BLOCK_ID);
                    pb = -1;
                }
            }
            if (lane == 0) mbar_arrive_expect_tx(full, 2 * S::kChunk);
            for (int pg = 0; pg < 8; ++pg) {
                const int blk = __shfl_sync(0xffffffffu, pb, pg);
                if (lane == 0) {
                    const int row = blk * kPageRows;             // -16: a box wholly outside the pool
                    tma_load_3d_reused(dst + pg * 2048, map, full, 0, g, row);
                    tma_load_3d_reused(dst + S::kChunk + pg * 2048, map, full, 64, g, row);
                }
            }
            issued = j + 1;
        }
        // nothing of ours may be in flight when the CTA leaves
        for (int j = max(0, issued - 2); j < issued; ++j) mbar_wait(is_k ? k_full(j & 1) : v_full(j & 1), (j >> 1) & 1);
    } else if (warp == S::kMmaWarp) {
        // ================================ MMA ================================
        constexpr uint32_t kIdescS = umma_idesc_f16(128, 128, 0);    // Q K^T: both K-major
        constexpr uint32_t kIdescPV = umma_idesc_f16(128, 128, 1);   // P V: V is MN-major
        constexpr uint32_t kIdescL = umma_idesc_f16(128, 16, 0);     // P 1: the row sums
        const int last_page = (L - 1) / kPageRows;
        const int valid_last = L - last_page * kPageRows;            // live rows of that page
        auto issue_pv = [&](int jp) -> bool {
            const int s = jp & 1;
            if (!__all_sync(0xffffffffu, wait(v_full(s), (jp >> 1) & 1))) return false;
            // rows past the context in the sequence's last page may hold anything
            // (NaN in free slots): zero their V before it meets a zero probability
            if (last_page >= 8 * jp && last_page < 8 * jp + 8 && last_page < npages && valid_last < kPageRows) {
                const int pg = last_page - 8 * jp;
                const int nz = (kPageRows - valid_last) * 8;          // 16-byte pieces per chunk
                for (int i = lane; i < 2 * nz; i += 32) {
                    const int c = i / nz, k = i % nz;
                    const uint32_t a = v_s(s) + c * S::kChunk + (pg * kPageRows + valid_last + k / 8) * 128 + (k % 8) * 16;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" :: "r"(a), "r"(0u) : "memory");
                }
                fence_proxy_async_shared();
            }
            __syncwarp();
            if (!__all_sync(0xffffffffu, wait(p_full, jp & 1))) return false;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = umma_desc_sw128(p_s + (kk >> 2) * S::kChunk + (kk & 3) * 32, 16, 1024);
                    const uint64_t bdesc = umma_desc_sw128(v_s(s) + kk * 2048, S::kChunk, 1024);
                    umma_f16_ss(tmem_o, a, bdesc, kIdescPV, (jp > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = umma_desc_sw128(p_s + (kk >> 2) * S::kChunk + (kk & 3) * 32, 16, 1024);
                    const uint64_t bdesc = umma_desc_sw128(ones_s + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
                    umma_f16_ss(tmem_l, a, bdesc, kIdescL, (jp > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(o_done);
                umma_commit(v_empty(s));
            }
            __syncwarp();
            return true;
        };
        bool ok = __all_sync(0xffffffffu, wait(q_full, 0));
        for (int j = 0; ok && j < ntiles; ++j) {
            const int s = j & 1;
            if (!(ok = __all_sync(0xffffffffu, wait(k_full(s), (j >> 1) & 1)))) break;
            if (j >= 1 && !(ok = __all_sync(0xffffffffu, wait(s_free, (j - 1) & 1)))) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = (kk >> 2) * S::kChunk + (kk & 3) * 32;
                    umma_f16_ss(tmem_s, umma_desc_sw128(q_s + koff, 16, 1024), umma_desc_sw128(k_s(s) + koff, 16, 1024),
                                kIdescS, kk > 0 ? 1u : 0u);
                }
                umma_commit(s_full);
                umma_commit(k_empty(s));
            }
            __syncwarp();
            if (j >= 1) ok = issue_pv(j - 1);
        }
        if (ok) issue_pv(ntiles - 1);
        // every MMA issued has completed before TMEM is freed
        if (lane == 0) umma_commit(drain);
        __syncwarp();
        mbar_wait(drain, 0);
    } else {
        // ============================== softmax ==============================
        const int quarter = warp & 3, half = warp >> 2;
        const int r = 32 * quarter + lane;                   // row = TMEM lane
        const int ti = r / G, hh = r - ti * G;              // token within the tile, head within g
        const bool valid = r < rows && ti < nq;
        const int prow = pos0 + min(ti, nq - 1);             // causal limit of the row
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const uint32_t s_cols = tmem_s + lane_base + 64 * half, o_cols = tmem_o + lane_base + 64 * half;
        const float sl = p.logit_scale_log2;
        float m_run = -INFINITY;                            // running maximum, exp2 domain (s * sl)
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            if (!(ok = __all_sync(0xffffffffu, wait(s_full, j & 1)))) break;
            tc_fence_after();
            float x[64];
            tmem_ld32(s_cols, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld32(s_cols + 32, *reinterpret_cast<float(*)[32]>(x + 32));
            tc_fence_before();
            mbar_arrive(s_free);
            // causal mask and maximum of the half row's raw logits (four independent chains);
            // the scale sl > 0 is applied to the maximum and inside the exponent's multiply-add
            const int t0 = j * S::kKvTok + 64 * half;
            const bool edge = j * S::kKvTok + S::kKvTok - 1 > pos0;   // some entries past a row's position
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (edge) {
#pragma unroll
                for (int c = 0; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], t0 + c <= prow ? x[c] : -INFINITY);
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], x[c]);
            }
            float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            mt = mt > -INFINITY ? mt * sl : -INFINITY;       // (a zero scale must not make -inf * 0)
            // the row's maximum: exchange with the other half of the row
            red[(j & 1) * 256 + half * 128 + r] = mt;
            mbar_arrive(xchg(quarter, j & 1));
            if (!(ok = __all_sync(0xffffffffu, wait(xchg(quarter, j & 1), (j >> 1) & 1)))) break;
            mt = fmaxf(mt, red[(j & 1) * 256 + (half ^ 1) * 128 + r]);
            // running maximum, raised only by more than the threshold
            const bool raise = mt > m_run + S::kRescaleThreshold;
            const float m_new = raise ? mt : m_run;
            // probabilities of this half row as f16 pairs (tokens 64 half + 2i, + 1):
            // exp2(s * sl - m_new), one fused multiply-add and the fp32 exp2; masked entries give 0
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float e0 = fmaf(x[2 * i], sl, -m_new), e1 = fmaf(x[2 * i + 1], sl, -m_new);
                if (edge) {
                    e0 = t0 + 2 * i <= prow ? e0 : -INFINITY;
                    e1 = t0 + 2 * i + 1 <= prow ? e1 : -INFINITY;
                }
                w[i] = pack_half2(fast_exp2(e0), fast_exp2(e1));
            }
            // O += P V of the previous tile has completed: the P buffer is free and O, l final for it
            if (j > 0) {
                if (!(ok = __all_sync(0xffffffffu, wait(o_done, (j - 1) & 1)))) break;
                tc_fence_after();
            }
            bool corrected = false;
            if (j > 0 && __any_sync(0xffffffffu, raise)) {
                const float alpha = raise ? fast_exp2(m_run - m_new) : 1.f;
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    float o[32];
                    tmem_ld32(o_cols + 32 * c, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(o_cols + 32 * c, o);
                }
                if (half == 0) tmem_st1(tmem_l + lane_base, tmem_ld1(tmem_l + lane_base) * alpha);
                tmem_wait_st();
                corrected = true;
            }
            m_run = m_new;
            // chunk `half` of row r of P: K-major operand layout, 16-byte pieces of 8 tokens
            const uint32_t prow_addr = p_s + half * S::kChunk + r * 128;
#pragma unroll
            for (int piece = 0; piece < 8; ++piece) {
                const uint32_t addr = prow_addr + ((piece ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "r"(w[4 * piece]),
                             "r"(w[4 * piece + 1]), "r"(w[4 * piece + 2]), "r"(w[4 * piece + 3]) : "memory");
            }
            fence_proxy_async_shared();
            if (corrected) tc_fence_before();
            mbar_arrive(p_full);
        }
        // ---- out = O / l ----
        if (ok) ok = __all_sync(0xffffffffu, wait(o_done, (ntiles - 1) & 1));
        if (ok) {
            tc_fence_after();
            const float inv = p.out_scale / tmem_ld1(tmem_l + lane_base);
            __half* dst = p.out + ((int64_t)(qs0 + i0 + ti) * p.Hq + (int64_t)g * G + hh) * kHeadDim + 64 * half;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                float o[32];
                tmem_ld32(o_cols + 32 * c, o);
                if (valid) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint4 u;
                        u.x = pack_half2(o[8 * k + 0] * inv, o[8 * k + 1] * inv);
                        u.y = pack_half2(o[8 * k + 2] * inv, o[8 * k + 3] * inv);
                        u.z = pack_half2(o[8 * k + 4] * inv, o[8 * k + 5] * inv);
                        u.w = pack_half2(o[8 * k + 6] * inv, o[8 * k + 7] * inv);
                        *reinterpret_cast<uint4*>(dst + 32 * c + 8 * k) = u;
                    }
                }
            }
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
