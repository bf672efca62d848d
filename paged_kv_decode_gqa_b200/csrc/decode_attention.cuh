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
//    last partition of (b, g) -- found by an atomic ticket, no waiting --
//    merges all partitions by the log-sum-exp rule and writes the output.
//
// FP8 E4M3 blocks are expanded to f16 in registers (exact), with k_scale
// folded into the logit scale and v_scale into the output.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr int kHeadDim = 128;
constexpr int kPageRows = 16;   // block_size
constexpr int kGroupPad = 8;    // query heads per KV head, padded to the mma N

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
    float logit_scale_log2;       // softmax_scale * log2(e) (* k_scale for FP8)
    float out_scale;              // 1 (v_scale for FP8)
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
    // Q^T as the B operand (16 channels x 8 heads per k-step); head r of g.
    uint32_t qf[8][2];
    {
        const bool live = r < G;
        const uint32_t* qh = reinterpret_cast<const uint32_t*>(
            p.q + ((int64_t)b * p.Hq + (int64_t)g * G + (live ? r : 0)) * kHeadDim);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            // f16 cache: channels 16j+2c(+1) and 16j+8+2c(+1);
            // FP8 cache: channels 16j+4c(+1) and 16j+4c+2(+1), matching the byte tile fragments.
            const int d0 = kFp8 ? 16 * j + 4 * c : 16 * j + 2 * c;
            const int d1 = kFp8 ? d0 + 2 : d0 + 8;
            qf[j][0] = live ? __ldg(qh + d0 / 2) : 0u;
            qf[j][1] = live ? __ldg(qh + d1 / 2) : 0u;
        }
    }
    const float sl = p.logit_scale_log2;
    float m0 = -INFINITY, m1 = -INFINITY;      // running max of heads 2c, 2c+1
    float l0 = 0.f, l1 = 0.f;                  // this lane's share of the running sums
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    for (int it = 0; it < n_iters; ++it) {
        const int s = it % kStages;
        const int ok = mbar_wait(full_bar(s), (it / kStages) & 1);
        // A timed-out wait (flagged) ends this warp's loop; the warp still
        // joins the merge barriers below so that no other warp waits for it.
        if (!__all_sync(0xffffffffu, ok)) break;
        const int blk = it * kConsumers + warp;
        if (blk < nblk) {
            const int valid = blk == nblk - 1 ? last_valid : kPageRows;
            const uint32_t kt = k_tile(s, warp), vt = v_tile(s, warp);

            // ---- S^T (16 tokens x 8 heads) = K (16 x 128) . Q^T ----
            float sacc[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (!kFp8) {
                const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int chunk = (kk & 3) * 2 + (lane >> 4);
                    const uint32_t addr = kt + (kk >> 2) * 2048 + row * 128 + ((chunk ^ (row & 7)) << 4);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(addr, a0, a1, a2, a3);
                    mma_16816(sacc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                }
            } else {
                const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                for (int J = 0; J < 4; ++J) {
                    const int chunk = 2 * J + (lane >> 4);
                    const uint32_t addr = kt + row * 128 + ((chunk ^ (row & 7)) << 4);
                    uint32_t r0, r1, r2, r3;            // 4 codes each: channels 16*chunk + 4c .. +3
                    ldsm_x4(addr, r0, r1, r2, r3);
                    mma_16816(sacc, e4m3x2_to_half2(r0), e4m3x2_to_half2(r1),
                              e4m3x2_to_half2(r0 >> 16), e4m3x2_to_half2(r1 >> 16),
                              qf[2 * J][0], qf[2 * J][1]);
                    mma_16816(sacc, e4m3x2_to_half2(r2), e4m3x2_to_half2(r3),
                              e4m3x2_to_half2(r2 >> 16), e4m3x2_to_half2(r3 >> 16),
                              qf[2 * J + 1][0], qf[2 * J + 1][1]);
                }
            }

            // ---- online softmax over this block's tokens (rows r, r+8) ----
            float x0 = sacc[0] * sl, x1 = sacc[1] * sl, x2 = sacc[2] * sl, x3 = sacc[3] * sl;
            if (valid < kPageRows) {                // rows past the context: excluded
                if (r >= valid) x0 = x1 = -INFINITY;
                if (r + 8 >= valid) x2 = x3 = -INFINITY;
            }
            float bm0 = fmaxf(x0, x2), bm1 = fmaxf(x1, x3);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
                bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
            }
            const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
            const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            const float p0 = fast_exp2(x0 - mn0), p1 = fast_exp2(x1 - mn1);
            const float p2 = fast_exp2(x2 - mn0), p3 = fast_exp2(x3 - mn1);
            l0 = l0 * al0 + (p0 + p2);
            l1 = l1 * al1 + (p1 + p3);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                o[i][0] *= al0; o[i][1] *= al1; o[i][2] *= al0; o[i][3] *= al1;
            }
            // P^T as the B operand: transpose the (token x head) accumulator layout.
            const uint32_t pb0 = movmatrix_trans(pack_half2(p0, p1));   // tokens 0..7
            const uint32_t pb1 = movmatrix_trans(pack_half2(p2, p3));   // tokens 8..15

            // ---- O^T (128 ch x 8 heads) += V^T (128 x 16 tokens) . P^T ----
            if constexpr (!kFp8) {
                uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;   // zero V of excluded rows
                if (valid < kPageRows) {
                    mlo = (2 * c < valid ? 0x0000ffffu : 0u) | (2 * c + 1 < valid ? 0xffff0000u : 0u);
                    mhi = (2 * c + 8 < valid ? 0x0000ffffu : 0u) | (2 * c + 9 < valid ? 0xffff0000u : 0u);
                }
                const int row = (lane & 7) + (lane >> 4) * 8;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int chunk = (i & 3) * 2 + ((lane >> 3) & 1);
                    const uint32_t addr = vt + (i >> 2) * 2048 + row * 128 + ((chunk ^ (row & 7)) << 4);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_trans(addr, a0, a1, a2, a3);
                    mma_16816(o[i], a0 & mlo, a1 & mlo, a2 & mhi, a3 & mhi, pb0, pb1);
                }
            } else {
                // lane (r, c) reads channels 16r..16r+15 of token rows 2c, 2c+1, 2c+8, 2c+9
                auto row_addr = [&](int t) { return vt + t * 128 + ((r ^ (t & 7)) << 4); };
                uint4 va = lds128(row_addr(2 * c)), vb = lds128(row_addr(2 * c + 1));
                uint4 vc = lds128(row_addr(2 * c + 8)), vd = lds128(row_addr(2 * c + 9));
                if (valid < kPageRows) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    if (2 * c >= valid) va = z;
                    if (2 * c + 1 >= valid) vb = z;
                    if (2 * c + 8 >= valid) vc = z;
                    if (2 * c + 9 >= valid) vd = z;
                }
                const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
                const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
                // m-tile i: rows r / r+8 are channels 16r+2i / 16r+2i+1 (bytes 2(i%2), +1 of word i/2)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t sel = (i & 1) ? 0x7362u : 0x5140u;
                    const uint32_t top = prmt(wa[i >> 1], wb[i >> 1], sel);   // tokens 2c, 2c+1
                    const uint32_t bot = prmt(wc[i >> 1], wd[i >> 1], sel);   // tokens 2c+8, 2c+9
                    mma_16816(o[i], e4m3x2_to_half2(top), e4m3x2_to_half2(top >> 16),
                              e4m3x2_to_half2(bot), e4m3x2_to_half2(bot >> 16), pb0, pb1);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
    }

    // ---- merge the consumer warps through shared memory (ring reused) ----
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    constexpr int kCT = 32 * kConsumers;
    consumer_sync(kCT);                           // every warp is done with the ring
    float* red_o = reinterpret_cast<float*>(ring_ptr);                 // [warp][head][D]
    float* red_m = red_o + kConsumers * kGroupPad * kHeadDim;          // [warp][head]
    float* red_l = red_m + kConsumers * kGroupPad;
    {
        float* ow = red_o + warp * kGroupPad * kHeadDim;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int d_lo = kFp8 ? 16 * r + 2 * i : 16 * i + r;
            const int d_hi = kFp8 ? d_lo + 1 : d_lo + 8;
            ow[(2 * c) * kHeadDim + d_lo] = o[i][0];
            ow[(2 * c + 1) * kHeadDim + d_lo] = o[i][1];
            ow[(2 * c) * kHeadDim + d_hi] = o[i][2];
            ow[(2 * c + 1) * kHeadDim + d_hi] = o[i][3];
        }
        if (r == 0) {
            red_m[warp * kGroupPad + 2 * c] = m0;
            red_m[warp * kGroupPad + 2 * c + 1] = m1;
            red_l[warp * kGroupPad + 2 * c] = l0;
            red_l[warp * kGroupPad + 2 * c + 1] = l1;
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
            out_g[h * kHeadDim + d] = __float2half_rn(acc / lsum * p.out_scale);
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
    __threadfence();
    consumer_sync(kCT);
    if (threadIdx.x == 0) {
        const unsigned int prev = atomicAdd(p.ws_count + (int64_t)b * p.Hkv + g, 1u);
        s_is_last = prev == (unsigned int)(nparts_b - 1);
    }
    consumer_sync(kCT);
    if (!s_is_last) return;
    __threadfence();
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
        out_g[h * kHeadDim + d] = __float2half_rn(acc / wsum * p.out_scale);
    }
    if (threadIdx.x == 0) p.ws_count[(int64_t)b * p.Hkv + g] = 0u;   // ready for the next call
}

}  // namespace pkv
