// Per-warp building blocks of paged GQA decode attention: the query-group
// fragments, and the online-softmax update of one 16-token page of K/V held in
// shared memory (a 128-byte-swizzled TMA tile).
//
// Layout of the tensor-core work (mma.sync m16n8k16, f16 in, f32 accumulate),
// chosen so that the KV tokens sit on the M side and the G <= 8 query heads of
// one KV head on N = 8 (G = 6 or 7 for Qwen2.5 wastes 1/4 or 1/8 of N, where
// putting the heads on M = 16 would waste 5/8):
//   S^T (16 tok x 8 heads) = K (16 tok x 128 ch) . Q^T (128 ch x 8 heads)
//   O^T (128 ch x 8 heads) += V^T (128 ch x 16 tok) . P^T (16 tok x 8 heads)
// Lane (r, c) = (lane / 4, lane % 4) holds the logits of tokens r, r+8 for
// heads 2c, 2c+1 and the output of the same two heads, so the softmax rescale
// is lane-local; P^T reaches the B-operand layout by an 8x8 transpose
// (movmatrix). The contraction over channels may use any channel order as long
// as K and Q agree; the FP8 path uses that freedom to read 4 codes per lane.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr int kHeadDim = 128;
constexpr int kPageRows = 16;   // block_size
constexpr int kGroupPad = 8;    // query heads per KV head, padded to the mma N

// Running softmax state of one warp over the tokens it has seen.
struct WarpState {
    float m0, m1;       // running max (exp2 domain) of heads 2c, 2c+1
    float l0, l1;       // this lane's share of the running sums
    float o[8][4];      // O^T fragments: m-tile i, rows r / r+8, heads 2c / 2c+1

    __device__ __forceinline__ void reset() {
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    }
    // Sums the lanes' shares of l over the 8 lanes that hold the same heads.
    __device__ __forceinline__ void reduce_l() {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        }
    }
};

// Channel held by lane (r, c) in m-tile i of O^T, rows r and r+8.
template <bool kFp8>
__device__ __forceinline__ int out_channel_lo(int r, int i) { return kFp8 ? 16 * r + 2 * i : 16 * i + r; }
template <bool kFp8>
__device__ __forceinline__ int out_channel_hi(int r, int i) { return kFp8 ? 16 * r + 2 * i + 1 : 16 * i + r + 8; }

// Q^T as the B operand of the logits (mma m16n8k16), for the query head of
// row r (lane (r, c) = (lane / 4, lane % 4)); `qrow` is that head's 128 f16
// channels, or nullptr for a padding head. The contraction may take the
// channels in any order as long as K and Q agree:
//  * f16 cache: channels 16j+2c(+1) and 16j+8+2c(+1) of k-step j;
//  * FP8 cache: channels 16j+4c(+1) and 16j+4c+2(+1), matching the four E4M3
//    codes per lane that ldmatrix delivers from the byte tile.
template <bool kFp8>
struct QOperand {
    uint32_t f[8][2];
};

template <bool kFp8>
__device__ __forceinline__ void load_q_fragments(QOperand<kFp8>& q, const __half* qrow, int lane) {
    const int c = lane & 3;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qrow);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int d0 = kFp8 ? 16 * j + 4 * c : 16 * j + 2 * c;
        const int d1 = kFp8 ? d0 + 2 : d0 + 8;
        q.f[j][0] = qrow ? __ldg(q32 + d0 / 2) : 0u;
        q.f[j][1] = qrow ? __ldg(q32 + d1 / 2) : 0u;
    }
}

// Logits S^T (16 tokens x 8 heads) = K (16 x 128) . Q^T of one page, times
// `sl`, with the rows at or past `valid` set to -inf: lane (r, c) gets tokens
// r (x[0], x[1]) and r + 8 (x[2], x[3]) of heads 2c, 2c + 1. K tile at shared
// address kt (f16: two 2 KiB boxes of 64 channels each; FP8: one 2 KiB box).
template <bool kFp8>
__device__ __forceinline__ void page_logits(float (&x)[4], uint32_t kt, int valid, const QOperand<kFp8>& qf,
                                            float sl, int lane) {
    const int r = lane >> 2;
    // Two independent accumulators (even and odd k-steps) halve the chain of
    // dependent tensor-core ops; their sum is the contraction over all channels.
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
    if constexpr (!kFp8) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int chunk = (kk & 3) * 2 + (lane >> 4);
            const uint32_t addr = kt + (kk >> 2) * 2048 + row * 128 + ((chunk ^ (row & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(addr, a0, a1, a2, a3);
            mma_16816(sacc[kk & 1], a0, a1, a2, a3, qf.f[kk][0], qf.f[kk][1]);
        }
    } else {
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            const int chunk = 2 * J + (lane >> 4);
            const uint32_t addr = kt + row * 128 + ((chunk ^ (row & 7)) << 4);
            uint32_t r0, r1, r2, r3;            // 4 codes each: channels 16*chunk + 4c .. +3
            ldsm_x4(addr, r0, r1, r2, r3);
            uint32_t h0l, h0h, h1l, h1h, h2l, h2h, h3l, h3h;
            e4m3x4_to_half2x2(r0, h0l, h0h);
            e4m3x4_to_half2x2(r1, h1l, h1h);
            e4m3x4_to_half2x2(r2, h2l, h2h);
            e4m3x4_to_half2x2(r3, h3l, h3h);
            mma_16816(sacc[0], h0l, h1l, h0h, h1h, qf.f[2 * J][0], qf.f[2 * J][1]);
            mma_16816(sacc[1], h2l, h3l, h2h, h3h, qf.f[2 * J + 1][0], qf.f[2 * J + 1][1]);
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = (sacc[0][k] + sacc[1][k]) * sl;
    if (valid < kPageRows) {                    // rows past the context: excluded
        if (r >= valid) x[0] = x[1] = -INFINITY;
        if (r + 8 >= valid) x[2] = x[3] = -INFINITY;
    }
}

// O^T (128 ch x 8 heads) += V^T (128 x 16 tokens) . P^T of one page, P^T given
// as the B operand (pb0: tokens 0..7, pb1: tokens 8..15); V tile at shared
// address vt, rows at or past `valid` read as zero.
template <bool kFp8>
__device__ __forceinline__ void page_pv(float (&o)[8][4], uint32_t vt, int valid, uint32_t pb0, uint32_t pb1,
                                        int lane) {
    const int r = lane >> 2, c = lane & 3;
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
            uint32_t tl, th, bl, bh;
            e4m3x4_to_half2x2(top, tl, th);
            e4m3x4_to_half2x2(bot, bl, bh);
            mma_16816(o[i], tl, th, bl, bh, pb0, pb1);
        }
    }
}

// Online-softmax step of `st` over the logits of `kPages` pages (16 tokens
// each): new running max, rescale of l and O by exp2(m_old - m_new), the
// probabilities of the new tokens added to l, and P^T of each page as the
// B operand (pb[2 * page], pb[2 * page + 1]).
template <int kPages>
__device__ __forceinline__ void softmax_step(WarpState& st, const float (&x)[kPages][4], uint32_t (&pb)[2 * kPages]) {
    float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
    for (int q = 0; q < kPages; ++q) {
        bm0 = fmaxf(bm0, fmaxf(x[q][0], x[q][2]));
        bm1 = fmaxf(bm1, fmaxf(x[q][1], x[q][3]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
        bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
    }
    const float mn0 = fmaxf(st.m0, bm0), mn1 = fmaxf(st.m1, bm1);
    const float al0 = fast_exp2(st.m0 - mn0), al1 = fast_exp2(st.m1 - mn1);
    st.m0 = mn0;
    st.m1 = mn1;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int q = 0; q < kPages; ++q) {
        const float p0 = fast_exp2(x[q][0] - mn0), p1 = fast_exp2(x[q][1] - mn1);
        const float p2 = fast_exp2(x[q][2] - mn0), p3 = fast_exp2(x[q][3] - mn1);
        s0 += p0 + p2;
        s1 += p1 + p3;
        // P^T as the B operand: transpose the (token x head) accumulator layout.
        pb[2 * q] = movmatrix_trans(pack_half2(p0, p1));       // tokens 0..7
        pb[2 * q + 1] = movmatrix_trans(pack_half2(p2, p3));   // tokens 8..15
    }
    st.l0 = st.l0 * al0 + s0;
    st.l1 = st.l1 * al1 + s1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        st.o[i][0] *= al0; st.o[i][1] *= al1; st.o[i][2] *= al0; st.o[i][3] *= al1;
    }
}

// Online-softmax update of `st` with one page: K tile at shared address kt,
// V tile at vt, the first `valid` rows live. `sl` = softmax scale * log2(e)
// (* k_scale for FP8).
template <bool kFp8>
__device__ __forceinline__ void attend_page(WarpState& st, uint32_t kt, uint32_t vt, int valid,
                                            const QOperand<kFp8>& qf, float sl, int lane) {
    float x[1][4];
    page_logits<kFp8>(x[0], kt, valid, qf, sl, lane);
    uint32_t pb[2];
    softmax_step<1>(st, x, pb);
    page_pv<kFp8>(st.o, vt, valid, pb[0], pb[1], lane);
}

// The same update with two consecutive pages of one segment in one softmax
// step: page A (all 16 rows live) at ka/va, page B (the first valid_b rows
// live) at kb/vb. Their logits are independent tensor-core chains and the
// max, rescale and shuffles are paid once for 32 tokens.
template <bool kFp8>
__device__ __forceinline__ void attend_page_pair(WarpState& st, uint32_t ka, uint32_t va, uint32_t kb,
                                                 uint32_t vb, int valid_b, const QOperand<kFp8>& qf, float sl,
                                                 int lane) {
    float x[2][4];
    page_logits<kFp8>(x[0], ka, kPageRows, qf, sl, lane);
    page_logits<kFp8>(x[1], kb, valid_b, qf, sl, lane);
    uint32_t pb[4];
    softmax_step<2>(st, x, pb);
    page_pv<kFp8>(st.o, va, kPageRows, pb[0], pb[1], lane);
    page_pv<kFp8>(st.o, vb, valid_b, pb[2], pb[3], lane);
}

}  // namespace pkv
