// Fused residual add + RMSNorm + QKV projection of one decode step.
//
// "rvLLM 소개" (discuss.pytorch.kr), §퓨즈드 CUDA 커널: each layer runs the
// residual add, the RMSNorm and the QKV projection as one kernel, so the
// normalised activations never travel through HBM. For T decode tokens:
//   s   = f16(x + residual)                 returned: the new residual stream
//   y   = s / sqrt(mean(s^2) + eps) * gamma
//   qkv = W y + bias                        W [N, H] f16, rows q heads | k | v
// and q, k, v leave in the layouts the cache write and the decode step take.
//
// At decode batch sizes this is a thin GEMM (N = 2048..4608 features, T =
// 64..256 tokens, K = H = 1536..3584) whose bytes are almost all W, so the
// grid reads W once from HBM and keeps the activations on chip:
//  * A CTA owns 64 tokens x one slice of H and streams W for a run of
//    consecutive feature tiles of kFT = 128 * kMT rows against them, so the
//    activation slice is built once for several tiles. The `split` slices of
//    a run are one thread-block cluster (split-K); after each feature tile
//    their partial sums meet in distributed shared memory, in rank order.
//  * W tiles [kFT rows x 64 k] come by TMA (128-byte swizzle) into a ring of
//    kStages slots that runs on across the feature tiles. With the overlap
//    flag the first ones are requested before the grid-dependency wait (W is
//    not written by the previous launch).
//  * The slice's activations are built once in shared memory: s = x + r in
//    f16 (stored to residual_out by the CTAs of the first run), the token's
//    sum of squares in fp32 and max |s| in f16, then the tensor-core operand
//    b = f16(s * gamma * 2^-e_t) with e_t the per-token power of two that puts
//    max |s| * max |gamma| (over the slice) in [2^14, 2^15). The division by
//    the RMS happens after the sum (the RMS needs all slices), so the operand
//    is scaled to neither overflow nor lose precision: s * gamma alone passes
//    65504 in residual streams with large channels.
//  * mma.sync m16n8k16 with features on M and tokens on N, fp32 accumulators.
//  * After each feature tile: partial * 2^e_t into shared memory; cluster
//    barrier; rank r sums its share of the tile's tokens over all ranks,
//    multiplies by 1 / sqrt(sum_s^2 / H + eps) (IEEE sqrt and division), adds
//    the bias and stores f16 (round to nearest even); cluster barrier.
#pragma once

#include <cooperative_groups.h>

#include "pkv_device.cuh"

namespace pkv {

constexpr int kQkvMaxCluster = 8;

struct QkvParams {
    const __half* x;           // [T, H]
    const __half* residual;    // [T, H]
    const __half* gamma;       // [H]
    const __half* bias;        // [N] or null
    __half* residual_out;      // [T, H]
    __half* q;                 // [T, q_cols]
    __half* k;                 // [T, kv_cols]
    __half* v;                 // [T, kv_cols]
    int32_t T, H, N;
    int32_t q_cols, kv_cols;   // Hq * D, Hkv * D
    int32_t kblocks;           // H / 64
    int32_t split;             // slices of H per run = cluster size (<= kQkvMaxCluster)
    int32_t slab_blocks;       // most 64-wide k blocks in one slice
    int32_t ftiles;            // feature tiles of kFT rows covering N
    int32_t tiles_per_cta;     // consecutive feature tiles one CTA streams
    float eps;
    int32_t prefetch_w;        // request W tiles before the grid-dependency wait
};

template <int kMT, int kStages>
struct QkvShape {
    static constexpr int kFT = 128 * kMT;                 // features per tile (8 warps x 16 kMT)
    static constexpr int kTT = 64;                        // tokens per CTA
    static constexpr int kThreads = 256;
    static constexpr int kStageBytes = kFT * 128;         // [kFT rows][64 k] f16
    static constexpr int kHeader = 1024;                  // barriers and per-token values
    static constexpr int kRedStride = kFT + 4;            // floats per token row of the partial tile
    static constexpr int kRedBytes = kTT * kRedStride * 4;
    static constexpr int kMaxSlabBytes = 232448 - 1024 - kHeader - kStages * kStageBytes - kRedBytes;
    static constexpr int kMaxSlabBlocks = kMaxSlabBytes / (kTT * 128);
    static_assert(kRedBytes % 1024 == 0, "the slab stays 1024-byte aligned");
    static size_t smem_bytes(int slab_blocks) {
        return 1024 + kHeader + (size_t)kStages * kStageBytes + kRedBytes + (size_t)kTT * slab_blocks * 128;
    }
};

// 2-D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                 :: "r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// 2^n as a float for -126 <= n <= 127.
__device__ __forceinline__ float exp2_int(int n) { return __int_as_float((127 + n) << 23); }

template <int kMT, int kStages>
__global__ void __launch_bounds__(256, 1)
add_rmsnorm_qkv_kernel(const __grid_constant__ CUtensorMap tm_w, const QkvParams p) {
    using S = QkvShape<kMT, kStages>;
    constexpr int kFT = S::kFT, kTT = S::kTT, kRS = S::kRedStride;
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const uint32_t bars = base;                                           // kStages x 8 bytes
    float* const ssq = reinterpret_cast<float*>(base_ptr + 64);           // [64] sum of s^2
    float* const up = reinterpret_cast<float*>(base_ptr + 320);           // [64] 2^e_t
    float* const rinv = reinterpret_cast<float*>(base_ptr + 576);         // [64] 1 / RMS
    const uint32_t ring = base + S::kHeader;
    float* const red = reinterpret_cast<float*>(base_ptr + S::kHeader + kStages * S::kStageBytes);
    const uint32_t slab = ring + kStages * S::kStageBytes + S::kRedBytes;
    const int slab_row = p.slab_blocks * 128;                             // bytes per token row

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = p.split;
    const int rank = (int)cluster.block_rank();                           // == blockIdx.x % split
    const int run = blockIdx.x / split;
    const int ft0 = run * p.tiles_per_cta;                                // first feature tile of the run
    const int nft = min(p.ftiles - ft0, p.tiles_per_cta);                 // >= 1
    const int t0 = blockIdx.y * kTT;
    const int kb0 = (int)((int64_t)rank * p.kblocks / split);
    const int nkb = (int)((int64_t)(rank + 1) * p.kblocks / split) - kb0; // >= 1: split <= kblocks
    const int total = nft * nkb;                                          // W blocks this CTA streams

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(bars + 8 * s, 1);
        mbar_init_fence();
    }
    __syncthreads();
    // W block i (feature tile i / nkb of the run, k block i % nkb of the slice)
    // into slot i % kStages (thread 0)
    auto issue = [&](int i) {
        const int s = i % kStages;
        const int j = i / nkb;
        mbar_arrive_expect_tx(bars + 8 * s, S::kStageBytes);
        tma_load_2d(ring + s * S::kStageBytes, &tm_w, bars + 8 * s, (kb0 + i - j * nkb) * 64, (ft0 + j) * kFT);
    };
    const int prologue = min(total, kStages);
    if (tid == 0) {
        prefetch_tensormap(&tm_w);
        if (p.prefetch_w)
            for (int i = 0; i < prologue; ++i) issue(i);
    }
    grid_dependency_wait();
    if (tid == 0 && !p.prefetch_w)
        for (int i = 0; i < prologue; ++i) issue(i);

    // ---- the slice's activations: warp w builds tokens w, w + 8, ..., w + 56 ----
    {
        const int cpt = nkb * 8;                  // 16-byte chunks per token row of the slice
        const bool write_res = run == 0;
        auto slab_addr = [&](int tl, int ch) {
            return slab + tl * slab_row + (((ch & ~7) | ((ch ^ tl) & 7)) << 4);
        };
        // max |gamma| over the slice (every warp, the same value)
        __half2 gm = __float2half2_rn(0.f);
        for (int ch = lane; ch < cpt; ch += 32) {
            const uint4 gv = __ldg(reinterpret_cast<const uint4*>(p.gamma + (int64_t)kb0 * 64 + ch * 8));
            const __half2* g2 = reinterpret_cast<const __half2*>(&gv);
#pragma unroll
            for (int e = 0; e < 4; ++e) gm = __hmax2(gm, __habs2(g2[e]));
        }
        float gmax = fmaxf(__low2float(gm), __high2float(gm));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));

        float sq[8];
        __half2 mx[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            sq[j] = 0.f;
            mx[j] = __float2half2_rn(0.f);
        }
        for (int ch = lane; ch < cpt; ch += 32) {
            const int64_t kg = (int64_t)kb0 * 64 + ch * 8;
            uint4 xv[8], rv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int t = t0 + warp + 8 * j;
                if (t < p.T) {
                    const int64_t off = (int64_t)t * p.H + kg;
                    xv[j] = ld_stream_16(reinterpret_cast<const uint4*>(p.x + off));
                    rv[j] = ld_stream_16(reinterpret_cast<const uint4*>(p.residual + off));
                } else {
                    xv[j] = rv[j] = make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int tl = warp + 8 * j;
                uint4 sv;
                __half2* s2 = reinterpret_cast<__half2*>(&sv);
                const __half2* x2 = reinterpret_cast<const __half2*>(&xv[j]);
                const __half2* r2 = reinterpret_cast<const __half2*>(&rv[j]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    s2[e] = __hadd2(x2[e], r2[e]);            // one rounding to f16, nearest even
                    mx[j] = __hmax2(mx[j], __habs2(s2[e]));
                    const float2 sf = __half22float2(s2[e]);
                    sq[j] = fmaf(sf.x, sf.x, sq[j]);
                    sq[j] = fmaf(sf.y, sf.y, sq[j]);
                }
                if (t0 + tl < p.T && write_res)
                    *reinterpret_cast<uint4*>(p.residual_out + (int64_t)(t0 + tl) * p.H + kg) = sv;
                sts128(slab_addr(tl, ch), sv);
            }
        }
        // per token: the sum of squares, and the operand's power-of-two scale
        float down[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float m = fmaxf(__low2float(mx[j]), __high2float(mx[j]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sq[j] += __shfl_xor_sync(0xffffffffu, sq[j], o);
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            }
            const float bound = m * gmax;                 // >= max |s * gamma| over the slice
            int e = 0;
            if (bound > 0.f && bound <= 3.402823466e38f) {
                const int E = (int)((__float_as_uint(bound) >> 23) & 0xFF) - 126;   // bound in [2^(E-1), 2^E)
                e = E - 15;                                                           // bound * 2^-e in [2^14, 2^15)
            }
            down[j] = exp2_int(-e);
            if (lane == 0) {
                ssq[warp + 8 * j] = sq[j];
                up[warp + 8 * j] = exp2_int(e);
            }
        }
        // b = f16(s * gamma * 2^-e): s * gamma is exact in fp32, the power of two too
        for (int ch = lane; ch < cpt; ch += 32) {
            const int64_t kg = (int64_t)kb0 * 64 + ch * 8;
            const uint4 gv = __ldg(reinterpret_cast<const uint4*>(p.gamma + kg));
            const __half2* g2 = reinterpret_cast<const __half2*>(&gv);
            float2 gf[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) gf[e] = __half22float2(g2[e]);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int tl = warp + 8 * j;
                const uint32_t a = slab_addr(tl, ch);
                uint4 sv = lds128(a), bv;
                const __half2* s2 = reinterpret_cast<const __half2*>(&sv);
                __half2* b2 = reinterpret_cast<__half2*>(&bv);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 sf = __half22float2(s2[e]);
                    b2[e] = __floats2half2_rn(sf.x * gf[e].x * down[j], sf.y * gf[e].y * down[j]);
                }
                sts128(a, bv);
            }
        }
    }
    __syncthreads();

    const int lr = lane & 15, lh = lane >> 4;     // A: row within 16, k half
    const int bm = lane >> 3, br = lane & 7;      // B: matrix of the x4 load, row within it
    const int g = lane >> 2, c = lane & 3;        // accumulator: feature row, token pair
    const int ta = rank * kTT / split, tb = (rank + 1) * kTT / split;   // this rank's tokens of a tile
    bool failed = false;
    int i = 0;                                    // W block counter over the run
    for (int j = 0; j < nft; ++j) {
        // ---- stream the tile's W blocks: 4 k16 steps per 64-wide block ----
        float acc[kMT][8][4];
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
        for (int kk = 0; kk < nkb; ++kk, ++i) {
            const int s = i % kStages;
            const bool ok = !failed && mbar_wait(bars + 8 * s, (i / kStages) & 1);
            if (ok) {
                const uint32_t wt = ring + s * S::kStageBytes;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    uint32_t a[kMT][4];
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        const int row = (warp * kMT + mt) * 16 + lr;
                        const int chunk = 2 * ks + lh;
                        ldsm_x4(wt + row * 128 + ((chunk ^ (row & 7)) << 4), a[mt][0], a[mt][1], a[mt][2],
                                a[mt][3]);
                    }
#pragma unroll
                    for (int np = 0; np < 4; ++np) {     // two n8 token tiles per x4 load
                        const int tl = np * 16 + (bm >> 1) * 8 + br;
                        const int ch = kk * 8 + 2 * ks + (bm & 1);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(slab + tl * slab_row + (((ch & ~7) | ((ch ^ tl) & 7)) << 4), b0, b1, b2, b3);
#pragma unroll
                        for (int mt = 0; mt < kMT; ++mt) {
                            mma_16816(acc[mt][2 * np], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
                            mma_16816(acc[mt][2 * np + 1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b2, b3);
                        }
                    }
                }
            }
            // a lost TMA is flagged by mbar_wait; every thread then skips the rest of the
            // stream but still takes every cluster barrier below
            if (__syncthreads_or(!ok)) failed = true;
            else if (tid == 0 && i + kStages < total) {
                fence_proxy_async_shared();       // the slot's reads by ldmatrix come first
                issue(i + kStages);
            }
        }
        if (j == nft - 1) grid_dependents_launch();

        // ---- partial tile, scaled back by 2^e_t, as red[token][feature] ----
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int f = (warp * kMT + mt) * 16 + g;
                const int tk = nt * 8 + 2 * c;
                const float u0 = up[tk], u1 = up[tk + 1];
                red[tk * kRS + f] = acc[mt][nt][0] * u0;
                red[(tk + 1) * kRS + f] = acc[mt][nt][1] * u1;
                red[tk * kRS + f + 8] = acc[mt][nt][2] * u0;
                red[(tk + 1) * kRS + f + 8] = acc[mt][nt][3] * u1;
            }
        cluster.sync();                           // every rank's partials (and sums of squares) are written

        if (j == 0) {                             // 1 / RMS of this rank's tokens, for every tile
            if (tid < tb - ta) {
                const int tk = ta + tid;
                float part[kQkvMaxCluster];
#pragma unroll
                for (int r = 0; r < kQkvMaxCluster; ++r)
                    part[r] = r < split ? *cluster.map_shared_rank(ssq + tk, r) : 0.f;
                float tot = 0.f;
#pragma unroll
                for (int r = 0; r < kQkvMaxCluster; ++r) tot += part[r];
                rinv[tk] = 1.0f / sqrtf(tot / (float)p.H + p.eps);
            }
            __syncthreads();
        }
        // ---- rank r finishes tokens [ta, tb) of feature tile ft0 + j ----
        constexpr int kQuads = kFT / 4;
        const int f0 = (ft0 + j) * kFT;
        for (int it = tid; it < (tb - ta) * kQuads; it += S::kThreads) {
            const int tk = ta + it / kQuads, fq = (it % kQuads) * 4;
            const int t = t0 + tk, n = f0 + fq;
            if (t >= p.T || n >= p.N) continue;
            float4 v[kQkvMaxCluster];
#pragma unroll
            for (int r = 0; r < kQkvMaxCluster; ++r)
                if (r < split)
                    v[r] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(red + tk * kRS + fq, r));
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < kQkvMaxCluster; ++r)
                if (r < split) {
                    sum.x += v[r].x;
                    sum.y += v[r].y;
                    sum.z += v[r].z;
                    sum.w += v[r].w;
                }
            const float ri = rinv[tk];
            float o[4] = {sum.x * ri, sum.y * ri, sum.z * ri, sum.w * ri};
            if (p.bias) {
                const uint2 bv = __ldg(reinterpret_cast<const uint2*>(p.bias + n));
                const float2 b01 = __half22float2(*reinterpret_cast<const __half2*>(&bv.x));
                const float2 b23 = __half22float2(*reinterpret_cast<const __half2*>(&bv.y));
                o[0] += b01.x;
                o[1] += b01.y;
                o[2] += b23.x;
                o[3] += b23.y;
            }
            __half* dst;
            if (n < p.q_cols) dst = p.q + (int64_t)t * p.q_cols + n;
            else if (n < p.q_cols + p.kv_cols) dst = p.k + (int64_t)t * p.kv_cols + (n - p.q_cols);
            else dst = p.v + (int64_t)t * p.kv_cols + (n - p.q_cols - p.kv_cols);
            uint2 ov;
            ov.x = pack_half2(o[0], o[1]);
            ov.y = pack_half2(o[2], o[3]);
            *reinterpret_cast<uint2*>(dst) = ov;
        }
        cluster.sync();                           // peers are done reading this CTA's partial tile
    }
}

}  // namespace pkv
