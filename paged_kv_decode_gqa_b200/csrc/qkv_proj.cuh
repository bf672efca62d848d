// Fused residual add + RMSNorm + QKV projection of one decode step, on the
// fifth-generation tensor cores (tcgen05, TMEM accumulators).
//
// "rvLLM 소개" (discuss.pytorch.kr), §퓨즈드 CUDA 커널: each layer runs the
// residual add, the RMSNorm and the QKV projection fused, so the normalised
// activations never travel through HBM. For T decode tokens:
//   s   = f16(x + residual)                 returned: the new residual stream
//   y   = s / sqrt(mean(s^2) + eps) * gamma
//   qkv = W y + bias                        W [N, H] f16, rows q heads | k | v
// and q, k, v leave in the layouts the cache write and the decode step take.
//
// At decode batch sizes this is a thin GEMM (N = 2048..4608 features, T =
// 64..256 tokens, K = H = 1536..3584) whose bytes are almost all W. Each SM
// keeps a fixed number of bytes in flight (its shared-memory ring), so the
// time is set by the bytes each SM must bring in; the design minimises them:
//  * Two launches. `add_residual_kernel` forms s = x + r (one f16 rounding,
//    nearest even) into residual_out, which the caller receives anyway. The
//    projection then reads one activation tile per k block (s, from L2)
//    instead of two (x and r), and every 128- or 256-feature tile reads it.
//    The projection is launched with programmatic dependent launch and, with
//    the overlap flag, requests its first W tiles while the add still runs.
//  * The normalisation is folded into the operands and the epilogue, never
//    materialised: 1/RMS is a per-token scalar applied after the sum, and
//    gamma scales the weight tile instead of the activations:
//      qkv[t][n] = (1 / rms_t) * sum_k f16(W[n][k] * gamma[k]) * s[t][k].
//    The activation operand is s itself, exact in f16 (no per-token scale,
//    no overflow); W * gamma is rounded once to f16 (relative 2^-11, as
//    rounding the activations would be).
//  * Work unit: (M = 128 or 256 features, token tile of TT = 64, 128 or 256
//    tokens, slice of H). The `split` slices of one (features, tokens) tile
//    are one thread-block cluster (split-K); their fp32 partial tiles meet in
//    distributed shared memory at the end.
//  * Per k block, one TMA warp brings the W tile [M rows x 64 k] and the s
//    tile [TT tokens x 64 k] (128-byte swizzle, the UMMA K-major layout) into
//    one stage of a ring. Eight warps multiply the W tile by gamma in place
//    and add each token's s^2 to its sum in fp32. One thread issues, per
//    128-row half of the W tile, D[128 x TT] += W' s^T (4 steps of K = 16,
//    `tcgen05.mma.kind::f16`) into its own TMEM columns and commits the
//    stage back to the TMA warp.
//  * Epilogue: the eight warps read the accumulators out of TMEM into shared
//    memory as fp32 [token][feature]; after a cluster barrier, rank r sums
//    its share of the tile's tokens over all ranks in rank order (every
//    remote load of two items in flight before the first sum), and the sums
//    of squares likewise, multiplies by 1 / sqrt(sum_s^2 / H + eps) (IEEE
//    square root and division), adds the bias and stores f16 (nearest even);
//    a second cluster barrier keeps every partial tile alive until its
//    readers are done.
// Every barrier wait has a time limit; one that runs out flags
// PKV_DEVERR_WAIT_TIMEOUT, and every role stops, waits for what it has in
// flight, still takes both cluster barriers, and TMEM is freed.
#pragma once

#include <cooperative_groups.h>

#include "pkv_device.cuh"
#include "umma.cuh"

namespace pkv {

constexpr int kQkvMaxCluster = 8;
constexpr int kQkvMaxStages = 8;

struct QkvParams {
    const __half* gamma;       // [H]
    const __half* bias;        // [N] or null
    __half* residual_out;      // [T, H]
    __half* q;                 // [T, q_cols]
    __half* k;                 // [T, kv_cols]
    __half* v;                 // [T, kv_cols]
    int32_t T, H, N;
    int32_t q_cols, kv_cols;   // Hq * D, Hkv * D
    int32_t kblocks;           // H / 64
    int32_t split;             // slices of H = cluster size (<= kQkvMaxCluster)
    int32_t tt;                // tokens per tile: 64, 128 or 256
    int32_t stages;            // ring depth (<= kQkvMaxStages)
    float eps;
    int32_t prefetch_w;        // request W tiles before the grid-dependency wait
};

struct QkvShape {
    static constexpr int kThreads = 320;               // warp 0 TMA, warp 1 MMA, warps 2-9 scale + epilogue
    static constexpr int kBuilders = 256;
    static constexpr int kHeader = 4096;               // barriers and per-token values
    static constexpr int kSmemMax = 232448 - 1024;     // the opt-in limit per block, less static room
    __host__ __device__ static int stage_bytes(int m, int tt) { return m * 128 + tt * 128; }
    __host__ __device__ static int gamma_bytes(int kblocks, int split) {   // the slice's gamma, 1024-aligned
        return ((kblocks + split - 1) / split * 128 + 1023) & ~1023;
    }
    static size_t smem_bytes(int m, int tt, int stages, int kblocks, int split) {
        return 1024 + kHeader + (size_t)gamma_bytes(kblocks, split) + (size_t)stages * stage_bytes(m, tt);
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

// Barrier among the 256 build/epilogue threads only (named barrier 1).
__device__ __forceinline__ void builders_sync() {
    asm volatile("bar.sync 1, %0;" :: "n"(QkvShape::kBuilders) : "memory");
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ float sumsq_half2(uint32_t a, float acc) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&a));
    return fmaf(f.y, f.y, fmaf(f.x, f.x, acc));
}


// s = f16(x + residual) into residual_out, 16 bytes per thread per step (the
// first launch of the projection). `chunks` = T * H / 8.
__global__ void __launch_bounds__(256)
add_residual_kernel(const __half* __restrict__ x, const __half* __restrict__ residual, __half* __restrict__ out,
                    int64_t chunks) {
    grid_dependents_launch();                    // the projection may start requesting W tiles
    grid_dependency_wait();                      // x and residual may come from the previous launch
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += stride) {
        const uint4 a = ld_stream_16(reinterpret_cast<const uint4*>(x) + i);
        const uint4 b = ld_stream_16(reinterpret_cast<const uint4*>(residual) + i);
        uint4 r;
        const __half2* a2 = reinterpret_cast<const __half2*>(&a);
        const __half2* b2 = reinterpret_cast<const __half2*>(&b);
        __half2* r2 = reinterpret_cast<__half2*>(&r);
#pragma unroll
        for (int e = 0; e < 4; ++e) r2[e] = __hadd2(a2[e], b2[e]);   // one rounding, nearest even
        reinterpret_cast<uint4*>(out)[i] = r;
    }
}

template <int kAcc>   // 128-row halves of the W tile: M = 128 kAcc features
__global__ void __launch_bounds__(QkvShape::kThreads, 1)
rmsnorm_qkv_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                   const QkvParams p) {
    using S = QkvShape;
    constexpr int kM = 128 * kAcc;
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = p.split, TT = p.tt, NS = p.stages;
    const int rank = (int)cluster.block_rank();                           // == blockIdx.x % split
    const int m0 = (int)(blockIdx.x / split) * kM;                        // first feature of the tile
    const int t0 = (int)blockIdx.y * TT;                                   // first token of the tile
    const int kb0 = (int)((int64_t)rank * p.kblocks / split);
    const int nkb = (int)((int64_t)(rank + 1) * p.kblocks / split) - kb0;  // >= 1: split <= kblocks

    // ---- shared memory ----
    const uint32_t bars = base;
    auto full = [&](int s) { return bars + 8u * s; };                    // TMA landed (transaction bytes)
    auto ready = [&](int s) { return bars + 64u + 8u * s; };             // W scaled (256 threads)
    auto empty = [&](int s) { return bars + 128u + 8u * s; };            // the MMAs that read it are done
    const uint32_t acc_full = bars + 192, tmem_slot = bars + 200;
    float* const sqp = reinterpret_cast<float*>(base_ptr + 1024);         // [256]: per-thread sums of s^2
    float* const sqt = reinterpret_cast<float*>(base_ptr + 2048);         // [TT]: over the slice, per token
    float* const rinv = reinterpret_cast<float*>(base_ptr + 3072);        // [TT]: 1 / RMS of rank's tokens
    const uint32_t gam = base + S::kHeader;                               // the slice's gamma [nkb][64]
    const uint32_t ring = gam + S::gamma_bytes(p.kblocks, split);
    const int stage = S::stage_bytes(kM, TT);
    auto w_s = [&](int s) { return ring + (uint32_t)(s * stage); };
    auto s_s = [&](int s) { return w_s(s) + kM * 128; };
    float* const red = reinterpret_cast<float*>(base_ptr + (ring - base)); // [TT][kM] after the MMAs

    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < NS; ++s) {
            mbar_init(full(s), 1);
            mbar_init(ready(s), S::kBuilders);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, (uint32_t)(kAcc * TT));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t tmem;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(tmem_slot) : "memory");
    grid_dependents_launch();

    // Bounded wait that also gives up once another role has given up.
    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        if (mbar_try_wait(bar, parity)) return true;
        const uint64_t t_start = global_timer_ns();
        for (uint32_t it = 0;; ++it) {
            if (mbar_try_wait(bar, parity)) return true;
            if ((it & 63u) == 63u) {
                if (*reinterpret_cast<volatile int*>(&s_abort)) return false;
                if (global_timer_ns() - t_start > kWaitLimitNs) {
                    flag_error(PKV_DEVERR_WAIT_TIMEOUT);
                    *reinterpret_cast<volatile int*>(&s_abort) = 1;
                    return false;
                }
            }
        }
    };

    bool ok = true;
    if (warp == 0) {
        // ================================ TMA ================================
        if (lane == 0) {
            prefetch_tensormap(&tm_w);
            prefetch_tensormap(&tm_s);
        }
        const uint32_t tx = (uint32_t)stage;
        const int pre = p.prefetch_w ? min(NS, nkb) : 0;
        if (lane == 0)
            for (int j = 0; j < pre; ++j) {
                mbar_arrive_expect_tx(full(j), tx);
                tma_load_2d(w_s(j), &tm_w, full(j), (kb0 + j) * 64, m0);
            }
        grid_dependency_wait();                                            // s is the first launch's output
        if (lane == 0)
            for (int j = 0; j < pre; ++j) tma_load_2d(s_s(j), &tm_s, full(j), (kb0 + j) * 64, t0);
        int j = pre;
        for (; j < nkb; ++j) {
            const int s = j % NS;
            if (j >= NS && !(ok = __all_sync(0xffffffffu, wait(empty(s), ((j / NS) - 1) & 1)))) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(full(s), tx);
                tma_load_2d(w_s(s), &tm_w, full(s), (kb0 + j) * 64, m0);
                tma_load_2d(s_s(s), &tm_s, full(s), (kb0 + j) * 64, t0);
            }
        }
        // nothing of ours may be in flight when the CTA leaves
        for (int i = max(0, j - NS); i < j; ++i) mbar_wait(full(i % NS), (i / NS) & 1);
    } else if (warp == 1) {
        // ================================ MMA ================================
        const uint32_t idesc = umma_idesc_f16(128, TT, 0);               // W' and s both K-major
        for (int j = 0; j < nkb; ++j) {
            const int s = j % NS;
            if (!(ok = __all_sync(0xffffffffu, wait(ready(s), (j / NS) & 1)))) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int a = 0; a < kAcc; ++a)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tmem + (uint32_t)(a * TT), umma_desc_sw128(w_s(s) + a * 16384 + kk * 32, 16, 1024),
                                    umma_desc_sw128(s_s(s) + kk * 32, 16, 1024), idesc, (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(empty(s));
            }
            __syncwarp();
        }
        // completes once every MMA issued above has (also after a timeout)
        if (lane == 0) umma_commit(acc_full);
        __syncwarp();
    } else {
        // ========================= scale, then epilogue ========================
        const int bt = tid - 64;                                           // 0 .. 255
        const int nsub = S::kBuilders / TT;                                // threads per token: 4, 2 or 1
        const int tok = bt % TT, sub = bt / TT, cpt = 8 / nsub;            // 16-byte chunks per k block
        grid_dependency_wait();
        // the slice's gamma, once
        for (int i = bt; i < nkb * 8; i += S::kBuilders)
            sts128(gam + 16 * i, __ldg(reinterpret_cast<const uint4*>(p.gamma + (int64_t)kb0 * 64) + i));
        builders_sync();
        float sq = 0.f;
        for (int j = 0; j < nkb; ++j) {
            const int s = j % NS;
            if (!(ok = __all_sync(0xffffffffu, wait(full(s), (j / NS) & 1)))) break;
            // this token's s^2 over this thread's chunks (logical chunk c sits at c ^ (row & 7))
            for (int c = sub * cpt; c < sub * cpt + cpt; ++c) {
                const uint4 sv = lds128(s_s(s) + (uint32_t)(tok * 128 + ((c ^ (tok & 7)) << 4)));
                sq = sumsq_half2(sv.w, sumsq_half2(sv.z, sumsq_half2(sv.y, sumsq_half2(sv.x, sq))));
            }
            // W' = f16(W * gamma) on this thread's share of the tile's kM x 8 chunks
#pragma unroll
            for (int i = bt; i < kM * 8; i += S::kBuilders) {
                const int row = i >> 3, c = i & 7;
                const uint32_t off = (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4));
                uint4 wv = lds128(w_s(s) + off);
                const uint4 gv = lds128(gam + j * 128 + 16 * c);
                wv.x = hmul2_u32(wv.x, gv.x);
                wv.y = hmul2_u32(wv.y, gv.y);
                wv.z = hmul2_u32(wv.z, gv.z);
                wv.w = hmul2_u32(wv.w, gv.w);
                sts128(w_s(s) + off, wv);
            }
            fence_proxy_async_shared();
            mbar_arrive(ready(s));
        }
        sqp[sub * TT + tok] = sq;
        if (ok) ok = __all_sync(0xffffffffu, wait(acc_full, 0));
        tc_fence_after();
        builders_sync();
        if (bt < TT) {                                                     // the slice's sum, in sub order
            float a = 0.f;
            for (int u = 0; u < nsub; ++u) a += sqp[u * TT + bt];
            sqt[bt] = a;
        }
        // the partial tile out of TMEM: red[token][feature] (every load landed, every MMA done)
        if (ok) {
            const int qd = warp & 3, hf = (warp - 2) >> 2;                 // TMEM lane quarter, column half
#pragma unroll 1
            for (int a = 0; a < kAcc; ++a) {
                const int f = 128 * a + 32 * qd + lane;
#pragma unroll 1
                for (int c0 = hf * (TT / 2); c0 < (hf + 1) * (TT / 2); c0 += 32) {
                    float v[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + (uint32_t)(a * TT + c0), v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) red[(c0 + i) * kM + f] = v[i];
                }
            }
        }
        tc_fence_before();
    }

    // ---- every rank's partial tile and sums of squares are in its shared memory ----
    cluster.sync();
    if (warp >= 2) {
        const int bt = tid - 64;
        const int tr0 = rank * TT / split, tr1 = (rank + 1) * TT / split;   // this rank's tokens of the tile
        // 1 / RMS of those tokens: the ranks' sums of squares, all requested before any is added
        for (int t = tr0 + bt; t < tr1; t += S::kBuilders) {
            float u[kQkvMaxCluster];
#pragma unroll
            for (int r = 0; r < kQkvMaxCluster; ++r) u[r] = r < split ? *cluster.map_shared_rank(sqt + t, r) : 0.f;
            float a = 0.f;
#pragma unroll
            for (int r = 0; r < kQkvMaxCluster; ++r) a += u[r];             // rank order (the rest add 0)
            rinv[t] = 1.f / sqrtf(a / (float)p.H + p.eps);
        }
        builders_sync();
        // (token, 4 features) items, two at a time: the partial tiles summed in rank order, / RMS,
        // + bias, f16; every remote load of both items is issued before the first sum
        constexpr int kChunks = kM / 4;
        const int items = (tr1 - tr0) * kChunks;
        for (int i0 = bt; i0 < items; i0 += 2 * S::kBuilders) {
            float4 u[2][kQkvMaxCluster];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int it = min(i0 + h * S::kBuilders, items - 1);
                const int t = tr0 + it / kChunks, fc = (it % kChunks) * 4;
#pragma unroll
                for (int r = 0; r < kQkvMaxCluster; ++r)
                    u[h][r] = r < split ? *reinterpret_cast<const float4*>(cluster.map_shared_rank(red + t * kM + fc, r))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int it = i0 + h * S::kBuilders;
                if (it >= items) continue;
                const int t = tr0 + it / kChunks, fc = (it % kChunks) * 4;
                const int tg = t0 + t, n = m0 + fc;
                if (tg >= p.T || n >= p.N) continue;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int r = 0; r < kQkvMaxCluster; ++r) {                 // rank order (the rest add 0)
                    acc.x += u[h][r].x;
                    acc.y += u[h][r].y;
                    acc.z += u[h][r].z;
                    acc.w += u[h][r].w;
                }
                const float ri = rinv[t];
                float2 b01 = make_float2(0.f, 0.f), b23 = b01;
                if (p.bias) {
                    const uint2 bv = __ldg(reinterpret_cast<const uint2*>(p.bias + n));
                    b01 = __half22float2(*reinterpret_cast<const __half2*>(&bv.x));
                    b23 = __half22float2(*reinterpret_cast<const __half2*>(&bv.y));
                }
                uint2 o;
                o.x = pack_half2(acc.x * ri + b01.x, acc.y * ri + b01.y);
                o.y = pack_half2(acc.z * ri + b23.x, acc.w * ri + b23.y);
                __half* dst;
                int64_t idx;
                if (n < p.q_cols) {
                    dst = p.q;
                    idx = (int64_t)tg * p.q_cols + n;
                } else if (n < p.q_cols + p.kv_cols) {
                    dst = p.k;
                    idx = (int64_t)tg * p.kv_cols + (n - p.q_cols);
                } else {
                    dst = p.v;
                    idx = (int64_t)tg * p.kv_cols + (n - p.q_cols - p.kv_cols);
                }
                *reinterpret_cast<uint2*>(dst + idx) = o;
            }
        }
    }
    cluster.sync();                                      // peers are done reading this CTA's partial tile
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)(kAcc * TT));
    }
}

}  // namespace pkv
