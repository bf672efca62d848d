// C ABI of the paged-KV decode library (declared in include/pagedkv.h):
// argument checks, TMA descriptors, launch planning and launches. The whole
// library is this one translation unit, so the device error word needs no
// relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "pagedkv.h"
#include "cache_write.cuh"
#include "decode_attention.cuh"
#include "decode_balanced.cuh"
#include "fp8_scales.cuh"
#include "qkv_proj.cuh"
#include "prefill_attention.cuh"
#include "prefill_tc.cuh"

namespace {

using pkv::kHeadDim;
using pkv::kPageRows;

constexpr int kConsumers = 4;
constexpr int kStagesF16 = 3;   // 3 x 32 KiB ring: two CTAs per SM
constexpr int kStagesFp8 = 6;   // 6 x 16 KiB ring

// Balanced streaming kernel: worker warps per CTA and page slots per worker
// ring (f16 pages are 8 KiB, FP8 pages 4 KiB), one CTA per SM. Measured best
// on the benchmark workloads with two-page softmax steps: f16 6 workers x 3
// slots (144 KiB of ring, 255 registers a thread; 8 x 3 took 17% longer on the
// 1.5B-shaped step and 25% on the skewed one, 7B-shaped steps were within 2%
// for 5..8 workers), FP8 12 workers x 3 slots (144 KiB; three warps per
// scheduler at 168 registers, 2.5% faster than 8 x 4 at 255 registers, while
// 10 x 4 and 10 x 3 were 10% slower). The macros exist for tuning builds.
#ifndef PKV_BAL_WARPS_F16
#define PKV_BAL_WARPS_F16 6
#endif
#ifndef PKV_BAL_WARPS_FP8
#define PKV_BAL_WARPS_FP8 12
#endif
#ifndef PKV_BAL_STAGES_F16
#define PKV_BAL_STAGES_F16 3
#endif
#ifndef PKV_BAL_STAGES_FP8
#define PKV_BAL_STAGES_FP8 3
#endif
// CTAs of one launch per SM (at most; fewer if they do not fit). One CTA per SM
// leaves room, when its shared memory allows, for the next launch's CTA to
// start its prologue beside it.
#ifndef PKV_BAL_CTAS_PER_SM
#define PKV_BAL_CTAS_PER_SM 8
#endif
constexpr int kBalWarpsF16 = PKV_BAL_WARPS_F16;
constexpr int kBalWarpsFp8 = PKV_BAL_WARPS_FP8;
constexpr int kBalStagesF16 = PKV_BAL_STAGES_F16;
constexpr int kBalStagesFp8 = PKV_BAL_STAGES_FP8;
constexpr int kBalMaxBatch = 8192;        // unit-order tables must fit in shared memory
constexpr int kBalMinUnits = 4;           // pages per worker at least (small batches)
// Barrier-wait limit of a launch under PKV_STEP_SELFTEST_WAIT_TIMEOUT.
constexpr uint64_t kSelftestWaitLimitNs = 2000000ull;   // 2 ms

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// FP8 scales held on the device ([1] or [Hkv] floats); null arrays mean the
// per-tensor scalar scales of the call.
struct DeviceScales {
    const float* k = nullptr;
    const float* v = nullptr;
    int32_t per_head = 0;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// View of one cache tensor [num_blocks, 16, Hkv, 128] as a 3-D TMA tensor
// (channel, head, pool row) with 16-row x 128-byte boxes, 128-byte swizzled.
// L2 fills are promoted to one KV head's row: 256 bytes in f16 (both boxes of
// the row), 128 bytes in FP8, where a wider fill would drag in the next KV
// head's row, which is streamed by another worker much later.
bool make_cache_map(CUtensorMap* map, const void* base, bool fp8, int num_blocks, int Hkv) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
    if (!encode) return false;
    const cuuint64_t esz = fp8 ? 1 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)Hkv, (cuuint64_t)num_blocks * kPageRows};
    cuuint64_t strides[2] = {kHeadDim * esz, (cuuint64_t)Hkv * kHeadDim * esz};
    cuuint32_t box[3] = {fp8 ? 128u : 64u, 1u, (cuuint32_t)kPageRows};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        fp8 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Small per-thread cache of encoded maps: serving loops reuse the same pool.
struct MapKey {
    const void* base;
    int num_blocks, Hkv;
    bool fp8;
    bool operator==(const MapKey& o) const {
        return base == o.base && num_blocks == o.num_blocks && Hkv == o.Hkv && fp8 == o.fp8;
    }
};

bool cached_cache_map(CUtensorMap* out, const void* base, bool fp8, int num_blocks, int Hkv) {
    constexpr int kSlots = 8;
    thread_local MapKey keys[kSlots];
    thread_local CUtensorMap maps[kSlots];
    thread_local int used = 0, next = 0;
    const MapKey key{base, num_blocks, Hkv, fp8};
    for (int i = 0; i < used; ++i)
        if (keys[i] == key) {
            *out = maps[i];
            return true;
        }
    CUtensorMap m;
    if (!make_cache_map(&m, base, fp8, num_blocks, Hkv)) return false;
    keys[next] = key;
    maps[next] = m;
    next = (next + 1) % kSlots;
    used = std::min(used + 1, kSlots);
    *out = m;
    return true;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous launch in the stream finishes; it waits (griddepcontrol.wait)
// before its first global-memory access.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Opt a kernel into its dynamic shared memory once per device.
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, int bytes, unsigned long long* done_mask) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) __atomic_fetch_or(done_mask, bit, __ATOMIC_ACQ_REL);
    return e;
}

template <bool kFp8, int kStages>
pkv_status launch_decode(const pkv::DecodeParams& prm, const CUtensorMap& mk, const CUtensorMap& mv,
                         int B, int Hkv, cudaStream_t stream) {
    using S = pkv::DecodeShape<kFp8, kConsumers, kStages>;
    auto kernel = pkv::decode_attention_kernel<kFp8, kConsumers, kStages>;
    static unsigned long long done = 0;
    if (ensure_smem(kernel, S::kSmemBytes, &done) != cudaSuccess) return PKV_ERR_CUDA;
    dim3 grid(prm.nparts, Hkv, B);
    return launch_pdl(kernel, grid, dim3(S::kThreads), S::kSmemBytes, stream, mk, mv, prm) == cudaSuccess
               ? PKV_OK : PKV_ERR_CUDA;
}

int bal_warps(bool fp8) { return fp8 ? kBalWarpsFp8 : kBalWarpsF16; }

template <bool kFp8>
using BalShape = pkv::BalancedShape<kFp8, kFp8 ? kBalWarpsFp8 : kBalWarpsF16, kFp8 ? kBalStagesFp8 : kBalStagesF16>;

template <bool kFp8, bool kFuse = false>
auto balanced_kernel() {
    return pkv::decode_balanced_kernel<kFp8, kFp8 ? kBalWarpsFp8 : kBalWarpsF16,
                                       kFp8 ? kBalStagesFp8 : kBalStagesF16, kFuse>;
}

// Persistent grid of the balanced kernel for batch B on the current device:
// as many CTAs as fit at once (0 on error). Both the plain and the fused
// variant are opted into their shared memory here.
template <bool kFp8>
int balanced_grid(int B) {
    static unsigned long long done = 0, done_fused = 0;
    auto kernel = balanced_kernel<kFp8>();
    int dev = 0, sms = 0, per_sm = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return 0;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return 0;
    const int dyn_max = optin - (int)fa.sharedSizeBytes;            // opt-in minus static shared
    if (BalShape<kFp8>::smem_bytes(B) > (size_t)dyn_max) return 0;  // tables do not fit
    if (ensure_smem(balanced_kernel<kFp8, true>(), dyn_max, &done_fused) != cudaSuccess) return 0;
    if (ensure_smem(kernel, dyn_max, &done) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, BalShape<kFp8>::kThreads,
                                                      BalShape<kFp8>::smem_bytes(B)) != cudaSuccess)
        return 0;
    return std::max(1, std::min(per_sm, PKV_BAL_CTAS_PER_SM)) * sms;
}

struct BalancedLayout {
    size_t o, ml, count, total;
};

BalancedLayout balanced_layout(int64_t workers, int64_t B, int64_t Hkv) {
    BalancedLayout w{};
    w.o = 0;
    w.ml = align256(2 * workers * 32 * 8 * sizeof(float4));
    w.count = w.ml + align256(2 * workers * 4 * sizeof(float4));
    w.total = w.count + align256(pkv::kMergeLevels * 2 * workers * sizeof(unsigned int));
    (void)B;
    (void)Hkv;
    return w;
}

// The balanced kernel serves AUTO unless the batch is too large for its tables.
bool use_balanced(int64_t B, int64_t Hkv, int64_t max_blocks_per_seq) {
    return B <= kBalMaxBatch && B * Hkv * max_blocks_per_seq < (int64_t(1) << 31);
}

struct WorkspaceLayout {
    size_t o, m, l, count, total;
};

// Launches the balanced kernel (fused with this step's cache write when
// k_new/v_new are given) after the workspace check.
pkv_status launch_balanced(bool fp8, int grid, const void* k_new, const void* v_new, void* out,
                           const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
                           int32_t Hq, int32_t Hkv, int32_t max_blocks_per_seq, int32_t num_blocks,
                           int32_t max_context_len, float softmax_scale, float k_scale, float v_scale,
                           const DeviceScales& ds, void* workspace, size_t workspace_bytes,
                           bool overlap_previous, cudaStream_t st, bool selftest_stall = false) {
    const BalancedLayout bl = balanced_layout((int64_t)grid * bal_warps(fp8), batch, Hkv);
    if (!workspace || workspace_bytes < bl.total) return PKV_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PKV_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    pkv::BalancedParams bp{};
    bp.out = static_cast<__half*>(out);
    bp.q = static_cast<const __half*>(q);
    bp.block_tables = block_tables;
    bp.context_lens = context_lens;
    bp.ws_o = reinterpret_cast<float4*>(ws + bl.o);
    bp.ws_ml = reinterpret_cast<float4*>(ws + bl.ml);
    bp.ws_count = reinterpret_cast<unsigned int*>(ws + bl.count);
    bp.k_new = static_cast<const __half*>(k_new);
    bp.v_new = static_cast<const __half*>(v_new);
    bp.k_cache = const_cast<void*>(k_cache);
    bp.v_cache = const_cast<void*>(v_cache);
    bp.k_scale = k_scale;
    bp.v_scale = v_scale;
    bp.B = batch;
    bp.Hq = Hq;
    bp.Hkv = Hkv;
    bp.G = Hq / Hkv;
    bp.max_blocks_per_seq = max_blocks_per_seq;
    bp.num_blocks = num_blocks;
    bp.max_context_len = max_context_len;
    bp.min_units_per_worker = kBalMinUnits;
    bp.overlap_previous = overlap_previous ? 1 : 0;
    const float log2e = 1.4426950408889634f;
    // per-tensor FP8 scales fold into these; device scales are applied per KV head in the kernel
    bp.logit_scale_log2 = softmax_scale * (fp8 && !ds.k ? k_scale : 1.f) * log2e;
    bp.out_scale = fp8 && !ds.k ? v_scale : 1.f;
    bp.k_scales = fp8 ? ds.k : nullptr;
    bp.v_scales = fp8 ? ds.v : nullptr;
    bp.scales_per_head = ds.per_head;
    bp.stall_worker = selftest_stall ? 0 : -1;
    bp.wait_limit_ns = selftest_stall ? kSelftestWaitLimitNs : pkv::kWaitLimitNs;
    CUtensorMap mk, mv;
    if (!cached_cache_map(&mk, k_cache, fp8, num_blocks, Hkv) ||
        !cached_cache_map(&mv, v_cache, fp8, num_blocks, Hkv))
        return PKV_ERR_CUDA;
    const bool fuse = k_new != nullptr;
    const dim3 g(grid), blk(fp8 ? BalShape<true>::kThreads : BalShape<false>::kThreads);
    cudaError_t e;
    if (fp8)
        e = fuse ? launch_pdl(balanced_kernel<true, true>(), g, blk, BalShape<true>::smem_bytes(batch), st, mk, mv, bp)
                 : launch_pdl(balanced_kernel<true, false>(), g, blk, BalShape<true>::smem_bytes(batch), st, mk, mv, bp);
    else
        e = fuse ? launch_pdl(balanced_kernel<false, true>(), g, blk, BalShape<false>::smem_bytes(batch), st, mk, mv, bp)
                 : launch_pdl(balanced_kernel<false, false>(), g, blk, BalShape<false>::smem_bytes(batch), st, mk, mv, bp);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

WorkspaceLayout workspace_layout(int64_t B, int64_t Hq, int64_t Hkv, int64_t nparts) {
    WorkspaceLayout w{};
    const int64_t rows = B * Hq * nparts;
    w.o = 0;
    w.m = w.o + align256(rows * kHeadDim * sizeof(float));
    w.l = w.m + align256(rows * sizeof(float));
    w.count = w.l + align256(rows * sizeof(float));
    w.total = w.count + align256(pkv::part_merge_levels((int)nparts) * B * Hkv * nparts * sizeof(unsigned int));
    return w;
}

// The plan paged_gqa_decode_attention runs for these sizes on the current
// device, and the scratch it needs: the balanced kernel for
// PKV_PARTITION_AUTO when the batch's tables fit (else fixed partitions of
// the suggested size); fixed partitions, rounded up to whole pages, when
// partition_tokens > 0, a single pass when one partition covers the longest
// context. `zero_off`/`zero_bytes` is the part of the scratch that must be
// zero when a call starts (the merge counters).
struct AttnPlan {
    bool balanced = false;
    int grid = 0;
    int32_t partition = 0;
    int nparts = 1;
    size_t ws_bytes = 0, zero_off = 0, zero_bytes = 0;
};

AttnPlan plan_attention(bool fp8, int32_t batch, int32_t Hq, int32_t Hkv, int32_t max_blocks_per_seq,
                        int32_t max_context_len, int32_t partition_tokens) {
    AttnPlan pl;
    if (partition_tokens == PKV_PARTITION_AUTO) {
        pl.grid = !use_balanced(batch, Hkv, max_blocks_per_seq) ? 0
                  : fp8 ? balanced_grid<true>(batch) : balanced_grid<false>(batch);
        if (pl.grid > 0) {
            const BalancedLayout bl = balanced_layout((int64_t)pl.grid * bal_warps(fp8), batch, Hkv);
            pl.balanced = true;
            pl.ws_bytes = bl.total;
            pl.zero_off = bl.count;
            pl.zero_bytes = bl.total - bl.count;
            return pl;
        }
        partition_tokens = paged_gqa_decode_suggest_partition(batch, Hkv, max_context_len, kPageRows, 0);
    }
    int32_t P = partition_tokens;
    if (P == 0 || P >= max_context_len) P = std::max(max_context_len, 1);
    P = (P + kPageRows - 1) / kPageRows * kPageRows;
    pl.partition = P;
    pl.nparts = std::max(1, (max_context_len + P - 1) / P);
    if (pl.nparts > 1) {
        const WorkspaceLayout wl = workspace_layout(batch, Hq, Hkv, pl.nparts);
        pl.ws_bytes = wl.total;
        pl.zero_off = wl.count;
        pl.zero_bytes = wl.total - wl.count;
    }
    return pl;
}

// Host-side argument checks shared by the attention entry points (PKV_OK for
// a valid call, also when batch == 0).
pkv_status check_attention_args(const void* out, const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
                                int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
                                int32_t max_context_len, float softmax_scale, int32_t kv_dtype,
                                float k_scale, float v_scale, int32_t partition_tokens) {
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_blocks_per_seq <= 0 || num_blocks <= 0 || max_context_len < 0 ||
        partition_tokens < PKV_PARTITION_AUTO)
        return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    if (kv_dtype != PKV_KV_F16 && kv_dtype != PKV_KV_FP8_E4M3) return PKV_ERR_INVALID_ARG;
    if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * block_size) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return PKV_ERR_INVALID_ARG;
    const bool fp8 = kv_dtype == PKV_KV_FP8_E4M3;
    if (fp8 && !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
        return PKV_ERR_INVALID_ARG;
    if (head_dim != kHeadDim || block_size != kPageRows) return PKV_ERR_UNSUPPORTED;
    if (num_q_heads / num_kv_heads > pkv::kGroupPad) return PKV_ERR_UNSUPPORTED;
    if (partition_tokens > 0 && partition_tokens % block_size != 0) return PKV_ERR_INVALID_ARG;
    if (batch == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
        return PKV_ERR_INVALID_ARG;
    if (batch > 65535 || num_kv_heads > 65535) return PKV_ERR_UNSUPPORTED;
    return PKV_OK;
}


// ---------------------------------------------------------------- the calls
// Bodies of the entry points, with FP8 scales either per tensor (host
// scalars) or on the device (DeviceScales).

pkv_status cache_write_impl(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                                const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                                int32_t head_dim, int32_t num_blocks, int32_t block_size,
                                int32_t kv_dtype, float k_scale, float v_scale, const DeviceScales& ds,
                            void* stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 || block_size <= 0)
        return PKV_ERR_INVALID_ARG;
    if (kv_dtype != PKV_KV_F16 && kv_dtype != PKV_KV_FP8_E4M3) return PKV_ERR_INVALID_ARG;
    if (head_dim % 8 != 0) return PKV_ERR_UNSUPPORTED;
    const bool fp8 = kv_dtype == PKV_KV_FP8_E4M3;
    if (fp8 && !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
        return PKV_ERR_INVALID_ARG;
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PKV_ERR_INVALID_ARG;
    pkv::CacheWriteParams prm;
    prm.k_new = static_cast<const uint4*>(k_new);
    prm.v_new = static_cast<const uint4*>(v_new);
    prm.k_cache = k_cache;
    prm.v_cache = v_cache;
    prm.slot_mapping = slot_mapping;
    prm.num_slots = (int64_t)num_blocks * block_size;
    prm.num_tokens = num_tokens;
    prm.chunks_per_token = num_kv_heads * (head_dim / 8);
    prm.chunks_per_head = head_dim / 8;
    prm.k_scale = k_scale;
    prm.v_scale = v_scale;
    prm.k_scales = fp8 ? ds.k : nullptr;
    prm.v_scales = fp8 ? ds.v : nullptr;
    prm.scales_per_head = ds.per_head;
    const int64_t total = (int64_t)num_tokens * prm.chunks_per_token;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 0x7fffffff) return PKV_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e =
        fp8 ? launch_pdl(pkv::cache_write_kernel<true>, dim3((unsigned)blocks), dim3(threads), 0, st, prm)
            : launch_pdl(pkv::cache_write_kernel<false>, dim3((unsigned)blocks), dim3(threads), 0, st, prm);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status attention_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, const int32_t* context_lens,
                                      int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                                      int32_t num_blocks, int32_t max_context_len, float softmax_scale,
                                      int32_t kv_dtype, float k_scale, float v_scale, const DeviceScales& ds,
                                      int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                                      void* stream) {
    {
        const pkv_status v = check_attention_args(out, q, k_cache, v_cache, block_tables, context_lens, batch,
                                                  num_q_heads, num_kv_heads, head_dim, block_size,
                                                  max_blocks_per_seq, num_blocks, max_context_len,
                                                  softmax_scale, kv_dtype, k_scale, v_scale,
                                                  partition_tokens);
        if (v != PKV_OK || batch == 0) return v;
    }
    const bool fp8 = kv_dtype == PKV_KV_FP8_E4M3;
    const int G = num_q_heads / num_kv_heads;

    const float log2e = 1.4426950408889634f;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const AttnPlan plan = plan_attention(fp8, batch, num_q_heads, num_kv_heads, max_blocks_per_seq,
                                         max_context_len, partition_tokens);
    if (plan.balanced) {
        return launch_balanced(fp8, plan.grid, nullptr, nullptr, out, q, k_cache, v_cache, block_tables,
                               context_lens, batch, num_q_heads, num_kv_heads, max_blocks_per_seq,
                               num_blocks, max_context_len, softmax_scale, k_scale, v_scale, ds,
                               workspace, workspace_bytes, false, st);
    }
    const int32_t P = plan.partition;
    const int nparts = plan.nparts;

    pkv::DecodeParams prm{};
    prm.out = static_cast<__half*>(out);
    prm.q = static_cast<const __half*>(q);
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    if (nparts > 1) {
        const WorkspaceLayout wl = workspace_layout(batch, num_q_heads, num_kv_heads, nparts);
        if (!workspace || workspace_bytes < wl.total) return PKV_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PKV_ERR_WORKSPACE;
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        prm.ws_o = reinterpret_cast<float*>(ws + wl.o);
        prm.ws_m = reinterpret_cast<float*>(ws + wl.m);
        prm.ws_l = reinterpret_cast<float*>(ws + wl.l);
        prm.ws_count = reinterpret_cast<unsigned int*>(ws + wl.count);
    }
    prm.Hq = num_q_heads;
    prm.Hkv = num_kv_heads;
    prm.G = G;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.max_context_len = max_context_len;
    prm.partition_tokens = P;
    prm.nparts = nparts;
    prm.logit_scale_log2 = softmax_scale * (fp8 && !ds.k ? k_scale : 1.f) * log2e;
    prm.out_scale = fp8 && !ds.k ? v_scale : 1.f;
    prm.k_scales = fp8 ? ds.k : nullptr;
    prm.v_scales = fp8 ? ds.v : nullptr;
    prm.scales_per_head = ds.per_head;

    CUtensorMap mk, mv;
    if (!cached_cache_map(&mk, k_cache, fp8, num_blocks, num_kv_heads) ||
        !cached_cache_map(&mv, v_cache, fp8, num_blocks, num_kv_heads))
        return PKV_ERR_CUDA;
    return fp8 ? launch_decode<true, kStagesFp8>(prm, mk, mv, batch, num_kv_heads, st)
               : launch_decode<false, kStagesF16>(prm, mk, mv, batch, num_kv_heads, st);
}

pkv_status step_impl(void* out, const void* q, const void* k_new, const void* v_new,
                                 void* k_cache, void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int32_t max_blocks_per_seq, int32_t num_blocks, int32_t max_context_len,
                                 float softmax_scale, int32_t kv_dtype, float k_scale, float v_scale,
                                 const DeviceScales& ds, void* workspace, size_t workspace_bytes,
                                 uint32_t flags, void* stream) {
    if (flags & ~(PKV_STEP_OVERLAP_PREVIOUS | PKV_STEP_SELFTEST_WAIT_TIMEOUT)) return PKV_ERR_INVALID_ARG;
    const pkv_status v = check_attention_args(out, q, k_cache, v_cache, block_tables, context_lens, batch,
                                              num_q_heads, num_kv_heads, head_dim, block_size,
                                              max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
                                              kv_dtype, k_scale, v_scale, PKV_PARTITION_AUTO);
    if (v != PKV_OK || batch == 0) return v;
    if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return PKV_ERR_INVALID_ARG;
    if (!use_balanced(batch, num_kv_heads, max_blocks_per_seq)) return PKV_ERR_UNSUPPORTED;
    const bool fp8 = kv_dtype == PKV_KV_FP8_E4M3;
    const int grid = fp8 ? balanced_grid<true>(batch) : balanced_grid<false>(batch);
    if (grid <= 0) return PKV_ERR_UNSUPPORTED;
    return launch_balanced(fp8, grid, k_new, v_new, out, q, k_cache, v_cache, block_tables, context_lens,
                           batch, num_q_heads, num_kv_heads, max_blocks_per_seq, num_blocks,
                           max_context_len, softmax_scale, k_scale, v_scale, ds, workspace, workspace_bytes,
                           (flags & PKV_STEP_OVERLAP_PREVIOUS) != 0, static_cast<cudaStream_t>(stream),
                           (flags & PKV_STEP_SELFTEST_WAIT_TIMEOUT) != 0);
}

// Validates a device-scale pair (a per-head set needs num_kv_heads entries).
pkv_status check_device_scales(const float* k_scales, const float* v_scales, int32_t per_head) {
    if (!k_scales || !v_scales) return PKV_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(k_scales) & 3u) || (reinterpret_cast<uintptr_t>(v_scales) & 3u))
        return PKV_ERR_INVALID_ARG;
    if (per_head != 0 && per_head != 1) return PKV_ERR_INVALID_ARG;
    return PKV_OK;
}

// ------------------------------------------------ fused add + RMSNorm + QKV
constexpr int kQkvMaxSplit = pkv::kQkvMaxCluster;   // portable cluster size
constexpr int kQkvMaxHidden = 8192;

// A [rows, H] f16 matrix as a 2-D TMA tensor (k, row) with [box_rows x 64]
// boxes, 128-byte swizzled (the UMMA K-major layout); rows past the end read
// as zeros.
bool make_rows_map(CUtensorMap* map, const void* ptr, int H, int rows, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
    if (!encode) return false;
    cuuint64_t dims[2] = {(cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)H * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct QkvPlan {
    int acc = 0, split = 0, tt = 0, stages = 0, mtiles = 0, ttiles = 0;
    size_t smem = 0;
    double cost = 0;
};

auto qkv_kernel(int acc) { return acc == 1 ? pkv::rmsnorm_qkv_kernel<1> : pkv::rmsnorm_qkv_kernel<2>; }

cudaLaunchConfig_t qkv_config(const QkvPlan& pl, cudaStream_t st, cudaLaunchAttribute (&attr)[2]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(pl.mtiles * pl.split), (unsigned)pl.ttiles);
    cfg.blockDim = dim3(pkv::QkvShape::kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)pl.split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cfg;
}

// The plan: token tiles of 64, 128 or 256 tokens (the MMA's N), feature
// tiles of 128 or 256 rows, and the split of H (cluster size). An SM keeps
// its ring's bytes in flight, so a CTA's time goes with the bytes it streams:
// cost = waves x (stages streamed x stage bytes + a share per cluster rank
// for the reduction), waves counted from the clusters the device reports it
// can hold at once.
bool qkv_plan(int T, int H, int N, QkvPlan* out) {
    using S = pkv::QkvShape;
    struct Entry {
        int dev, T, H, N;
        QkvPlan plan;
    };
    constexpr int kSlots = 8;
    thread_local Entry cache[kSlots];
    thread_local int used = 0, next = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    for (int i = 0; i < used; ++i)
        if (cache[i].dev == dev && cache[i].T == T && cache[i].H == H && cache[i].N == N) {
            *out = cache[i].plan;
            return true;
        }
    static unsigned long long done1 = 0, done2 = 0;
    if (ensure_smem(qkv_kernel(1), S::kSmemMax, &done1) != cudaSuccess ||
        ensure_smem(qkv_kernel(2), S::kSmemMax, &done2) != cudaSuccess)
        return false;
    const int kb = H / 64;
    const int tt = T <= 64 ? 64 : T <= 128 ? 128 : 256;
    const int ttiles = (T + tt - 1) / tt;
    bool found = false;
    for (int acc = 1; acc <= 2; ++acc) {
        const int m = 128 * acc;
        for (int split = 1; split <= std::min(kQkvMaxSplit, kb); ++split) {
            QkvPlan pl;
            pl.acc = acc;
            pl.split = split;
            pl.tt = tt;
            pl.mtiles = (N + m - 1) / m;
            pl.ttiles = ttiles;
            const size_t fixed = 1024 + S::kHeader + (size_t)S::gamma_bytes(kb, split);
            const int stage = S::stage_bytes(m, tt);
            pl.stages = (int)std::min<size_t>(pkv::kQkvMaxStages, (S::kSmemMax - fixed) / stage);
            // at least two stages, and the partial tile [tt][m] fp32 fits in the ring it reuses
            if (pl.stages < 2 || (size_t)pl.stages * stage < (size_t)tt * m * 4) continue;
            pl.smem = S::smem_bytes(m, tt, pl.stages, kb, split);
            cudaLaunchAttribute attr[2];
            cudaLaunchConfig_t cfg = qkv_config(pl, nullptr, attr);
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, qkv_kernel(acc), &cfg) != cudaSuccess) {
                (void)cudaGetLastError();
                continue;
            }
            if (clusters < 1) continue;
            const int64_t waves = ((int64_t)pl.mtiles * ttiles + clusters - 1) / clusters;
            const int per = (kb + split - 1) / split;
            pl.cost = (double)waves * ((double)per * stage + 16384.0 * split);
            if (!found || pl.cost < out->cost) {
                *out = pl;
                found = true;
            }
        }
    }
    if (!found) return false;
    cache[next] = Entry{dev, T, H, N, *out};
    next = (next + 1) % kSlots;
    used = std::min(used + 1, kSlots);
    return true;
}

// Two launches: s = x + r into residual_out, then the projection, which reads
// s back (from L2) and may request its first W tiles while the add runs.
pkv_status launch_qkv(const QkvPlan& pl, const pkv::QkvParams& prm, const void* w, const void* x,
                      const void* residual, cudaStream_t st) {
    CUtensorMap mw, ms;
    if (!make_rows_map(&mw, w, prm.H, prm.N, 128 * pl.acc) ||
        !make_rows_map(&ms, prm.residual_out, prm.H, prm.T, pl.tt))
        return PKV_ERR_CUDA;
    const int64_t chunks = (int64_t)prm.T * prm.H / 8;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return PKV_ERR_CUDA;
    const int64_t blocks = std::min<int64_t>((chunks + 255) / 256, (int64_t)sms * 4);
    if (launch_pdl(pkv::add_residual_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                   static_cast<const __half*>(x), static_cast<const __half*>(residual), prm.residual_out,
                   chunks) != cudaSuccess)
        return PKV_ERR_CUDA;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = qkv_config(pl, st, attr);
    return cudaLaunchKernelEx(&cfg, qkv_kernel(pl.acc), mw, ms, prm) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// ------------------------------------------------------------ paged prefill
// 8 query tokens per CTA (one per consumer warp), an 8-page ring.
constexpr int kPrefillConsumers = 8;
constexpr int kPrefillStages = 8;

template <bool kFp8>
pkv_status launch_prefill(const pkv::PrefillParams& prm, const CUtensorMap& mk, const CUtensorMap& mv,
                          int chunks, int Hkv, int B, cudaStream_t stream) {
    using S = pkv::PrefillShape<kFp8, kPrefillConsumers, kPrefillStages>;
    auto kernel = pkv::prefill_attention_kernel<kFp8, kPrefillConsumers, kPrefillStages>;
    static unsigned long long done = 0;
    if (ensure_smem(kernel, S::kSmemBytes, &done) != cudaSuccess) return PKV_ERR_CUDA;
    return launch_pdl(kernel, dim3((unsigned)chunks, Hkv, B), dim3(S::kThreads), S::kSmemBytes, stream, mk, mv,
                      prm) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// q [total, Hq, 128] f16 as a 3-D TMA tensor (channel, head, token) with
// boxes of 64 channels x the G heads of one KV head x `tokens` tokens,
// 128-byte swizzled: one box is the operand rows (token, head) of a prefill
// tile for one half of the channels; tokens past `total` read as zeros.
bool make_q_map(CUtensorMap* map, const void* q, int Hq, int total, int G, int tokens) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
    if (!encode) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)Hq, (cuuint64_t)total};
    cuuint64_t strides[2] = {kHeadDim * 2, (cuuint64_t)Hq * kHeadDim * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)G, (cuuint32_t)tokens};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Workspace of the stream-K prefill schedule for a device of `ctas` SMs (grids of up to one CTA
// per SM): two partial results (both query tiles) per CTA, then one ticket per (CTA, query tile,
// row quarter).
struct PrefillWorkspace {
    int64_t parts, counters, total;
};
PrefillWorkspace prefill_layout(int64_t ctas) {
    using S = pkv::PrefillTcShape;
    PrefillWorkspace w;
    w.parts = 0;
    w.counters = 2 * ctas * S::kQTiles * (int64_t)S::kPartBytes;
    w.total = (int64_t)align256((size_t)(w.counters + ctas * S::kQTiles * 4 * (int64_t)sizeof(unsigned int)));
    return w;
}

// f16 prefill on tcgen05: a persistent grid of one CTA per SM (its shared
// memory and TMEM) over items of (two tiles of 128 / G query tokens, KV head,
// sequence); whole items without a workspace, the load-balanced (stream-K)
// schedule with one.
pkv_status launch_prefill_tc(const pkv::PrefillParams& prm, const CUtensorMap& mk, const CUtensorMap& mv,
                             int max_query_len, int Hkv, int B, void* workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
    using S = pkv::PrefillTcShape;
    const int tokens = S::kRows / prm.G;
    CUtensorMap mq;
    if (!make_q_map(&mq, prm.q, prm.Hq, prm.total, prm.G, tokens)) return PKV_ERR_CUDA;
    auto kernel = workspace ? pkv::prefill_tc_kernel<true> : pkv::prefill_tc_kernel<false>;
    static unsigned long long done[2] = {0, 0};
    if (ensure_smem(kernel, S::kSmemBytes, &done[workspace ? 1 : 0]) != cudaSuccess) return PKV_ERR_CUDA;
    // persistent: one CTA per SM (or per item when there are fewer), items of two query tiles
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return PKV_ERR_CUDA;
    const int per_item = S::kQTiles * tokens;                    // queries per item: two tiles
    const int q_groups = (max_query_len + per_item - 1) / per_item;
    const int64_t items = (int64_t)q_groups * Hkv * B;
    if (items > INT32_MAX / 2) return PKV_ERR_UNSUPPORTED;      // item indices are int in the kernel
    const int ctas = (int)std::min<int64_t>(items, sms);
    uint8_t* ws = nullptr;
    unsigned int* counters = nullptr;
    if (workspace) {
        // laid out for the device (not this call's grid), so that calls of any size can share it
        const PrefillWorkspace w = prefill_layout(sms);
        if (workspace_bytes < (size_t)w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return PKV_ERR_WORKSPACE;
        ws = static_cast<uint8_t*>(workspace) + w.parts;
        counters = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(workspace) + w.counters);
    }
    return launch_pdl(kernel, dim3((unsigned)ctas), dim3(S::kThreads), S::kSmemBytes, stream, mq, mk, mv, prm,
                      tokens, q_groups, B, ws, counters) == cudaSuccess
               ? PKV_OK : PKV_ERR_CUDA;
}

bool ranges_overlap(const void* a, int64_t na, const void* b, int64_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na > 0 && nb > 0 && x < y + (uintptr_t)nb && y < x + (uintptr_t)na;
}

}  // namespace

extern "C" {

const char* pkv_status_string(pkv_status status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported shape or type";
        case PKV_ERR_WORKSPACE: return "workspace missing or too small";
        case PKV_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

pkv_status pkv_device_error(uint32_t* flags) {
    if (!flags) return PKV_ERR_INVALID_ARG;
    unsigned int v = 0, zero = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return PKV_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, pkv::g_device_error, sizeof(v)) != cudaSuccess) return PKV_ERR_CUDA;
    if (cudaMemcpyToSymbol(pkv::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return PKV_ERR_CUDA;
    *flags = v;
    return PKV_OK;
}

pkv_status paged_kv_cache_write(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                                const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                                int32_t head_dim, int32_t num_blocks, int32_t block_size,
                                int32_t kv_dtype, float k_scale, float v_scale, void* stream) {
    return cache_write_impl(k_new, v_new, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads, head_dim,
                            num_blocks, block_size, kv_dtype, k_scale, v_scale, DeviceScales{}, stream);
}

pkv_status paged_kv_fp8_scales(const void* x, int64_t rows, int32_t num_kv_heads, int32_t head_dim,
                               int32_t scales_per_head, float* scales, void* stream) {
    if (rows < 0 || num_kv_heads <= 0 || head_dim <= 0 || !scales) return PKV_ERR_INVALID_ARG;
    if (scales_per_head != 0 && scales_per_head != 1) return PKV_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(scales) & 3u) return PKV_ERR_INVALID_ARG;
    if (head_dim % 8 != 0 || (scales_per_head && num_kv_heads > 1024)) return PKV_ERR_UNSUPPORTED;
    if (rows > 0 && (!x || !aligned16(x))) return PKV_ERR_INVALID_ARG;
    const int n = scales_per_head ? num_kv_heads : 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the running maxima live in `scales` (as fp32 bit patterns) until the conversion
    if (cudaMemsetAsync(scales, 0, sizeof(float) * n, st) != cudaSuccess) return PKV_ERR_CUDA;
    if (rows > 0) {
        pkv::AmaxParams ap;
        ap.x = static_cast<const uint4*>(x);
        ap.chunks_per_head = head_dim / 8;
        ap.chunks = rows * num_kv_heads * (int64_t)ap.chunks_per_head;
        ap.Hkv = num_kv_heads;
        ap.per_head = scales_per_head;
        ap.amax_bits = reinterpret_cast<unsigned int*>(scales);
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return PKV_ERR_CUDA;
        constexpr int kThreads = 256;
        int64_t blocks = std::min<int64_t>((ap.chunks + kThreads - 1) / kThreads, 8 * (int64_t)sms);
        // a grid stride that is a multiple of one row's chunks keeps each thread on one head
        const int64_t row_chunks = (int64_t)num_kv_heads * ap.chunks_per_head;
        if (scales_per_head && blocks * kThreads >= row_chunks) {
            int64_t unit = row_chunks;                       // threads per whole number of rows
            while (unit % kThreads) unit += row_chunks;
            const int64_t unit_blocks = unit / kThreads;
            if (unit_blocks <= blocks) blocks = blocks / unit_blocks * unit_blocks;
        }
        if (launch_pdl(pkv::amax_kernel, dim3((unsigned)blocks), dim3(kThreads), sizeof(unsigned int) * n, st,
                       ap) != cudaSuccess)
            return PKV_ERR_CUDA;
    }
    return launch_pdl(pkv::scales_from_amax_kernel, dim3(1), dim3(256), 0, st, scales, n) == cudaSuccess
               ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status paged_kv_cache_write_fp8_scaled(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                                           const int64_t* slot_mapping, int32_t num_tokens,
                                           int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                                           int32_t block_size, const float* k_scales, const float* v_scales,
                                           int32_t scales_per_head, void* stream) {
    const pkv_status v = check_device_scales(k_scales, v_scales, scales_per_head);
    if (v != PKV_OK) return v;
    return cache_write_impl(k_new, v_new, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads, head_dim,
                            num_blocks, block_size, PKV_KV_FP8_E4M3, 1.f, 1.f,
                            DeviceScales{k_scales, v_scales, scales_per_head}, stream);
}

size_t paged_gqa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t max_context_len,
                                       int32_t partition_tokens) {
    if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim != kHeadDim ||
        max_context_len < 0 || partition_tokens < PKV_PARTITION_AUTO)
        return 0;
    auto fixed_size = [&](int32_t P) -> size_t {
        if (P == 0) return 0;
        const int64_t nparts = std::max<int64_t>(1, (max_context_len + P - 1) / P);
        return workspace_layout(batch, num_q_heads, num_kv_heads, nparts).total;
    };
    if (partition_tokens != PKV_PARTITION_AUTO) return fixed_size(partition_tokens);
    // AUTO: the cache type is not an argument, so cover both. Each runs the
    // balanced plan if its tables fit, else the suggested fixed partitions.
    const int64_t max_blocks = std::max(1, (max_context_len + kPageRows - 1) / kPageRows);
    const bool balanced = use_balanced(batch, num_kv_heads, max_blocks);
    const int g16 = balanced ? balanced_grid<false>(batch) : 0;
    const int g8 = balanced ? balanced_grid<true>(batch) : 0;
    size_t need = 0;
    if (g16 > 0) need = std::max(need, balanced_layout((int64_t)g16 * kBalWarpsF16, batch, num_kv_heads).total);
    if (g8 > 0) need = std::max(need, balanced_layout((int64_t)g8 * kBalWarpsFp8, batch, num_kv_heads).total);
    if (g16 <= 0 || g8 <= 0)
        need = std::max(need, fixed_size(paged_gqa_decode_suggest_partition(batch, num_kv_heads, max_context_len,
                                                                            kPageRows, 0)));
    return need;
}

int32_t paged_gqa_decode_suggest_partition(int32_t batch, int32_t num_kv_heads, int32_t max_context_len,
                                           int32_t block_size, int32_t sm_count) {
    if (batch <= 0 || num_kv_heads <= 0 || max_context_len <= 0 || block_size <= 0) return 0;
    if (sm_count <= 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sm_count = 148;
    }
    // Aim for about eight partitions per resident CTA slot (two per SM),
    // assuming contexts spread up to max_context_len (mean about half of it).
    const double work = (double)batch * num_kv_heads * (0.5 * max_context_len);
    const double want = 16.0 * sm_count;
    int32_t P = 128;
    while (P < 4096 && work / (2.0 * P) >= want) P *= 2;
    P = std::max(P, block_size);
    P -= P % block_size;
    if (P >= max_context_len) return 0;
    return P;
}

pkv_status paged_gqa_decode_attention(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, const int32_t* context_lens,
                                      int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                                      int32_t num_blocks, int32_t max_context_len, float softmax_scale,
                                      int32_t kv_dtype, float k_scale, float v_scale,
                                      int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                                      void* stream) {
    return attention_impl(out, q, k_cache, v_cache, block_tables, context_lens, batch, num_q_heads, num_kv_heads,
                          head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
                          kv_dtype, k_scale, v_scale, DeviceScales{}, partition_tokens, workspace,
                          workspace_bytes, stream);
}

pkv_status paged_gqa_decode_attention_fp8_scaled(
    void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks, int32_t max_context_len,
    float softmax_scale, const float* k_scales, const float* v_scales, int32_t scales_per_head,
    int32_t partition_tokens, void* workspace, size_t workspace_bytes, void* stream) {
    const pkv_status v = check_device_scales(k_scales, v_scales, scales_per_head);
    if (v != PKV_OK) return v;
    return attention_impl(out, q, k_cache, v_cache, block_tables, context_lens, batch, num_q_heads, num_kv_heads,
                          head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
                          PKV_KV_FP8_E4M3, 1.f, 1.f, DeviceScales{k_scales, v_scales, scales_per_head},
                          partition_tokens, workspace, workspace_bytes, stream);
}

pkv_status paged_gqa_decode_step(void* out, const void* q, const void* k_new, const void* v_new,
                                 void* k_cache, void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int32_t max_blocks_per_seq, int32_t num_blocks, int32_t max_context_len,
                                 float softmax_scale, int32_t kv_dtype, float k_scale, float v_scale,
                                 void* workspace, size_t workspace_bytes, uint32_t flags, void* stream) {
    return step_impl(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, batch, num_q_heads,
                     num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                     softmax_scale, kv_dtype, k_scale, v_scale, DeviceScales{}, workspace, workspace_bytes,
                     flags, stream);
}

pkv_status paged_gqa_decode_step_fp8_scaled(
    void* out, const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
    int32_t max_context_len, float softmax_scale, const float* k_scales, const float* v_scales,
    int32_t scales_per_head, void* workspace, size_t workspace_bytes, uint32_t flags, void* stream) {
    const pkv_status v = check_device_scales(k_scales, v_scales, scales_per_head);
    if (v != PKV_OK) return v;
    return step_impl(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, batch, num_q_heads,
                     num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                     softmax_scale, PKV_KV_FP8_E4M3, 1.f, 1.f, DeviceScales{k_scales, v_scales, scales_per_head},
                     workspace, workspace_bytes, flags, stream);
}

size_t paged_gqa_prefill_workspace_size(int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                        int32_t kv_dtype) {
    if (num_q_heads <= 0 || num_kv_heads <= 0 || head_dim != kHeadDim || num_q_heads % num_kv_heads != 0 ||
        num_q_heads / num_kv_heads > pkv::kGroupPad || (kv_dtype != PKV_KV_F16 && kv_dtype != PKV_KV_FP8_E4M3))
        return 0;
    if (kv_dtype == PKV_KV_FP8_E4M3) return 0;                  // the warp-level FP8 kernel takes none
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return 0;
    return (size_t)prefill_layout(sms).total;
}

pkv_status paged_gqa_prefill_attention(void* out, const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       const int32_t* query_start, int32_t batch, int32_t total_queries,
                                       int32_t max_query_len, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                                       int32_t num_blocks, int32_t max_context_len, float softmax_scale,
                                       int32_t kv_dtype, float k_scale, float v_scale, void* workspace,
                                       size_t workspace_bytes, void* stream) {
    if (total_queries < 0 || max_query_len < 0) return PKV_ERR_INVALID_ARG;
    const bool any = batch > 0 && total_queries > 0 && max_query_len > 0;
    {
        const pkv_status v = check_attention_args(out, q, k_cache, v_cache, block_tables, context_lens,
                                                  any ? batch : 0, num_q_heads, num_kv_heads, head_dim, block_size,
                                                  max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
                                                  kv_dtype, k_scale, v_scale, 0);
        if (v != PKV_OK || !any) return v;
    }
    if (!query_start || (reinterpret_cast<uintptr_t>(query_start) & 3u)) return PKV_ERR_INVALID_ARG;
    if (max_query_len > max_context_len) return PKV_ERR_INVALID_ARG;
    const bool fp8 = kv_dtype == PKV_KV_FP8_E4M3;
    pkv::PrefillParams prm{};
    prm.out = static_cast<__half*>(out);
    prm.q = static_cast<const __half*>(q);
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.query_start = query_start;
    prm.total = total_queries;
    prm.Hq = num_q_heads;
    prm.Hkv = num_kv_heads;
    prm.G = num_q_heads / num_kv_heads;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.max_context_len = max_context_len;
    prm.max_query_len = max_query_len;
    prm.logit_scale_log2 = softmax_scale * (fp8 ? k_scale : 1.f) * 1.4426950408889634f;
    prm.out_scale = fp8 ? v_scale : 1.f;
    CUtensorMap mk, mv;
    if (!cached_cache_map(&mk, k_cache, fp8, num_blocks, num_kv_heads) ||
        !cached_cache_map(&mv, v_cache, fp8, num_blocks, num_kv_heads))
        return PKV_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!fp8)
        return launch_prefill_tc(prm, mk, mv, max_query_len, num_kv_heads, batch, workspace, workspace_bytes, st);
    // an FP8 cache stays on the warp-level path: tcgen05 kind::f16 takes f16 operands only,
    // and an E4M3 query would not meet the attention tolerance
    const int chunks = (max_query_len + kPrefillConsumers - 1) / kPrefillConsumers;
    return launch_prefill<true>(prm, mk, mv, chunks, num_kv_heads, batch, st);
}

pkv_status fused_add_rmsnorm_qkv_plan(int32_t num_tokens, int32_t hidden, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t* plan) {
    if (!plan || num_tokens <= 0 || hidden <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return PKV_ERR_INVALID_ARG;
    const int64_t N = ((int64_t)num_q_heads + 2 * (int64_t)num_kv_heads) * head_dim;
    if (head_dim % 8 != 0 || hidden % 64 != 0 || hidden > kQkvMaxHidden || N > (1 << 24) ||
        num_tokens > 65535 * 64)
        return PKV_ERR_UNSUPPORTED;
    QkvPlan pl;
    if (!qkv_plan(num_tokens, hidden, (int)N, &pl)) return PKV_ERR_CUDA;
    plan[0] = 128 * pl.acc;
    plan[1] = pl.split;
    plan[2] = pl.tt;
    plan[3] = pl.mtiles * pl.split * pl.ttiles;
    plan[4] = pl.ttiles;
    return PKV_OK;
}

pkv_status fused_add_rmsnorm_qkv(const void* x, const void* residual, const void* gamma, const void* w_qkv,
                                 const void* bias, void* residual_out, void* q, void* k_new, void* v_new,
                                 int32_t num_tokens, int32_t hidden, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, float eps, uint32_t flags, void* stream) {
    if (flags & ~PKV_STEP_OVERLAP_PREVIOUS) return PKV_ERR_INVALID_ARG;
    if (num_tokens < 0 || hidden <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return PKV_ERR_INVALID_ARG;
    if (!(eps >= 0.f && eps <= 3.402823466e38f)) return PKV_ERR_INVALID_ARG;
    // the per-token buffers are empty (possibly null) when there are no tokens
    const void* weights[] = {gamma, w_qkv};
    const void* per_token[] = {x, residual, residual_out, q, k_new, v_new};
    for (const void* ptr : weights)
        if (!ptr || !aligned16(ptr)) return PKV_ERR_INVALID_ARG;
    for (const void* ptr : per_token)
        if ((num_tokens > 0 && !ptr) || !aligned16(ptr)) return PKV_ERR_INVALID_ARG;
    if (bias && !aligned16(bias)) return PKV_ERR_INVALID_ARG;
    const int64_t N = ((int64_t)num_q_heads + 2 * (int64_t)num_kv_heads) * head_dim;
    if (head_dim % 8 != 0 || hidden % 64 != 0 || hidden > kQkvMaxHidden || N > (1 << 24) ||
        num_tokens > 65535 * 64)
        return PKV_ERR_UNSUPPORTED;
    const int64_t T = num_tokens;
    const int64_t act = T * hidden * 2, qb = T * num_q_heads * head_dim * 2, kvb = T * num_kv_heads * head_dim * 2;
    const void* outs[] = {residual_out, q, k_new, v_new};
    const int64_t out_bytes[] = {act, qb, kvb, kvb};
    for (int i = 0; i < 4; ++i) {
        if (ranges_overlap(outs[i], out_bytes[i], x, act) || ranges_overlap(outs[i], out_bytes[i], residual, act))
            return PKV_ERR_INVALID_ARG;
        for (int j = 0; j < i; ++j)
            if (ranges_overlap(outs[i], out_bytes[i], outs[j], out_bytes[j])) return PKV_ERR_INVALID_ARG;
    }
    if (num_tokens == 0) return PKV_OK;
    QkvPlan pl;
    if (!qkv_plan(num_tokens, hidden, (int)N, &pl)) return PKV_ERR_CUDA;
    pkv::QkvParams prm;
    prm.gamma = static_cast<const __half*>(gamma);
    prm.bias = static_cast<const __half*>(bias);
    prm.residual_out = static_cast<__half*>(residual_out);
    prm.q = static_cast<__half*>(q);
    prm.k = static_cast<__half*>(k_new);
    prm.v = static_cast<__half*>(v_new);
    prm.T = num_tokens;
    prm.H = hidden;
    prm.N = (int32_t)N;
    prm.q_cols = num_q_heads * head_dim;
    prm.kv_cols = num_kv_heads * head_dim;
    prm.kblocks = hidden / 64;
    prm.split = pl.split;
    prm.tt = pl.tt;
    prm.stages = pl.stages;
    prm.eps = eps;
    prm.prefetch_w = (flags & PKV_STEP_OVERLAP_PREVIOUS) ? 1 : 0;
    return launch_qkv(pl, prm, w_qkv, x, residual, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------------------------------
// Split-KV scratch owned by the library, for callers that cannot allocate.
// The host name of this array is only a stand-in for it: kernels get its
// device address, looked up once per device below.
static __device__ __align__(256) uint8_t g_static_workspace[PKV_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_static_workspace_addr[kMaxDevices];

// Device address of g_static_workspace on the current device (looked up with
// that device current, once), or nullptr on failure.
void* static_workspace_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = g_static_workspace_addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return nullptr;
    g_static_workspace_addr[dev].store(p, std::memory_order_release);
    return p;
}

}  // namespace

extern "C" pkv_status paged_gqa_decode_attention_static_workspace(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
    int32_t num_blocks, int32_t max_context_len, float softmax_scale, int32_t kv_dtype,
    float k_scale, float v_scale, int32_t partition_tokens, void* stream) {
    const pkv_status v = check_attention_args(out, q, k_cache, v_cache, block_tables, context_lens, batch,
                                              num_q_heads, num_kv_heads, head_dim, block_size,
                                              max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
                                              kv_dtype, k_scale, v_scale, partition_tokens);
    if (v != PKV_OK || batch == 0) return v;
    // The scratch of the plan paged_gqa_decode_attention will run (the same
    // rule it applies): the balanced kernel's piece slots and tickets for
    // PKV_PARTITION_AUTO, the partitions' results and counters for fixed
    // partitions, nothing for a single pass.
    const AttnPlan plan = plan_attention(kv_dtype == PKV_KV_FP8_E4M3, batch, num_q_heads, num_kv_heads,
                                         max_blocks_per_seq, max_context_len, partition_tokens);
    void* ws = nullptr;
    size_t ws_bytes = 0;
    if (plan.ws_bytes > 0) {
        if (plan.ws_bytes > PKV_STATIC_WORKSPACE_BYTES) return PKV_ERR_WORKSPACE;
        ws = static_workspace_address();
        if (!ws) return PKV_ERR_CUDA;
        // the previous call may have left other data where this call's
        // counters go: clear them, in stream order
        if (plan.zero_bytes > 0 &&
            cudaMemsetAsync(static_cast<uint8_t*>(ws) + plan.zero_off, 0, plan.zero_bytes,
                            static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return PKV_ERR_CUDA;
        ws_bytes = PKV_STATIC_WORKSPACE_BYTES;
    }
    return paged_gqa_decode_attention(out, q, k_cache, v_cache, block_tables, context_lens, batch,
                                      num_q_heads, num_kv_heads, head_dim, block_size,
                                      max_blocks_per_seq, num_blocks, max_context_len, softmax_scale,
                                      kv_dtype, k_scale, v_scale, partition_tokens, ws, ws_bytes,
                                      stream);
}
