// reshape_and_cache for a paged KV cache [num_blocks, block_size, Hkv, D].
//
// Each step's new key/value vectors ([T, Hkv, D] f16) go to the rows named by
// slot_mapping (block = slot / block_size, row = slot % block_size), in f16 or
// as OCP E4M3 codes with per-tensor or per-KV-head scales. The pages describe the paged
// cache ("rvLLM 소개" (discuss.pytorch.kr), §PagedAttention과 FlashAttention-3)
// but not the write; the slot convention is the one vLLM-style engines use.
//
// One thread moves one 16-byte chunk (8 channels) of K and of V for one
// (token, head): 128-bit coalesced loads and stores, no shared memory. The
// kernel is launch-bound (a 7B-shaped step writes 256 KiB); its grid is the
// number of chunks, in 256-thread blocks.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

struct CacheWriteParams {
    const uint4* k_new;        // [T, Hkv, D] f16, as 16-byte chunks
    const uint4* v_new;
    void* k_cache;             // [NB, bs, Hkv, D] f16 or u8
    void* v_cache;
    const int64_t* slot_mapping;
    int64_t num_slots;         // num_blocks * block_size
    int32_t num_tokens;
    int32_t chunks_per_token;  // Hkv * D / 8
    int32_t chunks_per_head;   // D / 8
    float k_scale, v_scale;    // per-tensor scales, used when k_scales is null
    const float* k_scales;     // device scales: [1] or [Hkv] (scales_per_head)
    const float* v_scales;
    int32_t scales_per_head;
};

// Eight f16 values divided by `scale` in fp32 (IEEE division), rounded to
// nearest even E4M3 with saturation to +-448, as 8 bytes in channel order.
__device__ __forceinline__ uint2 quantize8_e4m3(uint4 x, float scale) {
    const __half2* h = reinterpret_cast<const __half2*>(&x);
    uint32_t out[2];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        uint32_t bytes = 0;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            float2 f = __half22float2(h[2 * w + p]);
            float lo = f.x / scale, hi = f.y / scale;
            uint16_t two;
            // the first source lands in the upper byte
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(hi), "f"(lo));
            bytes |= static_cast<uint32_t>(two) << (16 * p);
        }
        out[w] = bytes;
    }
    return make_uint2(out[0], out[1]);
}

template <bool kFp8>
__global__ void __launch_bounds__(256) cache_write_kernel(CacheWriteParams p) {
    grid_dependency_wait();
    grid_dependents_launch();
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t total = static_cast<int64_t>(p.num_tokens) * p.chunks_per_token;
    if (kFp8 && p.k_scales && idx == 0)
        check_scales(p.k_scales, p.v_scales, p.scales_per_head ? p.chunks_per_token / p.chunks_per_head : 1, 0, 1);
    if (idx >= total) return;
    const int32_t tok = static_cast<int32_t>(idx / p.chunks_per_token);
    const int32_t chunk = static_cast<int32_t>(idx - static_cast<int64_t>(tok) * p.chunks_per_token);
    const int64_t slot = __ldg(p.slot_mapping + tok);
    if (slot < 0) return;                                   // padding token
    if (slot >= p.num_slots) {
        if (chunk == 0) flag_error(PKV_DEVERR_SLOT);
        return;
    }
    const uint4 k = __ldg(p.k_new + idx);
    const uint4 v = __ldg(p.v_new + idx);
    // chunk c of (slot) is at chunk index slot * chunks_per_token + c in both layouts
    const int64_t dst = slot * p.chunks_per_token + chunk;
    if constexpr (kFp8) {
        float ks = p.k_scale, vs = p.v_scale;
        if (p.k_scales) {                                   // device scales of this chunk's head
            const int head = chunk / p.chunks_per_head;
            ks = head_scale(p.k_scales, p.scales_per_head, head);
            vs = head_scale(p.v_scales, p.scales_per_head, head);
        }
        reinterpret_cast<uint2*>(p.k_cache)[dst] = quantize8_e4m3(k, ks);
        reinterpret_cast<uint2*>(p.v_cache)[dst] = quantize8_e4m3(v, vs);
    } else {
        reinterpret_cast<uint4*>(p.k_cache)[dst] = k;
        reinterpret_cast<uint4*>(p.v_cache)[dst] = v;
    }
}

}  // namespace pkv
