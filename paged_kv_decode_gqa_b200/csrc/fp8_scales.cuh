// E4M3 cache scales computed from data, on the device.
//
// The pages name an FP8 E4M3 KV cache ("rvLLM 소개" (discuss.pytorch.kr),
// §PagedAttention과 FlashAttention-3) and say nothing of its scales. The
// library's reading: a scale maps the largest magnitude of the data onto the
// largest finite E4M3 value, scale = amax / 448 in fp32 (1 when amax is 0),
// with amax taken over the non-NaN elements of each KV head or of the whole
// tensor. Doing it on the device lets a step be calibrated and replayed from a
// CUDA graph without a host round trip.
//
// amax_kernel streams x [rows, Hkv, D] f16 once in 16-byte chunks (HBM
// bound). The grid stride is a multiple of one row's chunks whenever the grid
// allows it, so a thread meets one KV head only and keeps its running maximum
// in a register; block maxima meet in shared memory, and one atomicMax per
// block and head on the fp32 bit pattern (non-negative floats order like their
// bits) combines the blocks. scales_from_amax_kernel then turns the maxima
// into scales in place.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

struct AmaxParams {
    const uint4* x;            // [rows, Hkv, D] f16 as 16-byte chunks
    int64_t chunks;            // rows * Hkv * D / 8
    int32_t chunks_per_head;   // D / 8
    int32_t Hkv;
    int32_t per_head;          // 1: one maximum per KV head; 0: one overall
    unsigned int* amax_bits;   // [per_head ? Hkv : 1], zero before the launch
};

__global__ void __launch_bounds__(256) amax_kernel(AmaxParams p) {
    extern __shared__ unsigned int s_max[];  // [per_head ? Hkv : 1]
    const int n = p.per_head ? p.Hkv : 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x) s_max[i] = 0u;
    grid_dependency_wait();
    grid_dependents_launch();
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int head = -1;
    float m = 0.f;
    auto fold = [&](int64_t c, const uint4& v) {
        const int h = p.per_head ? (int)((c / p.chunks_per_head) % p.Hkv) : 0;
        if (h != head) {                      // a new head for this thread: flush the old one
            if (head >= 0) atomicMax(&s_max[head], __float_as_uint(m));
            head = h;
            m = 0.f;
        }
        const __half2* h2 = reinterpret_cast<const __half2*>(&v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(h2[k]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));   // fmaxf ignores a NaN operand
        }
    };
    // four independent 16-byte loads in flight per thread, then their maxima
    constexpr int kUnroll = 4;
    int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; c + (kUnroll - 1) * stride < p.chunks; c += kUnroll * stride) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) v[u] = ld_stream_16(p.x + c + u * stride);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) fold(c + u * stride, v[u]);
    }
    for (; c < p.chunks; c += stride) fold(c, ld_stream_16(p.x + c));
    if (head >= 0) atomicMax(&s_max[head], __float_as_uint(m));
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        if (s_max[i]) atomicMax(p.amax_bits + i, s_max[i]);
}

// scales[i] = amax_i / 448 (IEEE fp32 division), or 1 when amax_i is 0; the
// maxima are read from the same words as fp32 bit patterns.
__global__ void __launch_bounds__(256) scales_from_amax_kernel(float* scales, int n) {
    grid_dependency_wait();
    grid_dependents_launch();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const float a = __uint_as_float(reinterpret_cast<const unsigned int*>(scales)[i]);
        scales[i] = a > 0.f ? a / 448.f : 1.f;
    }
}

}  // namespace pkv
