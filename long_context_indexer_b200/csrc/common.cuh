// common.cuh -- small device helpers shared by the lci kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lci {

// Sticky device status word: bit flags, set with atomicOr, read and cleared
// by lci_get_device_status. The library is one translation unit (lci.cu
// includes every kernel header), so this is its only definition.
__device__ unsigned int g_device_status = 0u;

enum : unsigned int {
    kStatusBadBlockId = 1u << 0,  // block id outside [-1, nb_max)
    kStatusBadPage = 1u << 1,     // table entry outside [0, num_pages)
    kStatusTimeout = 1u << 2,     // a bounded device wait gave up
};

// A published (block id << 32 | page) pick not yet written: both INT_MIN.
constexpr unsigned long long kPickPending = 0x8000000080000000ull;

// Limit of every bounded device wait, in nanoseconds of global time. Set from
// the host (lci_set_wait_limit_ns) between launches; 2 s unless changed.
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;

__device__ __forceinline__ void raise_status(unsigned int bits) {
    atomicOr(&g_device_status, bits);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Order-preserving map of an fp32 score onto uint32: a > b  <=>  key(a) > key(b).
// -0.0 is folded onto +0.0 first so that equal scores give equal keys.
__device__ __forceinline__ uint32_t score_key(float s) {
    s = s + 0.0f;
    uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Causal-visible block count for a query at absolute position p.
__device__ __forceinline__ int visible_blocks(long long p, long long ctx, int bs, int nb_max) {
    long long last = p < ctx - 1 ? p : ctx - 1;
    if (last < 0) return 0;
    long long v = last / bs + 1;
    return (int)(v < nb_max ? v : nb_max);
}

__device__ __forceinline__ float2 bf16x2_to_f32(uint32_t w) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w);
    return __bfloat1622float2(h);
}

}  // namespace lci
