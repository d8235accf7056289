// common.cuh -- small device helpers shared by the kernels of libmoeq4.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moeq4.h"

namespace moeq4 {

constexpr int kGroup = 64;     // weights per quantisation group

// Byte offsets of the six sections of an expert blob (layout in moeq4.h).
struct BlobLayout {
    size_t gu_q, gu_s, gu_b, dn_q, dn_s, dn_b, bytes;
    __host__ __device__ BlobLayout(int H, int I) {
        size_t rows = 2 * (size_t)I;
        gu_q = 0;
        gu_s = gu_q + rows * (size_t)H / 2;
        gu_b = gu_s + rows * (size_t)(H / kGroup) * 2;
        dn_q = gu_b + rows * (size_t)(H / kGroup) * 2;
        dn_s = dn_q + (size_t)H * (size_t)I / 2;
        dn_b = dn_s + (size_t)H * (size_t)(I / kGroup) * 2;
        bytes = dn_b + (size_t)H * (size_t)(I / kGroup) * 2;
    }
};

// fp16 value * 2^24 as an exact integer (|v| < 2^40 for every finite half).
__device__ __forceinline__ long long half_fixed24(__half v) {
    return __float2ll_rn(__half2float(v) * 16777216.0f);
}

// Correctly rounded (nearest-even) conversion of an unsigned 128-bit integer
// to double: keep the top 64 bits with a sticky bit for what was dropped.
__device__ __forceinline__ double u128_to_double_rn(unsigned __int128 v) {
    unsigned long long hi = (unsigned long long)(v >> 64);
    unsigned long long lo = (unsigned long long)v;
    if (hi == 0) return __ull2double_rn(lo);
    int shift = 64 - __clzll((long long)hi);          // 1..64
    unsigned long long top = (unsigned long long)(v >> shift);
    unsigned long long mask = shift == 64 ? ~0ull : ((1ull << shift) - 1);
    top |= (lo & mask) ? 1ull : 0ull;
    return scalbn(__ull2double_rn(top), shift);
}

__device__ __forceinline__ float gelu_f(float g, int variant) {
    if (variant == MOE_GELU_ERF)
        return 0.5f * g * (1.0f + erff(g * 0.70710678118654752f));
    const float k = 0.79788456080286536f;             // sqrt(2/pi)
    return 0.5f * g * (1.0f + tanhf(k * (g + 0.044715f * g * g * g)));
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ unsigned __int128 warp_sum_u128(unsigned __int128 v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        unsigned long long hi = (unsigned long long)(v >> 64);
        unsigned long long lo = (unsigned long long)v;
        hi = __shfl_xor_sync(0xffffffffu, hi, o);
        lo = __shfl_xor_sync(0xffffffffu, lo, o);
        v += ((unsigned __int128)hi << 64) | lo;
    }
    return v;
}

}  // namespace moeq4
