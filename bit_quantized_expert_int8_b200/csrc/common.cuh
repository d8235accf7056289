// common.cuh -- small device helpers shared by the kernels of libmoeq4.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moeq4.h"

namespace moeq4 {

constexpr int kGroup = 64;     // weights per quantisation group

// Tiled expert blob (layout in moeq4.h): I/16 gate/up tiles of 18 H bytes
// (gate codes [16][H/8] u32, up codes [16][H/8], gate scales [16][H/64]
// fp16, up scales, gate biases, up biases), then H/16 down tiles of 9 I
// bytes (codes [16][I/8] u32, scales [16][I/64] fp16, biases).  Byte offsets
// of one row's codes, scales and biases.
struct BlobLayout {
    int H, I;
    size_t gu_tile, dn_base, dn_tile, bytes;
    __host__ __device__ BlobLayout(int H_, int I_) : H(H_), I(I_) {
        gu_tile = 18 * (size_t)H;
        dn_base = (size_t)(I / 16) * gu_tile;
        dn_tile = 9 * (size_t)I;
        bytes = dn_base + (size_t)(H / 16) * dn_tile;
    }
    // row r of the gate/up matrix: gate rows 0..I-1, up rows I..2I-1
    __host__ __device__ size_t gu_row(int r) const {      // 16 * up + position in the tile
        const int up = r >= I ? 1 : 0, i = r - up * I;
        return (size_t)(16 * up + i % 16);
    }
    __host__ __device__ size_t gu_base(int r) const {
        const int i = r >= I ? r - I : r;
        return (size_t)(i / 16) * gu_tile;
    }
    __host__ __device__ size_t gu_codes(int r) const { return gu_base(r) + gu_row(r) * (H / 2); }
    __host__ __device__ size_t gu_scales(int r) const {
        return gu_base(r) + 16 * (size_t)H + gu_row(r) * (H / 32);
    }
    __host__ __device__ size_t gu_biases(int r) const {
        return gu_base(r) + 17 * (size_t)H + gu_row(r) * (H / 32);
    }
    // row r of the down matrix
    __host__ __device__ size_t dn_codes(int r) const {
        return dn_base + (size_t)(r / 16) * dn_tile + (size_t)(r % 16) * (I / 2);
    }
    __host__ __device__ size_t dn_scales(int r) const {
        return dn_base + (size_t)(r / 16) * dn_tile + 8 * (size_t)I + (size_t)(r % 16) * (I / 32);
    }
    __host__ __device__ size_t dn_biases(int r) const {
        return dn_base + (size_t)(r / 16) * dn_tile + 17 * (size_t)I / 2 + (size_t)(r % 16) * (I / 32);
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
