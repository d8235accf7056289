// router.cuh -- int8 router GEMV, top-k and softmax.
//
// 8-bit router choosing the top 8 experts: "Gemma 4 26B : Comment faire
// tourner un LLM en 2 Go de RAM", section 04, pipeline step 1; daily.steinslab
// TurboFieldfare article, "L'atout cache des modeles MoE" (8 of 128) and
// "Trois optimisations cles" item 1 (router kept at 8 bits).
//
// Exactness: x (fp16) * 2^24 is an integer X below 2^40, so every product
// with an int8 weight and the whole row sum fit in int64; the sum is exact
// and is rounded once to fp64.  The routing decision therefore does not
// depend on summation order.  X is held as NL balanced base-256 digits
// (X = sum_d digit_d 256^d, digit_d in [-128, 127]; NL covers the token's
// largest |X|), so the row sum is sum_d 256^d (W . digit_d), each inner sum
// formed exactly in int32 by DP4A (at most H * 128 * 128 < 2^31).
#pragma once
#include "common.cuh"

namespace moeq4 {

constexpr int kRouterWarps = 8;          // expert rows per CTA
constexpr int kRouterDigits = 6;         // base-256 digits of |X| < 2^40 (6 * 8 > 40 + sign)

// grid (ceil(E / 8), T), block 256, dynamic shared memory of at least
// kRouterDigits * H bytes.  Each warp forms one logit; the last CTA
// to finish a token selects its top-k and computes the routing weights.
__global__ void __launch_bounds__(256)
k_router(const int8_t* __restrict__ W, const __half* __restrict__ scale,
         const float* __restrict__ bias, const __half* __restrict__ x,
         int E, int H, int k, int renorm, double* __restrict__ logits,
         int* __restrict__ done_counter, int32_t* __restrict__ topk_idx,
         float* __restrict__ topk_w) {
    extern __shared__ __align__(16) uint8_t sDig[];   // [kRouterDigits][H] digits of x * 2^24
    __shared__ unsigned s_mx;
    const int t = blockIdx.y;
    const __half* xr = x + (size_t)t * H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // digits needed for the largest |x| of this token
    if (threadIdx.x == 0) s_mx = 0u;
    __syncthreads();
    float mx = 0.f;
    for (int c = threadIdx.x; c < H; c += blockDim.x) mx = fmaxf(mx, fabsf(__half2float(xr[c])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) atomicMax(&s_mx, __float_as_uint(mx));   // non-negative floats order as integers
    __syncthreads();
    int NL = 1;
    {
        const double xmax = (double)__uint_as_float(s_mx) * 16777216.0;
        double cap = 127.0;                           // largest |X| of NL digits: 127 (256^NL - 1) / 255
        while (NL < kRouterDigits && xmax > cap) { NL++; cap = cap * 256.0 + 127.0; }
    }
    for (int c4 = threadIdx.x; c4 < H / 4; c4 += blockDim.x) {
        uint32_t packed[kRouterDigits];
#pragma unroll
        for (int d = 0; d < kRouterDigits; d++) packed[d] = 0u;
#pragma unroll
        for (int q = 0; q < 4; q++) {
            long long X = __float2ll_rn(__half2float(xr[4 * c4 + q]) * 16777216.0f);   // exact
#pragma unroll
            for (int d = 0; d < kRouterDigits; d++) {
                const int digit = (int)((X + 128) & 255) - 128;
                packed[d] |= (uint32_t)(digit & 255) << (8 * q);
                X = (X - digit) >> 8;
            }
        }
#pragma unroll
        for (int d = 0; d < kRouterDigits; d++)
            if (d < NL) reinterpret_cast<uint32_t*>(sDig + (size_t)d * H)[c4] = packed[d];
    }
    __syncthreads();

    const int e = blockIdx.x * kRouterWarps + warp;
    if (e < E) {
        const int8_t* wr = W + (size_t)e * H;
        int acc[kRouterDigits];
#pragma unroll
        for (int d = 0; d < kRouterDigits; d++) acc[d] = 0;
        for (int c0 = lane * 16; c0 < H; c0 += 32 * 16) {
            const int4 v = *reinterpret_cast<const int4*>(wr + c0);
#pragma unroll
            for (int d = 0; d < kRouterDigits; d++) {
                if (d < NL) {
                    const int4 l = *reinterpret_cast<const int4*>(sDig + (size_t)d * H + c0);
                    acc[d] = __dp4a(v.x, l.x, acc[d]);
                    acc[d] = __dp4a(v.y, l.y, acc[d]);
                    acc[d] = __dp4a(v.z, l.z, acc[d]);
                    acc[d] = __dp4a(v.w, l.w, acc[d]);
                }
            }
        }
        long long S = 0;
#pragma unroll
        for (int d = 0; d < kRouterDigits; d++)
            if (d < NL) S += (long long)warp_sum(acc[d]) * (1ll << (8 * d));
        if (lane == 0) {
            double l = __ll2double_rn(S);
            l = __dmul_rn(l, 0x1p-24);
            l = __dmul_rn(l, (double)__half2float(scale[e]));
            if (bias) l = __dadd_rn(l, (double)bias[e]);
            logits[(size_t)t * E + e] = l;
        }
    }

    // Last CTA of this token does the selection.
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        int prev = atomicAdd(&done_counter[t], 1);
        s_last = (prev == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last || warp != 0) return;
    __threadfence();

    const volatile double* lg = logits + (size_t)t * E;
    constexpr int kPer = MOE_MAX_EXPERTS / 32;        // logits per lane
    double v[kPer];
    bool taken[kPer];
#pragma unroll
    for (int i = 0; i < kPer; i++) {
        int ee = lane + 32 * i;
        v[i] = ee < E ? lg[ee] : 0.0;
        taken[i] = !(ee < E);
    }
    int sel[MOE_MAX_TOPK];
    double sel_l[MOE_MAX_TOPK];
    for (int j = 0; j < k; j++) {
        // lane-local best: largest value, lowest index on ties
        double bv = 0.0;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kPer; i++) {
            int ee = lane + 32 * i;
            if (!taken[i] && (bi == 0x7fffffff || v[i] > bv)) { bv = v[i]; bi = ee; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            double ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            bool better = (oi != 0x7fffffff) &&
                          (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi));
            if (better) { bv = ov; bi = oi; }
        }
        sel[j] = bi;
        sel_l[j] = bv;
        if ((bi & 31) == lane) taken[bi >> 5] = true;
    }
    // softmax over all E logits (fp64), then the selected probabilities
    const double m = sel_l[0];
    double z = 0.0;
#pragma unroll
    for (int i = 0; i < kPer; i++) {
        int ee = lane + 32 * i;
        if (ee < E) z += exp(v[i] - m);
    }
    z = warp_sum(z);
    if (lane == 0) {
        double p[MOE_MAX_TOPK], zs = 0.0;
        for (int j = 0; j < k; j++) { p[j] = exp(sel_l[j] - m) / z; zs += p[j]; }
        for (int j = 0; j < k; j++) {
            topk_idx[(size_t)t * k + j] = sel[j];
            topk_w[(size_t)t * k + j] = (float)(renorm ? p[j] / zs : p[j]);
        }
        done_counter[t] = 0;                          // ready for the next launch
    }
}

}  // namespace moeq4
