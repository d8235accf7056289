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

// Digits needed for a token whose largest |x| is xmax_f (X = x * 2^24).
__device__ __forceinline__ int router_ndigits(float xmax_f) {
    int NL = 1;
    const double xmax = (double)xmax_f * 16777216.0;
    double cap = 127.0;                               // largest |X| of NL digits: 127 (256^NL - 1) / 255
    while (NL < kRouterDigits && xmax > cap) { NL++; cap = cap * 256.0 + 127.0; }
    return NL;
}

// Four consecutive values of x (columns 4 c4 ..) as NL packed digit words:
// digit d of X = x * 2^24 (balanced base 256) of value q in byte q of word d.
__device__ __forceinline__ void router_digits4(const __half* xr, int c4, int NL, uint8_t* dig, int H) {
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
        if (d < NL) reinterpret_cast<uint32_t*>(dig + (size_t)d * H)[c4] = packed[d];
}

// Logit of expert e from its exact integer row sum S = sum_c W[e][c] X[c].
__device__ __forceinline__ double router_logit(long long S, const __half* scale, const float* bias, int e) {
    double l = __ll2double_rn(S);
    l = __dmul_rn(l, 0x1p-24);
    l = __dmul_rn(l, (double)__half2float(scale[e]));
    if (bias) l = __dadd_rn(l, (double)bias[e]);
    return l;
}

// Top-k of one token's E logits by one warp (largest value, lowest index on
// ties), then the softmax over all E logits in fp64 and the selected
// probabilities (renormalised over the k when renorm).
template <typename LP>
__device__ __forceinline__ void router_select(LP lg, int E, int k, int renorm, int lane,
                                              int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
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
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; j++) {
        if (j >= k) break;
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
#pragma unroll
        for (int i = 0; i < kPer; i++)
            if (bi == lane + 32 * i) taken[i] = true;
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
    // lane j < k forms p_j; every lane sums them in selection order
    double lj = 0.0;
    int ij = 0;
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; j++)
        if (j == lane) { lj = sel_l[j]; ij = sel[j]; }
    const double pj = lane < k ? exp(lj - m) / z : 0.0;
    double zs = 0.0;
    for (int j = 0; j < k; j++) zs += __shfl_sync(0xffffffffu, pj, j);
    if (lane < k) {
        topk_idx[lane] = ij;
        topk_w[lane] = (float)(renorm ? pj / zs : pj);
    }
}

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
    const int NL = router_ndigits(__uint_as_float(s_mx));
    for (int c4 = threadIdx.x; c4 < H / 4; c4 += blockDim.x) router_digits4(xr, c4, NL, sDig, H);
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
        if (lane == 0) logits[(size_t)t * E + e] = router_logit(S, scale, bias, e);
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
    router_select(lg, E, k, renorm, lane, topk_idx + (size_t)t * k, topk_w + (size_t)t * k);
    if (lane == 0) {
        done_counter[t] = 0;                          // ready for the next launch
    }
}

// Steps of many tokens: CTA (token pair, block of eper experts).  The pair's x
// rows come into shared memory with one pass; their digits are formed there;
// each warp takes two expert rows of the block (lanes read consecutive
// 16-byte chunks, several in flight) and reduces its digit sums across the
// lanes.  The last CTA of a pair (a counter per pair) selects its tokens'
// experts.  The arithmetic (digits, exact integer row sums, fp64 logits,
// selection) is that of k_router, so the two kernels choose the same experts
// with the same weights.  grid (ceil(T / 2), ceil(E / eper)), eper a multiple
// of 32 (the host picks it so that the grid stays within one wave of CTAs:
// every CTA forms its pair's digits, so more blocks than SMs cost a second
// round of that), block kRouterBatchThreads, dynamic shared memory
// router_batch_smem(2, H, E).
constexpr int kRouterBatchThreads = 512;
constexpr int kRouterBatchExperts = 32;     // expert rows per CTA and pass (two per warp)
constexpr int kRouterBatchMinTokens = 40;   // steps from which the batched router runs (measured)
__host__ __device__ constexpr size_t router_batch_smem(int TB, int H, int E) {
    return (size_t)TB * kRouterDigits * H + (size_t)TB * H * 2;
}
template <int TB>
__global__ void __launch_bounds__(kRouterBatchThreads)
k_router_batch(const int8_t* __restrict__ W, const __half* __restrict__ scale,
               const float* __restrict__ bias, const __half* __restrict__ x, int T, int E, int H,
               int k, int renorm, int eper, double* __restrict__ logits,
               int* __restrict__ done_counter, int32_t* __restrict__ topk_idx,
               float* __restrict__ topk_w) {
    extern __shared__ __align__(16) uint8_t sDig[];   // [TB][kRouterDigits][H], then x [TB][H]
    __half* sx = reinterpret_cast<__half*>(sDig + (size_t)TB * kRouterDigits * H);
    __shared__ unsigned s_mx[TB];
    __shared__ int s_last;
    const int t0 = blockIdx.x * TB, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = min(TB, T - t0);
    if (tid < TB) s_mx[tid] = 0u;
    // the pair's rows, one 16-byte load per chunk
    for (int i = tid; i < nt * (H / 8); i += blockDim.x) {
        const int t = i / (H / 8), c = i % (H / 8);
        reinterpret_cast<uint4*>(sx + (size_t)t * H)[c] = reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * H)[c];
    }
    __syncthreads();
    for (int t = 0; t < nt; t++) {
        float mx = 0.f;
        for (int c = tid; c < H; c += blockDim.x) mx = fmaxf(mx, fabsf(__half2float(sx[(size_t)t * H + c])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) atomicMax(&s_mx[t], __float_as_uint(mx));
    }
    __syncthreads();
    int NL[TB];
#pragma unroll
    for (int t = 0; t < TB; t++) NL[t] = t < nt ? router_ndigits(__uint_as_float(s_mx[t])) : 0;
    for (int t = 0; t < nt; t++)
        for (int c4 = tid; c4 < H / 4; c4 += blockDim.x)
            router_digits4(sx + (size_t)t * H, c4, NL[t], sDig + (size_t)t * kRouterDigits * H, H);
    __syncthreads();
    // two expert rows per warp, up to 6 chunks of 16 bytes per lane and row in
    // flight before their dot products
    constexpr int kCh = 6;
    const int eb = blockIdx.y * eper, ee = min(E, eb + eper);
    for (int e0 = eb + 2 * warp; e0 < ee; e0 += 2 * (kRouterBatchThreads / 32)) {
        const bool two = e0 + 1 < ee;
        const int8_t* wr0 = W + (size_t)e0 * H;
        const int8_t* wr1 = W + (size_t)(two ? e0 + 1 : e0) * H;
        int acc[2][TB][kRouterDigits];
#pragma unroll
        for (int r = 0; r < 2; r++)
#pragma unroll
            for (int t = 0; t < TB; t++)
#pragma unroll
                for (int d = 0; d < kRouterDigits; d++) acc[r][t][d] = 0;
        for (int cb = lane * 16; cb < H; cb += kCh * 32 * 16) {
            int4 w[2][kCh];
#pragma unroll
            for (int i = 0; i < kCh; i++) {
                const int c0 = cb + i * 32 * 16;
                if (c0 < H) {
                    w[0][i] = *reinterpret_cast<const int4*>(wr0 + c0);
                    w[1][i] = *reinterpret_cast<const int4*>(wr1 + c0);
                }
            }
#pragma unroll
            for (int i = 0; i < kCh; i++) {
                const int c0 = cb + i * 32 * 16;
                if (c0 < H) {
#pragma unroll
                    for (int t = 0; t < TB; t++) {
#pragma unroll
                        for (int d = 0; d < kRouterDigits; d++) {
                            if (d < NL[t]) {
                                const int4 l = *reinterpret_cast<const int4*>(
                                    sDig + ((size_t)t * kRouterDigits + d) * H + c0);
#pragma unroll
                                for (int r = 0; r < 2; r++) {
                                    acc[r][t][d] = __dp4a(w[r][i].x, l.x, acc[r][t][d]);
                                    acc[r][t][d] = __dp4a(w[r][i].y, l.y, acc[r][t][d]);
                                    acc[r][t][d] = __dp4a(w[r][i].z, l.z, acc[r][t][d]);
                                    acc[r][t][d] = __dp4a(w[r][i].w, l.w, acc[r][t][d]);
                                }
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 2; r++) {
            if (r == 1 && !two) break;
            const int e = e0 + r;
#pragma unroll
            for (int t = 0; t < TB; t++) {
                if (t < nt) {
                    long long S = 0;
#pragma unroll
                    for (int d = 0; d < kRouterDigits; d++)
                        if (d < NL[t]) S += (long long)warp_sum(acc[r][t][d]) * (1ll << (8 * d));
                    if (lane == 0) logits[(size_t)(t0 + t) * E + e] = router_logit(S, scale, bias, e);
                }
            }
        }
    }
    // the last CTA of this token pair selects
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int prev = atomicAdd(&done_counter[blockIdx.x], 1);
        s_last = prev == (int)gridDim.y - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (warp < nt) {
        const volatile double* lg = logits + (size_t)(t0 + warp) * E;
        router_select(lg, E, k, renorm, lane, topk_idx + (size_t)(t0 + warp) * k,
                      topk_w + (size_t)(t0 + warp) * k);
    }
    if (tid == 0) done_counter[blockIdx.x] = 0;       // ready for the next launch
}

}  // namespace moeq4
