// grouped.cuh -- multi-token (T > 1) expert FFN grouped by expert.
//
// For a step of T tokens each routed expert is read from memory once and
// applied to every token routed to it (chunked prefill reads one fetched
// expert for many rows: "Gemma 4 26B : Comment faire tourner un LLM en 2 Go
// de RAM", section 04 "Chunked Prefill"); the shared expert is read once for
// all T tokens.  Arithmetic: a 4-bit code is an exact fp32 value, fp16 scales,
// biases and activations are exact in fp32, and every product is accumulated
// in fp32 (per 32-column chunk, then scaled per 64-column group: scale * sum
// code * x + bias * sum x).
//
// Layout of the outputs follows the pair convention of the direct kernels:
// row p < T of h_ws / y_pairs is the shared expert for token p, row T + q the
// routed pair q = t * k + j (token t, routing slot j).
#pragma once
#include "common.cuh"

namespace moeq4 {

constexpr int kGrpTokens = 4;          // tokens per pass of a grouped kernel
constexpr int kGrpThreads = 256;
constexpr int kGrpChunk = 16;          // shared expert: tokens per CTA (grid z splits the step)

// Groups the P routed pairs by expert: e_off[E + 1] (prefix counts) and
// list[P] (pair indices q of expert e at e_off[e] .. e_off[e + 1]).
// "Experts" may be cache slots (idx = slot_of, E = the slot count); with
// sel, only the pairs q with sel[q] == sel_val take part (a batch of a
// streaming chunk).  One CTA.
__global__ void __launch_bounds__(1024) k_group_pairs(const int32_t* __restrict__ idx, int P, int E,
                                                      int* __restrict__ e_off, int* __restrict__ list,
                                                      const int32_t* __restrict__ sel = nullptr,
                                                      int sel_val = 0) {
    __shared__ int cnt[MOE_MAX_EXPERTS + 1];
    const int tid = threadIdx.x;
    for (int e = tid; e <= E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int q = tid; q < P; q += blockDim.x) {
        const int e = idx[q];
        if (e >= 0 && e < E && (!sel || sel[q] == sel_val)) atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int e = 0; e < E; e++) {
            const int c = cnt[e];
            cnt[e] = run;
            e_off[e] = run;
            run += c;
        }
        e_off[E] = run;
    }
    __syncthreads();
    for (int q = tid; q < P; q += blockDim.x) {
        const int e = idx[q];
        if (e >= 0 && e < E && (!sel || sel[q] == sel_val)) list[atomicAdd(&cnt[e], 1)] = q;
    }
}

// Token of the i-th pair of an expert's group (shared expert: token i).
__device__ __forceinline__ int grp_token(bool shared, const int* list, int base, int i, int k) {
    return shared ? i : list[base + i] / k;
}

// Output row of the i-th pair of an expert's group in h_ws / y_pairs.
__device__ __forceinline__ int grp_row(bool shared, const int* list, int base, int i, int T) {
    return shared ? i : T + list[base + i];
}

// Dot products of one 8-column word w: NR rows of 4-bit codes (row r's word
// at sm + rowq[r] + 4 w, its group's fp16 scale and bias at rows[r] / rowb[r]
// + 2 (w / 8)) with kGrpTokens activation rows held as fp32 in shared memory
// (xsf[t * K + column]); accumulates scale * sum(code * x) + bias * sum(x)
// into acc[r][t].  Lanes take consecutive words, so the code reads are
// contiguous across the warp.  A code becomes an exact float through its bit
// pattern (2^23 + q, minus 2^23), which keeps the conversion unit free.
template <int NR>
__device__ __forceinline__ void grp_word(const uint8_t* sm, const uint32_t (&rowq)[NR],
                                         const uint32_t (&rows)[NR], const uint32_t (&rowb)[NR],
                                         const float* xsf, int K, int w,
                                         float (&acc)[NR][kGrpTokens]) {
    float xv[kGrpTokens][8];
    float sx[kGrpTokens];
#pragma unroll
    for (int t = 0; t < kGrpTokens; t++) {
        const float4* xp = reinterpret_cast<const float4*>(xsf + (size_t)t * K + 8 * w);
        const float4 p0 = xp[0], p1 = xp[1];
        xv[t][0] = p0.x; xv[t][1] = p0.y; xv[t][2] = p0.z; xv[t][3] = p0.w;
        xv[t][4] = p1.x; xv[t][5] = p1.y; xv[t][6] = p1.z; xv[t][7] = p1.w;
        sx[t] = ((xv[t][0] + xv[t][1]) + (xv[t][2] + xv[t][3])) +
                ((xv[t][4] + xv[t][5]) + (xv[t][6] + xv[t][7]));
    }
    const uint32_t g2 = 2u * (uint32_t)(w >> 3);
#pragma unroll
    for (int r = 0; r < NR; r++) {
        const uint32_t word = *reinterpret_cast<const uint32_t*>(sm + rowq[r] + 4u * w);
        float d[kGrpTokens];
#pragma unroll
        for (int t = 0; t < kGrpTokens; t++) d[t] = 0.f;
#pragma unroll
        for (int n = 0; n < 8; n++) {
            const float q = __uint_as_float(0x4B000000u | ((word >> (4 * n)) & 0xFu)) - 8388608.0f;
#pragma unroll
            for (int t = 0; t < kGrpTokens; t++) d[t] = fmaf(q, xv[t][n], d[t]);
        }
        const float s = __half2float(*reinterpret_cast<const __half*>(sm + rows[r] + g2));
        const float b = __half2float(*reinterpret_cast<const __half*>(sm + rowb[r] + g2));
#pragma unroll
        for (int t = 0; t < kGrpTokens; t++) acc[r][t] = fmaf(s, d[t], fmaf(b, sx[t], acc[r][t]));
    }
}

// Sum over the 32 lanes of v[0..16): lane l ends with the total of v[l / 2].
__device__ __forceinline__ float grp_reduce16(const float (&v)[16], int lane) {
    float u[16];
#pragma unroll
    for (int i = 0; i < 16; i++) u[i] = v[i];
#pragma unroll
    for (int n = 16, bit = 16; n > 1; n >>= 1, bit >>= 1) {
        const bool upper = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; i++) {
            const float send = upper ? u[i] : u[i + n / 2];
            const float keep = upper ? u[i + n / 2] : u[i];
            u[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
        }
    }
    return u[0] + __shfl_xor_sync(0xffffffffu, u[0], 1);
}

// Copies n16 16-byte words global -> shared with cp.async (all in flight at
// once); the caller waits with cp.async.wait_all and a barrier.
__device__ __forceinline__ void grp_tile_async(void* dst, const void* src, int n16) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    const uint8_t* s = static_cast<const uint8_t*>(src);
    for (int i = threadIdx.x; i < n16; i += blockDim.x)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + 16u * i),
                     "l"(s + 16 * (size_t)i) : "memory");
}

__device__ __forceinline__ void grp_tile_wait() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Token and output row of the pass's pairs g0 .. g0 + kGrpTokens - 1 into
// shared memory (-1 past the end of the group).  Call between barriers.
__device__ __forceinline__ void grp_pass_rows(bool shared, const int* list, int base, int g0, int ng,
                                              int k, int T, int* s_tok, int* s_row) {
    if (threadIdx.x < kGrpTokens) {
        const int t = threadIdx.x;
        const bool v = t < ng;
        s_tok[t] = v ? grp_token(shared, list, base, g0 + t, k) : -1;
        s_row[t] = v ? grp_row(shared, list, base, g0 + t, T) : -1;
    }
}

// fp16 activation rows (x[tok * K ...]) of the pass as fp32 rows of K values
// (zeros for absent tokens): independent 8-byte loads.
__device__ __forceinline__ void grp_stage_half(float* xsf, int K, const __half* x, const int* s_tok) {
    const int q4 = K / 4;
#pragma unroll 4
    for (int i = threadIdx.x; i < kGrpTokens * q4; i += blockDim.x) {
        const int t = i / q4, q = i - t * q4;
        const int tok = s_tok[t];
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (tok >= 0) {
            const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + (size_t)tok * K) + q);
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
            const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
            v = make_float4(a.x, a.y, b.x, b.y);
        }
        reinterpret_cast<float4*>(xsf)[i] = v;
    }
}

// fp32 rows (src[row * stride ...], K values) of the pass: independent 16-byte loads.
__device__ __forceinline__ void grp_stage_float(float* xsf, int K, const float* src, int stride,
                                                const int* s_row) {
    const int q4 = K / 4;
#pragma unroll 4
    for (int i = threadIdx.x; i < kGrpTokens * q4; i += blockDim.x) {
        const int t = i / q4, q = i - t * q4;
        const int row = s_row[t];
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row >= 0) v = __ldcg(reinterpret_cast<const float4*>(src + (size_t)row * stride) + q);
        reinterpret_cast<float4*>(xsf)[i] = v;
    }
}

// Gate/up of one gate/up tile (16 intermediate indices) of one expert for all
// of its tokens (the shared expert: for kGrpChunk tokens, grid z over the
// step's tokens).  grid (Ie / 16, n_experts or 1, 1 or chunks), block 256; dynamic shared
// memory 18 H + kGrpTokens * H * 4 bytes.  Warp w: indices 2w, 2w + 1 (gate
// rows w-pair, up rows w-pair); lane l: 8-column words l, l + 32, ...
// A routed expert whose bucket holds n_cap or more pairs is skipped (the
// tensor-core kernel takes it).
template <bool SHARED>
__global__ void __launch_bounds__(kGrpThreads, 2)
k_gateup_grouped(const uint8_t* __restrict__ experts, size_t stride, const uint8_t* __restrict__ shared_blob,
                 int H, int Ie, const __half* __restrict__ x, int T, int k,
                 const int* __restrict__ e_off, const int* __restrict__ list, int n_cap, int gelu,
                 float* __restrict__ h_ws, int h_stride) {
    extern __shared__ __align__(16) uint8_t gsm[];
    int n = T, base = 0, z0 = 0;
    const uint8_t* blob = shared_blob;
    if (!SHARED) {
        base = e_off[blockIdx.y];
        n = e_off[blockIdx.y + 1] - base;
        if (n == 0 || n >= n_cap) return;                 // empty, or left to the tensor cores
        blob = experts + (size_t)blockIdx.y * stride;
    } else {
        z0 = blockIdx.z * kGrpChunk;                      // this CTA's tokens
        if (z0 >= n) return;
        n = min(n, z0 + kGrpChunk);
    }
    const int tile_bytes = 18 * H;
    grp_tile_async(gsm, blob + (size_t)blockIdx.x * tile_bytes, tile_bytes / 16);
    float* xsf = reinterpret_cast<float*>(gsm + tile_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t rq[4], rs[4], rb[4];
#pragma unroll
    for (int r = 0; r < 4; r++) {
        const int tr = 16 * (r >> 1) + 2 * warp + (r & 1);        // gate 2w, 2w+1, then up
        rq[r] = (uint32_t)tr * (H / 2);
        rs[r] = 16u * H + (uint32_t)tr * (H / 32);
        rb[r] = 17u * H + (uint32_t)tr * (H / 32);
    }
    __shared__ int s_tok[kGrpTokens], s_row[kGrpTokens];
    for (int g0 = z0; g0 < n; g0 += kGrpTokens) {
        const int ng = min(kGrpTokens, n - g0);
        __syncthreads();                                  // previous pass done with xsf
        grp_pass_rows(SHARED, list, base, g0, ng, k, T, s_tok, s_row);
        __syncthreads();
        grp_stage_half(xsf, H, x, s_tok);
        if (g0 == z0) grp_tile_wait();                    // the tile, issued before the first pass
        __syncthreads();
        float acc[4][kGrpTokens];
#pragma unroll
        for (int r = 0; r < 4; r++)
#pragma unroll
            for (int t = 0; t < kGrpTokens; t++) acc[r][t] = 0.f;
        for (int w = lane; w < H / 8; w += 32) grp_word<4>(gsm, rq, rs, rb, xsf, H, w, acc);
        float flat[16];
#pragma unroll
        for (int r = 0; r < 4; r++)
#pragma unroll
            for (int t = 0; t < kGrpTokens; t++) flat[r * kGrpTokens + t] = acc[r][t];
        const float tot = grp_reduce16(flat, lane);       // lane l: element l / 2 = (row, token)
        const float up = __shfl_sync(0xffffffffu, tot, (lane + 4 * kGrpTokens) & 31);
        const int e = lane >> 1;
        if ((lane & 1) == 0 && e < 2 * kGrpTokens) {
            const int r = e / kGrpTokens, t = e - r * kGrpTokens;
            if (t < ng) {
                const int i = 16 * blockIdx.x + 2 * warp + r;
                h_ws[(size_t)s_row[t] * h_stride + i] = gelu_f(tot, gelu) * up;
            }
        }
    }
}

// Down projection of one 16-row down tile of one expert for all of its
// tokens (the shared expert: kGrpChunk tokens per CTA, grid z).  grid
// (H / 16, n_experts or 1, 1 or chunks), block 256; dynamic shared memory
// 9 Ie + kGrpTokens * Ie * 4 bytes.  Warp w: tile rows 2w, 2w + 1; lane l:
// 8-column words l, l + 32, ... of the intermediate.  Routed buckets of n_cap or more
// pairs are skipped, as in the gate/up kernel.
template <bool SHARED>
__global__ void __launch_bounds__(kGrpThreads, 2)
k_down_grouped(const uint8_t* __restrict__ experts, size_t stride, const uint8_t* __restrict__ shared_blob,
               int H, int Ie, int T, const int* __restrict__ e_off, const int* __restrict__ list,
               int n_cap, const float* __restrict__ h_ws, int h_stride, float* __restrict__ y_pairs) {
    extern __shared__ __align__(16) uint8_t gsm[];
    int n = T, base = 0, z0 = 0;
    const uint8_t* blob = shared_blob;
    if (!SHARED) {
        base = e_off[blockIdx.y];
        n = e_off[blockIdx.y + 1] - base;
        if (n == 0 || n >= n_cap) return;                 // empty, or left to the tensor cores
        blob = experts + (size_t)blockIdx.y * stride;
    } else {
        z0 = blockIdx.z * kGrpChunk;                      // this CTA's tokens
        if (z0 >= n) return;
        n = min(n, z0 + kGrpChunk);
    }
    const BlobLayout L(H, Ie);
    const int tile_bytes = 9 * Ie;
    grp_tile_async(gsm, blob + L.dn_base + (size_t)blockIdx.x * tile_bytes, tile_bytes / 16);
    float* hsf = reinterpret_cast<float*>(gsm + tile_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t rq[2], rs[2], rb[2];
#pragma unroll
    for (int r = 0; r < 2; r++) {
        const int tr = 2 * warp + r;
        rq[r] = (uint32_t)tr * (Ie / 2);
        rs[r] = 8u * Ie + (uint32_t)tr * (Ie / 32);
        rb[r] = 8u * Ie + Ie / 2 + (uint32_t)tr * (Ie / 32);
    }
    __shared__ int s_tok[kGrpTokens], s_row[kGrpTokens];
    for (int g0 = z0; g0 < n; g0 += kGrpTokens) {
        const int ng = min(kGrpTokens, n - g0);
        __syncthreads();
        grp_pass_rows(SHARED, list, base, g0, ng, 1, T, s_tok, s_row);
        __syncthreads();
        grp_stage_float(hsf, Ie, h_ws, h_stride, s_row);
        if (g0 == z0) grp_tile_wait();
        __syncthreads();
        float acc[2][kGrpTokens];
#pragma unroll
        for (int r = 0; r < 2; r++)
#pragma unroll
            for (int t = 0; t < kGrpTokens; t++) acc[r][t] = 0.f;
        for (int w = lane; w < Ie / 8; w += 32) grp_word<2>(gsm, rq, rs, rb, hsf, Ie, w, acc);
        float flat[16];
#pragma unroll
        for (int r = 0; r < 2; r++)
#pragma unroll
            for (int t = 0; t < kGrpTokens; t++) {
                flat[r * kGrpTokens + t] = acc[r][t];
                flat[8 + r * kGrpTokens + t] = 0.f;
            }
        const float tot = grp_reduce16(flat, lane);
        const int e = lane >> 1;
        if ((lane & 1) == 0 && e < 2 * kGrpTokens) {
            const int r = e / kGrpTokens, t = e - r * kGrpTokens;
            if (t < ng) y_pairs[(size_t)s_row[t] * H + 16 * blockIdx.x + 2 * warp + r] = tot;
        }
    }
}

}  // namespace moeq4
