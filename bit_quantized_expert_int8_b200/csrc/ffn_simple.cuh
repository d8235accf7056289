// ffn_simple.cuh -- grouped 4-bit expert FFN, direct form.
//
// Gated expert FFN g = Wg x, u = Wu x, h = GELU(g) u, y = Wd h with weights
// stored as 4-bit affine groups ("MLX affine" 4-bit experts: remio.ai
// TurboFieldfare article, "L'affirmation des 2 Go ..."; daily.steinslab
// article, "Trois optimisations cles" item 1).  One warp per output row,
// 128-bit loads of packed codes, fp32 accumulation.  This form serves any
// list of (expert, token) pairs; the single-token layer path uses the fused
// kernel in layer_fused.cuh.
//
// The activation row sits in shared memory chunk-interleaved: element
// 32 j + m of the row at xs[m * nch + j] (nch = K / 32 chunks), so that when
// lane j works on chunk j the 32 lanes of a load read 32 consecutive floats
// (a row-major copy would put every lane of the warp on one bank).
#pragma once
#include "common.cuh"

namespace moeq4 {

// Element c of a K-long row in the chunk-interleaved shared-memory layout.
__device__ __forceinline__ int q4_xs_pos(int c, int K) { return (c & 31) * (K / 32) + (c >> 5); }

// Dot product of one 32-column chunk of a q4 row with x (fp32 in shared
// memory, chunk-interleaved: xs points at the chunk's first element, its
// element m at xs[m * nch]): returns scale * sum(code * x) + bias * sum(x).
__device__ __forceinline__ float q4_chunk_dot(uint4 w, const float* xs, int nch,
                                              float s, float b) {
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    float dq = 0.f, dx = 0.f;
#pragma unroll
    for (int i = 0; i < 4; i++) {
#pragma unroll
        for (int n = 0; n < 8; n++) {
            float xv = xs[(i * 8 + n) * nch];
            dq = fmaf((float)((words[i] >> (4 * n)) & 0xFu), xv, dq);
            dx += xv;
        }
    }
    return fmaf(s, dq, b * dx);
}

// Row r of a q4 matrix with K columns, dotted with the chunk-interleaved
// xs[K] by one warp.
__device__ __forceinline__ float q4_row_dot_warp(const uint8_t* q, const __half* sc,
                                                 const __half* bi, int K, int r,
                                                 const float* xs, int lane) {
    const uint4* row = reinterpret_cast<const uint4*>(q + (size_t)r * (K / 2));
    const __half* srow = sc + (size_t)r * (K / kGroup);
    const __half* brow = bi + (size_t)r * (K / kGroup);
    const int nch = K / 32;
    float acc = 0.f;
    for (int j = lane; j < nch; j += 32) {
        uint4 w = __ldg(row + j);
        int g = j >> 1;
        acc += q4_chunk_dot(w, xs + j, nch, __half2float(srow[g]), __half2float(brow[g]));
    }
    return warp_sum(acc);
}

// grid (ceil(maxI / 8), n_pairs), block 256: warp w of block b computes
// h[p][i] for i = 8b + w.
__global__ void __launch_bounds__(256)
k_ffn_gateup_simple(const MoeFfnPair* __restrict__ pairs, const __half* __restrict__ x,
                    int T, int H, int I_a, int I_b, int gelu, float* __restrict__ h_ws,
                    int h_stride) {
    extern __shared__ float xs[];
    const MoeFfnPair pr = pairs[blockIdx.y];
    const int I = pr.inter;
    // a pair whose size or token is out of range is skipped (never indexed)
    if ((I != I_a && I != I_b) || pr.token < 0 || pr.token >= T) return;
    if ((int)blockIdx.x * 8 >= I) return;
    const __half* xr = x + (size_t)pr.token * H;
    for (int c = threadIdx.x; c < H; c += blockDim.x) xs[q4_xs_pos(c, H)] = __half2float(xr[c]);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * 8 + warp;
    if (i >= I) return;
    const BlobLayout L(H, I);
    const uint8_t* blob = static_cast<const uint8_t*>(pr.blob);
    const float g = q4_row_dot_warp(blob + L.gu_codes(i),
                                    reinterpret_cast<const __half*>(blob + L.gu_scales(i)),
                                    reinterpret_cast<const __half*>(blob + L.gu_biases(i)), H, 0,
                                    xs, lane);
    const float u = q4_row_dot_warp(blob + L.gu_codes(I + i),
                                    reinterpret_cast<const __half*>(blob + L.gu_scales(I + i)),
                                    reinterpret_cast<const __half*>(blob + L.gu_biases(I + i)), H,
                                    0, xs, lane);
    if (lane == 0) h_ws[(size_t)blockIdx.y * h_stride + i] = gelu_f(g, gelu) * u;
}

// grid (H / 8, n_pairs), block 256: warp w of block b computes y[p][8b + w].
__global__ void __launch_bounds__(256)
k_ffn_down_simple(const MoeFfnPair* __restrict__ pairs, const float* __restrict__ h_ws,
                  int h_stride, int H, int I_a, int I_b, float* __restrict__ y) {
    extern __shared__ float hs[];
    const MoeFfnPair pr = pairs[blockIdx.y];
    const int I = pr.inter;
    if (I != I_a && I != I_b) return;
    const float* hr = h_ws + (size_t)blockIdx.y * h_stride;
    for (int c = threadIdx.x; c < I; c += blockDim.x) hs[q4_xs_pos(c, I)] = hr[c];
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + warp;
    if (r >= H) return;
    const BlobLayout L(H, I);
    const uint8_t* blob = static_cast<const uint8_t*>(pr.blob);
    const float v = q4_row_dot_warp(blob + L.dn_codes(r),
                                    reinterpret_cast<const __half*>(blob + L.dn_scales(r)),
                                    reinterpret_cast<const __half*>(blob + L.dn_biases(r)), I, 0,
                                    hs, lane);
    if (lane == 0) y[(size_t)blockIdx.y * H + r] = v;
}

}  // namespace moeq4
