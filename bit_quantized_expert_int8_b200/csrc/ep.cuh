// ep.cuh -- expert-parallel dispatch over ranks (experts partitioned, rank r
// owning experts r * epr .. r * epr + epr - 1).
//
// A rank's T tokens choose k experts each; every (token, expert) pair is sent
// to the rank that owns the expert, which applies the expert and sends the
// row back.  These kernels are the device side of one rank's step: sort the
// pairs by destination (stable in pair order), pack the x rows to send, and
// put the returned rows back in pair order for the combine.  The exchange
// itself is two all-to-alls between the kernels (the host owns them).
#pragma once
#include "common.cuh"

namespace moeq4 {

// One CTA, one warp per destination rank (n_ranks <= 32): counts[d] pairs go
// to rank d; order[pos] is the pair index q (= t * k + j) at send position
// pos, destinations in rank order, pairs in index order within each.  An
// expert index outside [0, E) sets *status to MOE_ERR_INVALID_ARG and the
// pair is not sent.
__global__ void k_ep_plan(const int32_t* __restrict__ idx, int P, int E, int epr, int n_ranks,
                          int32_t* __restrict__ counts, int32_t* __restrict__ order,
                          int* __restrict__ status) {
    __shared__ int s_off[33];
    const int d = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int cnt = 0;
    for (int q0 = 0; q0 < P; q0 += 32) {
        const int q = q0 + lane;
        const int e = q < P ? idx[q] : 0;
        if (d == 0 && q < P && (e < 0 || e >= E)) atomicExch(status, MOE_ERR_INVALID_ARG);
        const bool mine = q < P && e >= 0 && e < E && e / epr == d;
        cnt += __popc(__ballot_sync(0xffffffffu, mine));
    }
    if (lane == 0) s_off[d + 1] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        s_off[0] = 0;
        for (int r = 0; r < n_ranks; r++) {
            counts[r] = s_off[r + 1];
            s_off[r + 1] += s_off[r];
        }
    }
    __syncthreads();
    int run = s_off[d];
    for (int q0 = 0; q0 < P; q0 += 32) {
        const int q = q0 + lane;
        const int e = q < P ? idx[q] : 0;
        const bool mine = q < P && e >= 0 && e < E && e / epr == d;
        const unsigned b = __ballot_sync(0xffffffffu, mine);
        if (mine) order[run + __popc(b & ((1u << lane) - 1u))] = q;
        run += __popc(b);
    }
}

// Send rows: send_x[pos] = x[order[pos] / k], send_expert[pos] = the expert's
// index at its owner.  grid (ceil(n / 8)), block 256: one warp per row.
__global__ void k_ep_gather(const __half* __restrict__ x, const int32_t* __restrict__ idx,
                            const int32_t* __restrict__ order, int n, int k, int H, int epr,
                            __half* __restrict__ send_x, int32_t* __restrict__ send_expert) {
    const int pos = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (pos >= n) return;
    const int q = order[pos];
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(q / k) * H);
    uint4* dst = reinterpret_cast<uint4*>(send_x + (size_t)pos * H);
    for (int c = lane; c < H / 8; c += 32) dst[c] = src[c];
    if (lane == 0) send_expert[pos] = idx[q] % epr;
}

// Returned rows back in pair order: y_pairs[order[pos]] = y_sorted[pos].
// grid (ceil(n / 8)), block 256: one warp per row.
__global__ void k_ep_unpermute(const float* __restrict__ y_sorted, const int32_t* __restrict__ order,
                               int n, int H, float* __restrict__ y_pairs) {
    const int pos = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (pos >= n) return;
    const float4* src = reinterpret_cast<const float4*>(y_sorted + (size_t)pos * H);
    float4* dst = reinterpret_cast<float4*>(y_pairs + (size_t)order[pos] * H);
    for (int c = lane; c < H / 4; c += 32) dst[c] = src[c];
}

}  // namespace moeq4
