// misc.cuh -- RMSNorm, combine, LFU cache lookup and small glue kernels.
#pragma once
#include "common.cuh"

namespace moeq4 {

// ------------------------------------------------------------- RMSNorm --
// Unit-weight RMSNorm between layers (a RMSNorm kernel is among the engine's
// kernels: devtrends.cc article, "Geen afhankelijkheden van llama.cpp en
// MLX").  x = fp16(h / sqrt(mean(h^2) + eps)).  The sum of squares is exact
// (fp16 * 2^24 is an integer below 2^40; squares summed in 128 bits) and is
// rounded once to fp64, so the fp16 result does not depend on the reduction
// order.  grid T, block 256.
__global__ void __launch_bounds__(256)
k_rmsnorm(const __half* __restrict__ h, __half* __restrict__ x, int H, double eps) {
    const __half* hr = h + (size_t)blockIdx.x * H;
    __half* xr = x + (size_t)blockIdx.x * H;
    unsigned __int128 acc = 0;
    for (int c = threadIdx.x; c < H; c += blockDim.x) {
        long long X = half_fixed24(hr[c]);
        acc += (unsigned __int128)((__int128)X * (__int128)X);
    }
    acc = warp_sum_u128(acc);
    __shared__ unsigned long long s_hi[8], s_lo[8];
    __shared__ double s_r;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) { s_hi[warp] = (unsigned long long)(acc >> 64); s_lo[warp] = (unsigned long long)acc; }
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned __int128 tot = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++)
            tot += ((unsigned __int128)s_hi[w] << 64) | s_lo[w];
        double s = __dmul_rn(u128_to_double_rn(tot), 0x1p-48);
        double ms = __ddiv_rn(s, (double)H);
        s_r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, eps)));
    }
    __syncthreads();
    const double r = s_r;
    for (int c = threadIdx.x; c < H; c += blockDim.x)
        xr[c] = __double2half(__dmul_rn((double)__half2float(hr[c]), r));
}

// ------------------------------------------------------------- combine --
// y = y_shared + sum_j w_j y_routed[j] (j in order, fp32): the shared and
// routed branch outputs combine ("Gemma 4 26B : Comment faire tourner un LLM
// en 2 Go de RAM", "Concurrence pour masquer la latence").  Optional fp16
// residual update h <- fp16(h + y).  grid (ceil(H/256), T), block 256.
__global__ void __launch_bounds__(256)
k_combine(const float* __restrict__ y_routed, size_t routed_tok_stride,
          const float* __restrict__ y_shared, size_t shared_tok_stride,
          const float* __restrict__ w, int k, int H, float* __restrict__ y_out,
          __half* __restrict__ residual) {
    const int t = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= H) return;
    float acc = y_shared[(size_t)t * shared_tok_stride + c];
    const float* yr = y_routed + (size_t)t * routed_tok_stride;
    for (int j = 0; j < k; j++) acc = fmaf(w[(size_t)t * k + j], yr[(size_t)j * H + c], acc);
    y_out[(size_t)t * H + c] = acc;
    if (residual) {
        __half* hp = residual + (size_t)t * H + c;
        *hp = __float2half_rn(__half2float(*hp) + acc);
    }
}

// ----------------------------------------------------------------- LFU --
// One layer's 16-slot LFU expert cache ("daily.steinslab" TurboFieldfare
// article, "Trois optimisations cles" item 3; remio.ai article, "Mac Gemma 4
// 26B tient en memoire ..."): hits first in ascending expert order, then each
// miss in ascending order takes the lowest empty slot, else the slot unused by
// this token with the lowest count, ties to the oldest insertion.  The table
// is tiny and the walk is sequential: one thread.  grid 1, block 32.
// An invalid table (an earlier fill failed) changes nothing: n_miss = -1,
// slot_of is set to slot 0 (a valid index, so later kernels stay in bounds)
// and, when status is given, MOE_ERR_CACHE_STATE is recorded there.
__global__ void k_lfu_lookup(MoeLfuTable* __restrict__ tb, const int32_t* __restrict__ idx,
                             int T, int k, int32_t* __restrict__ slot_of,
                             int32_t* __restrict__ miss_list, int32_t* __restrict__ n_miss,
                             int* __restrict__ status = nullptr) {
    if (threadIdx.x != 0) return;
    if (!tb->valid) {
        for (int i = 0; i < T * k; i++) slot_of[i] = 0;
        if (status) atomicCAS(status, 0, MOE_ERR_CACHE_STATE);
        __threadfence_system();
        *n_miss = -1;
        return;
    }
    const int S = tb->n_slots;
    int nm = 0;
    for (int t = 0; t < T; t++) {
        const int32_t* it = idx + (size_t)t * k;
        int ord[MOE_MAX_TOPK];
        for (int j = 0; j < k; j++) ord[j] = j;
        for (int a = 1; a < k; a++)              // sort positions by expert id
            for (int b = a; b > 0 && it[ord[b - 1]] > it[ord[b]]; b--) {
                int tmp = ord[b]; ord[b] = ord[b - 1]; ord[b - 1] = tmp;
            }
        uint32_t used = 0;                       // bit s: slot used by this token
        uint32_t hitmask = 0;                    // bit j: idx j was a hit
        for (int a = 0; a < k; a++) {
            int j = ord[a];
            for (int s = 0; s < S; s++)
                if (tb->expert[s] == it[j]) {
                    tb->count[s] += 1;
                    used |= 1u << s;
                    hitmask |= 1u << j;
                    slot_of[(size_t)t * k + j] = s;
                    tb->hits += 1;
                    break;
                }
        }
        for (int a = 0; a < k; a++) {
            int j = ord[a];
            if (hitmask & (1u << j)) continue;
            int v = -1;
            for (int s = 0; s < S && v < 0; s++)
                if (tb->expert[s] < 0) v = s;
            if (v < 0)
                for (int s = 0; s < S; s++) {
                    if (used & (1u << s)) continue;
                    if (v < 0 || tb->count[s] < tb->count[v] ||
                        (tb->count[s] == tb->count[v] && tb->seq[s] < tb->seq[v]))
                        v = s;
                }
            // top_k < n_slots guarantees a victim (checked on the host)
            tb->counter += 1;
            tb->expert[v] = it[j];
            tb->count[v] = 1;
            tb->seq[v] = tb->counter;
            used |= 1u << v;
            slot_of[(size_t)t * k + j] = v;
            miss_list[2 * nm] = it[j];
            miss_list[2 * nm + 1] = v;
            nm++;
            tb->misses += 1;
        }
    }
    __threadfence_system();
    *n_miss = nm;
}

// LFU lookup of a chunk of tokens (chunked prefill: "Gemma 4 26B : Comment
// faire tourner un LLM en 2 Go de RAM", section 04 "Chunked Prefill" -- one
// expert fetched into the cache serves every row of the chunk that uses it).
// The per-token rule of k_lfu_lookup applied to the chunk's distinct experts,
// each weighted by its uses, served in batches that fit the slots:
//   - the distinct experts in ascending id order: a resident one is a hit,
//     its count grows by its number of (token, choice) pairs, and its slot
//     is pinned to batch 0;
//   - then each missing one takes the lowest empty slot, else, among the
//     slots not pinned by the current batch, the lowest count, ties to the
//     oldest insertion; when every slot is pinned the next batch starts with
//     no slot pinned; the newcomer starts at its number of uses;
//   - hits and misses count distinct experts (a miss is one copy).
// Outputs: slot_of and batch_of [n_tok][k] (device), and in `plan` (ints,
// mapped host memory) the number of batches nb, then nb + 1 offsets and nb
// counts into the miss list, then the misses as (expert, slot) pairs in
// insertion order (batch by batch): plan = [nb, off[0..max_b], cnt[0..max_b),
// pairs...] with max_b = n_experts + 1.  An invalid table gives nb = -1, slot
// 0 everywhere and MOE_ERR_CACHE_STATE in the status word.  One thread.
__global__ void k_lfu_chunk(MoeLfuTable* __restrict__ tb, const int32_t* __restrict__ idx, int n_tok,
                            int k, int n_experts, int32_t* __restrict__ slot_of,
                            int32_t* __restrict__ batch_of, int32_t* __restrict__ plan,
                            int* __restrict__ status) {
    if (threadIdx.x != 0) return;
    const int P = n_tok * k, max_b = n_experts + 1;
    int32_t* off = plan + 1;
    int32_t* cnt = off + max_b + 1;
    int32_t* pairs = cnt + max_b;
    if (!tb->valid) {
        for (int q = 0; q < P; q++) { slot_of[q] = 0; batch_of[q] = 0; }
        if (status) atomicCAS(status, 0, MOE_ERR_CACHE_STATE);
        __threadfence_system();
        plan[0] = -1;
        return;
    }
    const int S = tb->n_slots;
    // uses per expert id (n_experts <= MOE_MAX_EXPERTS), then slot and batch per id
    int uses[MOE_MAX_EXPERTS], where[MOE_MAX_EXPERTS], bat[MOE_MAX_EXPERTS];
    for (int e = 0; e < n_experts; e++) { uses[e] = 0; where[e] = -1; bat[e] = 0; }
    for (int q = 0; q < P; q++) {
        const int e = idx[q];
        if (e < 0 || e >= n_experts) {           // not a routing: refuse the chunk
            for (int r = 0; r < P; r++) { slot_of[r] = 0; batch_of[r] = 0; }
            if (status) atomicCAS(status, 0, MOE_ERR_CACHE_STATE);
            __threadfence_system();
            plan[0] = -1;
            return;
        }
        uses[e] += 1;
    }
    uint32_t pinned = 0;
    for (int e = 0; e < n_experts; e++) {
        if (!uses[e]) continue;
        for (int s = 0; s < S; s++)
            if (tb->expert[s] == e) {
                tb->count[s] += uses[e];
                pinned |= 1u << s;
                where[e] = s;
                tb->hits += 1;
                break;
            }
    }
    int batch = 0, nm = 0;
    off[0] = 0;
    for (int e = 0; e < n_experts; e++) {
        if (!uses[e] || where[e] >= 0) continue;
        int v = -1;
        for (int pass = 0; pass < 2 && v < 0; pass++) {
            if (pass == 1) {                     // every slot pinned: the next batch
                cnt[batch] = nm - off[batch];
                batch += 1;
                off[batch] = nm;
                pinned = 0;
            }
            for (int s = 0; s < S && v < 0; s++)
                if (tb->expert[s] < 0) v = s;
            if (v < 0)
                for (int s = 0; s < S; s++) {
                    if (pinned & (1u << s)) continue;
                    if (v < 0 || tb->count[s] < tb->count[v] ||
                        (tb->count[s] == tb->count[v] && tb->seq[s] < tb->seq[v]))
                        v = s;
                }
        }
        tb->counter += 1;
        tb->expert[v] = e;
        tb->count[v] = uses[e];
        tb->seq[v] = tb->counter;
        pinned |= 1u << v;
        where[e] = v;
        bat[e] = batch;
        pairs[2 * nm] = e;
        pairs[2 * nm + 1] = v;
        nm++;
        tb->misses += 1;
    }
    cnt[batch] = nm - off[batch];
    off[batch + 1] = nm;
    for (int q = 0; q < P; q++) {
        slot_of[q] = where[idx[q]];
        batch_of[q] = bat[idx[q]];
    }
    __threadfence_system();
    plan[0] = batch + 1;
}

// Device-initiated cache fill: the blobs of the miss list, copied from pinned
// host memory (read over the bus by plain 16-byte loads) into their cache
// slots, with no host involvement ("Gemma 4 26B : Comment faire tourner un LLM
// en 2 Go de RAM", section 04 "Le pipeline de traitement": only the missing
// experts are loaded).  grid (parts, max misses), block 256: blockIdx.y is the
// miss, blockIdx.x a part of its blob; nothing to do for misses beyond n_miss
// (or when n_miss < 0).
constexpr int kFillParts = 16;
constexpr int kFillThreads = 256;

__global__ void __launch_bounds__(kFillThreads)
k_fill_from_host(const uint8_t* __restrict__ store, uint8_t* __restrict__ slots, size_t stride,
                 const int32_t* __restrict__ miss_list, const int32_t* __restrict__ n_miss, int E, int S) {
    const int j = blockIdx.y;
    if (j >= *n_miss) return;
    const int e = miss_list[2 * j], s = miss_list[2 * j + 1];
    if (e < 0 || e >= E || s < 0 || s >= S) return;
    const uint4* src = reinterpret_cast<const uint4*>(store + (size_t)e * stride);
    uint4* dst = reinterpret_cast<uint4*>(slots + (size_t)s * stride);
    const size_t n16 = stride / 16;
    const size_t per = (n16 + gridDim.x - 1) / gridDim.x;
    const size_t b0 = (size_t)blockIdx.x * per;
    const size_t b1 = b0 + per < n16 ? b0 + per : n16;
    constexpr int U = 4;                          // 16-byte loads in flight per thread
    for (size_t i = b0 + threadIdx.x; i < b1; i += (size_t)kFillThreads * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const size_t q = i + (size_t)u * kFillThreads;
            v[u] = q < b1 ? __ldg(src + q) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            const size_t q = i + (size_t)u * kFillThreads;
            if (q < b1) dst[q] = v[u];
        }
    }
}

__global__ void k_lfu_init(MoeLfuTable* tb, int S) {
    int s = threadIdx.x;
    if (s < MOE_MAX_SLOTS) { tb->expert[s] = -1; tb->count[s] = 0; tb->seq[s] = 0; }
    if (s == 0) { tb->counter = 0; tb->hits = 0; tb->misses = 0; tb->n_slots = S; tb->valid = 1; }
}

__global__ void k_lfu_invalidate(MoeLfuTable* tb) { tb->valid = 0; }

// --------------------------------------------------------------- glue --
// Pair lists for a layer: pairs [0, T) are the shared expert of each token,
// pairs T + t*k + j the routed expert j of token t (resident: experts base +
// idx * stride; streaming: slots base + slot * stride).
__global__ void k_build_pairs(const void* shared_blob, int Is, const uint8_t* base,
                              size_t stride, const int32_t* __restrict__ sel, int I,
                              int T, int k, MoeFfnPair* __restrict__ pairs) {
    int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p < T) {
        pairs[p] = MoeFfnPair{shared_blob, Is, p};
    } else if (p < T + T * k) {
        int q = p - T;
        pairs[p] = MoeFfnPair{base + (size_t)sel[q] * stride, I, q / k};
    }
}

__global__ void k_copy_half_row(const __half* __restrict__ src, __half* __restrict__ dst,
                                const int* __restrict__ cursor, int H, int src_indexed) {
    const int t = *cursor;
    const __half* s = src + (src_indexed ? (size_t)t * H : 0);
    __half* d = dst + (src_indexed ? 0 : (size_t)t * H);
    for (int c = threadIdx.x; c < H; c += blockDim.x) d[c] = s[c];
}

__global__ void k_copy_rows(const __half* __restrict__ src, __half* __restrict__ dst, int n) {
    for (int c = threadIdx.x; c < n; c += blockDim.x) dst[c] = src[c];
}

__global__ void k_store_token(const __half* __restrict__ h_cur, const float* __restrict__ y,
                              __half* __restrict__ h_all, float* __restrict__ y_all,
                              int* __restrict__ cursor, int H) {
    const int t = *cursor;
    for (int c = threadIdx.x; c < H; c += blockDim.x) {
        h_all[(size_t)t * H + c] = h_cur[c];
        if (y_all) y_all[(size_t)t * H + c] = y[c];
    }
    __syncthreads();
    if (threadIdx.x == 0) *cursor = t + 1;
}

}  // namespace moeq4
