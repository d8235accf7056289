// ffn_mma.cuh -- expert FFN on the tensor cores (tcgen05, accumulators in
// tensor memory) for experts that receive many tokens in one step.
//
// Chunked prefill applies one fetched expert to many token rows at once
// ("Gemma 4 26B : Comment faire tourner un LLM en 2 Go de RAM", section 04
// "Chunked Prefill").  Once an expert's bucket holds at least the configured
// number of tokens (32 by default; the pages, written for another GPU, name
// no threshold), its product with the bucket is a small GEMM.  With the
// affine 4-bit weight w = s_g q + b_g of group g (64 columns):
//
//   D[m][t] = sum_g ( s_g[m] P_g[m][t] + b_g[m] S_g[t] ),
//   P_g[m][t] = sum_{c in g} q[m][c] X[t][c],   S_g[t] = sum_{c in g} X[t][c]
//
// The tensor cores compute P_g with the raw codes q as A (0..15 are exact in
// bf16) and X as B split into two bf16 planes, X = hi + lo (hi = bf16(X),
// lo = bf16(X - hi); exact for an fp16 x, 16 significant bits for the fp32
// intermediate h): P_g = q*hi + q*lo, every product exact, sums in fp32.
// Each group g has its own TMEM accumulator; the CUDA cores fold it into the
// fp32 result with the group's scale and bias.  S_g comes with the B planes
// (k_split_x for x, the gate/up epilogue for h).
//
// Per CTA (512 threads, one per SM): M = 128 weight rows (one TMEM lane
// each), N = 64 tokens, one 64-column group per stage.  The CTA stages the
// 128 rows' scales and biases for all groups and the tile's S_g; a ring of
// six slots, filled by cp.async four stages ahead, holds each stage's codes
// and B planes.  Per stage every thread turns its own 16 codes into bf16 in
// one of two A buffers (no-swizzle K-major core matrices of 8 rows x 16
// bytes) and folds the accumulator of the stage two back; thread 0 issues
// 4 x 2 MMAs of K = 16 into one of three TMEM buffers and commits them to
// the A buffer's mbarrier.  Every wait is bounded (2 s); on expiry the kernel
// records MOE_ERR_TIMEOUT, waits (bounded) for its issued MMAs, frees its
// tensor memory and returns.
#pragma once
#include <cuda_bf16.h>
#include "common.cuh"
#include "grouped.cuh"
#include "layer_fused.cuh"
#include "ptx.cuh"

namespace moeq4 {

constexpr int kMmaRows = 128;                          // M
constexpr int kMmaTok = 64;                            // N
constexpr int kMmaK = 64;                              // K per stage (one scale group)
constexpr int kMmaThreads = 512;
constexpr int kMmaRing = 6;                            // ring slots (4 stages in flight ahead)
constexpr int kMmaABytes = kMmaRows * kMmaK * 2;       // one bf16 A tile (16 KB)
constexpr int kMmaBBytes = kMmaTok * kMmaK * 2;        // one bf16 B tile (8 KB)
constexpr int kMmaRawA = kMmaRows * kMmaK / 2;         // one stage of 4-bit codes (4 KB)
constexpr int kMmaSlotBytes = 2 * kMmaBBytes + kMmaRawA;   // B hi, B lo, codes
constexpr int kMmaAccBufs = 3;                         // TMEM accumulators (one per stage)
constexpr int kMmaTmemCols = 256;                      // allocation (power of two >= 3 x 64)
constexpr int kMmaDefaultMinTokens = 32;

// Dynamic shared memory of k_ffn_mma for reduction length K: two A buffers,
// the ring, scales and biases of 128 rows (4 K bytes each), the tile's S_g
// (64 rows x K / 64 floats = 4 K bytes), alignment slack.
__host__ __device__ constexpr size_t mma_smem_bytes(int K) {
    return (size_t)2 * kMmaABytes + (size_t)kMmaRing * kMmaSlotBytes + 12 * (size_t)K + 1024;
}

// Instruction descriptor of kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9, 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bit 17,
// M >> 4 at bit 24.
constexpr uint32_t kMmaIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                               ((uint32_t)(kMmaTok >> 3) << 17) | ((uint32_t)(kMmaRows >> 4) << 24);

// Byte offset of the 16-byte granule (row r, 8-column group g) inside one
// operand tile: core matrices of 8 rows x 16 bytes, the 8 column groups of a
// row block side by side (128 B apart), row blocks 1024 B apart.
__device__ __forceinline__ uint32_t mma_granule(int r, int g) {
    return (uint32_t)(((r >> 3) * 8 + g) * 128 + (r & 7) * 16);
}

// Shared-memory matrix descriptor, no swizzle, K-major: start address >> 4
// (bits 0-13), leading byte offset 128 >> 4 (the next 8 columns, bits
// 16-29), stride byte offset 1024 >> 4 (the next 8 rows, bits 32-45),
// descriptor version 1 (bit 46), base offset 0, layout type 0.
__device__ __forceinline__ uint64_t mma_sdesc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | (1ull << 46);
}

__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kMmaIdesc), "r"(accum)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}

// hi/lo bf16 pair of two values, packed two per word (first value in the low half).
__device__ __forceinline__ void mma_split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h2);
    const __nv_bfloat162 l2 = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h2);
    lo = *reinterpret_cast<const uint32_t*>(&l2);
}

// Eight 4-bit codes of one word (low nibble first) as eight exact bf16
// values: nibble q sits in the mantissa of bf16 128 + q (0x4300 | q), then
// 128 is subtracted (exact).  Result: one granule of 8 bf16 in column order.
__device__ __forceinline__ uint4 mma_codes_bf16(uint32_t w) {
    const __nv_bfloat162 k128 = __floats2bfloat162_rn(128.f, 128.f);
    uint32_t o[4];
#pragma unroll
    for (int p = 0; p < 4; p++) {
        // codes 2p (low half) and 2p + 1 (high half)
        const uint32_t q0 = (w >> (8 * p)) & 0xFu, q1 = (w >> (8 * p + 4)) & 0xFu;
        const uint32_t v = 0x43004300u | q0 | (q1 << 16);
        const __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v), k128);
        o[p] = *reinterpret_cast<const uint32_t*>(&q);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float4 lds128f(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// cp.async global -> shared of 16 (or 8, 4) bytes; src_bytes 0 writes zeros.
__device__ __forceinline__ void cpa16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cpa8(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa4(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cpa_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Waits for an mbarrier phase with a time bound only (used while draining
// after a failure, when the status word is already set).
__device__ __forceinline__ void mma_drain_wait(uint64_t* bar, uint32_t parity) {
    const unsigned long long t0 = gtimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (gtimer_ns() - t0 > kWaitNs) return;
    }
}

// x (fp16 [rows][H]) as two bf16 planes (hi = bf16(x), lo = bf16(x - hi);
// an fp16 value has 11 significant bits, so hi + lo equals it) and the
// 64-column group sums S[row][g] = sum of the group's x (fp32).  One thread
// per 8 columns; 8 consecutive threads make a group.  n8 = rows * H / 8.
__global__ void k_split_x(const uint4* __restrict__ x, size_t n8, uint4* __restrict__ hi,
                          uint4* __restrict__ lo, float* __restrict__ gsum) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t n_iter = (n8 + stride - 1) / stride;     // same count in every thread
    for (size_t it = 0; it < n_iter; it++) {
        const size_t i = it * stride + (size_t)blockIdx.x * blockDim.x + threadIdx.x;
        float s = 0.f;
        if (i < n8) {
            const uint4 v = x[i];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t h[4], l[4];
#pragma unroll
            for (int p = 0; p < 4; p++) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[p]));
                mma_split2(f.x, f.y, h[p], l[p]);
                s += f.x + f.y;
            }
            hi[i] = make_uint4(h[0], h[1], h[2], h[3]);
            lo[i] = make_uint4(l[0], l[1], l[2], l[3]);
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if (i < n8 && (i & 7) == 0) gsum[i >> 3] = s;
    }
}

// Tensor-core FFN half over expert token buckets.
//   DOWN = false (gate/up): CTA strip sb takes 4 gate/up tiles; A row 32 j + r
//     is tile 4 sb + j, row r (r < 16: gate, else up) of intermediate index
//     i = 64 sb + 16 j + r % 16; K = H; B rows are tokens of the x planes.
//     Writes h = GELU(gate) * up as bf16 hi/lo planes h_hi / h_lo [row][i]
//     and, the strip being one 64-column group of the down projection, the
//     group sums h_sum[row * h_stride / 64 + sb] = sum over its 64 i of
//     (hi + lo).
//   DOWN = true: CTA strip sb takes output rows o = 128 sb + m; K = Ie; B rows
//     are pair rows of the h planes.  Writes y_pairs[row][o] (fp32).
// b_sum[row * bs_stride + g] holds S_g of B row `row`.  Rows follow
// the grouped kernels' pair convention (row p < T: shared expert of token p;
// row T + q: routed pair q).  Routed (SHARED = false): expert blockIdx.y,
// skipped unless its bucket holds at least min_tok pairs.  Token tiles of 64:
// z = blockIdx.z, + gridDim.z, ...  grid (Ie / 64 or H / 128, experts or 1,
// tiles), block 512, dynamic shared memory mma_smem_bytes(K).
template <bool DOWN, bool SHARED>
__global__ void __launch_bounds__(kMmaThreads, 1)
k_ffn_mma(const uint8_t* __restrict__ experts, size_t stride, const uint8_t* __restrict__ shared_blob,
          int H, int Ie, int T, int k, const int* __restrict__ e_off, const int* __restrict__ list,
          int min_tok, int gelu, const __nv_bfloat16* __restrict__ b_hi,
          const __nv_bfloat16* __restrict__ b_lo, int b_stride, const float* __restrict__ b_sum,
          int bs_stride, __nv_bfloat16* __restrict__ h_hi, __nv_bfloat16* __restrict__ h_lo, int h_stride,
          float* __restrict__ h_sum, float* __restrict__ y_pairs, int* __restrict__ status) {
    extern __shared__ uint8_t msm_raw[];
    __shared__ __align__(8) uint64_t mbar[2];
    __shared__ uint32_t s_tmem;
    __shared__ int s_src[kMmaTok], s_row[kMmaTok];
    __shared__ float s_red[4][kMmaTok];

    int n = T, base = 0;
    const uint8_t* blob = shared_blob;
    if (!SHARED) {
        base = e_off[blockIdx.y];
        n = e_off[blockIdx.y + 1] - base;
        if (n < min_tok) return;
        blob = experts + (size_t)blockIdx.y * stride;
    }
    if ((int)blockIdx.z * kMmaTok >= n) return;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = DOWN ? Ie : H, nk = K / kMmaK;
    const uint32_t sbase = (smem_u32(msm_raw) + 1023u) & ~1023u;
    const uint32_t s_a = sbase, s_ring = sbase + 2 * kMmaABytes;
    const uint32_t s_sc = s_ring + kMmaRing * kMmaSlotBytes, s_bi = s_sc + 4 * K, s_gs = s_bi + 4 * K;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s_tmem)),
                     "r"(kMmaTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&mbar[0], 1);
        mbar_init(&mbar[1], 1);
        fence_mbar_init();
    }

    // Scales and biases of the 128 rows for all groups (fp16): row m at
    // m * K / 32 bytes.  They sit in the blob as whole blocks per tile
    // (gate/up: 32 rows x H / 32 bytes; down: 16 rows x Ie / 32 bytes).
    const BlobLayout L(H, Ie);
    if (!DOWN) {
        const int per = H / 16;                           // 16-byte pieces per tile block
        for (int p = tid; p < 8 * per; p += kMmaThreads) {
            const int which = p / (4 * per), rem = p - which * 4 * per;
            const int j = rem / per, o = rem - j * per;
            const uint8_t* src = blob + (size_t)(4 * blockIdx.x + j) * L.gu_tile +
                                 (size_t)(16 + which) * H + 16 * o;
            cpa16((which ? s_bi : s_sc) + j * H + 16 * o, src, 16);
        }
    } else {
        const int per = Ie / 32;
        for (int p = tid; p < 16 * per; p += kMmaThreads) {
            const int which = p / (8 * per), rem = p - which * 8 * per;
            const int j = rem / per, o = rem - j * per;
            const uint8_t* src = blob + L.dn_base + (size_t)(8 * blockIdx.x + j) * L.dn_tile +
                                 8 * (size_t)Ie + which * (Ie / 2) + 16 * o;
            cpa16((which ? s_bi : s_sc) + j * (Ie / 2) + 16 * o, src, 16);
        }
    }
    cpa_commit();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    // Copy roles.  Codes: row dm = 8 warp + lane % 8, bytes 8 dq .. 8 dq + 7
    // (dq = lane / 8) of the row's 32 bytes per stage; the same thread turns
    // them into bf16, so no barrier sits between copy and use.  B: rows
    // tid >> 4 and 32 + (tid >> 4), plane (tid >> 3) & 1, 8-column group tid & 7.
    const int dm = 8 * warp + (lane & 7), dq = lane >> 3;
    size_t oc;
    if (!DOWN) {
        const int j = dm >> 5, r = dm & 31;
        const int i = 64 * (int)blockIdx.x + 16 * j + (r & 15);
        oc = L.gu_codes(r < 16 ? i : Ie + i);
    } else {
        oc = L.dn_codes(kMmaRows * (int)blockIdx.x + dm);
    }
    const uint8_t* a_src = blob + oc + 8 * dq;
    const uint32_t a_raw = 2 * kMmaBBytes + (uint32_t)dm * 32 + 8 * dq;
    const uint32_t a_g0 = mma_granule(dm, 2 * dq), a_g1 = mma_granule(dm, 2 * dq + 1);
    const int bt0 = tid >> 4, bpl = (tid >> 3) & 1, bg = tid & 7;
    const __nv_bfloat16* bplane = bpl ? b_lo : b_hi;
    const uint32_t b_dst0 = bpl * kMmaBBytes + mma_granule(bt0, bg);
    const uint32_t b_dst1 = bpl * kMmaBBytes + mma_granule(bt0 + 32, bg);
    // Fold role: TMEM lane quarter j (rows 32 j + lane), columns 16 cg .. + 15.
    const int fj = warp & 3, cg = warp >> 2, fm = 32 * fj + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * fj) << 16) + 16u * cg;

    bool ok = true;
    uint32_t g = 0;                                       // stages issued
    for (int z = blockIdx.z; z * kMmaTok < n; z += gridDim.z) {
        const int t0 = z * kMmaTok, nt = min(kMmaTok, n - t0);
        const bool fold_on = 16 * cg < nt;                // warp-uniform
        __syncthreads();                                  // the previous tile is done with s_row, s_gs
        if (tid < kMmaTok) {
            int src = -1, row = -1;
            if (tid < nt) {
                row = grp_row(SHARED, list, base, t0 + tid, T);
                src = DOWN ? row : grp_token(SHARED, list, base, t0 + tid, k);
            }
            s_src[tid] = src;
            s_row[tid] = row;
        }
        __syncthreads();
        // S_g of the tile's rows, stored [g][t]
        for (int p = tid; p < kMmaTok * nk; p += kMmaThreads) {
            const int t = p & (kMmaTok - 1), gg = p >> 6, r = s_src[t];
            cpa4(s_gs + 4u * p, r >= 0 ? b_sum + (size_t)r * bs_stride + gg : b_sum, r >= 0 ? 4u : 0u);
        }
        cpa_commit();
        const int r0 = s_src[bt0], r1 = s_src[bt0 + 32];
        auto issue = [&](int c) {
            const uint32_t sl = s_ring + (uint32_t)(c % kMmaRing) * kMmaSlotBytes;
            cpa8(sl + a_raw, a_src + 32 * c);
            const size_t col = (size_t)kMmaK * c + 8 * bg;
            cpa16(sl + b_dst0, r0 >= 0 ? bplane + (size_t)r0 * b_stride + col : bplane, r0 >= 0 ? 16u : 0u);
            cpa16(sl + b_dst1, r1 >= 0 ? bplane + (size_t)r1 * b_stride + col : bplane, r1 >= 0 ? 16u : 0u);
        };
        float acc[16];
#pragma unroll
        for (int q = 0; q < 16; q++) acc[q] = 0.f;
        // acc += s_gg * P_gg + b_gg * S_gg from TMEM buffer buf
        auto fold = [&](int gg, uint32_t buf) {
            if (!fold_on) return;
            float P[16];
            tmem_ld16(t_lane + 64u * buf, P);
            const uint32_t so = (uint32_t)fm * (K / 32) + 2 * gg;
            const float sc = __half2float(__ushort_as_half(lds16(s_sc + so)));
            const float bi = __half2float(__ushort_as_half(lds16(s_bi + so)));
            const uint32_t ga = s_gs + 4u * (gg * kMmaTok + 16 * cg);
#pragma unroll
            for (int v = 0; v < 4; v++) {
                const float4 S = lds128f(ga + 16 * v);
                acc[4 * v + 0] = fmaf(sc, P[4 * v + 0], fmaf(bi, S.x, acc[4 * v + 0]));
                acc[4 * v + 1] = fmaf(sc, P[4 * v + 1], fmaf(bi, S.y, acc[4 * v + 1]));
                acc[4 * v + 2] = fmaf(sc, P[4 * v + 2], fmaf(bi, S.z, acc[4 * v + 2]));
                acc[4 * v + 3] = fmaf(sc, P[4 * v + 3], fmaf(bi, S.w, acc[4 * v + 3]));
            }
        };
#pragma unroll 1
        for (int c = 0; c < kMmaRing - 2; c++) {
            if (c < nk) issue(c);
            cpa_commit();
        }
#pragma unroll 1
        for (int c = 0; c < nk; c++, g++) {
            const uint32_t s = g & 1u;
            // the MMAs of stage c - 2 are done: A buffer s, ring slot (c - 2) % ring
            // and TMEM buffer (g - 2) % 3 are free to reuse or read
            const bool w_ok = c < 2 || fused_wait_bar(&mbar[s], ((g - 2) >> 1) & 1u, status);
            tc_fence_after();
            if (w_ok && c + kMmaRing - 2 < nk) issue(c + kMmaRing - 2);
            cpa_commit();
            cpa_wait<kMmaRing - 2>();                     // this thread's copies of stage c landed
            const uint32_t sl = s_ring + (uint32_t)(c % kMmaRing) * kMmaSlotBytes;
            const uint32_t ab = s_a + s * kMmaABytes;
            if (w_ok) {
                const uint2 w2 = lds64(sl + a_raw);
                sts128(ab + a_g0, mma_codes_bf16(w2.x));
                sts128(ab + a_g1, mma_codes_bf16(w2.y));
                if (c >= 2) fold(c - 2, (g - 2) % kMmaAccBufs);
            }
            fence_proxy_async_smem();                     // codes and cp.async data -> tensor core
            tc_fence_before();
            if (!__syncthreads_and(w_ok)) { ok = false; break; }
            if (tid == 0) {
                tc_fence_after();
                const uint32_t d = tmem + 64u * (g % kMmaAccBufs);
#pragma unroll
                for (int kk = 0; kk < kMmaK / 16; kk++) {
                    const uint32_t ko = 256u * kk;        // two 8-column granules per K = 16
                    const uint64_t da = mma_sdesc(ab + ko);
                    mma_bf16_ss(d, da, mma_sdesc(sl + ko), kk > 0 ? 1u : 0u);
                    mma_bf16_ss(d, da, mma_sdesc(sl + kMmaBBytes + ko), 1u);
                }
                mma_commit(&mbar[s]);
            }
        }
        cpa_wait<0>();
        if (!ok) break;
        // the last two stages: wait for the final commit, then fold them
        const bool d_ok = fused_wait_bar(&mbar[(g - 1) & 1u], ((g - 1) >> 1) & 1u, status);
        if (!__syncthreads_and(d_ok)) { ok = false; break; }
        tc_fence_after();
        if (nk >= 2) fold(nk - 2, (g - 2) % kMmaAccBufs);
        fold(nk - 1, (g - 1) % kMmaAccBufs);
        if (!DOWN) {
            const int i = 64 * (int)blockIdx.x + 16 * fj + (lane & 15);
            if (fold_on) {
#pragma unroll
                for (int q = 0; q < 16; q++) {
                    const float up = __shfl_xor_sync(0xffffffffu, acc[q], 16);
                    const int col = 16 * cg + q;
                    float part = 0.f;
                    if (lane < 16 && col < nt) {
                        uint32_t hh, hl;
                        const float hv = gelu_f(acc[q], gelu) * up;
                        mma_split2(hv, 0.f, hh, hl);
                        const __nv_bfloat16 bh = __ushort_as_bfloat16((unsigned short)(hh & 0xFFFFu));
                        const __nv_bfloat16 bl = __ushort_as_bfloat16((unsigned short)(hl & 0xFFFFu));
                        const size_t o = (size_t)s_row[col] * h_stride + i;
                        h_hi[o] = bh;
                        h_lo[o] = bl;
                        part = __bfloat162float(bh) + __bfloat162float(bl);
                    }
                    part += __shfl_xor_sync(0xffffffffu, part, 8);
                    part += __shfl_xor_sync(0xffffffffu, part, 4);
                    part += __shfl_xor_sync(0xffffffffu, part, 2);
                    part += __shfl_xor_sync(0xffffffffu, part, 1);
                    if (lane == 0) s_red[fj][col] = part;
                }
            }
            __syncthreads();
            if (tid < nt)
                h_sum[(size_t)s_row[tid] * (h_stride / 64) + blockIdx.x] =
                    ((s_red[0][tid] + s_red[1][tid]) + s_red[2][tid]) + s_red[3][tid];
        } else if (fold_on) {
            const int o = kMmaRows * (int)blockIdx.x + fm;
#pragma unroll
            for (int q = 0; q < 16; q++) {
                const int col = 16 * cg + q;
                if (col < nt) y_pairs[(size_t)s_row[col] * H + o] = acc[q];
            }
        }
        tc_fence_before();
    }
    cpa_wait<0>();
    if (!ok && g > 0 && tid == 0) mma_drain_wait(&mbar[(g - 1) & 1u], ((g - 1) >> 1) & 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kMmaTmemCols)
                     : "memory");
    }
}

}  // namespace moeq4
