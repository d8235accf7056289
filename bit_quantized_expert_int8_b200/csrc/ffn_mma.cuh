// ffn_mma.cuh -- expert FFN on the tensor cores (tcgen05, accumulators in
// tensor memory) for experts that receive many tokens in one step.
//
// Chunked prefill applies one fetched expert to many token rows at once
// ("Gemma 4 26B : Comment faire tourner un LLM en 2 Go de RAM", section 04
// "Chunked Prefill").  Once an expert's bucket holds at least the configured
// number of tokens (32 by default; the pages, written for another GPU, name
// no threshold), its product with the bucket is a small GEMM:
//
//   D[m][t] = sum_c W[m][c] * X[t][c]     m: 128 weight rows, t: 64 tokens
//
// W is the 4-bit affine weight, dequantised per 64-column group (one K stage)
// into shared memory by CUDA cores; X is the token tile (x rows for gate/up,
// h rows for down).  Both are split into two bf16 terms, v = hi + lo with
// hi = bf16(v) and lo = bf16(v - hi), and the MMA sums hi_W*hi_X + hi_W*lo_X
// + lo_W*hi_X in fp32: each product then carries about 16 significant bits
// (the dropped lo*lo term is below 2^-16 of it), well inside the layer's
// 1e-3 relative tolerance.  An fp16 x is exact as hi + lo.
//
// Per CTA: M = 128 weight rows (one TMEM lane each), N = 64 tokens (fp32
// TMEM columns), K loop over 64-column stages with two shared-memory stages
// of 48 KB (A hi, A lo, B hi, B lo; no-swizzle K-major core matrices of
// 8 rows x 16 bytes).  All 256 threads stage; thread 0 issues 4 x 3 MMAs of
// K = 16 per stage and commits them to the stage's mbarrier.  Every wait is
// bounded (2 s); on expiry the kernel records MOE_ERR_TIMEOUT, waits (bounded)
// for its issued MMAs, frees its tensor memory and returns.
#pragma once
#include <cuda_bf16.h>
#include "common.cuh"
#include "ptx.cuh"
#include "grouped.cuh"
#include "layer_fused.cuh"

namespace moeq4 {

constexpr int kMmaRows = 128;                          // M
constexpr int kMmaTok = 64;                            // N
constexpr int kMmaK = 64;                              // K per stage (one scale group)
constexpr int kMmaThreads = 256;
constexpr int kMmaABytes = kMmaRows * kMmaK * 2;       // one bf16 A tile (16 KB)
constexpr int kMmaBBytes = kMmaTok * kMmaK * 2;        // one bf16 B tile (8 KB)
constexpr int kMmaStageBytes = 2 * kMmaABytes + 2 * kMmaBBytes;
constexpr int kMmaSmem = 2 * kMmaStageBytes + 1024;    // two stages + alignment slack
constexpr int kMmaTmemCols = kMmaTok;                  // fp32 accumulator columns
constexpr int kMmaDefaultMinTokens = 32;

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

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// hi/lo bf16 pair of v, packed two values per word (lower column in the low half).
__device__ __forceinline__ void mma_split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat16 ah = __float2bfloat16_rn(a), bh = __float2bfloat16_rn(b);
    const __nv_bfloat16 al = __float2bfloat16_rn(a - __bfloat162float(ah));
    const __nv_bfloat16 bl = __float2bfloat16_rn(b - __bfloat162float(bh));
    hi = (uint32_t)__bfloat16_as_ushort(ah) | ((uint32_t)__bfloat16_as_ushort(bh) << 16);
    lo = (uint32_t)__bfloat16_as_ushort(al) | ((uint32_t)__bfloat16_as_ushort(bl) << 16);
}

// One 8-code word w (low nibble first) of a row with scale s, bias b, as
// hi and lo granules of 8 bf16 weights.
__device__ __forceinline__ void mma_dequant_word(uint32_t w, float s, float b, uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int p = 0; p < 4; p++) {
        const float q0 = __uint_as_float(0x4B000000u | ((w >> (8 * p)) & 15u)) - 8388608.f;
        const float q1 = __uint_as_float(0x4B000000u | ((w >> (8 * p + 4)) & 15u)) - 8388608.f;
        mma_split2(fmaf(s, q0, b), fmaf(s, q1, b), h[p], l[p]);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// Waits for an mbarrier phase with a time bound only (used while draining
// after a failure, when the status word is already set).
__device__ __forceinline__ void mma_drain_wait(uint64_t* bar, uint32_t parity) {
    const unsigned long long t0 = gtimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (gtimer_ns() - t0 > kWaitNs) return;
    }
}

// Tensor-core FFN half over expert token buckets.
//   DOWN = false (gate/up): CTA strip sb takes 4 gate/up tiles; A row 32 j + r
//     is tile 4 sb + j, row r (r < 16: gate, else up) of intermediate index
//     i = 64 sb + 16 j + r % 16; K = H.  Writes h_ws[row][i] = GELU(gate) * up.
//   DOWN = true: CTA strip sb takes output rows o = 128 sb + m; K = Ie.
//     Writes y_pairs[row][o].
// Rows of h_ws / y_pairs follow the grouped kernels' pair convention.
// Routed (SHARED = false): expert blockIdx.y, skipped unless its bucket holds
// at least min_tok pairs.  Token tiles of 64: z = blockIdx.z, + gridDim.z, ...
// grid (Ie / 64 or H / 128, experts or 1, tiles), block 256, dynamic shared
// memory kMmaSmem bytes.
template <bool DOWN, bool SHARED>
__global__ void __launch_bounds__(kMmaThreads, 2)
k_ffn_mma(const uint8_t* __restrict__ experts, size_t stride, const uint8_t* __restrict__ shared_blob,
          int H, int Ie, const __half* __restrict__ x, int T, int k, const int* __restrict__ e_off,
          const int* __restrict__ list, int min_tok, int gelu, float* __restrict__ h_ws, int h_stride,
          float* __restrict__ y_pairs, int* __restrict__ status) {
    extern __shared__ uint8_t msm_raw[];
    __shared__ __align__(8) uint64_t mbar[2];
    __shared__ uint32_t s_tmem;
    __shared__ int s_tok[kMmaTok], s_row[kMmaTok];

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
    const uint32_t sbase = (smem_u32(msm_raw) + 1023u) & ~1023u;
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
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    // This thread's A row (tid >> 1, columns 32 (tid & 1) .. + 31 of a stage).
    const BlobLayout L(H, Ie);
    const int am = tid >> 1, ah = tid & 1;
    size_t oc, os, ob;
    if (!DOWN) {
        const int j = am >> 5, r = am & 31;
        const int i = 64 * (int)blockIdx.x + 16 * j + (r & 15);
        const int gr = r < 16 ? i : Ie + i;
        oc = L.gu_codes(gr);
        os = L.gu_scales(gr);
        ob = L.gu_biases(gr);
    } else {
        const int o = kMmaRows * (int)blockIdx.x + am;
        oc = L.dn_codes(o);
        os = L.dn_scales(o);
        ob = L.dn_biases(o);
    }
    const uint8_t* a_codes = blob + oc + 16 * ah;
    const __half* a_sc = reinterpret_cast<const __half*>(blob + os);
    const __half* a_bi = reinterpret_cast<const __half*>(blob + ob);
    const uint32_t a_off = mma_granule(am, 4 * ah);       // granules 4 ah .. 4 ah + 3 follow at +128
    // This thread's B slot: token bt, columns 16 bq .. + 15 of a stage.
    const int bt = tid >> 2, bq = tid & 3;
    const uint32_t b_off = mma_granule(bt, 2 * bq);

    const int K = DOWN ? Ie : H;
    const int nk = K / kMmaK;
    bool ok = true;
    uint32_t g = 0;                                       // stages issued (stage = g & 1)
    for (int z = blockIdx.z; z * kMmaTok < n; z += gridDim.z) {
        const int t0 = z * kMmaTok, nt = min(kMmaTok, n - t0);
        __syncthreads();                                  // the previous epilogue is done with s_row
        if (tid < kMmaTok) {
            int tok = -1, row = -1;
            if (tid < nt) {
                tok = grp_token(SHARED, list, base, t0 + tid, k);
                row = grp_row(SHARED, list, base, t0 + tid, T);
            }
            s_tok[tid] = tok;
            s_row[tid] = row;
        }
        __syncthreads();
        const int bsrc = DOWN ? s_row[bt] : s_tok[bt];

        // registers of the current stage
        uint4 acode;
        float asc, abi;
        uint4 bv[4];
        auto load = [&](int c, uint4& code, float& sc, float& bi, uint4 (&v)[4]) {
            code = __ldg(reinterpret_cast<const uint4*>(a_codes + 32 * c));
            sc = __half2float(a_sc[c]);
            bi = __half2float(a_bi[c]);
            if (bsrc < 0) {
                v[0] = v[1] = v[2] = v[3] = make_uint4(0u, 0u, 0u, 0u);
            } else if (DOWN) {
                const uint4* p = reinterpret_cast<const uint4*>(h_ws + (size_t)bsrc * h_stride +
                                                                kMmaK * c + 16 * bq);
                v[0] = __ldg(p); v[1] = __ldg(p + 1); v[2] = __ldg(p + 2); v[3] = __ldg(p + 3);
            } else {
                const uint4* p =
                    reinterpret_cast<const uint4*>(x + (size_t)bsrc * H + kMmaK * c + 16 * bq);
                v[0] = __ldg(p); v[1] = __ldg(p + 1);
            }
        };
        load(0, acode, asc, abi, bv);
#pragma unroll 1
        for (int c = 0; c < nk; c++, g++) {
            uint4 ncode = acode, nbv[4] = {bv[0], bv[1], bv[2], bv[3]};
            float nsc = asc, nbi = abi;
            if (c + 1 < nk) load(c + 1, ncode, nsc, nbi, nbv);
            const uint32_t s = g & 1u;
            bool w_ok = g < 2 || fused_wait_bar(&mbar[s], ((g - 2) >> 1) & 1u, status);
            const uint32_t st = sbase + s * kMmaStageBytes;
            if (w_ok) {
                const uint32_t ahi = st + a_off, alo = st + kMmaABytes + a_off;
                const uint32_t w4[4] = {acode.x, acode.y, acode.z, acode.w};
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    uint4 hi, lo;
                    mma_dequant_word(w4[q], asc, abi, hi, lo);
                    sts128(ahi + 128 * q, hi);
                    sts128(alo + 128 * q, lo);
                }
                const uint32_t bhi = st + 2 * kMmaABytes + b_off, blo = bhi + kMmaBBytes;
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    float f[8];
                    if (DOWN) {
                        const uint4 p0 = bv[2 * u], p1 = bv[2 * u + 1];
                        f[0] = __uint_as_float(p0.x); f[1] = __uint_as_float(p0.y);
                        f[2] = __uint_as_float(p0.z); f[3] = __uint_as_float(p0.w);
                        f[4] = __uint_as_float(p1.x); f[5] = __uint_as_float(p1.y);
                        f[6] = __uint_as_float(p1.z); f[7] = __uint_as_float(p1.w);
                    } else {
                        const uint32_t hw[4] = {bv[u].x, bv[u].y, bv[u].z, bv[u].w};
#pragma unroll
                        for (int p = 0; p < 4; p++) {
                            const __half2 h2 = *reinterpret_cast<const __half2*>(&hw[p]);
                            const float2 f2 = __half22float2(h2);
                            f[2 * p] = f2.x;
                            f[2 * p + 1] = f2.y;
                        }
                    }
                    uint32_t h[4], l[4];
#pragma unroll
                    for (int p = 0; p < 4; p++) mma_split2(f[2 * p], f[2 * p + 1], h[p], l[p]);
                    sts128(bhi + 128 * u, make_uint4(h[0], h[1], h[2], h[3]));
                    sts128(blo + 128 * u, make_uint4(l[0], l[1], l[2], l[3]));
                }
            }
            fence_proxy_async_smem();
            if (!__syncthreads_and(w_ok)) { ok = false; break; }
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kMmaK / 16; kk++) {
                    const uint32_t ko = 256u * kk;        // two 8-column granules per K = 16
                    const uint64_t dah = mma_sdesc(st + ko), dal = mma_sdesc(st + kMmaABytes + ko);
                    const uint64_t dbh = mma_sdesc(st + 2 * kMmaABytes + ko);
                    const uint64_t dbl = mma_sdesc(st + 2 * kMmaABytes + kMmaBBytes + ko);
                    mma_bf16_ss(tmem, dah, dbh, (c > 0 || kk > 0) ? 1u : 0u);
                    mma_bf16_ss(tmem, dah, dbl, 1u);
                    mma_bf16_ss(tmem, dal, dbh, 1u);
                }
                mma_commit(&mbar[s]);
            }
            acode = ncode;
            asc = nsc;
            abi = nbi;
#pragma unroll
            for (int q = 0; q < 4; q++) bv[q] = nbv[q];
        }
        if (!ok) break;
        // the tile's accumulator: wait for the last commit, then read TMEM
        const bool d_ok = fused_wait_bar(&mbar[(g - 1) & 1u], ((g - 1) >> 1) & 1u, status);
        if (!__syncthreads_and(d_ok)) { ok = false; break; }
        tc_fence_after();
        const int j = warp & 3, ch = warp >> 2;
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * j) << 16) + (uint32_t)(32 * ch), v);
        if (!DOWN) {
            const int i = 64 * (int)blockIdx.x + 16 * j + (lane & 15);
#pragma unroll
            for (int q = 0; q < 32; q++) {
                const float up = __shfl_xor_sync(0xffffffffu, v[q], 16);
                const int col = 32 * ch + q;
                if (lane < 16 && col < nt)
                    h_ws[(size_t)s_row[col] * h_stride + i] = gelu_f(v[q], gelu) * up;
            }
        } else {
            const int o = kMmaRows * (int)blockIdx.x + 32 * j + lane;
#pragma unroll
            for (int q = 0; q < 32; q++) {
                const int col = 32 * ch + q;
                if (col < nt) y_pairs[(size_t)s_row[col] * H + o] = v[q];
            }
        }
        tc_fence_before();
    }
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
