// ffn_tc.cuh -- expert FFN on the tensor cores (tcgen05 MMAs, accumulators in
// tensor memory, operands staged by TMA) for steps of many tokens.
//
// Chunked prefill applies one fetched expert to many token rows at once
// ("Gemma 4 26B : Comment faire tourner un LLM en 2 Go de RAM", section 04
// "Chunked Prefill").  With the affine 4-bit weight w = s_g q + b_g of the
// 64-column group g, an expert applied to its bucket of token rows X is
//
//   D[m][t] = sum_g ( s_g[m] P_g[m][t] + b_g[m] S_g[t] ),
//   P_g[m][t] = sum_{c in g} q[m][c] X[t][c],   S_g[t] = sum_{c in g} X[t][c].
//
// The tensor cores form P_g from the raw codes (0..15, exact in fp16 and
// bf16) and the token rows, one TMEM accumulator per group; CUDA cores fold
// it into fp32 with the group's scale and bias.  Gate/up runs kind::f16 on
// fp16 operands (codes and the fp16 x are both exact: one MMA per K = 16,
// every product exact, sums in fp32).  The down projection takes the fp32
// intermediate h as two bf16 planes, h = hi + lo (hi = bf16(h),
// lo = bf16(h - hi), 16 significant bits), and runs two bf16 MMAs per K = 16.
//
// One CTA per SM, 18 warps in four roles that meet only at mbarriers:
//   warp 0       TMA producer: per stage one tiled copy of the 128 rows'
//                codes (4 KB) and one of the 64-row B tile (128-byte swizzle)
//                into a ring slot;
//   warp 1       MMA issuer: 4 (or 8) MMAs per stage into one of four TMEM
//                buffers, then commits that free the A tile and the ring
//                slot and publish the accumulator;
//   warps 2..9   converters: codes -> fp16/bf16 A tile (no-swizzle K-major
//                core matrices) in one of three A buffers;
//   warps 10..17 folders: accumulator -> registers (acc += s P + b S), and the
//                epilogue of each token tile.
// B rows of a bucket are contiguous: x rows are gathered into bucket order
// once per step (k_gather_x) and the gate/up epilogue writes h in the same
// order, so one tiled copy fetches a stage's B tile.
// Every wait is bounded (2 s); on expiry the kernel records MOE_ERR_TIMEOUT,
// the other roles see it and stop, in-flight copies and MMAs are waited for
// (bounded) and the tensor memory is freed.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include "common.cuh"
#include "grouped.cuh"
#include "layer_fused.cuh"
#include "ptx.cuh"

namespace moeq4 {

constexpr int kMmaRows = 128;                          // M: weight rows per CTA (TMEM lanes)
constexpr int kMmaTok = 64;                            // N: tokens per tile
constexpr int kMmaK = 64;                              // K per stage (one scale group)
constexpr int kMmaABytes = kMmaRows * kMmaK * 2;       // one 16-bit A tile (16 KB)
constexpr int kMmaBBytes = kMmaTok * kMmaK * 2;        // one 16-bit B plane tile (8 KB)
constexpr int kMmaDefaultMinTokens = 4;                // bucket size from which a routed expert runs here
constexpr int kMmaMinStep = 32;                        // tokens in a step before any expert runs here

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

__device__ __forceinline__ float4 lds128f(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// Waits for an mbarrier phase with a time bound only (used while draining
// after a failure, when the status word is already set).
__device__ __forceinline__ void mma_drain_wait(uint64_t* bar, uint32_t parity) {
    const unsigned long long t0 = gtimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (gtimer_ns() - t0 > kWaitNs) return;
    }
}


constexpr int kTcWarps = 18;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcABufs = 3;                            // A tiles (one per stage in flight)
constexpr int kTcAccBufs = 4;                          // TMEM accumulators of 64 columns
constexpr int kTcCodes = kMmaRows * kMmaK / 2;         // codes of one stage (4 KB)

template <bool DOWN>
struct TcShape {
    static constexpr int kRing = DOWN ? 6 : 8;                         // ring slots
    static constexpr int kBBytes = DOWN ? 2 * kMmaBBytes : kMmaBBytes;  // B tile (hi, lo planes)
    static constexpr int kSlot = kBBytes + kTcCodes;                   // multiple of 1024
};

// Dynamic shared memory of k_ffn_tc for reduction length K: ring, A tiles,
// scales and biases (4 K bytes each), the tile's group sums (4 K bytes),
// alignment slack.
template <bool DOWN>
__host__ __device__ constexpr size_t tc_smem_bytes(int K) {
    return (size_t)TcShape<DOWN>::kRing * TcShape<DOWN>::kSlot + (size_t)kTcABufs * kMmaABytes +
           12 * (size_t)K + 1024;
}

// kind::f16 instruction descriptors (M = 128, N = 64, D fp32, K-major A/B):
// fp16 operands (A/B format 0) and bf16 operands (format 1).
constexpr uint32_t kTcIdescF16 = (1u << 4) | ((uint32_t)(kMmaTok >> 3) << 17) |
                                 ((uint32_t)(kMmaRows >> 4) << 24);
constexpr uint32_t kTcIdescBF16 = kTcIdescF16 | (1u << 7) | (1u << 10);

// Shared-memory descriptor of a K-major tile written by a tiled copy with
// 128-byte swizzle (rows of 128 bytes, 8-row atoms of 1024 bytes): start
// address >> 4, leading byte offset 1 (unused within one swizzle atom of K),
// stride byte offset 1024 >> 4, version 1, layout type 2 (128-byte swizzle).
// The tile base is 1024-byte aligned; a K step of 16 elements adds 32 bytes
// to the start address.
__device__ __forceinline__ uint64_t tc_sdesc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) |
           (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accum)
        : "memory");
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

// Tiled global -> shared copies (no cluster multicast), completion counted on bar.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}
// Untiled bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s_u32(uint32_t dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void sts32f(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Eight 4-bit codes of one word as eight exact fp16 values (1024 + q in the
// mantissa, minus 1024).
__device__ __forceinline__ uint4 tc_codes_f16(uint32_t w) {
    const __half2 k1024 = __floats2half2_rn(1024.f, 1024.f);
    uint32_t o[4];
#pragma unroll
    for (int p = 0; p < 4; p++) {
        const uint32_t q0 = (w >> (8 * p)) & 0xFu, q1 = (w >> (8 * p + 4)) & 0xFu;
        const uint32_t v = 0x64006400u | q0 | (q1 << 16);
        const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&v), k1024);
        o[p] = *reinterpret_cast<const uint32_t*>(&q);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Rows r < T + T k of the gate/up B operand: r < T is token r (shared
// expert), r = T + i is the token of the i-th pair in bucket order
// (list[i] / k).  Copies the fp16 row into xs[r] and writes its 64-column
// group sums gsum[r][g] (fp32).  One warp per 256 columns; grid y strides
// over the rows.
__global__ void k_gather_x(const __half* __restrict__ x, int H, int T, int k, int rows,
                           const int* __restrict__ list, __half* __restrict__ xs,
                           float* __restrict__ gsum) {
    const int lane = threadIdx.x & 31;
    const int c0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 256 + 8 * lane;
    if (c0 - 8 * lane >= H) return;                       // whole warp past the row end
    for (int r = blockIdx.y; r < rows; r += gridDim.y) {
        const int tok = r < T ? r : list[r - T] / k;
        float s = 0.f;
        if (c0 < H) {
            const uint4 v = *reinterpret_cast<const uint4*>(x + (size_t)tok * H + c0);
            *reinterpret_cast<uint4*>(xs + (size_t)r * H + c0) = v;
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int p = 0; p < 4; p++) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[p]));
                s += f.x + f.y;
            }
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if (c0 < H && (lane & 7) == 0) gsum[(size_t)r * (H / 64) + c0 / 64] = s;
    }
}

struct TcArgs {
    int H, Ie, T, k, min_tok, gelu;
    const int* e_off;
    const int* list;
    const float* b_sum;      // group sums of the B rows [rows][bs_stride]
    int bs_stride;
    __nv_bfloat16* h_hi;     // gate/up output planes [rows][hs]
    __nv_bfloat16* h_lo;
    float* h_sum;            // gate/up output group sums [rows][hs / 64]
    int hs;
    float* y_pairs;          // down output [pair rows][H]
    int* status;
};

// Tensor-core FFN half over expert token buckets, warp-specialised.
//   DOWN = false (gate/up): strip sb = 4 gate/up tiles (A row 32 j + r: tile
//     4 sb + j, row r; r < 16 gate, else up, of intermediate index
//     i = 64 sb + 16 j + r % 16); K = H; B = gathered x rows (fp16).  Writes
//     h = GELU(gate) * up as bf16 hi/lo planes at row `brow` (the B row of
//     the token: t for the shared expert, T + bucket position for a routed
//     pair) and the group sums h_sum[brow][sb].
//   DOWN = true: strip sb = output rows 128 sb .. + 127; K = Ie; B = the h
//     planes; writes y_pairs[pair row][o] (fp32).
// tm_codes: the 128 rows' codes ([tile][row][32 bytes] per stage, experts as
// the last dimension); tm_b: the B rows (64 columns x 64 rows per stage,
// 128-byte swizzle; down: both planes).  Routed (SHARED = false): expert
// blockIdx.y, skipped unless its bucket holds at least min_tok pairs.  Token
// tiles of 64: z = blockIdx.z, + gridDim.z, ...  grid (Ie / 64 or H / 128,
// experts or 1, tiles), block kTcThreads, dynamic shared memory
// tc_smem_bytes<DOWN>(K).
template <bool DOWN, bool SHARED>
__global__ void __launch_bounds__(kTcThreads, 1)
k_ffn_tc(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_b,
         const uint8_t* __restrict__ experts, size_t stride, const uint8_t* __restrict__ shared_blob,
         const TcArgs a) {
    using S = TcShape<DOWN>;
    constexpr int R = S::kRing;
    extern __shared__ uint8_t tsm_raw[];
    __shared__ __align__(8) uint64_t full_slot[R], empty_slot[R], full_a[kTcABufs], empty_a[kTcABufs];
    __shared__ __align__(8) uint64_t acc_full[kTcAccBufs], acc_empty[kTcAccBufs], sc_full;
    __shared__ uint32_t s_tmem;
    __shared__ int s_row[kMmaTok];
    __shared__ float s_red[4][kMmaTok];

    const int H = a.H, Ie = a.Ie, T = a.T;
    int n = T, base = 0, e = 0;
    const uint8_t* blob = shared_blob;
    if (!SHARED) {
        e = blockIdx.y;
        base = a.e_off[e];
        n = a.e_off[e + 1] - base;
        if (n < a.min_tok) return;
        blob = experts + (size_t)e * stride;
    }
    if ((int)blockIdx.z * kMmaTok >= n) return;
    const int brow0 = SHARED ? 0 : T + base;              // first B row of the bucket

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = DOWN ? Ie : H, nk = K / kMmaK;
    const uint32_t sbase = (smem_u32(tsm_raw) + 1023u) & ~1023u;
    const uint32_t s_ring = sbase, s_a = sbase + R * S::kSlot;
    const uint32_t s_sc = s_a + kTcABufs * kMmaABytes, s_bi = s_sc + 4 * K, s_gs = s_bi + 4 * K;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s_tmem)),
                     "r"(256)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int i = 0; i < R; i++) {
            mbar_init(&full_slot[i], 1);
            mbar_init(&empty_slot[i], 8 + 1);             // 8 converter warps + the MMA commit
        }
        for (int i = 0; i < kTcABufs; i++) {
            mbar_init(&full_a[i], 8);                     // converter warps
            mbar_init(&empty_a[i], 1);                    // MMA commit
        }
        for (int i = 0; i < kTcAccBufs; i++) {
            mbar_init(&acc_full[i], 1);                   // MMA commit
            mbar_init(&acc_empty[i], 8);                  // folder warps
        }
        mbar_init(&sc_full, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const BlobLayout L(H, Ie);
    int* status = a.status;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0) {
            // scales and biases of the strip: whole per-tile blocks
            mbar_arrive_expect_tx(&sc_full, 8u * K);
            if (!DOWN) {
                for (int j = 0; j < 4; j++) {
                    const uint8_t* tb = blob + (size_t)(4 * blockIdx.x + j) * L.gu_tile;
                    bulk_g2s_u32(s_sc + j * H, tb + 16 * (size_t)H, H, &sc_full);
                    bulk_g2s_u32(s_bi + j * H, tb + 17 * (size_t)H, H, &sc_full);
                }
            } else {
                for (int j = 0; j < 8; j++) {
                    const uint8_t* tb = blob + L.dn_base + (size_t)(8 * blockIdx.x + j) * L.dn_tile;
                    bulk_g2s_u32(s_sc + j * (Ie / 2), tb + 8 * (size_t)Ie, Ie / 2, &sc_full);
                    bulk_g2s_u32(s_bi + j * (Ie / 2), tb + 8 * (size_t)Ie + Ie / 2, Ie / 2, &sc_full);
                }
            }
            uint32_t g = 0;
            for (int z = blockIdx.z; ok && z * kMmaTok < n; z += gridDim.z) {
                const int brow = brow0 + z * kMmaTok;
                for (int c = 0; c < nk; c++, g++) {
                    const uint32_t slot = g % R, use = g / R;
                    if (!fused_wait_bar(&empty_slot[slot], (use & 1u) ^ 1u, status)) { ok = false; break; }
                    const uint32_t sl = s_ring + slot * S::kSlot;
                    mbar_arrive_expect_tx(&full_slot[slot], (uint32_t)S::kSlot);
                    tma_load_4d(sl + S::kBBytes, &tm_codes, 32 * c, 0, (DOWN ? 8 : 4) * (int)blockIdx.x,
                                e, &full_slot[slot]);
                    tma_load_3d(sl, &tm_b, kMmaK * c, brow, 0, &full_slot[slot]);   // both planes (down)
                }
            }
            // copies still in flight land before the CTA ends
            if (g > 0) mma_drain_wait(&full_slot[(g - 1) % R], ((g - 1) / R) & 1u);
            mma_drain_wait(&sc_full, 0);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer --
        if (lane == 0) {
            uint32_t g = 0;
            for (int z = blockIdx.z; ok && z * kMmaTok < n; z += gridDim.z) {
                for (int c = 0; c < nk; c++, g++) {
                    const uint32_t slot = g % R, ab = g % kTcABufs, tb = g % kTcAccBufs;
                    if (!fused_wait_bar(&full_slot[slot], (g / R) & 1u, status) ||
                        !fused_wait_bar(&full_a[ab], (g / kTcABufs) & 1u, status) ||
                        !fused_wait_bar(&acc_empty[tb], ((g / kTcAccBufs) & 1u) ^ 1u, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sl = s_ring + slot * S::kSlot;
                    const uint32_t aa = s_a + ab * kMmaABytes;
                    const uint32_t d = tmem + 64u * tb;
#pragma unroll
                    for (int kk = 0; kk < kMmaK / 16; kk++) {
                        const uint64_t da = mma_sdesc(aa + 256u * kk);
                        if (DOWN) {
                            tc_mma(d, da, tc_sdesc_sw128(sl + 32u * kk), kTcIdescBF16, kk > 0 ? 1u : 0u);
                            tc_mma(d, da, tc_sdesc_sw128(sl + kMmaBBytes + 32u * kk), kTcIdescBF16, 1u);
                        } else {
                            tc_mma(d, da, tc_sdesc_sw128(sl + 32u * kk), kTcIdescF16, kk > 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(&empty_a[ab]);
                    mma_commit(&empty_slot[slot]);
                    mma_commit(&acc_full[tb]);
                }
            }
            if (g > 0) {                                  // every commit has arrived before the CTA ends
                mma_drain_wait(&acc_full[(g - 1) % kTcAccBufs], ((g - 1) / kTcAccBufs) & 1u);
                mma_drain_wait(&empty_a[(g - 1) % kTcABufs], ((g - 1) / kTcABufs) & 1u);
                mma_drain_wait(&empty_slot[(g - 1) % R], ((g - 1) / R) & 1u);
            }
        }
    } else if (warp < 10) {
        // ---------------------------------------------------- converters --
        const int u = tid - 64, m = u & 127, hh = u >> 7;  // row m, 32 columns 32 hh .. + 31
        uint32_t g = 0;
        for (int z = blockIdx.z; ok && z * kMmaTok < n; z += gridDim.z) {
            for (int c = 0; c < nk; c++, g++) {
                const uint32_t slot = g % R, ab = g % kTcABufs;
                if (!fused_wait_bar(&full_slot[slot], (g / R) & 1u, status) ||
                    !fused_wait_bar(&empty_a[ab], ((g / kTcABufs) & 1u) ^ 1u, status)) {
                    ok = false;
                    break;
                }
                const uint32_t sl = s_ring + slot * S::kSlot;
                const uint4 w = lds128(sl + S::kBBytes + m * 32 + 16 * hh);
                const uint32_t aa = s_a + ab * kMmaABytes;
                const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q = 0; q < 4; q++)
                    sts128(aa + mma_granule(m, 4 * hh + q), DOWN ? mma_codes_bf16(wv[q]) : tc_codes_f16(wv[q]));
                fence_proxy_async_smem();                 // A tile -> tensor core
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&full_a[ab]);
                    mbar_arrive(&empty_slot[slot]);
                }
            }
        }
    } else {
        // ------------------------------------------------------- folders --
        const int v = tid - 320;                          // 0 .. 255
        const int fj = warp & 3, ch = (warp - 10) >> 2;   // TMEM lane quarter, column half
        const int fm = 32 * fj + lane;                    // A row (TMEM lane)
        const uint32_t t_lane = tmem + ((uint32_t)(32 * fj) << 16) + 32u * ch;
        if (!fused_wait_bar(&sc_full, 0, status)) ok = false;
        uint32_t g = 0;
        for (int z = blockIdx.z; ok && z * kMmaTok < n; z += gridDim.z) {
            const int t0 = z * kMmaTok, nt = min(kMmaTok, n - t0);
            const int brow = brow0 + t0;
            named_sync(1, 256);                           // the previous tile is done with s_gs, s_row
            for (int p = v; p < kMmaTok * nk; p += 256) {
                const int t = p & (kMmaTok - 1), gg = p >> 6;
                sts32f(s_gs + 4u * p, t < nt ? a.b_sum[(size_t)(brow + t) * a.bs_stride + gg] : 0.f);
            }
            if (DOWN && v < kMmaTok)
                s_row[v] = v < nt ? grp_row(SHARED, a.list, base, t0 + v, T) : -1;
            named_sync(1, 256);
            const bool on = 32 * ch < nt;                 // warp-uniform
            float acc[32];
#pragma unroll
            for (int q = 0; q < 32; q++) acc[q] = 0.f;
            for (int c = 0; c < nk; c++, g++) {
                const uint32_t tb = g % kTcAccBufs;
                if (!fused_wait_bar(&acc_full[tb], (g / kTcAccBufs) & 1u, status)) { ok = false; break; }
                tc_fence_after();
                if (on) {
                    float P[32];
                    tmem_ld32(t_lane + 64u * tb, P);
                    const uint32_t so = (uint32_t)fm * (K / 32) + 2 * c;
                    const float sc = __half2float(__ushort_as_half(lds16(s_sc + so)));
                    const float bi = __half2float(__ushort_as_half(lds16(s_bi + so)));
                    const uint32_t ga = s_gs + 4u * (c * kMmaTok + 32 * ch);
#pragma unroll
                    for (int q4 = 0; q4 < 8; q4++) {
                        const float4 Sg = lds128f(ga + 16 * q4);
                        acc[4 * q4 + 0] = fmaf(sc, P[4 * q4 + 0], fmaf(bi, Sg.x, acc[4 * q4 + 0]));
                        acc[4 * q4 + 1] = fmaf(sc, P[4 * q4 + 1], fmaf(bi, Sg.y, acc[4 * q4 + 1]));
                        acc[4 * q4 + 2] = fmaf(sc, P[4 * q4 + 2], fmaf(bi, Sg.z, acc[4 * q4 + 2]));
                        acc[4 * q4 + 3] = fmaf(sc, P[4 * q4 + 3], fmaf(bi, Sg.w, acc[4 * q4 + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[tb]);
            }
            if (!ok) break;
            if (!DOWN) {
                const int i = 64 * (int)blockIdx.x + 16 * fj + (lane & 15);
                const int hs = a.hs;
                if (on) {
#pragma unroll
                    for (int q = 0; q < 32; q++) {
                        const float up = __shfl_xor_sync(0xffffffffu, acc[q], 16);
                        const int col = 32 * ch + q;
                        float part = 0.f;
                        if (lane < 16 && col < nt) {
                            uint32_t hh2, hl2;
                            mma_split2(gelu_f(acc[q], a.gelu) * up, 0.f, hh2, hl2);
                            const __nv_bfloat16 bh = __ushort_as_bfloat16((unsigned short)(hh2 & 0xFFFFu));
                            const __nv_bfloat16 bl = __ushort_as_bfloat16((unsigned short)(hl2 & 0xFFFFu));
                            const size_t o = (size_t)(brow + col) * hs + i;
                            a.h_hi[o] = bh;
                            a.h_lo[o] = bl;
                            part = __bfloat162float(bh) + __bfloat162float(bl);
                        }
                        part += __shfl_xor_sync(0xffffffffu, part, 8);
                        part += __shfl_xor_sync(0xffffffffu, part, 4);
                        part += __shfl_xor_sync(0xffffffffu, part, 2);
                        part += __shfl_xor_sync(0xffffffffu, part, 1);
                        if (lane == 0) s_red[fj][col] = part;
                    }
                }
                named_sync(1, 256);
                if (v < nt)
                    a.h_sum[(size_t)(brow + v) * (hs / 64) + blockIdx.x] =
                        ((s_red[0][v] + s_red[1][v]) + s_red[2][v]) + s_red[3][v];
            } else if (on) {
                const int o = kMmaRows * (int)blockIdx.x + fm;
#pragma unroll
                for (int q = 0; q < 32; q++) {
                    const int col = 32 * ch + q;
                    if (col < nt) a.y_pairs[(size_t)s_row[col] * H + o] = acc[q];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256)
                     : "memory");
    }
}

}  // namespace moeq4
