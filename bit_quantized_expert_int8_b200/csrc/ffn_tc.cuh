// ffn_tc.cuh -- expert FFN on the tensor cores (tcgen05 MMAs, operands and
// accumulators in tensor memory, tiles staged by TMA) for steps of many
// tokens.
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
// fp16 operands (codes and the fp16 x are both exact: every product exact,
// sums in fp32).  The down projection takes the fp32 intermediate h as two
// bf16 planes, h = hi + lo (hi = bf16(h), lo = bf16(h - hi), 16 significant
// bits), and runs two bf16 MMAs per K = 16.  Rounding the dequantised
// weight s q + b to one 16-bit value instead would miss the absolute
// tolerance on heavy-tailed rows, which is why the fold stays.
//
// On B200 a 128 x N x 16 MMA costs the same ~24 ns for every N up to 64, so
// the MMA count (rows / 128 x K / 16 per token tile) sets the floor, and the
// kernel is built so that nothing else waits: one persistent CTA per SM walks
// a list of work items (expert, 128-row strip, token tile of <= 64) without
// draining its pipeline between items, in stages of 128 columns (two scale
// groups, one MMA commit per stage).  Roles, meeting only at mbarriers:
//   warp 0       TMA producer: per item the strip's scales and biases and the
//                tile's group sums (one bulk copy each block, into one of three
//                item buffers); per stage one tiled copy of the 128 rows'
//                codes (8 KB, 64-byte swizzle) and two of the B tile (two
//                64-column halves, 128-byte swizzle; down: both planes) sized
//                to the tile (16, 32 or 64 rows);
//   warp 1       MMA issuers (lanes 0 and 1, one scale group each): per
//                stage 4 (down: 8) MMAs per group with A in tensor memory,
//                then each lane's commit; the two publish the stage's
//                accumulators and free its ring slot and A buffer;
//   warps 2..5   converters: codes -> 16-bit A straight into tensor memory
//                (tcgen05.st, one row per thread), so A costs no shared-
//                memory bandwidth;
//   warps 6..13  folders: accumulator -> registers (acc += s P + b S), and the
//                epilogue of each item; the two warps of a TMEM lane quarter
//                take half of the item's columns each.
// Within each 8 columns the A operand holds the codes in the order
// 0 4 1 5 2 6 3 7 (two shifts and a mask per pair); every B operand is
// written in that order (k_gather_x for x, the gate/up epilogue for h).
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

constexpr int kMmaRows = 128;                          // M: weight rows per item (TMEM lanes)
constexpr int kMmaTok = 64;                            // tokens per item at most (N: rounded up to 16)
constexpr int kMmaDefaultMinTokens = 1;                // bucket size from which a routed expert runs here
constexpr int kMmaMinStep = 2;                         // tokens in a step before any expert runs here (measured)
constexpr int kTcStageK = 128;                         // K per pipeline stage: two scale groups
constexpr int kTcCodeBytes = kMmaRows * kTcStageK / 2; // codes of one stage (8 KB)
constexpr int kTcWarps = 14;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcAcc = 8;                              // accumulator stages in flight at most
constexpr uint32_t kTcAccCols = 256;                   // TMEM columns of the accumulator ring
constexpr int kTcItemBufs = 3;                         // per-item scale / group-sum buffers
constexpr uint32_t kTcAccCol = 256;                    // first TMEM column of the accumulators

template <bool DOWN>
struct TcShape {
    static constexpr int kRing = DOWN ? 3 : 4;                         // ring slots (and A buffers)
    static constexpr int kPlanes = DOWN ? 2 : 1;                       // B planes (h hi, lo)
    static constexpr int kBBytes = 2 * kMmaTok * 128 * kPlanes;         // two 64-column halves
    static constexpr int kSlot = kTcCodeBytes + kBBytes;               // multiple of 1024
};

// Per-item buffer: scales and biases of the strip (8 K bytes: 128 rows x
// K / 64 groups x 2 values x 2 bytes) and the tile's group sums (64 rows of
// gs_stride floats).
__host__ __device__ constexpr size_t tc_item_bytes(int K, int gs_stride) {
    return ((size_t)8 * K + (size_t)kMmaTok * gs_stride * 4 + 1023) / 1024 * 1024;
}

// Dynamic shared memory of k_ffn_tc for the longest reduction kmax.
template <bool DOWN>
__host__ __device__ constexpr size_t tc_smem_bytes(int kmax, int gs_stride) {
    return (size_t)TcShape<DOWN>::kRing * TcShape<DOWN>::kSlot +
           (size_t)kTcItemBufs * tc_item_bytes(kmax, gs_stride) + 1024;
}

// kind::f16 instruction descriptors (M = 128, D fp32, K-major A and B; N is
// or-ed in per item as N / 8 at bit 17): fp16 operands (A/B format 0) and
// bf16 operands (format 1).
constexpr uint32_t kTcIdescF16 = (1u << 4) | ((uint32_t)(kMmaRows >> 4) << 24);
constexpr uint32_t kTcIdescBF16 = kTcIdescF16 | (1u << 7) | (1u << 10);

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

// D (TMEM) (+)= A (TMEM, 128 lanes x 16 K) * B (shared memory descriptor).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                          uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum)
        : "memory");
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

// 8 consecutive fp32 columns of this thread's TMEM lane (column a multiple
// of 8), without waiting (tmem_ld_wait() before the registers are read).
__device__ __forceinline__ void tmem_ld8_nw(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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

// Waits for an mbarrier phase with a time bound only (used while draining
// after a failure, when the status word is already set).
__device__ __forceinline__ void mma_drain_wait(uint64_t* bar, uint32_t parity) {
    const unsigned long long t0 = gtimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (gtimer_ns() - t0 > kWaitNs) return;
    }
}

// Eight 4-bit codes of one word (column 8 w + i in nibble i) as four 16-bit
// pairs, pair j = (column j, column j + 4): the tensor-core K order within
// each 8 columns is 0 4 1 5 2 6 3 7.  1024 + q (fp16) or 128 + q (bf16)
// carries q in its mantissa; the offset is subtracted exactly.
template <bool BF16>
__device__ __forceinline__ void tc_codes(uint32_t w, uint32_t* o) {
#pragma unroll
    for (int j = 0; j < 4; j++) {
        uint32_t v = ((w >> (4 * j)) & 0x000F000Fu) | (BF16 ? 0x43004300u : 0x64006400u);
        if (BF16) {
            const __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v),
                                             __floats2bfloat162_rn(128.f, 128.f));
            o[j] = *reinterpret_cast<const uint32_t*>(&q);
        } else {
            const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&v), __floats2half2_rn(1024.f, 1024.f));
            o[j] = *reinterpret_cast<const uint32_t*>(&q);
        }
    }
}

// GELU of the gate for the tensor-core epilogue.  The tanh form uses
// tanh(u) = 1 - 2 / (e^(2u) + 1) with the hardware exponential (absolute
// error of tanh near 1e-6, far below the tolerance); 2u is capped at 60,
// where tanh is 1 in fp32.  The erf form calls erff.
__device__ __forceinline__ float tc_gelu(float g, int variant) {
    if (variant == MOE_GELU_ERF) return 0.5f * g * (1.0f + erff(g * 0.70710678118654752f));
    const float u = 0.79788456080286536f * (g + 0.044715f * g * g * g);
    const float e = __expf(fminf(2.0f * u, 60.0f));
    return 0.5f * g * (2.0f - __fdividef(2.0f, e + 1.0f));
}

// Position of column c in a B row: the tensor-core order within each 8.
__device__ __forceinline__ int tc_col_pos(int c) {
    return (c & ~7) | ((c & 3) << 1) | ((c >> 2) & 1);
}

// Rows r < T + T k of the gate/up B operand: r < T is token r (shared
// expert), r = T + i is the token of the i-th pair in bucket order
// (list[i] / k).  Copies the fp16 row into xs[r] with each 8 columns in the
// tensor-core order and writes its 64-column group sums gsum[r][g] (fp32,
// row stride gs_stride).  n_pairs (device, or null for all T k): the pairs
// the list holds, when a grouping selected only some of them.  One warp per
// 256 columns; grid y strides over the rows.
__global__ void k_gather_x(const __half* __restrict__ x, int H, int T, int k, int rows,
                           const int* __restrict__ list, __half* __restrict__ xs,
                           float* __restrict__ gsum, int gs_stride, const int* __restrict__ n_pairs) {
    const int lane = threadIdx.x & 31;
    const int c0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 256 + 8 * lane;
    if (c0 - 8 * lane >= H) return;                       // whole warp past the row end
    if (n_pairs) rows = min(rows, T + *n_pairs);
    for (int r = blockIdx.y; r < rows; r += gridDim.y) {
        const int tok = r < T ? r : list[r - T] / k;
        float s = 0.f;
        if (c0 < H) {
            const uint4 v = *reinterpret_cast<const uint4*>(x + (size_t)tok * H + c0);
            uint4 o;
            o.x = __byte_perm(v.x, v.z, 0x5410);          // columns 0, 4
            o.y = __byte_perm(v.x, v.z, 0x7632);          // 1, 5
            o.z = __byte_perm(v.y, v.w, 0x5410);          // 2, 6
            o.w = __byte_perm(v.y, v.w, 0x7632);          // 3, 7
            *reinterpret_cast<uint4*>(xs + (size_t)r * H + c0) = o;
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
        if (c0 < H && (lane & 7) == 0) gsum[(size_t)r * gs_stride + c0 / 64] = s;
    }
}

struct TcArgs {
    int H, T, k, E, gelu;
    int Ir, Is;              // intermediate sizes: routed experts, shared expert
    int kmax;                // longest reduction of the launch (sizes the item buffers)
    int min_tok;             // routed buckets with fewer pairs stay on the CUDA cores
    int do_shared;           // shared expert items included
    const int* e_off;
    const int* list;
    const float* b_sum;      // group sums of the B rows [rows][bs_stride] (bs_stride % 4 == 0)
    int bs_stride;
    __nv_bfloat16* h_hi;     // gate/up output planes [rows][hs]
    __nv_bfloat16* h_lo;
    float* h_sum;            // gate/up output group sums [rows][hsum_stride]
    int hs, hsum_stride;
    float* y_pairs;          // down output [pair rows][H]
    int* status;
};

// One work item: expert (or the shared expert), strip of 128 weight rows
// (gate/up: 64 intermediate indices as 4 tiles of 16 gate + 16 up rows;
// down: 128 output rows), token tile t0 .. t0 + nt of its bucket.
struct TcItem {
    int shared, e, sb, n, base, t0, nt, npad, brow, K, ng, nst;
};

// Item `it` of the launch: s_ioff[0] = 0, s_ioff[j + 1] = s_ioff[j] + items
// of entry j (entry 0 the shared expert, entry e + 1 routed expert e).
template <bool DOWN>
__device__ __forceinline__ TcItem tc_item(int it, const int* s_ioff, const int* s_eoff, const TcArgs& a) {
    int lo = 0, hi = a.E;                                 // largest j with s_ioff[j] <= it
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_ioff[mid] <= it) lo = mid;
        else hi = mid - 1;
    }
    TcItem d;
    d.shared = lo == 0;
    d.e = lo - 1;
    const int Ie = d.shared ? a.Is : a.Ir;
    const int strips = DOWN ? a.H / kMmaRows : Ie / 64;
    const int rem = it - s_ioff[lo];
    d.sb = rem % strips;
    d.base = d.shared ? 0 : s_eoff[d.e];
    d.n = d.shared ? a.T : s_eoff[d.e + 1] - d.base;
    d.t0 = (rem / strips) * kMmaTok;
    d.nt = min(kMmaTok, d.n - d.t0);
    d.npad = (d.nt + 15) & ~15;
    d.brow = (d.shared ? 0 : a.T + d.base) + d.t0;
    d.K = DOWN ? Ie : a.H;
    d.ng = d.K / 64;
    d.nst = (d.ng + 1) / 2;
    return d;
}

__device__ __forceinline__ int tc_brows(int npad) { return npad <= 16 ? 16 : npad <= 32 ? 32 : 64; }

// Accumulator ring: each stage takes two group accumulators of gstride
// columns (npad for 16 and 32 tokens, 64 above) from a circular run of
// kTcAccCols TMEM columns; a stage that would wrap starts at column 0 and
// the skipped tail counts as consumed.  `cum` counts consumed columns, so
// the stages between the last one released and stage g fit while
// cum(g) - cum(released) <= kTcAccCols.  Every role advances the same state.
struct TcAccRing {
    uint32_t cur = 0, cum = 0;
    __device__ __forceinline__ uint32_t take(uint32_t w) {
        if (cur + w > kTcAccCols) { cum += kTcAccCols - cur; cur = 0; }
        const uint32_t start = cur;
        cur += w;
        cum += w;
        return start;
    }
};
__device__ __forceinline__ uint32_t tc_gstride(int npad) { return npad <= 32 ? (uint32_t)npad : 64u; }

// State of one folder thread (warps 6..13).
struct TcFold {
    const TcArgs* a;
    int* status;
    uint32_t g;              // stages consumed so far
    int m, q4, half, lane, tid;
    uint32_t t_acc0;         // TMEM address of this lane quarter's accumulators
    uint64_t* acc_empty;
    uint64_t* acc_full;
    TcAccRing ring;
    uint64_t* red_full;
    float (*s_red)[2][4][32];
};

// One item of a folder thread: CW = npad / 2 columns from column half * CW,
// both groups of every stage, then the epilogue (gate/up: h planes and their
// group sums; down: y rows).  ibp: the item's scale / group-sum buffer.
// Returns the updated stage count, or -1 after a failed wait.  Up to CW
// columns are loaded and folded, in chunks of 16 (8 for CW = 8) that start
// below the warp's own npad / 2 columns: every load stays inside the stage's
// group accumulators (a 24-column half of 48 tokens reads 32 columns of its
// 64-column group).  The epilogue stores the npad / 2 columns.
template <bool DOWN, int R, int CW>
__device__ __forceinline__ int tc_fold_item(TcFold& f, const TcItem& d, int j, const uint8_t* ibp) {
    const TcArgs& a = *f.a;
    const int cw = d.npad >> 1;                       // columns of this warp (8, 16, 24 or 32)
    const int c0 = f.half * cw;                       // its first column (a multiple of 8)
    const bool on = c0 < d.nt;                        // warp-uniform
    uint32_t g = f.g;
    const uint32_t gst = tc_gstride(d.npad);        // column stride of the stage's two groups
    const int ngr = d.K / 64;                         // groups per row
    const __half* scp = reinterpret_cast<const __half*>(ibp) + f.m * ngr;   // [row][group]
    const __half* bip = reinterpret_cast<const __half*>(ibp + 4 * d.K) + f.m * ngr;
    const float* gsp = reinterpret_cast<const float*>(ibp + 8 * d.K) + c0 * a.bs_stride;  // [t][group]
    const bool pair_sc = (ngr & 1) == 0;              // a row's scale pairs are 4-byte aligned
    const int bs = a.bs_stride;
    int rrow = 0;                                     // down: output row of column c0 + lane
    if (DOWN && on && f.lane < cw) {
        const int i = d.t0 + c0 + f.lane;
        if (i < d.n) rrow = grp_row(d.shared, a.list, d.base, i, a.T);
    }
    float acc[CW];
#pragma unroll
    for (int q = 0; q < CW; q++) acc[q] = 0.f;
    const uint32_t t_acc = f.t_acc0 + (uint32_t)c0;
    if (CW == 8) {
        // 8 columns: up to 2 stages per TMEM load batch (one wait on the last
        // stage's commit, which follows every earlier MMA)
        constexpr int NB = 2;
        for (int c = 0; c < d.nst;) {
            const int nb = min(NB, d.nst - c);
            uint32_t acol[NB];
#pragma unroll
            for (int b = 0; b < NB; b++) acol[b] = b < nb ? f.ring.take(2 * gst) : 0u;
            const uint32_t gl = g + (uint32_t)nb - 1;
            if (!fused_wait_bar(&f.acc_full[gl % kTcAcc], (gl / kTcAcc) & 1u, f.status)) return -1;
            tc_fence_after();
            uint32_t P[NB][2][8];
            if (on) {
#pragma unroll
                for (int b = 0; b < NB; b++) {
                    if (b < nb) {
                        tmem_ld8_nw(t_acc + acol[b], P[b][0]);
                        if (d.ng - 2 * (c + b) > 1) tmem_ld8_nw(t_acc + acol[b] + gst, P[b][1]);
                    }
                }
                tmem_ld_wait();
            }
            tc_fence_before();                        // the accumulators are free once in registers
            __syncwarp();
            if (f.lane == 0) {
                for (int b = 0; b < nb; b++) mbar_arrive(&f.acc_empty[(g + b) % kTcAcc]);
            }
            if (on) {
#pragma unroll
                for (int b = 0; b < NB; b++) {
                    if (b < nb) {
                        const int G = 2 * (c + b);
                        if (d.ng - G > 1) {
                            float s0, s1, b0, b1;
                            if (pair_sc) {
                                const float2 sc2 = __half22float2(*reinterpret_cast<const __half2*>(scp + G));
                                const float2 bi2 = __half22float2(*reinterpret_cast<const __half2*>(bip + G));
                                s0 = sc2.x; s1 = sc2.y; b0 = bi2.x; b1 = bi2.y;
                            } else {
                                s0 = __half2float(scp[G]); s1 = __half2float(scp[G + 1]);
                                b0 = __half2float(bip[G]); b1 = __half2float(bip[G + 1]);
                            }
#pragma unroll
                            for (int q = 0; q < 8; q++) {
                                const float2 S2 = *reinterpret_cast<const float2*>(gsp + q * bs + G);
                                float v = fmaf(b0, S2.x, acc[q]);
                                v = fmaf(s0, __uint_as_float(P[b][0][q]), v);
                                v = fmaf(b1, S2.y, v);
                                acc[q] = fmaf(s1, __uint_as_float(P[b][1][q]), v);
                            }
                        } else {
                            const float s0 = __half2float(scp[G]), b0 = __half2float(bip[G]);
#pragma unroll
                            for (int q = 0; q < 8; q++)
                                acc[q] = fmaf(s0, __uint_as_float(P[b][0][q]), fmaf(b0, gsp[q * bs + G], acc[q]));
                        }
                    }
                }
            }
            c += nb;
            g += (uint32_t)nb;
        }
    } else {
    for (int c = 0; c < d.nst; c++, g++) {
        const uint32_t ab = g % kTcAcc;
        const uint32_t acol = f.ring.take(2 * gst);
        if (!fused_wait_bar(&f.acc_full[ab], (g / kTcAcc) & 1u, f.status)) return -1;
        tc_fence_after();
        const bool two = d.ng - 2 * c > 1;            // the second group of the stage exists
        const int G = 2 * c;
        float s0 = 0.f, s1 = 0.f, b0 = 0.f, b1 = 0.f;
        if (on) {
            if (two && pair_sc) {
                const float2 sc2 = __half22float2(*reinterpret_cast<const __half2*>(scp + G));
                const float2 bi2 = __half22float2(*reinterpret_cast<const __half2*>(bip + G));
                s0 = sc2.x; s1 = sc2.y; b0 = bi2.x; b1 = bi2.y;
            } else {
                s0 = __half2float(scp[G]); b0 = __half2float(bip[G]);
                if (two) { s1 = __half2float(scp[G + 1]); b1 = __half2float(bip[G + 1]); }
            }
        }
        // chunks of LC columns: both groups loaded, one wait, then folded; the
        // accumulator is released after the last chunk's wait
        constexpr int LC = CW < 16 ? CW : 16;
        const uint32_t ta = t_acc + acol;
#pragma unroll
        for (int k = 0; k < CW / LC; k++) {
            uint32_t P0[LC], P1[LC];
            const bool ck = on && (k == 0 || LC * k < cw);   // warp-uniform
            if (ck) {
#pragma unroll
                for (int u = 0; u < LC / 8; u++) tmem_ld8_nw(ta + (uint32_t)(LC * k + 8 * u), P0 + 8 * u);
                if (two) {
#pragma unroll
                    for (int u = 0; u < LC / 8; u++) tmem_ld8_nw(ta + gst + (uint32_t)(LC * k + 8 * u), P1 + 8 * u);
                }
                tmem_ld_wait();
            }
            if (k == CW / LC - 1) {
                tc_fence_before();                    // the accumulator is free once in registers
                __syncwarp();
                if (f.lane == 0) mbar_arrive(&f.acc_empty[ab]);
            }
            if (!ck) continue;
            if (two) {
#pragma unroll
                for (int q = 0; q < LC; q++) {
                    const int qq = LC * k + q;
                    const float2 S2 = *reinterpret_cast<const float2*>(gsp + qq * bs + G);
                    float v = fmaf(b0, S2.x, acc[qq]);
                    v = fmaf(s0, __uint_as_float(P0[q]), v);
                    v = fmaf(b1, S2.y, v);
                    acc[qq] = fmaf(s1, __uint_as_float(P1[q]), v);
                }
            } else {
#pragma unroll
                for (int q = 0; q < LC; q++) {
                    const int qq = LC * k + q;
                    acc[qq] = fmaf(s0, __uint_as_float(P0[q]), fmaf(b0, gsp[qq * bs + G], acc[qq]));
                }
            }
        }
    }
    }
    if (!DOWN) {
        // lanes < 16 hold gate rows, lanes >= 16 the up rows of the same 16
        // intermediate indices (tile q4 of the strip)
        const int i = 64 * d.sb + 16 * f.q4 + (f.lane & 15);
        const int pos = tc_col_pos(i);
        float (*red)[4][32] = f.s_red[j & 1];
        if (on) {
            // column pairs: lanes < 16 take column q (their gate, the up of
            // lane + 16), lanes >= 16 column q + 1 (their up, the gate of
            // lane - 16); one exchange per pair
            const int hi_half = f.lane >> 4;
            __nv_bfloat16* hh = a.h_hi;
            __nv_bfloat16* hl = a.h_lo;
#pragma unroll
            for (int q = 0; q < CW; q += 2) {
                const float give = hi_half ? acc[q] : acc[q + 1];
                const float got = __shfl_xor_sync(0xffffffffu, give, 16);
                const float gate = hi_half ? got : acc[q];
                const float up = hi_half ? acc[q + 1] : got;
                const int qq = q + hi_half, t = c0 + qq;
                float part = 0.f;
                if (qq < cw && t < d.nt) {
                    const float hv = tc_gelu(gate, a.gelu) * up;
                    const __nv_bfloat16 bh = __float2bfloat16_rn(hv);
                    const __nv_bfloat16 bl = __float2bfloat16_rn(hv - __bfloat162float(bh));
                    const size_t o = (size_t)(d.brow + t) * a.hs + pos;
                    hh[o] = bh;
                    hl[o] = bl;
                    part = __bfloat162float(bh) + __bfloat162float(bl);
                }
                part += __shfl_xor_sync(0xffffffffu, part, 8);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                if ((f.lane & 15) == 0) red[f.half][f.q4][qq] = part;
            }
        }
        __syncwarp();
        if (f.lane == 0) mbar_arrive(&f.red_full[j & 1]);
        if (!fused_wait_bar(&f.red_full[j & 1], (uint32_t)((j >> 1) & 1), f.status)) return -1;
        const int v = f.tid - 6 * 32;                 // 0 .. 255: one token column each
        if (v < d.nt) {
            const int hf = v >= cw ? 1 : 0, q = v - hf * cw;
            a.h_sum[(size_t)(d.brow + v) * a.hsum_stride + d.sb] =
                ((red[hf][0][q] + red[hf][1][q]) + red[hf][2][q]) + red[hf][3][q];
        }
    } else if (on) {
        const int o = kMmaRows * d.sb + f.m;
#pragma unroll
        for (int q = 0; q < CW; q++) {
            const int rr = __shfl_sync(0xffffffffu, rrow, q);
            if (q < cw && c0 + q < d.nt) a.y_pairs[(size_t)rr * a.H + o] = acc[q];
        }
    }
    return (int)g;
}

// Tensor-core FFN half over all work items of a step, persistent.
//   DOWN = false (gate/up): K = H, B = gathered x rows (fp16).  Writes
//     h = GELU(gate) * up as bf16 hi/lo planes at row `brow` + t (the B row of
//     the token: t for the shared expert, T + bucket position for a routed
//     pair), columns in the tensor-core order, and the group sums
//     h_sum[row][strip] (a strip's 64 indices are one down group).
//   DOWN = true: K = Ie, B = the h planes; writes y_pairs[pair row][o] (fp32).
// tm_cr / tm_cs: codes of the routed experts / the shared expert ([tile]
// [row][64 bytes] per stage, experts as the last dimension, 64-byte swizzle);
// tm_b16 / 32 / 64: the B rows, boxes of 64 columns x 16 / 32 / 64 rows
// (down: both planes), 128-byte swizzle.  Grid: one CTA per SM; block
// kTcThreads; dynamic shared memory tc_smem_bytes<DOWN>(kmax, bs_stride).
template <bool DOWN>
__global__ void __launch_bounds__(kTcThreads, 1)
k_ffn_tc(const __grid_constant__ CUtensorMap tm_cr, const __grid_constant__ CUtensorMap tm_cs,
         const __grid_constant__ CUtensorMap tm_b16, const __grid_constant__ CUtensorMap tm_b32,
         const __grid_constant__ CUtensorMap tm_b64, const uint8_t* __restrict__ experts, size_t stride,
         const uint8_t* __restrict__ shared_blob, const __grid_constant__ TcArgs a) {
    using S = TcShape<DOWN>;
    constexpr int R = S::kRing;
    extern __shared__ uint8_t tsm_raw[];
    __shared__ __align__(8) uint64_t full_slot[R], a_full[R];
    __shared__ __align__(8) uint64_t acc_empty[kTcAcc], acc_full[kTcAcc], ib_full[kTcItemBufs], ib_empty[kTcItemBufs];
    __shared__ __align__(8) uint64_t red_full[2];
    __shared__ uint32_t s_tmem;
    __shared__ int s_eoff[MOE_MAX_EXPERTS + 1];
    __shared__ int s_ioff[MOE_MAX_EXPERTS + 2];
    __shared__ float s_red[2][2][4][32];                  // [item parity][token half][quarter][column]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E;
    for (int i = tid; i <= E; i += kTcThreads) s_eoff[i] = a.e_off[i];
    __syncthreads();
    if (warp == 0) {                                      // items per entry, prefix sums
        int carry = 0;
        for (int j0 = 0; j0 <= E; j0 += 32) {
            const int j = j0 + lane;
            int c = 0;
            if (j == 0) {
                if (a.do_shared) c = (DOWN ? a.H / kMmaRows : a.Is / 64) * ((a.T + kMmaTok - 1) / kMmaTok);
            } else if (j <= E) {
                const int n = s_eoff[j] - s_eoff[j - 1];
                if (n > 0 && n >= a.min_tok) c = (DOWN ? a.H / kMmaRows : a.Ir / 64) * ((n + kMmaTok - 1) / kMmaTok);
            }
            int v = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (j <= E) s_ioff[j + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) s_ioff[0] = 0;
    }
    __syncthreads();
    const int n_items = s_ioff[E + 1];
    if ((int)blockIdx.x >= n_items) return;

    const uint32_t sbase = (smem_u32(tsm_raw) + 1023u) & ~1023u;
    const uint32_t s_ring = sbase;
    const uint32_t ib_bytes = (uint32_t)tc_item_bytes(a.kmax, a.bs_stride);
    const uint32_t s_items = s_ring + R * S::kSlot;
    // the same buffers through generic pointers (plain loads the compiler can batch)
    const uint8_t* g_ring = tsm_raw + (sbase - smem_u32(tsm_raw));
    const uint8_t* g_items = g_ring + R * S::kSlot;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s_tmem)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int i = 0; i < R; i++) {
            mbar_init(&full_slot[i], 1);
            mbar_init(&a_full[i], 4);                     // converter warps
        }
        for (int i = 0; i < kTcAcc; i++) {
            mbar_init(&acc_empty[i], 8);                  // folder warps
            mbar_init(&acc_full[i], 2);                   // the two MMA issuers' commits
        }
        for (int i = 0; i < kTcItemBufs; i++) {
            mbar_init(&ib_full[i], 1);
            mbar_init(&ib_empty[i], 8);
        }
        mbar_init(&red_full[0], 8);
        mbar_init(&red_full[1], 8);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    int* status = a.status;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0) {
            uint32_t g = 0;
            int j = 0, ib_last = -1, j_last = 0;
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x, j++) {
                const TcItem d = tc_item<DOWN>(it, s_ioff, s_eoff, a);
                const uint8_t* blob = d.shared ? shared_blob : experts + (size_t)d.e * stride;
                const int ib = j % kTcItemBufs;
                if (!fused_wait_bar(&ib_empty[ib], (uint32_t)((j / kTcItemBufs) & 1) ^ 1u, status)) {
                    ok = false;
                    break;
                }
                const uint32_t sc = s_items + ib * ib_bytes;
                const uint32_t gbytes = (uint32_t)d.nt * a.bs_stride * 4;
                mbar_arrive_expect_tx(&ib_full[ib], 8u * d.K + gbytes);
                if (!DOWN) {
                    const BlobLayout L(a.H, d.shared ? a.Is : a.Ir);
                    for (int t4 = 0; t4 < 4; t4++) {
                        const uint8_t* tb = blob + (size_t)(4 * d.sb + t4) * L.gu_tile;
                        bulk_g2s_u32(sc + t4 * d.K, tb + 16 * (size_t)a.H, a.H, &ib_full[ib]);
                        bulk_g2s_u32(sc + 4 * d.K + t4 * d.K, tb + 17 * (size_t)a.H, a.H, &ib_full[ib]);
                    }
                } else {
                    const BlobLayout L(a.H, d.K);
                    for (int t8 = 0; t8 < 8; t8++) {
                        const uint8_t* tb = blob + L.dn_base + (size_t)(8 * d.sb + t8) * L.dn_tile;
                        bulk_g2s_u32(sc + t8 * (d.K / 2), tb + 8 * (size_t)d.K, d.K / 2, &ib_full[ib]);
                        bulk_g2s_u32(sc + 4 * d.K + t8 * (d.K / 2), tb + 8 * (size_t)d.K + d.K / 2, d.K / 2,
                                     &ib_full[ib]);
                    }
                }
                bulk_g2s_u32(sc + 8 * d.K, a.b_sum + (size_t)d.brow * a.bs_stride, gbytes, &ib_full[ib]);
                ib_last = ib;
                j_last = j;
                const int brows = tc_brows(d.npad);
                const uint32_t bbytes = (uint32_t)brows * 128 * S::kPlanes;
                const CUtensorMap* mb = brows == 16 ? &tm_b16 : brows == 32 ? &tm_b32 : &tm_b64;
                const CUtensorMap* mc = d.shared ? &tm_cs : &tm_cr;
                for (int c = 0; c < d.nst; c++, g++) {
                    const uint32_t slot = g % R;
                    // the slot's previous stage (g - R) has completed its MMAs
                    if (g >= (uint32_t)R &&
                        !fused_wait_bar(&acc_full[(g - R) % kTcAcc], ((g - R) / kTcAcc) & 1u, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sl = s_ring + slot * S::kSlot;
                    mbar_arrive_expect_tx(&full_slot[slot], kTcCodeBytes + 2u * bbytes);
                    tma_load_4d(sl, mc, 64 * c, 0, (DOWN ? 8 : 4) * d.sb, d.shared ? 0 : d.e, &full_slot[slot]);
                    tma_load_3d(sl + kTcCodeBytes, mb, kTcStageK * c, d.brow, 0, &full_slot[slot]);
                    tma_load_3d(sl + kTcCodeBytes + bbytes, mb, kTcStageK * c + 64, d.brow, 0, &full_slot[slot]);
                }
            }
            // copies still in flight land before the CTA ends
            if (g > 0) mma_drain_wait(&full_slot[(g - 1) % R], ((g - 1) / R) & 1u);
            if (ib_last >= 0) mma_drain_wait(&ib_full[ib_last], (uint32_t)((j_last / kTcItemBufs) & 1));
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuers --
        // Lanes 0 and 1 run the same loop; lane gi issues the MMAs of scale
        // group gi of every stage (its own accumulator, A columns and B
        // half), so each MMA instruction of the warp issues two, and each
        // lane commits its own (the stage barrier takes both arrivals).
        if (lane < 2) {
            const int gi = lane;
            uint32_t g = 0, rel = 0, cum_rel = 0;        // stages released, their consumed columns
            uint32_t cumq[kTcAcc];                        // consumed columns after each stage in flight
            TcAccRing ring;
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const TcItem d = tc_item<DOWN>(it, s_ioff, s_eoff, a);
                const uint32_t gst = tc_gstride(d.npad);
                const int brows = tc_brows(d.npad);
                const uint32_t bbytes = (uint32_t)brows * 128 * S::kPlanes;
                const uint32_t idesc = (DOWN ? kTcIdescBF16 : kTcIdescF16) | ((uint32_t)(d.npad >> 3) << 17);
                for (int c = 0; c < d.nst; c++, g++) {
                    const uint32_t slot = g % R;
                    const uint32_t acol = ring.take(2 * gst);
                    // free accumulator columns: release stages in order until this one fits
                    while (rel < g && (ring.cum - cum_rel > kTcAccCols || g - rel >= (uint32_t)kTcAcc)) {
                        if (!fused_wait_bar(&acc_empty[rel % kTcAcc], (rel / kTcAcc) & 1u, status)) { ok = false; break; }
                        cum_rel = cumq[rel % kTcAcc];
                        rel++;
                    }
                    if (!ok) break;
                    cumq[g % kTcAcc] = ring.cum;
                    if (!fused_wait_bar(&full_slot[slot], (g / R) & 1u, status) ||
                        !fused_wait_bar(&a_full[slot], (g / R) & 1u, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // one descriptor per stage; a K step of 16 elements is 32 bytes (2 in
                    // the descriptor's address field), a group's half bbytes, a plane brows * 128
                    const uint64_t bdg = tc_sdesc_sw128(s_ring + slot * S::kSlot + kTcCodeBytes + gi * bbytes);
                    const uint32_t a0 = tmem + 64u * slot + 32u * gi;
                    const uint32_t dacc = tmem + kTcAccCol + acol + gst * gi;
                    if (gi < d.ng - 2 * c) {                  // the stage's group gi exists
#pragma unroll
                        for (int kk = 0; kk < 4; kk++) {
                            const uint32_t at = a0 + 8u * kk;
                            tc_mma_ts(dacc, at, bdg + 2u * kk, idesc, kk > 0 ? 1u : 0u);
                            if (DOWN) tc_mma_ts(dacc, at, bdg + (uint64_t)((brows * 128) >> 4) + 2u * kk, idesc, 1u);
                        }
                    }
                    mma_commit(&acc_full[g % kTcAcc]);
                }
            }
            // every commit has arrived before the CTA ends
            if (g > 0) {
                mma_drain_wait(&acc_full[(g - 1) % kTcAcc], ((g - 1) / kTcAcc) & 1u);
            }
        }
    } else if (warp < 6) {
        // ---------------------------------------------------- converters --
        const int q4 = warp & 3, m = 32 * q4 + lane;      // TMEM lane quarter of this warp, A row
        const uint32_t t_row = tmem + ((uint32_t)(32 * q4) << 16);
        const uint32_t sw = (uint32_t)((m >> 1) & 3);     // 64-byte swizzle of the row's chunks
        uint32_t g = 0;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            const TcItem d = tc_item<DOWN>(it, s_ioff, s_eoff, a);
            for (int c = 0; c < d.nst; c++, g++) {
                const uint32_t slot = g % R;
                if (!fused_wait_bar(&full_slot[slot], (g / R) & 1u, status) ||
                    (g >= (uint32_t)R &&
                     !fused_wait_bar(&acc_full[(g - R) % kTcAcc], ((g - R) / kTcAcc) & 1u, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint4* row = reinterpret_cast<const uint4*>(g_ring + slot * S::kSlot + m * 64);
                uint4 w[4];
#pragma unroll
                for (int cc = 0; cc < 4; cc++) w[cc] = row[cc ^ sw];
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    uint32_t r[32];
#pragma unroll
                    for (int cc = 0; cc < 2; cc++) {
                        const uint4 v = w[2 * h + cc];
                        tc_codes<DOWN>(v.x, r + 16 * cc + 0);
                        tc_codes<DOWN>(v.y, r + 16 * cc + 4);
                        tc_codes<DOWN>(v.z, r + 16 * cc + 8);
                        tc_codes<DOWN>(v.w, r + 16 * cc + 12);
                    }
                    tmem_st32(t_row + 64u * slot + 32u * h, r);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[slot]);
            }
        }
    } else {
        // ------------------------------------------------------- folders --
        // The two warps of a lane quarter split each item's columns in halves
        // (8, 16, 24 or 32 each, both groups of every stage).
        const int q4 = warp & 3, half = (warp - 6) >> 2;  // TMEM lane quarter, column half
        const int m = 32 * q4 + lane;                     // weight row (TMEM lane)
        const uint32_t t_acc0 = tmem + ((uint32_t)(32 * q4) << 16) + kTcAccCol;
        TcFold f;
        f.a = &a; f.status = status; f.g = 0; f.m = m; f.q4 = q4; f.half = half; f.lane = lane;
        f.tid = tid; f.t_acc0 = t_acc0; f.acc_empty = acc_empty;
        f.acc_full = acc_full;
        f.red_full = red_full; f.s_red = s_red;
        int j = 0;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x, j++) {
            const TcItem d = tc_item<DOWN>(it, s_ioff, s_eoff, a);
            const int ib = j % kTcItemBufs;
            if (!fused_wait_bar(&ib_full[ib], (uint32_t)((j / kTcItemBufs) & 1), status)) { ok = false; break; }
            const uint8_t* ibp = g_items + ib * ib_bytes;
            int ng;
            switch (d.npad) {
                case 16: ng = tc_fold_item<DOWN, R, 8>(f, d, j, ibp); break;
                default: ng = tc_fold_item<DOWN, R, 32>(f, d, j, ibp); break;   // 32, 48, 64
            }
            if (ng < 0) { ok = false; break; }
            f.g = (uint32_t)ng;
            __syncwarp();
            if (lane == 0) mbar_arrive(&ib_empty[ib]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                     : "memory");
    }
}

}  // namespace moeq4
