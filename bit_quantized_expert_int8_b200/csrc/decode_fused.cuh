// decode_fused.cuh -- one persistent kernel for a run of single-token MoE
// decode steps (T tokens one after another, each through L layers).
//
// Per step (token, layer) the engine's per-layer flow ("Gemma 4 26B : Comment
// faire tourner un LLM en 2 Go de RAM", section 04 "Le pipeline de traitement"
// and "Concurrence pour masquer la latence"; remio.ai TurboFieldfare article,
// "L'affirmation des 2 Go ...": router top-8, shared expert, routed experts,
// combine, then the next layer):
//
//   [RMSNorm]  x = fp16(h / sqrt(mean(h^2) + eps)), exact sum of squares
//   router     S_e = sum_c W[e,c] x_c * 2^24 exactly (integers), then
//              logit_e = S_e 2^-24 scale_e (+bias_e) in fp64; top-k (ties to
//              the lower index); softmax weights
//   gate/up    h = w_e * GELU(Wg_e x) * (Wu_e x), for the shared expert (w = 1)
//              and the k routed experts
//   down       y = sum_e Wd_e h_e (routing weights already in h, so this is the
//              combine), h_next = fp16(h + y)
//
// The kernel is shaped by what a memory round trip costs on this part: about
// 0.5 us when the memory system is quiet, several microseconds when many
// bytes are in flight.  A step therefore crosses the grid only three times,
// each a single hop of data: (1) the exact router sums, written as tagged
// 64-bit words that every CTA polls directly; (2) one counter of finished
// gate/up items, after which every CTA reads the intermediate h; (3) the next
// step's h rows, written as tagged words.  Weights stream with plain 16-byte
// loads issued by every warp (a warp holds one item's loads in flight), which
// keeps the bytes in flight near what the bandwidth needs; the down weights are
// copied into shared memory (cp.async) as soon as the routing is known, while
// the gate/up items finish and the counter travels.
//
// Work of a step, spread statically over CTAs and claimed dynamically by the
// warps of a CTA: router rows (one warp per expert row), gate/up items (the
// gate and up rows of one intermediate index of one expert: shared indices
// first, then routed), down blocks (8 output rows of the shared and all routed
// experts together, so the combine stays inside the CTA).
//
// Arithmetic: weight codes (0..15) times activations held as fixed point in
// int8 digits, summed exactly with DP4A and scaled in fp32 per 32-column chunk;
// each group's fp16 bias multiplies the fp32 sum of its activations.  x uses
// 24-bit fixed point (three digits) per 64-column group; h uses 16-bit fixed
// point per 8 values.  The router dot product is exact (balanced base-256
// digits of x * 2^24).
//
// Steps of one launch are numbered from a per-context step count, so tags
// never repeat; the last CTA to leave a launch advances the step count and,
// when the launch consumed the gate/up counter (it had down blocks), resets
// it.  A step may also be split over three launches (router; shared expert;
// routed experts and down blocks), as the expert cache needs: the shared
// launch's gate/up items stay in the counter for the routed launch.  Every wait is bounded; on expiry the kernel records
// MOE_ERR_TIMEOUT in the status word and leaves.  The launch is cooperative
// (all CTAs resident), one CTA per SM.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace moeq4 {

constexpr int kDecWarps = 12;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecRouteWarp = kDecWarps - 1;    // router rows, routing, down copies
constexpr int kDecGWarps = 11;                  // warps on the gate/up tiles
constexpr int kDecGThreads = kDecGWarps * 32;
constexpr int kDecGChunks = kDecGWarps * 8;     // 32-column chunks per round of a tile
constexpr int kDecSbVec = 2;                    // 16-byte words of a tile's scales/biases per thread
constexpr int kDecRouterVec = 8;                // 16-byte words of a router row per lane (hidden <= 4096)
constexpr int kDecMaxLayers = 64;               // layers per launch (kernel parameter table)
constexpr int kDecRouterLimbs = 6;
constexpr int kDecDownRows = 8;                 // output rows per down block
constexpr int kDecXWords = 28;                  // x digit words per 32-column chunk
constexpr int kDecHWords = 24;                  // h limb words per 32-value chunk
constexpr int kDecMaxBlocks = 4;                // down blocks per CTA and step
constexpr int kDecTraceSteps = 4;
constexpr int kDecTraceStride = 12;             // words per traced step

enum : int { kDecRouter = 1, kDecShared = 2, kDecRouted = 4, kDecFull = 7 };

// trace slots of a step
enum { kDtStart = 0, kDtInput = 1, kDtX = 2, kDtRouterRow = 3, kDtRouting = 4, kDtGDone = 5,
       kDtHSync = 6, kDtHPacked = 7, kDtDownDone = 8 };

struct DecLayer {
    const int8_t* Wr;          // router int8 [E][H]
    const __half* rscale;      // [E]
    const float* rbias;        // [E] or null
    const uint8_t* shared;     // shared-expert blob
    const uint8_t* experts;    // routed blobs [E], stride bytes apart
};

struct DecSync {                    // per context
    unsigned long long steps;       // steps run by earlier launches (tag base)
    unsigned long long exits;       // CTAs that left (launches x grid)
    unsigned long long gu_done;     // gate/up items finished in the running launch
    unsigned long long pad[5];
};

struct DecArgs {
    DecLayer layer[kDecMaxLayers];
    const __half* hin;           // [T][H] token rows (residual h with prenorm, else x)
    __half* hout;                // [T][H] or null: residual after the last layer (may alias hin)
    float* y;                    // [T][H] or null: MoE output of the last layer
    int32_t* idx_out;            // [k] or null: routing of the first step
    float* w_out;
    __half* x_norm_out;          // [H] or null: normalised input of the first step
    int32_t* idx_ws;             // [k]: routing of the latest step (router launches)
    float* w_ws;
    const int32_t* sel_src;      // launches without router items: expert (or slot) per position
    const float* w_src;
    const uint8_t* routed_base;  // non-null: routed blobs at routed_base + sel_src[j] * stride
    unsigned long long* rsum;    // [2][E][2] tagged halves of the exact router sums
    unsigned long long* hbuf;    // [2][H/2] tagged fp16 pairs of the residual between steps
    uint32_t* dlimb;             // [(Is + k I) / 32][24] packed intermediate h: shared, then routed
    DecSync* sync;
    int* status;
    unsigned long long* trace;   // optional
    unsigned long long wait_ns;
    unsigned long long stride;   // bytes between routed blobs
    double eps;
    int n_layers, n_tokens, mode, prenorm;
    int H, E, k, I, Is, gelu, renorm;
    int max_blocks;              // down blocks per CTA and step at most (shared-memory stage)
};

// ------------------------------------------------------------- helpers --
__device__ __forceinline__ unsigned long long dec_now() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void dec_trace(const DecArgs& a, int s, int slot) {
    if (a.trace && s < kDecTraceSteps)
        a.trace[(size_t)blockIdx.x * 160 + s * kDecTraceStride + slot] = dec_now();
}

__device__ __forceinline__ void dec_fail(int* status) { atomicCAS(status, 0, MOE_ERR_TIMEOUT); }

__device__ __forceinline__ bool dec_aborted(const int* status) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(status) : "memory");
    return v != 0;
}

__device__ __forceinline__ uint4 ldg_stream128(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_stream16(const void* p) {
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ unsigned long long ld_rlx64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_rlx64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void red_release_add(unsigned long long* p, unsigned long long v) {
    asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ float dec_h2f(uint32_t b) { return __half2float(__ushort_as_half((unsigned short)b)); }

// Exponent E with |v| < 2^E for a block whose largest |v| is m (clamped).
__device__ __forceinline__ int dec_block_exp(float m) {
    const int E = (int)((__float_as_uint(m) >> 23) & 0xff) - 126;
    return max(-100, min(E, 120));
}

__device__ __forceinline__ float dec_exp2(int e) {      // 2^e, e in [-126, 127]
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

// ------------------------------------------------------ x digits (24 bit) --
// x of one 32-column chunk as X = rint(x * 2^(23 - E)) (E of the 64-column
// group), split X = 65536 d2 + 256 b1 + b0 (d2 signed, b1 and b0 bytes); for
// each of the chunk's four 8-column code words, the even columns' digits and
// the odd columns' digits sit in the four bytes of one word.
struct XDigits {
    uint32_t d2e[4], d2o[4], b1e[4], b1o[4], b0e[4], b0o[4];
    float fexp;    // 2^(E - 23)
    float sx;      // sum of the chunk's 32 x (fp32)
};

// sum over a 32-column chunk of code * X, as fp32 (the three partial sums
// are exact integers; one rounding combines them)
__device__ __forceinline__ float dec_dot_x(uint4 q, const XDigits& L) {
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
    int a2 = 0;
    unsigned a1 = 0, a0 = 0;
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint32_t lo = wv[w] & 0x0F0F0F0Fu;
        const uint32_t hi = (wv[w] >> 4) & 0x0F0F0F0Fu;
        a2 = __dp4a((int)lo, (int)L.d2e[w], a2);
        a2 = __dp4a((int)hi, (int)L.d2o[w], a2);
        a1 = __dp4a(lo, L.b1e[w], a1);
        a1 = __dp4a(hi, L.b1o[w], a1);
        a0 = __dp4a(lo, L.b0e[w], a0);
        a0 = __dp4a(hi, L.b0o[w], a0);
    }
    return fmaf((float)a2, 65536.0f, (float)(a1 * 256u + a0));
}

// ------------------------------------------------------ h limbs (16 bit) --
struct HLimbs16 {
    uint32_t eh[4], oh[4], el[4], ol[4];
    float fexp[4];    // 2^(E - 15) of each 8-value word
    float sx;         // sum of the chunk's 32 values
};

__device__ __forceinline__ float dec_dot_h(uint4 q, const HLimbs16& L) {
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint32_t lo = wv[w] & 0x0F0F0F0Fu;
        const uint32_t hi = (wv[w] >> 4) & 0x0F0F0F0Fu;
        int ah = __dp4a((int)lo, (int)L.eh[w], 0);
        ah = __dp4a((int)hi, (int)L.oh[w], ah);
        unsigned al = __dp4a(lo, L.el[w], 0u);
        al = __dp4a(hi, L.ol[w], al);
        acc = fmaf((float)(ah * 256 + (int)al), L.fexp[w], acc);
    }
    return acc;
}

__device__ __forceinline__ HLimbs16 dec_load_h(uint32_t src) {
    HLimbs16 L;
    const uint4 t0 = lds128(src), t1 = lds128(src + 16), t2 = lds128(src + 32), t3 = lds128(src + 48),
                t4 = lds128(src + 64), t5 = lds128(src + 80);
    L.eh[0] = t0.x; L.eh[1] = t0.y; L.eh[2] = t0.z; L.eh[3] = t0.w;
    L.oh[0] = t1.x; L.oh[1] = t1.y; L.oh[2] = t1.z; L.oh[3] = t1.w;
    L.el[0] = t2.x; L.el[1] = t2.y; L.el[2] = t2.z; L.el[3] = t2.w;
    L.ol[0] = t3.x; L.ol[1] = t3.y; L.ol[2] = t3.z; L.ol[3] = t3.w;
    L.fexp[0] = __uint_as_float(t4.x); L.fexp[1] = __uint_as_float(t4.y);
    L.fexp[2] = __uint_as_float(t4.z); L.fexp[3] = __uint_as_float(t4.w);
    L.sx = __uint_as_float(t5.x) + __uint_as_float(t5.y) + __uint_as_float(t5.z) + __uint_as_float(t5.w);
    return L;
}

// Sum over the 32 lanes of v[0..N): afterwards lane l holds the total of
// element l / (32 / N).
template <int N>
__device__ __forceinline__ float dec_reduce_scatter(const float (&v)[N], int lane) {
    float u[N];
#pragma unroll
    for (int i = 0; i < N; i++) u[i] = v[i];
#pragma unroll
    for (int n = N, bit = 16; n > 1; n >>= 1, bit >>= 1) {
        const bool upper = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; i++) {
            const float send = upper ? u[i] : u[i + n / 2];
            const float keep = upper ? u[i + n / 2] : u[i];
            u[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
        }
    }
    float t = u[0];
#pragma unroll
    for (int bit = 16 / N; bit > 0; bit >>= 1) t += __shfl_xor_sync(0xffffffffu, t, bit);
    return t;
}

// ---------------------------------------------------------------- top-k --
__device__ __forceinline__ unsigned long long dec_order_key(double d) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(d);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Top-k of the E logits held by the warp (lane l holds experts l + 32 i in
// v[i]), largest first, ties to the lower index; then the routing weights:
// softmax over all E renormalised over the k picks (which needs only the k
// selected logits: the full normaliser cancels; fp32) or the raw softmax
// probabilities (fp64 over all E).  Lane j < k returns pick j.
//
// Fast path (E <= 128): each lane sorts its four experts by a packed word
// (24-bit monotone key of the logit, 255 - index) and each round takes the
// warp maximum of the lane heads; the picks are exact unless an unpicked
// expert shares the k-th pick's 24-bit key (then full exact rounds over the
// fp64 keys) or two picks share a key (then an exact rank sort of the picks).
__device__ __noinline__ void dec_topk(const double (&v)[8], int E, int k, int renorm, int lane,
                                         int& sel, float& w) {
    constexpr int kPer = 8;
    double sel_l = 0.0, m = 0.0;
    sel = 0;
    bool exact_rounds = E > 128;
    if (!exact_rounds) {
        unsigned pk[4];
        double vv[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int e = lane + 32 * i;
            vv[i] = v[i];
            pk[i] = e < E ? ((unsigned)(dec_order_key(v[i]) >> 40) << 8) | (unsigned)(255 - e) : 0u;
        }
#define MOEQ4_DSWAP(i, j)                                                  \
        if (pk[j] > pk[i]) {                                               \
            const unsigned tk = pk[i]; pk[i] = pk[j]; pk[j] = tk;          \
            const double tv = vv[i]; vv[i] = vv[j]; vv[j] = tv;            \
        }
        MOEQ4_DSWAP(0, 1) MOEQ4_DSWAP(2, 3) MOEQ4_DSWAP(0, 2) MOEQ4_DSWAP(1, 3) MOEQ4_DSWAP(1, 2)
#undef MOEQ4_DSWAP
        unsigned mk = 0, last = 0;
        for (int j = 0; j < k; j++) {
            const unsigned wmax = __reduce_max_sync(0xffffffffu, pk[0]);
            const int e = 255 - (int)(wmax & 255u);
            const int wl = e & 31;
            const double wv = __shfl_sync(0xffffffffu, vv[0], wl);
            if (lane == j) { sel = e; sel_l = wv; mk = wmax; }
            if (lane == wl) {
                pk[0] = pk[1]; pk[1] = pk[2]; pk[2] = pk[3]; pk[3] = 0u;
                vv[0] = vv[1]; vv[1] = vv[2]; vv[2] = vv[3];
            }
            last = wmax >> 8;
        }
        exact_rounds = __any_sync(0xffffffffu, pk[0] != 0u && (pk[0] >> 8) == last);
        if (!exact_rounds) {
            const unsigned nx = __shfl_down_sync(0xffffffffu, mk, 1);
            if (__any_sync(0xffffffffu, lane + 1 < k && (mk >> 8) == (nx >> 8))) {
                int rank = 0;
                for (int i = 0; i < k; i++) {
                    const double vi = __shfl_sync(0xffffffffu, sel_l, i);
                    const int ei = __shfl_sync(0xffffffffu, sel, i);
                    if (lane < k && (vi > sel_l || (vi == sel_l && ei < sel))) rank++;
                }
                int s2 = sel;
                double l2 = sel_l;
                for (int i = 0; i < k; i++) {
                    const double vi = __shfl_sync(0xffffffffu, sel_l, i);
                    const int ei = __shfl_sync(0xffffffffu, sel, i);
                    const int ri = __shfl_sync(0xffffffffu, rank, i);
                    if (ri == lane) { s2 = ei; l2 = vi; }
                }
                sel = s2;
                sel_l = l2;
            }
            m = __shfl_sync(0xffffffffu, sel_l, 0);
        }
    }
    if (exact_rounds) {
        unsigned long long key[kPer];
#pragma unroll
        for (int i = 0; i < kPer; i++) key[i] = lane + 32 * i < E ? dec_order_key(v[i]) : 0ull;
        unsigned taken = 0;
        for (int j = 0; j < k; j++) {
            unsigned long long bk = 0;
            int bi = 0;
            double bv = 0.0;
#pragma unroll
            for (int i = 0; i < kPer; i++)
                if (!((taken >> i) & 1u) && key[i] > bk) { bk = key[i]; bi = i; bv = v[i]; }
            const unsigned hi = (unsigned)(bk >> 32), lo = (unsigned)bk;
            const unsigned mhi = __reduce_max_sync(0xffffffffu, hi);
            const unsigned mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
            const bool tie = hi == mhi && lo == mlo && bk != 0;
            const unsigned e = (unsigned)(lane + 32 * bi);
            const unsigned wi = 256u - __reduce_max_sync(0xffffffffu, tie ? 256u - e : 0u);
            const int wl = (int)(wi & 31u);
            const double wv = __shfl_sync(0xffffffffu, bv, wl);
            if (lane == wl) taken |= 1u << (wi >> 5);
            if (j == 0) m = wv;
            if (lane == j) { sel = (int)wi; sel_l = wv; }
        }
    }
    if (renorm) {
        const float p = lane < k ? expf((float)(sel_l - m)) : 0.f;
        float z = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        w = p / z;
    } else {
        double zz = 0.0;
#pragma unroll
        for (int i = 0; i < kPer; i++)
            if (lane + 32 * i < E) zz += exp(v[i] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
        w = lane < k ? (float)(exp(sel_l - m) / zz) : 0.f;
    }
}

// ---------------------------------------------------------- shared memory --
struct DecShared {
    const uint8_t* blob[MOE_MAX_TOPK];   // routed blobs of the current step
    float rw[MOE_MAX_TOPK];              // routing weights
    int route_tag;                       // step + 1 once blob / rw hold the step's routing
    int issued_tag;                      // step + 1 once the gate/up warps issued their last tile
    int abort;                           // a wait of this CTA gave up
    unsigned xmax_bits;                  // largest |x| of the step (router digits)
    long long ss[kDecWarps * 3];         // exact sum of squares, three int64 parts per warp
};

struct DecSmemLayout {
    size_t xs, hs, xl, xt, ht, dst, sbt, red2, hb, red, hnew, rsc, rbs, cs, total;
    size_t blk_bytes, rblk;
    __host__ __device__ DecSmemLayout(int H, int E, int k, int I, int Is, int n_blocks) {
        rblk = (size_t)kDecDownRows * (I / 2 + I / 16);                    // one routed expert's rows
        blk_bytes = (size_t)k * rblk + (size_t)kDecDownRows * (Is / 2 + Is / 16);
        size_t off = 0;
        auto take = [&](size_t b) { size_t o = off; off = (off + b + 127) / 128 * 128; return o; };
        xs = take((size_t)H * 2);
        hs = take((size_t)H * 2);
        xl = take((size_t)kDecRouterLimbs * H);
        xt = take((size_t)(H / 32) * kDecXWords * 4);
        ht = take((size_t)((Is + k * I) / 32) * kDecHWords * 4);
        dst = take((size_t)n_blocks * blk_bytes);
        sbt = take((size_t)2 * 2 * H);                                    // tile scales/biases, two tiles
        red2 = take((size_t)kDecGWarps * 32 * 4);
        hb = take(64);
        red = take((size_t)(MOE_MAX_TOPK + 1) * kDecDownRows * 4);
        hnew = take((size_t)kDecDownRows * 2);
        rsc = take((size_t)E * 8);
        rbs = take((size_t)E * 8);
        cs = take(sizeof(DecShared));
        total = off;
    }
};

// Number of q in [0, n) with q = r (mod G), r in [0, G).
__device__ __forceinline__ int dec_count(int n, int r, int G) { return n > r ? (n - 1 - r) / G + 1 : 0; }

// Bounded wait until a shared-memory word equals `want`; lane 0 polls, the
// warp learns the outcome.  Gives up on the CTA's or the kernel's abort.
__device__ __forceinline__ bool dec_wait_smem_eq(const DecArgs& a, DecShared* cs, const int* p, int want,
                                                 int lane) {
    bool ok = true;
    if (lane == 0 && *(volatile const int*)p != want) {
        const unsigned long long t0 = dec_now();
        for (unsigned q = 0; *(volatile const int*)p != want; q++) {
            __nanosleep(64);
            if ((q & 15) == 15 && (*(volatile int*)&cs->abort || dec_aborted(a.status) ||
                                   dec_now() - t0 > a.wait_ns)) {
                dec_fail(a.status);
                ok = false;
                break;
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    fence_acq_rel_cta();                      // every lane reads what the flag publishes
    return ok;
}

// Named barrier among `n` threads that also ORs a predicate over them, so that
// every participant leaves with the same answer.
__device__ __forceinline__ bool dec_bar_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// cp.async of `bytes` (a multiple of 16) from global to shared memory by one warp.
__device__ __forceinline__ void dec_copy_warp(uint32_t dst, const uint8_t* src, int bytes, int lane) {
    for (int u = lane; u < bytes / 16; u += 32) cp_async16(dst + 16 * u, src + 16 * u);
}

// ----------------------------------------------------------------- kernel --
// Thread roles: warps 0..10 (352 threads) take the gate/up tiles, warp 11
// the router rows, the routing and the copies of the down weights; all 12
// take the down blocks.  A gate/up thread owns one 32-column chunk of x
// (chunk 8 w + (lane & 7), and + 88 m for wider rows) and 8 of the tile's 32
// rows (lane >> 3, + 4, + 8, ...).
template <int MAXC>
__global__ void __launch_bounds__(kDecThreads, 1) k_moe_decode(const __grid_constant__ DecArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int H = a.H, E = a.E, k = a.k, I = a.I, Is = a.Is;
    const DecSmemLayout lay(H, E, k, I, Is, a.max_blocks);
    __half* xs = reinterpret_cast<__half*>(smem + lay.xs);
    __half* hs = reinterpret_cast<__half*>(smem + lay.hs);
    int8_t* xl = reinterpret_cast<int8_t*>(smem + lay.xl);
    uint32_t* xt = reinterpret_cast<uint32_t*>(smem + lay.xt);
    uint32_t* ht = reinterpret_cast<uint32_t*>(smem + lay.ht);
    uint8_t* dst = smem + lay.dst;
    uint8_t* sbt = smem + lay.sbt;
    float* red2 = reinterpret_cast<float*>(smem + lay.red2);
    uint32_t* hb = reinterpret_cast<uint32_t*>(smem + lay.hb);
    float* red = reinterpret_cast<float*>(smem + lay.red);
    __half* hnew = reinterpret_cast<__half*>(smem + lay.hnew);
    double* rsc = reinterpret_cast<double*>(smem + lay.rsc);
    double* rbs = reinterpret_cast<double*>(smem + lay.rbs);
    DecShared* cs = reinterpret_cast<DecShared*>(smem + lay.cs);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const int nch = H / 32;
    const bool m_router = (a.mode & kDecRouter) != 0, m_shared = (a.mode & kDecShared) != 0,
               m_routed = (a.mode & kDecRouted) != 0;
    // this CTA's share of a step: router rows e = c (mod G); gate/up tiles
    // (16 intermediate indices of one expert) dealt round-robin, the shared
    // expert's first, then the routed ones (slot j, tile q) as f = j I/16 + q;
    // down blocks b = c (mod G)
    const int nR = m_router ? dec_count(E, c, G) : 0;
    const int n_sh = m_shared ? Is / 16 : 0, n_rt = m_routed ? k * I / 16 : 0;
    const int nSG = dec_count(n_sh, c, G);
    const int rt0 = ((c - n_sh % G) % G + G) % G;          // first routed f with n_sh + f = c (mod G)
    const int nRG = dec_count(n_rt, rt0, G);
    const int nGt = nSG + nRG;
    const int NB = H / kDecDownRows;
    const int nB = m_routed ? dec_count(NB, c, G) : 0;
    const bool need_x = nR + nGt > 0;
    const bool need_input = need_x || nB > 0;
    // the routing is computed where routed work needs it, and by CTA 0 of a
    // router launch for the caller's outputs
    const bool need_route = nRG > 0 || nB > 0 || (m_router && c == 0);
    // intermediate indices of a step over the grid, shared and routed: a
    // launch with down blocks waits for all of them (in a split step the shared
    // ones come from the preceding shared launch, whose count the counter holds)
    const unsigned long long ngu_step = (unsigned long long)(Is + k * I);
    const int tpe = I / 16;                                 // gate/up tiles per routed expert
    const BlobLayout Lr(H, I), Lsh(H, Is);

    const unsigned long long base = ld_rlx64(&a.sync->steps);
    const int S = a.n_layers * a.n_tokens;
    if (tid == 0) { cs->abort = 0; cs->route_tag = 0; cs->issued_tag = 0; }
    __syncthreads();

#pragma unroll 1
    for (int s = 0; s < S; s++) {
        const int t = s / a.n_layers, l = s % a.n_layers;
        const DecLayer& Ly = a.layer[l];
        const unsigned tag = (unsigned)(base + s + 1);
        dec_trace(a, s, kDtStart);

        // ---- input-independent loads, issued while the input is awaited:
        // the router warp's first row, router scales and biases, the shared
        // expert's down rows of this CTA's blocks; the gate/up warps' first tile
        // when it belongs to the shared expert
        uint4 wpre[kDecRouterVec];
        if (warp == kDecRouteWarp) {
            if (nR > 0) {
                const uint4* wrow = reinterpret_cast<const uint4*>(Ly.Wr + (size_t)c * H);
#pragma unroll
                for (int m = 0; m < kDecRouterVec; m++) {
                    const int j = lane + 32 * m;
                    wpre[m] = j < H / 16 ? ldg_stream128(wrow + j) : make_uint4(0, 0, 0, 0);
                }
            }
            if (need_route && m_router)
                for (int e = lane; e < E; e += 32) {
                    rsc[e] = (double)__half2float(Ly.rscale[e]);
                    rbs[e] = Ly.rbias ? (double)Ly.rbias[e] : 0.0;
                }
#pragma unroll 1
            for (int q = 0; q < nB; q++) {
                const int row0 = (c + G * q) * kDecDownRows;
                const uint8_t* tile = Ly.shared + Lsh.dn_base + (size_t)(row0 >> 4) * Lsh.dn_tile;
                const int rin = row0 & 15;
                const uint32_t d = smem_u32(dst + (size_t)q * lay.blk_bytes + (size_t)k * lay.rblk);
                dec_copy_warp(d, tile + (size_t)rin * (Is / 2), kDecDownRows * Is / 2, lane);
                dec_copy_warp(d + kDecDownRows * Is / 2, tile + (size_t)8 * Is + (size_t)rin * (Is / 32),
                              kDecDownRows * Is / 32, lane);
                dec_copy_warp(d + kDecDownRows * Is / 2 + kDecDownRows * Is / 32,
                              tile + (size_t)8 * Is + Is / 2 + (size_t)rin * (Is / 32), kDecDownRows * Is / 32, lane);
            }
        }
        const bool gw = warp < kDecGWarps && nGt > 0;
        const int rg = lane >> 3;                           // row group of a gate/up thread
        uint4 qc[MAXC][8];                                  // the current tile's codes of this thread
        uint4 sbc[kDecSbVec];                               // and its share of the tile's scales/biases
        float wc = 1.f;
        int hpc = 0;
        bool have_route = false;
        // loads of tile `it` of this CTA's list (false: the routing never came)
        auto issue = [&](int it, uint4 (&q)[MAXC][8], uint4 (&sb)[kDecSbVec], float& w, int& hp) -> bool {
            const uint8_t* tb;
            if (it < nSG) {
                const int qt = c + G * it;
                tb = Ly.shared + (size_t)qt * 18 * H;
                w = 1.f;
                hp = 16 * qt;
            } else {
                if (!have_route) {
                    if (!dec_wait_smem_eq(a, cs, &cs->route_tag, s + 1, lane)) return false;
                    have_route = true;
                }
                const int f = rt0 + G * (it - nSG);
                const int j = f / tpe, qt = f - j * tpe;
                tb = cs->blob[j] + (size_t)qt * 18 * H;
                w = cs->rw[j];
                hp = Is + j * I + 16 * qt;
            }
#pragma unroll
            for (int m = 0; m < MAXC; m++) {
                const int cc = 8 * warp + (lane & 7) + kDecGChunks * m;
#pragma unroll
                for (int n = 0; n < 8; n++)
                    q[m][n] = cc < nch ? ldg_stream128(tb + (size_t)(rg + 4 * n) * (H / 2) + 16 * cc)
                                       : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int v = 0; v < kDecSbVec; v++) {
                const int u = tid + kDecGThreads * v;
                sb[v] = u < H / 8 ? ldg_stream128(tb + (size_t)16 * H + 16 * u) : make_uint4(0, 0, 0, 0);
            }
            return true;
        };
        bool cur_loaded = false;
        if (gw && nSG > 0) { issue(0, qc, sbc, wc, hpc); cur_loaded = true; }

        // ---- step input: the previous step's tagged residual, or the caller's row
        if (need_input) {
            if (tid == 0) cs->xmax_bits = 0;
            if (s > 0) {
                // wait for every word of the previous step's output (sequential
                // decode: also at token boundaries, where the data is the next row)
                const unsigned long long* hbp = a.hbuf + (size_t)((base + s - 1) & 1) * (H / 2);
                const unsigned want = (unsigned)(base + s);
                bool ok = true;
                for (int i = tid; i < H / 2; i += kDecThreads) {
                    unsigned long long wd = ld_rlx64(hbp + i);
                    if ((unsigned)(wd >> 32) != want) {
                        const unsigned long long t0 = dec_now();
                        for (unsigned it = 0; (unsigned)(wd >> 32) != want; it++) {
                            __nanosleep(32);
                            wd = ld_rlx64(hbp + i);
                            if ((it & 15) == 15 && (dec_aborted(a.status) || dec_now() - t0 > a.wait_ns)) {
                                dec_fail(a.status);
                                ok = false;
                                break;
                            }
                        }
                    }
                    if (!ok) break;
                    if (l > 0) reinterpret_cast<uint32_t*>(hs)[i] = (uint32_t)wd;
                }
                if (!ok) cs->abort = 1;
            }
            if (s == 0 || l == 0) {
                const uint4* src = reinterpret_cast<const uint4*>(a.hin + (size_t)t * H);
                for (int i = tid; i < H / 8; i += kDecThreads) reinterpret_cast<uint4*>(hs)[i] = __ldcg(src + i);
            }
            // exact sum of squares: X = h 2^24 (|X| < 2^40) split as
            // X = xh 2^20 + xl; X^2 = xh^2 2^40 + 2 xh xl 2^20 + xl^2, three
            // int64 sums combined once in 128 bits
            if (__syncthreads_or(*(volatile int*)&cs->abort)) break;
            dec_trace(a, s, kDtInput);
            double r = 1.0;
            if (a.prenorm) {
                long long s2 = 0, s1 = 0, s0 = 0;
                for (int cc = tid; cc < H; cc += kDecThreads) {
                    const long long X = half_fixed24(hs[cc]);
                    const int xh = (int)(X >> 20);
                    const unsigned xl0 = (unsigned)(X & 0xFFFFF);
                    s2 += (long long)xh * xh;
                    s1 += (long long)xh * (long long)xl0;
                    s0 += (long long)((unsigned long long)xl0 * xl0);
                }
                s2 = warp_sum(s2);
                s1 = warp_sum(s1);
                s0 = warp_sum(s0);
                if (lane == 0) { cs->ss[3 * warp] = s2; cs->ss[3 * warp + 1] = s1; cs->ss[3 * warp + 2] = s0; }
                __syncthreads();
                __int128 tot = 0;
                for (int w = 0; w < kDecWarps; w++)
                    tot += (__int128)cs->ss[3 * w] * ((__int128)1 << 40) +
                           (__int128)cs->ss[3 * w + 1] * ((__int128)1 << 21) + (__int128)cs->ss[3 * w + 2];
                const double sm = __dmul_rn(u128_to_double_rn((unsigned __int128)tot), 0x1p-48);
                const double ms = __ddiv_rn(sm, (double)H);
                r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, a.eps)));
            }
            // x, the router's digits of x * 2^24 and the gate/up digit table:
            // one thread per 8-column word (the 64-column group's largest |x|
            // by shuffles over 8 consecutive threads)
            float mx = 0.f;
            for (int b0 = 0; b0 < H / 8; b0 += kDecThreads) {
                const int wd = b0 + tid;
                const bool valid = wd < H / 8;
                float v[8];
                uint4 xv = make_uint4(0, 0, 0, 0);
                if (valid) {
                    const uint4 hv = reinterpret_cast<const uint4*>(hs)[wd];
                    if (a.prenorm) {
                        const uint32_t hh[4] = {hv.x, hv.y, hv.z, hv.w};
                        uint32_t xo[4];
#pragma unroll
                        for (int u = 0; u < 4; u++) {
                            const __half2 p = *reinterpret_cast<const __half2*>(&hh[u]);
                            const __half lo = __double2half(__dmul_rn((double)__low2float(p), r));
                            const __half hi = __double2half(__dmul_rn((double)__high2float(p), r));
                            xo[u] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
                        }
                        xv = make_uint4(xo[0], xo[1], xo[2], xo[3]);
                    } else {
                        xv = hv;
                    }
                    reinterpret_cast<uint4*>(xs)[wd] = xv;
                }
                const uint32_t xq[4] = {xv.x, xv.y, xv.z, xv.w};
                float m = 0.f, sx = 0.f;
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xq[u]));
                    v[2 * u] = f.x;
                    v[2 * u + 1] = f.y;
                    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
                    sx += f.x + f.y;
                }
                mx = fmaxf(mx, m);
                if (valid && nR > 0) {
                    // balanced base-256 digits of x * 2^24 (exact integers)
                    uint32_t pk[2][kDecRouterLimbs];
#pragma unroll
                    for (int n = 0; n < 8; n++) {
                        long long X = __float2ll_rn(v[n] * 16777216.0f);
#pragma unroll
                        for (int dg = 0; dg < kDecRouterLimbs; dg++) {
                            const int digit = (int)((X + 128) & 255) - 128;
                            const uint32_t byte = (uint32_t)(digit & 255) << (8 * (n & 3));
                            if (n & 3) pk[n >> 2][dg] |= byte; else pk[n >> 2][dg] = byte;
                            X = (X - digit) >> 8;
                        }
                    }
#pragma unroll
                    for (int dg = 0; dg < kDecRouterLimbs; dg++) {
                        reinterpret_cast<uint32_t*>(xl + dg * H)[2 * wd] = pk[0][dg];
                        reinterpret_cast<uint32_t*>(xl + dg * H)[2 * wd + 1] = pk[1][dg];
                    }
                }
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
                sx += __shfl_xor_sync(0xffffffffu, sx, 1);
                sx += __shfl_xor_sync(0xffffffffu, sx, 2);
                if (valid && nGt > 0) {
                    const int Eg = dec_block_exp(m);
                    const float sc = dec_exp2(23 - Eg);
                    uint32_t d2e = 0, d2o = 0, b1e = 0, b1o = 0, b0e = 0, b0o = 0;
#pragma unroll
                    for (int n = 0; n < 8; n++) {
                        int X = __float2int_rn(v[n] * sc);
                        X = max(-8388608, min(X, 8388607));
                        const uint32_t c0 = (uint32_t)X & 0xffu, c1 = ((uint32_t)X >> 8) & 0xffu,
                                       c2 = (uint32_t)(X >> 16) & 0xffu;
                        const int sh = 8 * (n >> 1);
                        if (n & 1) { d2o |= c2 << sh; b1o |= c1 << sh; b0o |= c0 << sh; }
                        else       { d2e |= c2 << sh; b1e |= c1 << sh; b0e |= c0 << sh; }
                    }
                    const int cch = wd >> 2, j = wd & 3;
                    uint32_t* d = xt + (size_t)cch * kDecXWords;
                    d[j] = d2e; d[4 + j] = d2o; d[8 + j] = b1e; d[12 + j] = b1o; d[16 + j] = b0e;
                    d[20 + j] = b0o;
                    if (j == 0) {
                        d[24] = __float_as_uint(dec_exp2(Eg - 23));
                        d[25] = __float_as_uint(sx);
                    }
                }
            }
            if (nR > 0) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (lane == 0) atomicMax(&cs->xmax_bits, __float_as_uint(mx));
            }
            __syncthreads();
            if (c == 0 && s == 0 && a.x_norm_out)
                for (int cc = tid; cc < H; cc += kDecThreads) a.x_norm_out[cc] = xs[cc];
            dec_trace(a, s, kDtX);
        }

        // ---- router rows, the routing, the routed down copies (router warp)
        if (warp == kDecRouteWarp) {
            const int slot = (int)((base + s) & 1);
            if (nR > 0) {
                int NL = 1;
                {
                    const double xmax = (double)__uint_as_float(cs->xmax_bits) * 16777216.0;
                    double cap = 127.0;
                    while (NL < kDecRouterLimbs && xmax > cap) { NL++; cap = cap * 256.0 + 127.0; }
                }
#pragma unroll 1
                for (int e = c; e < E; e += G) {
                    const uint4* wrow = reinterpret_cast<const uint4*>(Ly.Wr + (size_t)e * H);
                    int acc[kDecRouterLimbs];
#pragma unroll
                    for (int dg = 0; dg < kDecRouterLimbs; dg++) acc[dg] = 0;
#pragma unroll
                    for (int m = 0; m < kDecRouterVec; m++) {
                        const int j = lane + 32 * m;
                        if (j < H / 16) {
                            const uint4 w4 = e == c ? wpre[m] : ldg_stream128(wrow + j);
#pragma unroll
                            for (int dg = 0; dg < kDecRouterLimbs; dg++) {
                                if (dg < NL) {
                                    const uint4 l4 = lds128(smem_u32(xl + dg * H) + 16 * j);
                                    int sacc = acc[dg];
                                    sacc = __dp4a((int)w4.x, (int)l4.x, sacc);
                                    sacc = __dp4a((int)w4.y, (int)l4.y, sacc);
                                    sacc = __dp4a((int)w4.z, (int)l4.z, sacc);
                                    sacc = __dp4a((int)w4.w, (int)l4.w, sacc);
                                    acc[dg] = sacc;
                                }
                            }
                        }
                    }
                    long long Ssum = 0;
#pragma unroll
                    for (int dg = 0; dg < kDecRouterLimbs; dg++)
                        if (dg < NL) Ssum += (long long)acc[dg] * (1ll << (8 * dg));
                    Ssum = warp_sum(Ssum);
                    if (lane == 0) {
                        unsigned long long* rw = a.rsum + ((size_t)slot * E + e) * 2;
                        const unsigned long long tg = (unsigned long long)tag << 32;
                        st_rlx64(rw, tg | (unsigned)((unsigned long long)Ssum >> 32));
                        st_rlx64(rw + 1, tg | (unsigned)(unsigned long long)Ssum);
                    }
                }
                dec_trace(a, s, kDtRouterRow);
            }
            if (need_route) {
                int sel = 0;
                float wgt = 0.f;
                bool ok = true;
                if (m_router) {
                    // every expert's tagged sum halves of this step
                    const unsigned long long* rb = a.rsum + (size_t)slot * E * 2;
                    double v[8];
                    const unsigned long long t0 = dec_now();
#pragma unroll
                    for (int i = 0; i < 8; i++) v[i] = 0.0;
#pragma unroll 1
                    for (int i = 0; i < 8 && ok; i++) {
                        const int e = lane + 32 * i;
                        if (e < E) {
                            unsigned long long w0 = ld_rlx64(rb + 2 * e), w1 = ld_rlx64(rb + 2 * e + 1);
                            for (unsigned it = 0; (unsigned)(w0 >> 32) != tag || (unsigned)(w1 >> 32) != tag; it++) {
                                __nanosleep(32);
                                w0 = ld_rlx64(rb + 2 * e);
                                w1 = ld_rlx64(rb + 2 * e + 1);
                                if ((it & 15) == 15 && (dec_aborted(a.status) || dec_now() - t0 > a.wait_ns)) {
                                    dec_fail(a.status);
                                    ok = false;
                                    break;
                                }
                            }
                            if (ok) {
                                const long long Sv = (long long)(((w0 & 0xffffffffull) << 32) | (w1 & 0xffffffffull));
                                double lg = __ll2double_rn(Sv);
                                lg = __dmul_rn(lg, 0x1p-24);
                                lg = __dmul_rn(lg, rsc[e]);
                                if (Ly.rbias) lg = __dadd_rn(lg, rbs[e]);
                                if (i == 0) v[0] = lg; else if (i == 1) v[1] = lg; else if (i == 2) v[2] = lg;
                                else if (i == 3) v[3] = lg; else if (i == 4) v[4] = lg; else if (i == 5) v[5] = lg;
                                else if (i == 6) v[6] = lg; else v[7] = lg;
                            }
                        }
                    }
                    ok = __all_sync(0xffffffffu, ok);
                    if (ok) {
                        dec_topk(v, E, k, a.renorm, lane, sel, wgt);
                        if (c == 0 && lane < k) {
                            a.idx_ws[lane] = sel;
                            a.w_ws[lane] = wgt;
                            if (s == 0 && a.idx_out) a.idx_out[lane] = sel;
                            if (s == 0 && a.w_out) a.w_out[lane] = wgt;
                        }
                    }
                } else {
                    if (lane < k) { sel = __ldcg(a.sel_src + lane); wgt = __ldcg(a.w_src + lane); }
                }
                if (!ok) {
                    cs->abort = 1;
                } else {
                    if (lane < k) {
                        const uint8_t* bb = a.routed_base ? a.routed_base : Ly.experts;
                        cs->blob[lane] = bb + (size_t)sel * a.stride;
                        cs->rw[lane] = wgt;
                    }
                    __syncwarp();
                    if (lane == 0) {
                        fence_acq_rel_cta();
                        *(volatile int*)&cs->route_tag = s + 1;
                    }
                    __syncwarp();
                    dec_trace(a, s, kDtRouting);
                    // the routed experts' down rows of this CTA's blocks, queued
                    // behind the gate/up tiles (which the step needs first)
                    if (nB > 0 && (nGt == 0 || dec_wait_smem_eq(a, cs, &cs->issued_tag, s + 1, lane))) {
#pragma unroll 1
                        for (int q = 0; q < nB; q++) {
                            const int row0 = (c + G * q) * kDecDownRows;
                            const int rin = row0 & 15;
#pragma unroll 1
                            for (int j = 0; j < k; j++) {
                                const uint8_t* tile = cs->blob[j] + Lr.dn_base + (size_t)(row0 >> 4) * Lr.dn_tile;
                                const uint32_t d = smem_u32(dst + (size_t)q * lay.blk_bytes + (size_t)j * lay.rblk);
                                dec_copy_warp(d, tile + (size_t)rin * (I / 2), kDecDownRows * I / 2, lane);
                                dec_copy_warp(d + kDecDownRows * I / 2, tile + (size_t)8 * I + (size_t)rin * (I / 32),
                                              kDecDownRows * I / 32, lane);
                                dec_copy_warp(d + kDecDownRows * I / 2 + kDecDownRows * I / 32,
                                              tile + (size_t)8 * I + I / 2 + (size_t)rin * (I / 32),
                                              kDecDownRows * I / 32, lane);
                            }
                        }
                    }
                }
            }
        }

        // ---- gate/up tiles (gate/up warps): register double buffer over the
        // CTA's tiles; per tile, 8 rows x 32 columns per thread, partial row
        // sums reduced over the warp's 8 chunks and then over the 11 warps in
        // a fixed order; warp 0 forms h = w GELU(gate) up for the 16 indices
        // and publishes them packed (16-bit fixed point per 8 values)
        if (gw) {
            XDigits X[MAXC];
#pragma unroll
            for (int m = 0; m < MAXC; m++) {
                const int cc = 8 * warp + (lane & 7) + kDecGChunks * m;
                const uint32_t src = smem_u32(xt + (size_t)(cc < nch ? cc : 0) * kDecXWords);
                const uint4 t0 = lds128(src), t1 = lds128(src + 16), t2 = lds128(src + 32),
                            t3 = lds128(src + 48), t4 = lds128(src + 64), t5 = lds128(src + 80),
                            t6 = lds128(src + 96);
                X[m].d2e[0] = t0.x; X[m].d2e[1] = t0.y; X[m].d2e[2] = t0.z; X[m].d2e[3] = t0.w;
                X[m].d2o[0] = t1.x; X[m].d2o[1] = t1.y; X[m].d2o[2] = t1.z; X[m].d2o[3] = t1.w;
                X[m].b1e[0] = t2.x; X[m].b1e[1] = t2.y; X[m].b1e[2] = t2.z; X[m].b1e[3] = t2.w;
                X[m].b1o[0] = t3.x; X[m].b1o[1] = t3.y; X[m].b1o[2] = t3.z; X[m].b1o[3] = t3.w;
                X[m].b0e[0] = t4.x; X[m].b0e[1] = t4.y; X[m].b0e[2] = t4.z; X[m].b0e[3] = t4.w;
                X[m].b0o[0] = t5.x; X[m].b0o[1] = t5.y; X[m].b0o[2] = t5.z; X[m].b0o[3] = t5.w;
                X[m].fexp = __uint_as_float(t6.x);
                X[m].sx = __uint_as_float(t6.y);
            }
            bool ok = true;
            if (!cur_loaded) ok = issue(0, qc, sbc, wc, hpc);
#pragma unroll 1
            for (int it = 0; it < nGt; it++) {
                uint4 qn[MAXC][8], sbn[kDecSbVec];
                float wn = 1.f;
                int hpn = 0;
                const bool more = it + 1 < nGt;
                if (more && ok) ok = issue(it + 1, qn, sbn, wn, hpn);
                if (warp == 0 && lane == 0 && (!more || !ok)) {
                    fence_acq_rel_cta();
                    *(volatile int*)&cs->issued_tag = s + 1;
                }
                if (!ok && lane == 0) cs->abort = 1;
                // this tile's scales and biases into shared memory
                uint8_t* sbs = sbt + (size_t)(it & 1) * 2 * H;
#pragma unroll
                for (int v = 0; v < kDecSbVec; v++) {
                    const int u = tid + kDecGThreads * v;
                    if (u < H / 8) reinterpret_cast<uint4*>(sbs)[u] = sbc[v];
                }
                if (dec_bar_or(1, kDecGThreads, !ok || *(volatile int*)&cs->abort)) break;
                float acc[8];
#pragma unroll
                for (int n = 0; n < 8; n++) acc[n] = 0.f;
                const uint32_t sbs_s = smem_u32(sbs);
#pragma unroll
                for (int m = 0; m < MAXC; m++) {
                    const int cc = 8 * warp + (lane & 7) + kDecGChunks * m;
                    if (cc < nch) {
                        const uint32_t g2 = 2u * (uint32_t)(cc >> 1);
#pragma unroll
                        for (int n = 0; n < 8; n++) {
                            const int R = rg + 4 * n;
                            const float d = dec_dot_x(qc[m][n], X[m]);
                            const float sv = dec_h2f(lds16(sbs_s + (uint32_t)(R * (H / 32)) + g2));
                            const float bv = dec_h2f(lds16(sbs_s + (uint32_t)(H + R * (H / 32)) + g2));
                            acc[n] = fmaf(sv * X[m].fexp, d, acc[n]);
                            acc[n] = fmaf(bv, X[m].sx, acc[n]);
                        }
                    }
                }
                // reduce over the 8 lanes of a row group: lane l ends with row
                // group (l >> 3)'s sum of row l & 7 (tile row (l >> 3) + 4 (l & 7))
#pragma unroll
                for (int nn = 8, bit = 4; nn > 1; nn >>= 1, bit >>= 1) {
                    const bool upper = (lane & bit) != 0;
#pragma unroll
                    for (int i = 0; i < nn / 2; i++) {
                        const float send = upper ? acc[i] : acc[i + nn / 2];
                        const float keep = upper ? acc[i + nn / 2] : acc[i];
                        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
                    }
                }
                red2[warp * 32 + rg + 4 * (lane & 7)] = acc[0];
                named_bar(1, kDecGThreads);
                if (warp == 0) {
                    // row `lane` over the 11 warps, fixed order; lanes 0..15 gate, 16..31 up
                    float tot = 0.f;
#pragma unroll
                    for (int w = 0; w < kDecGWarps; w++) tot += red2[w * 32 + lane];
                    const float up = __shfl_down_sync(0xffffffffu, tot, 16);
                    const float h = lane < 16 ? gelu_f(tot, a.gelu) * up * wc : 0.f;
                    // two 8-value words (lanes 0..7, 8..15): exponent, 16-bit fixed point
                    float m = fabsf(h), sx = h;
#pragma unroll
                    for (int o = 1; o < 8; o <<= 1) {
                        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        sx += __shfl_xor_sync(0xffffffffu, sx, o);
                    }
                    const int Eg = dec_block_exp(m);
                    int Xv = __float2int_rn(h * dec_exp2(15 - Eg));
                    Xv = max(-32768, min(Xv, 32767));
                    uint8_t* bytes = reinterpret_cast<uint8_t*>(hb);      // [2 words][eh oh el ol][4]
                    if (lane < 16) {
                        const int wdx = lane >> 3, n = lane & 7;
                        const int kind = (n & 1) ? 4 : 0;
                        bytes[32 * wdx + kind + (n >> 1)] = (uint8_t)((Xv >> 8) & 0xff);
                        bytes[32 * wdx + 8 + kind + (n >> 1)] = (uint8_t)(Xv & 0xff);
                    }
                    __syncwarp();
                    if (lane == 0 || lane == 8) {
                        const int wdx = lane >> 3;
                        const uint32_t* wv = hb + 8 * wdx;
                        const int gidx = hpc / 8 + wdx;                    // 8-value group of h
                        uint32_t* d = a.dlimb + (size_t)(gidx >> 2) * kDecHWords + (gidx & 3);
                        d[0] = wv[0];
                        d[4] = wv[1];
                        d[8] = wv[2];
                        d[12] = wv[3];
                        d[16] = __float_as_uint(dec_exp2(Eg - 15));
                        d[20] = __float_as_uint(sx);
                    }
                    __syncwarp();
                    if (lane == 0 && !more) {
                        fence_acq_rel_gpu();
                        red_release_add(&a.sync->gu_done, 16ull * (unsigned long long)nGt);
                        dec_trace(a, s, kDtGDone);
                    }
                }
                if (more) {
#pragma unroll
                    for (int m = 0; m < MAXC; m++)
#pragma unroll
                        for (int n = 0; n < 8; n++) qc[m][n] = qn[m][n];
#pragma unroll
                    for (int v = 0; v < kDecSbVec; v++) sbc[v] = sbn[v];
                    wc = wn;
                    hpc = hpn;
                }
            }
        }

        // ---- down blocks: every gate/up item of the step, then h, compute, combine
        if (nB > 0) {
            if (tid == 0 && !*(volatile int*)&cs->abort) {
                const unsigned long long target = (unsigned long long)(s + 1) * ngu_step;
                unsigned long long v;
                asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(&a.sync->gu_done) : "memory");
                if (v < target) {
                    const unsigned long long t0 = dec_now();
                    for (unsigned q = 0;; q++) {
                        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(&a.sync->gu_done) : "memory");
                        if (v >= target) break;
                        __nanosleep(32);
                        if ((q & 15) == 15 && (dec_aborted(a.status) || dec_now() - t0 > a.wait_ns)) {
                            dec_fail(a.status);
                            cs->abort = 1;
                            break;
                        }
                    }
                }
                dec_trace(a, s, kDtHSync);
            }
            if (__syncthreads_or(*(volatile int*)&cs->abort)) { cp_async_commit_wait_all(); break; }
            // the packed h of the step (all experts) into shared memory
            {
                const int nw = (Is + k * I) / 32 * kDecHWords / 4;       // uint4 words
                for (int i = tid; i < nw; i += kDecThreads)
                    reinterpret_cast<uint4*>(ht)[i] = __ldcg(reinterpret_cast<const uint4*>(a.dlimb) + i);
            }
            cp_async_commit_wait_all();
            __syncthreads();
            dec_trace(a, s, kDtHPacked);
            const int nsw = kDecWarps - k;                  // warps on the shared rows
            const uint32_t ht_s = smem_u32(ht);
#pragma unroll 1
            for (int q = 0; q < nB; q++) {
                const int b = c + G * q;
                const int row0 = b * kDecDownRows;
                const uint32_t st = smem_u32(dst + (size_t)q * lay.blk_bytes);
                if (warp < k) {
                    // routed expert `warp`: lane = 32-value chunk of its h
                    float acc[kDecDownRows];
#pragma unroll
                    for (int r = 0; r < kDecDownRows; r++) acc[r] = 0.f;
                    const int cpe = I / 32;
                    if (lane < cpe) {
                        const HLimbs16 L = dec_load_h(ht_s + (uint32_t)((Is / 32 + warp * cpe + lane) * kDecHWords * 4));
                        const uint32_t cb = st + (uint32_t)(warp * lay.rblk);
                        const uint32_t sb = cb + (uint32_t)(kDecDownRows * I / 2) + 2u * (uint32_t)(lane >> 1);
                        const uint32_t bb = sb + (uint32_t)(kDecDownRows * I / 32);
#pragma unroll
                        for (int r = 0; r < kDecDownRows; r++) {
                            const uint4 qv = lds128(cb + (uint32_t)(r * (I / 2) + 16 * lane));
                            const float dd = dec_dot_h(qv, L);
                            acc[r] = fmaf(dec_h2f(lds16(sb + (uint32_t)(r * (I / 32)))), dd, acc[r]);
                            acc[r] = fmaf(dec_h2f(lds16(bb + (uint32_t)(r * (I / 32)))), L.sx, acc[r]);
                        }
                    }
                    const float tot = dec_reduce_scatter<kDecDownRows>(acc, lane);
                    if ((lane & 3) == 0) red[warp * kDecDownRows + (lane >> 2)] = tot;
                } else {
                    // shared rows r with r % nsw == warp - k; lane = chunks of the shared h
                    const int w0 = warp - k;
                    float acc[kDecDownRows];
#pragma unroll
                    for (int r = 0; r < kDecDownRows; r++) acc[r] = 0.f;
                    const uint32_t cb = st + (uint32_t)(k * lay.rblk);
                    const uint32_t sb0 = cb + (uint32_t)(kDecDownRows * Is / 2);
                    const uint32_t bb0 = sb0 + (uint32_t)(kDecDownRows * Is / 32);
#pragma unroll 1
                    for (int cc = lane; cc < Is / 32; cc += 32) {
                        const HLimbs16 L = dec_load_h(ht_s + (uint32_t)(cc * kDecHWords * 4));
                        const uint32_t go = 2u * (uint32_t)(cc >> 1);
#pragma unroll
                        for (int r = 0; r < kDecDownRows; r++) {
                            if (r % nsw == w0) {
                                const uint4 qv = lds128(cb + (uint32_t)(r * (Is / 2) + 16 * cc));
                                const float dd = dec_dot_h(qv, L);
                                acc[r] = fmaf(dec_h2f(lds16(sb0 + (uint32_t)(r * (Is / 32)) + go)), dd, acc[r]);
                                acc[r] = fmaf(dec_h2f(lds16(bb0 + (uint32_t)(r * (Is / 32)) + go)), L.sx, acc[r]);
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < kDecDownRows; r++) {
                        if (r % nsw == w0) {
                            const float tot = warp_sum(acc[r]);
                            if (lane == 0) red[k * kDecDownRows + r] = tot;
                        }
                    }
                }
                __syncthreads();
                if (tid < kDecDownRows) {
                    const int row = row0 + tid;
                    float yv = red[k * kDecDownRows + tid];
                    for (int j = 0; j < k; j++) yv += red[j * kDecDownRows + tid];
                    const bool last_layer = l == a.n_layers - 1;
                    if (a.y && last_layer) a.y[(size_t)t * H + row] = yv;
                    const __half hn = __float2half_rn(__half2float(hs[row]) + yv);
                    hnew[tid] = hn;
                    if (a.prenorm && last_layer && a.hout) a.hout[(size_t)t * H + row] = hn;
                }
                __syncthreads();
                if (s + 1 < S && tid < kDecDownRows / 2) {
                    const uint32_t pair = (uint32_t)__half_as_ushort(hnew[2 * tid]) |
                                          ((uint32_t)__half_as_ushort(hnew[2 * tid + 1]) << 16);
                    st_rlx64(a.hbuf + (size_t)((base + s) & 1) * (H / 2) + row0 / 2 + tid,
                             ((unsigned long long)tag << 32) | pair);
                }
            }
            dec_trace(a, s, kDtDownDone);
        }
        if (__syncthreads_or(*(volatile int*)&cs->abort)) break;
    }
    // leave: the launch's last CTA advances the context's step count and, when
    // the launch consumed the gate/up counter, resets it (read by the next
    // launch on this context)
    cp_async_commit_wait_all();
    __syncthreads();
    if (tid == 0) {
        fence_acq_rel_gpu();
        const unsigned long long old = atomicAdd(&a.sync->exits, 1ull);
        if ((old + 1) % (unsigned long long)G == 0) {
            fence_acq_rel_gpu();
            if (m_routed) a.sync->gu_done = 0;
            a.sync->steps = base + (unsigned long long)S;
        }
        if (a.trace) {
            unsigned smid;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
            a.trace[(size_t)blockIdx.x * 160 + 159] = smid;
        }
    }
}

__host__ inline size_t dec_smem_bytes(int H, int E, int k, int I, int Is, int max_blocks) {
    return DecSmemLayout(H, E, k, I, Is, max_blocks).total;
}

}  // namespace moeq4
