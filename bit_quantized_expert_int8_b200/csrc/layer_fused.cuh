// layer_fused.cuh -- one persistent kernel per MoE layer and decode token.
//
// The whole per-layer flow of the decode engine ("Gemma 4 26B : Comment faire
// tourner un LLM en 2 Go de RAM", section 04 "Le pipeline de traitement" and
// "Concurrence pour masquer la latence"; remio.ai TurboFieldfare article,
// "L'affirmation des 2 Go ...": router top-8, shared expert, routed experts,
// combine) in one launch:
//
//   [RMSNorm]  x = fp16(h / sqrt(mean(h^2) + eps)), exact sum of squares
//   router     logit_e = scale_e * sum_c W[e,c] x_c (+bias), exact integer
//              dot; top-k (ties to the lower index); softmax weights
//   gate/up    h_e = w_e * GELU(Wg_e x) * (Wu_e x) for the shared expert
//              (w = 1) and the k routed experts
//   down       y = sum_e Wd_e h_e  (the routing weights are already folded
//              into h_e, so this is the combine), h_out = fp16(h + y)
//
// Work items, in this order: router (2 expert rows each), shared-expert
// gate/up (one gate/up tile: 16 intermediate indices = 32 rows), routed
// gate/up (same), shared-expert down (32 output rows: two down tiles), routed
// down (16 output rows of all k routed experts: one down tile of each; the
// routing weights are folded into h, so this is the combine, and the shared
// expert's output for the rows is added).  Item i belongs to CTA i mod grid,
// whose producer warp streams its items' weights, in increasing order, into a
// shared-memory ring with bulk asynchronous copies (TMA; the blob is tiled
// so that an item is one copy, or k for a routed down item) and mbarriers;
// eight consumer warps compute.  An item waits only on items of lower index
// (routed items on the router, down items on their class's gate/up items,
// routed down rows on the shared down rows).  Every wait is bounded; on
// expiry the kernel records MOE_ERR_TIMEOUT in the status word and drains.
//
// Counters are monotonic (64-bit): a launch derives its epoch from one entry
// count per CTA, so nothing has to be reset between launches.  Programmatic
// dependent launch lets the next layer's CTAs start as SMs free up and
// prefetch the router and shared-expert weights (which do not depend on this
// layer) before they wait for this layer's output.
//
// Arithmetic of the expert dot products: a weight code q (0..15) times an
// activation held as a 16-bit fixed-point value (two int8 limbs, X = 256*hi +
// lo, x ~= X * 2^(E-15) with 2^E above the largest |x| of its block),
// accumulated exactly in int32 with DP4A and scaled in fp32; the fp16 group
// bias multiplies the fp32 sum of the activations.  The input x shares one
// exponent per 64-column group; the intermediate h shares one per 8 values,
// packed by the warp that finishes the gate/up item, and reaches the down
// items by one bulk copy per CTA and class once the class is published.  The
// router dot product is exact: x * 2^24 is an integer below 2^40, split into
// balanced base-256 digits.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace moeq4 {

constexpr int kFusedConsumerWarps = 8;
constexpr int kFusedThreads = (kFusedConsumerWarps + 1) * 32;
constexpr int kFusedMaxStages = 8;
constexpr int kRouterMaxLimbs = 6;
constexpr int kGuRows = 16;                 // intermediate indices per gate/up item
constexpr int kRouterRows = 2;              // expert rows per router item (4 warps per row)
constexpr int kDLimbWords = 24;             // per 32-value chunk of h: 4 x (eh oh el ol fexp sx)
constexpr int kLimbWords = 28;              // per 32-column chunk of x in shared memory (16-byte rows)
constexpr int kMaxDownItems = 4;            // routed down items one CTA keeps residual rows for
constexpr int kRdRows = 16;                 // output rows per routed down item (one down tile)
constexpr int kSdRows = 32;                 // output rows per shared down item (two down tiles)
constexpr int kRedFloats = kFusedConsumerWarps * kRdRows;   // per-stage cross-warp sums
constexpr unsigned long long kWaitNs = 2000000000ull;   // bound of every device wait (2 s)

// Work classes a launch may include (bit mask).
enum : int { kModeRouter = 1, kModeShared = 2, kModeRouted = 4, kModeDown = 8,
             kModeFull = 15 };

struct FusedSync {               // one per launch parity; never reset
    unsigned long long entries;         // CTAs that entered: epoch = entries / grid
    unsigned long long router_done;     // router items finished
    unsigned long long gu_done[2];      // gate/up items finished: [0] shared, [1] routed
    unsigned long long pad[4];
    // routing of the launch: word j < k holds expert j, word 8 + j its weight
    // bits, each tagged with (epoch + 1) in the high 32 bits, so one read of
    // the record tells whether it is current and what it says
    unsigned long long route[2 * MOE_MAX_TOPK];
};

struct FusedArgs {
    const int8_t* Wr;
    const __half* rscale;
    const float* rbias;
    const uint8_t* shared;
    const uint8_t* experts;      // routed blobs: experts + sel_src[j] * stride
    unsigned long long stride;   // bytes between routed expert blobs
    const int32_t* sel_src;      // routing indices (idx_ws) or cache slots
    const __half* x_in;          // x, or the residual h when prenorm
    __half* h_out;               // new residual (prenorm) or nullptr
    __half* x_norm_out;          // optional copy of the normalised input
    float* y;                    // [H]
    int32_t* idx_ws;
    float* w_ws;
    int32_t* idx_out;
    float* w_out;
    double* logits;              // [E]
    uint32_t* dlimb;             // [(k*I + Is) / 32][kDLimbWords] packed h
    // shared-expert down output, one tagged word per row: (launch tag << 32)
    // | fp32 bits, written by one relaxed 64-bit store
    unsigned long long* ysh;     // [H]
    int sync_id;                 // index of this launch's sync block (0..7), part of the tag
    FusedSync* sync;
    int* status;
    unsigned long long* trace;   // optional: kTraceWords per CTA
    unsigned long long wait_ns;  // bound of every device wait
    // hand-off of a split layer: a launch with the shared gate/up items but
    // not their down rows writes shared_seq to *shared_tag once the shared h
    // is complete; a launch with the shared down rows but not the gate/up
    // items waits for it (both null / 0 when unused)
    unsigned long long* shared_tag;
    unsigned long long shared_seq;
    double eps;
    int H, E, k, I, Is, gelu, renorm, prenorm;
    int n_stages, stage_bytes;
    // item counts: router, shared gate/up, shared down, routed gate/up,
    // routed down
    int NR, NSG, NSD, NRG, NRD, NTOT;
};

struct FusedDesc {
    int type;                    // -1 end, 0 router, 1 gate/up, 2 routed down, 3 shared down
    int e_slot;                  // gate/up: 0..k-1 routed, k shared
    int blk;                     // row block
    int rows;                    // router rows in this item
    float w;                     // routing weight of e_slot (1 for shared)
    int item;                    // CTA-local index of a down item (residual rows)
    int pad[2];
};

// ----------------------------------------------------------------- trace --
// Phase stamps written when tracing is on (globaltimer ns; word 8 counts
// items by type in 16-bit fields, word 9 the SM id).
enum { kTrEntry = 0, kTrPrologue = 1, kTrFirstItem = 2, kTrRouting = 3, kTrDownReady = 4,
       kTrConsumerEnd = 5, kTrProducerEnd = 6, kTrTopk = 7, kTrCounts = 8, kTrSm = 9,
       kTrRouterItem = 10, kTrTopkStart = 11, kTrTopkLoaded = 12, kTrTopkSelected = 14,
       kTrProX = 16, kTrProRouterLimbs = 17, kTrProTable = 18, kTrDownLimbs = 19 };

constexpr int kTraceWords = 160;            // per CTA: 32 phase words + items
constexpr int kTracePhase = 32;
constexpr int kTraceItems = (kTraceWords - kTracePhase) / 3;
constexpr unsigned long long kTraceTimeMask = (1ull << 56) - 1;

__device__ __forceinline__ unsigned long long gtimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void fused_trace(const FusedArgs& a, int slot) {
    if (a.trace) a.trace[(size_t)blockIdx.x * kTraceWords + slot] = gtimer_ns();
}

// Per-item stamps: what = 0 copies issued, 1 data ready, 2 item done.
__device__ __forceinline__ void fused_trace_item(const FusedArgs& a, int item, int what,
                                                 int type) {
    if (a.trace && item < kTraceItems)
        a.trace[(size_t)blockIdx.x * kTraceWords + kTracePhase + 3 * item + what] =
            (gtimer_ns() & kTraceTimeMask) | ((unsigned long long)(type + 1) << 56);
}

// ------------------------------------------------------------- waiting --
__device__ __forceinline__ void fused_fail(int* status) { atomicCAS(status, 0, MOE_ERR_TIMEOUT); }

__device__ __forceinline__ bool fused_aborted(const int* status) {
    return ld_relaxed_s32(status) != 0;
}

// Waits longer than this look at the status word in global memory (a load
// that can take microseconds under load, so ordinary waits never issue it).
constexpr unsigned long long kAbortCheckNs = 20000;

// Wait on an mbarrier phase, bounded in time; once the wait is long, gives up
// early when another thread has already recorded a failure.
__device__ __forceinline__ bool fused_wait_bar(uint64_t* bar, uint32_t parity, int* status,
                                               unsigned long long bound = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = gtimer_ns();
    for (unsigned it = 1;; it++) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31) == 0) {
            const unsigned long long el = gtimer_ns() - t0;
            if (el > bound) { fused_fail(status); return false; }
            if (el > kAbortCheckNs && fused_aborted(status)) return false;
        }
    }
}

// Wait until *p >= target, bounded in time.
__device__ __forceinline__ bool fused_wait_ge(const unsigned long long* p,
                                              unsigned long long target, int* status,
                                              unsigned long long bound = kWaitNs) {
    const unsigned long long t0 = gtimer_ns();
    for (unsigned it = 0;; it++) {
        if (ld_acquire_u64(p) >= target) return true;
        __nanosleep(64);
        if ((it & 31) == 31) {
            if (fused_aborted(status)) return false;
            if (gtimer_ns() - t0 > bound) { fused_fail(status); return false; }
        }
    }
}

// ------------------------------------------------------- limb arithmetic --
// Exponent E (m < 2^E, clamped) for a block whose largest |v| is m:
// activations are held as X = rint(v * 2^(15-E)) in [-32768, 32767].
__device__ __forceinline__ int block_exp(float m) {
    const int E = (int)((__float_as_uint(m) >> 23) & 0xff) - 126;
    return max(-100, min(E, 120));
}

__device__ __forceinline__ float exp2_int(int e) {     // 2^e, e in [-126, 127]
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

__device__ __forceinline__ int to_fixed16(float v, int E) {
    const int X = __float2int_rn(v * exp2_int(15 - E));
    return max(-32768, min(X, 32767));
}

// Digit words of 8 activations held as 24-bit fixed point, X = rint(v *
// 2^(23-E)) = 65536 d2 + 256 b1 + b0 (d2 signed, b1 and b0 bytes): each
// digit's bytes of the even and of the odd columns (the nibble extraction
// below yields even and odd columns separately).
__device__ __forceinline__ void word_digits24(const float* v, int E, uint32_t (&d)[6]) {
#pragma unroll
    for (int i = 0; i < 6; i++) d[i] = 0;
    const float sc = exp2_int(23 - E);
#pragma unroll
    for (int n = 0; n < 8; n++) {
        int X = __float2int_rn(v[n] * sc);
        X = max(-8388608, min(X, 8388607));
        const uint32_t b0 = (uint32_t)X & 0xffu, b1 = ((uint32_t)X >> 8) & 0xffu,
                       d2 = (uint32_t)(X >> 16) & 0xffu;
        const int sh = 8 * (n >> 1), o = n & 1;
        d[0 + o] |= d2 << sh;
        d[2 + o] |= b1 << sh;
        d[4 + o] |= b0 << sh;
    }
}

// x digits of one 32-column chunk (one exponent per 64-column group): 24-bit
// fixed point, so a group whose one channel dwarfs the rest keeps the small
// channels to 2^-23 of the group's largest |x|.
struct XLimbs {
    uint32_t d2e[4], d2o[4], b1e[4], b1o[4], b0e[4], b0o[4];
    float fexp;   // 2^(E - 23)
    float sx;     // sum of the 32 activations
};

// h limbs of one 32-value chunk (one exponent per 8 values).
struct HLimbs {
    uint32_t eh[4], oh[4], el[4], ol[4];
    float fexp[4];
    float sx;
};

// sum over a 32-column chunk of code * X: three exact integer partial sums
// (one per digit), combined with one fp32 rounding
__device__ __forceinline__ float chunk_dot_x(uint4 q, const XLimbs& L) {
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
    int a2 = 0;
    unsigned a1 = 0, a0 = 0;
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint32_t lob = wv[w] & 0x0F0F0F0Fu;
        const uint32_t hib = (wv[w] >> 4) & 0x0F0F0F0Fu;
        a2 = __dp4a((int)lob, (int)L.d2e[w], a2);
        a2 = __dp4a((int)hib, (int)L.d2o[w], a2);
        a1 = __dp4a(lob, L.b1e[w], a1);
        a1 = __dp4a(hib, L.b1o[w], a1);
        a0 = __dp4a(lob, L.b0e[w], a0);
        a0 = __dp4a(hib, L.b0o[w], a0);
    }
    return fmaf((float)a2, 65536.0f, (float)(a1 * 256u + a0));
}

// sum over a 32-value chunk of code * h, each 8-value word with its exponent
__device__ __forceinline__ float chunk_dot_h(uint4 q, const HLimbs& L) {
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint32_t lob = wv[w] & 0x0F0F0F0Fu;
        const uint32_t hib = (wv[w] >> 4) & 0x0F0F0F0Fu;
        int ah = __dp4a((int)lob, (int)L.eh[w], 0);
        ah = __dp4a((int)hib, (int)L.oh[w], ah);
        unsigned al = __dp4a(lob, L.el[w], 0u);
        al = __dp4a(hib, L.ol[w], al);
        acc = fmaf((float)(ah * 256 + (int)al), L.fexp[w], acc);
    }
    return acc;
}

__device__ __forceinline__ float h2f_bits(uint16_t b) {
    return __half2float(__ushort_as_half(b));
}

// Sum over the 32 lanes of v[0..N) (N = 4 or 8): afterwards lane l holds the
// total of element l / (32 / N).
template <int N>
__device__ __forceinline__ float reduce_scatter(const float (&v)[N], int lane) {
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
// One warp: top-k of logits[0..E) (largest first, ties to the lower index),
// then the softmax weights of the selected experts, published as the
// launch's tagged routing record (and to the caller's outputs).  Logits become
// order-preserving 64-bit keys; a round is three warp max-reductions (key
// high word, key low word among the leaders, lowest index among exact ties).
// Renormalised weights need only the k selected terms (the full normaliser
// cancels) and are formed in fp32; raw weights use the fp64 softmax over all E.
__device__ __forceinline__ unsigned long long order_key(double d) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(d);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Exact selection by rounds of three max-reductions over the 64-bit keys.
__device__ __forceinline__ void topk_exact_rounds(const FusedArgs& a, const double* v,
                                                  const unsigned long long* key, int lane,
                                                  int& sel, double& sel_l, double& m) {
    constexpr int kPer = MOE_MAX_EXPERTS / 32;
    unsigned taken = 0;
    for (int j = 0; j < a.k; j++) {
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

// Top-k of logits[0..E), largest first, ties to the lower index, then the
// softmax weights of the selected experts, published as the launch's tagged
// routing record and to the caller's outputs.
//
// Fast path (E <= 128): each lane sorts its four experts by a packed word
// (24-bit order key << 8 | 255 - index), and each round takes the maximum of
// the lane heads with one reduction, the winning lane popping its head.  The
// 24-bit key is a monotone function of the logit, so the picked set is the
// exact top-k unless an unpicked expert shares the k-th pick's key, and the
// pick order is exact unless two picks share a key; those cases are settled
// by exact fp64 comparisons (a rank sort of the k picks, or the exact rounds
// over all experts).
__device__ __forceinline__ void fused_topk_publish(const FusedArgs& a, unsigned long long epoch,
                                                   int lane) {
    constexpr int kPer = MOE_MAX_EXPERTS / 32;
    int sel = 0;
    double sel_l = 0.0, m = 0.0;
    bool exact_rounds = a.E > 128;
    if (!exact_rounds) {
        unsigned pk[4];
        double vv[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int e = lane + 32 * i;
            vv[i] = e < a.E ? __ldcg(a.logits + e) : 0.0;
            pk[i] = e < a.E ? ((unsigned)(order_key(vv[i]) >> 40) << 8) | (unsigned)(255 - e) : 0u;
        }
        if (lane == 0) fused_trace(a, kTrTopkLoaded);
        // sorting network, descending: (0,1) (2,3) (0,2) (1,3) (1,2)
#define MOEQ4_CSWAP(i, j)                                                  \
        if (pk[j] > pk[i]) {                                               \
            const unsigned tk = pk[i]; pk[i] = pk[j]; pk[j] = tk;          \
            const double tv = vv[i]; vv[i] = vv[j]; vv[j] = tv;            \
        }
        MOEQ4_CSWAP(0, 1) MOEQ4_CSWAP(2, 3) MOEQ4_CSWAP(0, 2) MOEQ4_CSWAP(1, 3) MOEQ4_CSWAP(1, 2)
#undef MOEQ4_CSWAP
        unsigned mk = 0, last = 0;
        for (int j = 0; j < a.k; j++) {
            const unsigned w = __reduce_max_sync(0xffffffffu, pk[0]);
            const int e = 255 - (int)(w & 255u);
            const int wl = e & 31;
            const double wv = __shfl_sync(0xffffffffu, vv[0], wl);
            if (lane == j) { sel = e; sel_l = wv; mk = w; }
            if (lane == wl) {
                pk[0] = pk[1]; pk[1] = pk[2]; pk[2] = pk[3]; pk[3] = 0u;
                vv[0] = vv[1]; vv[1] = vv[2]; vv[2] = vv[3];
            }
            last = w >> 8;
        }
        // a lane's head is its largest unpicked expert
        exact_rounds = __any_sync(0xffffffffu, pk[0] != 0u && (pk[0] >> 8) == last);
        if (!exact_rounds) {
            const unsigned nx = __shfl_down_sync(0xffffffffu, mk, 1);
            if (__any_sync(0xffffffffu, lane + 1 < a.k && (mk >> 8) == (nx >> 8))) {
                // order the k picks exactly: rank by (logit desc, index asc)
                int rank = 0;
                for (int i = 0; i < a.k; i++) {
                    const double vi = __shfl_sync(0xffffffffu, sel_l, i);
                    const int ei = __shfl_sync(0xffffffffu, sel, i);
                    if (lane < a.k && (vi > sel_l || (vi == sel_l && ei < sel))) rank++;
                }
                int s2 = sel;
                double l2 = sel_l;
                for (int i = 0; i < a.k; i++) {
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
    double v[kPer];
    if (exact_rounds || !a.renorm) {
#pragma unroll
        for (int i = 0; i < kPer; i++) {
            const int e = lane + 32 * i;
            v[i] = e < a.E ? __ldcg(a.logits + e) : 0.0;
        }
    }
    if (exact_rounds) {
        unsigned long long key[kPer];
#pragma unroll
        for (int i = 0; i < kPer; i++)
            key[i] = lane + 32 * i < a.E ? order_key(v[i]) : 0ull;   // 0 sorts below every logit
        topk_exact_rounds(a, v, key, lane, sel, sel_l, m);
    }
    if (lane == 0) fused_trace(a, kTrTopkSelected);
    float w = 0.f;
    if (a.renorm) {
        const float p = lane < a.k ? expf((float)(sel_l - m)) : 0.f;
        w = p / warp_sum(p);
    } else {
        double zz = 0.0;
#pragma unroll
        for (int i = 0; i < kPer; i++)
            if (lane + 32 * i < a.E) zz += exp(v[i] - m);
        const double z = warp_sum(zz);
        w = lane < a.k ? (float)(exp(sel_l - m) / z) : 0.f;
    }
    if (lane < a.k) {
        const unsigned long long tag = (epoch + 1) << 32;
        a.sync->route[lane] = tag | (unsigned)sel;
        a.sync->route[MOE_MAX_TOPK + lane] = tag | __float_as_uint(w);
        a.idx_ws[lane] = sel;
        a.w_ws[lane] = w;
        if (a.idx_out) a.idx_out[lane] = sel;
        if (a.w_out) a.w_out[lane] = w;
    }
    __syncwarp();
}

// Number of q in [lo, hi) with q = b (mod G).
__device__ __forceinline__ int count_mod(int lo, int hi, int b, int G) {
    if (hi <= lo) return 0;
    const int first = lo + ((b - lo % G) % G + G) % G;
    return first >= hi ? 0 : (hi - 1 - first) / G + 1;
}

// Stage layouts (bytes): router item: kRouterRows rows of int8 [H];
// gate/up item: one gate/up tile (gate codes [16][H/2], up codes [16][H/2],
// gate scales [16][H/64] fp16, up scales, gate biases, up biases: 18 H);
// shared down item: two down tiles of the shared expert (codes [16][Is/2],
// scales [16][Is/64], biases [16][Is/64]: 9 Is each); routed down item: one
// down tile (9 I) of each of the k routed experts, expert j at j * 9 I.

// ------------------------------------------------------------- producer --
struct ProducerShared {
    int32_t sel[MOE_MAX_TOPK];
    float selw[MOE_MAX_TOPK];
};

// The producer warp learns the routing: from this launch's routing record
// (one read per lane, current once every word carries this epoch's tag), or,
// when the launch has no router items, from an earlier launch on the same
// stream (sel_src, w_ws).
__device__ __forceinline__ bool fused_get_routing(const FusedArgs& a,
                                                  volatile unsigned long long* ep_slot,
                                                  ProducerShared* ps, int lane) {
    if (a.NR > 0) {
        bool ok = true;
        if (lane == 0) {
            const unsigned long long t0 = gtimer_ns();
            while (*ep_slot == 0)
                if (gtimer_ns() - t0 > a.wait_ns) { fused_fail(a.status); ok = false; break; }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) return false;
        const unsigned long long tag = *ep_slot;             // epoch + 1
        const bool mine = lane < a.k || (lane >= MOE_MAX_TOPK && lane < MOE_MAX_TOPK + a.k);
        unsigned long long word = 0;
        const unsigned long long t0 = gtimer_ns();
        for (unsigned it = 0;; it++) {
            if (mine) word = ld_relaxed_u64(&a.sync->route[lane]);
            if (__all_sync(0xffffffffu, !mine || (word >> 32) == tag)) break;
            __nanosleep(32);
            if ((it & 31) == 31) {
                const bool bad = lane == 0 && (fused_aborted(a.status) || gtimer_ns() - t0 > a.wait_ns);
                if (__any_sync(0xffffffffu, bad)) {
                    if (lane == 0) fused_fail(a.status);
                    return false;
                }
            }
        }
        if (lane < a.k) ps->sel[lane] = (int32_t)(unsigned)word;
        if (lane >= MOE_MAX_TOPK && lane < MOE_MAX_TOPK + a.k)
            ps->selw[lane - MOE_MAX_TOPK] = __uint_as_float((unsigned)word);
    } else {
        if (lane < a.k) {
            ps->sel[lane] = __ldcg(a.sel_src + lane);
            ps->selw[lane] = __ldcg(a.w_ws + lane);
        }
    }
    __syncwarp();
    if (lane == 0) fused_trace(a, kTrRouting);
    return true;
}

__device__ __forceinline__ void fused_producer(const FusedArgs& a, uint8_t* stages, FusedDesc* desc,
                                               uint64_t* full, uint64_t* empty,
                                               volatile unsigned long long* ep_slot,
                                               ProducerShared* ps, int lane) {
    const int H = a.H;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t outstanding = 0, issued_parity = 0;     // bit per stage
    bool have_routing = false, ok = true;
    int n_issued = 0, n_down = 0;
    for (int q = blockIdx.x; q < a.NTOT; q += gridDim.x) {
        ok = __shfl_sync(0xffffffffu, (lane == 0 && fused_aborted(a.status)) ? 0 : 1, 0) != 0;
        if (!ok) break;
        FusedDesc d;
        d.w = 1.f;
        d.rows = kRouterRows;
        d.e_slot = 0;
        d.item = 0;
        d.pad[0] = d.pad[1] = 0;
        bool needs_routing = false;
        const int q1 = a.NR + a.NSG, q2 = q1 + a.NRG, q3 = q2 + a.NSD;
        if (q < a.NR) {
            d.type = 0; d.blk = q; d.rows = min(kRouterRows, a.E - kRouterRows * q);
        } else if (q < q1) {                                // shared gate/up tile
            d.type = 1; d.e_slot = a.k; d.blk = q - a.NR;
        } else if (q < q2) {                                // routed gate/up tile
            const int r = q - q1;
            const int per = a.I / kGuRows;
            d.type = 1; d.e_slot = r / per; d.blk = r % per;
            needs_routing = true;
        } else if (q < q3) {                                // shared down: 32 rows
            d.type = 3; d.e_slot = a.k; d.blk = q - q2;
        } else {                                            // routed down: 16 rows x k
            d.type = 2; d.blk = q - q3; d.item = n_down++;
            needs_routing = true;
        }
        if (needs_routing && !have_routing) {
            if (!fused_get_routing(a, ep_slot, ps, lane)) { ok = false; break; }
            have_routing = true;
        }
        if (d.type == 1 && d.e_slot < a.k) d.w = ps->selw[d.e_slot];
        if (lane == 0) {
            ok = fused_wait_bar(&empty[stage], phase ^ 1u, a.status, a.wait_ns);
            if (ok) {
                desc[stage] = d;
                uint8_t* dst = stages + (size_t)stage * a.stage_bytes;
                uint64_t* bar = &full[stage];
                if (d.type == 0) {
                    const uint32_t bytes = (uint32_t)d.rows * H;
                    mbar_arrive_expect_tx(bar, bytes);
                    bulk_g2s(dst, a.Wr + (size_t)d.blk * kRouterRows * H, bytes, bar);
                } else if (d.type == 1) {                   // one gate/up tile: one copy
                    const int Ie = d.e_slot < a.k ? a.I : a.Is;
                    const uint8_t* blob = d.e_slot < a.k
                                              ? a.experts + (size_t)ps->sel[d.e_slot] * a.stride
                                              : a.shared;
                    const BlobLayout L(H, Ie);
                    mbar_arrive_expect_tx(bar, (uint32_t)L.gu_tile);
                    bulk_g2s(dst, blob + (size_t)d.blk * L.gu_tile, (uint32_t)L.gu_tile, bar);
                } else if (d.type == 3) {                   // two shared down tiles: one copy
                    const BlobLayout L(H, a.Is);
                    const uint32_t bytes = 2u * (uint32_t)L.dn_tile;
                    mbar_arrive_expect_tx(bar, bytes);
                    bulk_g2s(dst, a.shared + L.dn_base + (size_t)(2 * d.blk) * L.dn_tile, bytes, bar);
                } else {                                    // one down tile of each routed expert
                    const BlobLayout L(H, a.I);
                    mbar_arrive_expect_tx(bar, (uint32_t)(a.k * L.dn_tile));
                    for (int e = 0; e < a.k; e++)
                        bulk_g2s(dst + (size_t)e * L.dn_tile,
                                 a.experts + (size_t)ps->sel[e] * a.stride + L.dn_base +
                                     (size_t)d.blk * L.dn_tile,
                                 (uint32_t)L.dn_tile, bar);
                }
                fused_trace_item(a, n_issued, 0, d.type);
            }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        n_issued++;
        outstanding |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == a.n_stages) { stage = 0; phase ^= 1u; }
    }
    if (lane != 0) return;
    fused_trace(a, kTrProducerEnd);
    // end marker for the consumers
    if (ok && fused_wait_bar(&empty[stage], phase ^ 1u, a.status, a.wait_ns)) {
        desc[stage].type = -1;
        outstanding &= ~(1u << stage);   // its data phase was consumed before release
        mbar_arrive(&full[stage]);
    }
    // never leave while a bulk copy into shared memory is in flight
    for (int s = 0; s < a.n_stages; s++)
        if ((outstanding >> s) & 1u) {
            const unsigned long long t0 = gtimer_ns();
            while (!mbar_try_wait(&full[s], (issued_parity >> s) & 1u))
                if (gtimer_ns() - t0 > a.wait_ns) { fused_fail(a.status); break; }
        }
}

// ------------------------------------------------------------- consumers --
struct ConsumerShared {
    unsigned long long rsum[kFusedMaxStages][kRouterRows];   // exact router row sums
    double rscale[kRouterRows];          // row scales / biases of the first router item
    double rbias[kRouterRows];
    int item_cnt[kFusedMaxStages];       // warps done with the stage's item
    int down_flag;                       // all gate/up items of the launch done
    int gu_cls_done[2];                  // this CTA's finished shared / routed gate/up items
    unsigned long long ep1;              // epoch + 1 (for the producer)
    unsigned long long sc[20];           // reductions
    __half h_rows[kMaxDownItems * kRdRows];   // residual rows of this CTA's routed down items
};

__device__ __forceinline__ FusedDesc fused_read_desc(const FusedDesc* p) {
    FusedDesc d;
    const uint32_t ds = smem_u32(p);
    const uint4 d0 = lds128(ds);
    const uint4 d1 = lds128(ds + 16);
    d.type = (int)d0.x; d.e_slot = (int)d0.y; d.blk = (int)d0.z; d.rows = (int)d0.w;
    d.w = __uint_as_float(d1.x); d.item = (int)d1.y;
    d.pad[0] = d.pad[1] = 0;
    return d;
}

template <int MAXC, int MAXD>
__device__ __forceinline__ void fused_consumers(const FusedArgs& a, uint8_t* stages, FusedDesc* desc,
                                                uint64_t* full, uint64_t* empty, __half* xs,
                                                int8_t* xl, float* red, uint32_t* glimb,
                                                uint8_t* hl, uint64_t* hl_bar, uint8_t* hls,
                                                uint64_t* hls_bar, ConsumerShared* cs) {
    const int tid = threadIdx.x;                 // 0..255
    const int warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int nthr = kFusedConsumerWarps * 32;
    unsigned long long* sc = cs->sc;

    // ---- prologue: this launch's epoch (the atomic's latency hides behind
    // the wait below), then this layer's input (waits for the previous layer)
    unsigned long long ent = 0;
    if (tid == 0) ent = atomicAdd(&a.sync->entries, 1ull);
    // this CTA's first router item's row scales and biases (weights: they do
    // not depend on the previous layer)
    if (tid < kRouterRows && (int)blockIdx.x < a.NR) {
        const int e = kRouterRows * (int)blockIdx.x + tid;
        cs->rscale[tid] = e < a.E ? (double)__half2float(a.rscale[e]) : 0.0;
        cs->rbias[tid] = (e < a.E && a.rbias) ? (double)a.rbias[e] : 0.0;
    }
    griddep_wait();
    constexpr int kHPer = 16;                    // h values per thread (H <= 4096)
    if (a.prenorm) {
        // residual row of this CTA's routed down items (for the final h + y),
        // loaded with the input so that both round trips overlap
        __half hres = __float2half(0.f);
        int hres_t = -1;
        if (a.NRD > 0 && tid < kMaxDownItems * kRdRows) {
            const int d0 = a.NR + a.NSG + a.NSD + a.NRG;
            int q0 = blockIdx.x;
            while (q0 < d0) q0 += gridDim.x;
            const int q = q0 + (tid / kRdRows) * gridDim.x;
            if (q < a.NTOT) {
                hres_t = tid;
                hres = __ushort_as_half(__ldcg((const unsigned short*)a.x_in + kRdRows * (q - d0) + (tid % kRdRows)));
            }
        }
        __half hv[kHPer];
        unsigned __int128 acc = 0;
#pragma unroll
        for (int i = 0; i < kHPer; i++) {
            const int c = tid + nthr * i;
            hv[i] = c < H ? __ushort_as_half(__ldcg((const unsigned short*)a.x_in + c))
                          : __float2half(0.f);
            const long long X = half_fixed24(hv[i]);
            acc += (unsigned __int128)((__int128)X * (__int128)X);
        }
        acc = warp_sum_u128(acc);
        if (lane == 0) { sc[2 * warp] = (unsigned long long)(acc >> 64); sc[2 * warp + 1] = (unsigned long long)acc; }
        named_bar(1, nthr);
        // every thread forms the same exact total and the same 1 / rms
        double r;
        {
            unsigned __int128 tot = 0;
            for (int w = 0; w < kFusedConsumerWarps; w++)
                tot += ((unsigned __int128)sc[2 * w] << 64) | sc[2 * w + 1];
            const double s = __dmul_rn(u128_to_double_rn(tot), 0x1p-48);
            const double ms = __ddiv_rn(s, (double)H);
            r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, a.eps)));
        }
#pragma unroll
        for (int i = 0; i < kHPer; i++) {
            const int c = tid + nthr * i;
            if (c < H) xs[c] = __double2half(__dmul_rn((double)__half2float(hv[i]), r));
        }
        if (hres_t >= 0) cs->h_rows[hres_t] = hres;
    } else {
        for (int c = tid; c < H / 8; c += nthr)
            reinterpret_cast<uint4*>(xs)[c] = __ldcg(reinterpret_cast<const uint4*>(a.x_in) + c);
    }
    if (tid == 0) {
        sc[17] = 0;
        sc[18] = ent / gridDim.x;                                   // epoch
        *(volatile unsigned long long*)&cs->ep1 = ent / gridDim.x + 1;
    }
    named_bar(1, nthr);
    const unsigned long long ep = sc[18];
    if (tid == 0) fused_trace(a, kTrProX);
    // the next layer may start scheduling now that this one has its input
    if (tid == 0) griddep_launch_dependents();
    if (blockIdx.x == 0 && a.x_norm_out)
        for (int c = tid; c < H; c += nthr) a.x_norm_out[c] = xs[c];

    // ---- exact router limbs: x * 2^24 in balanced base-256 digits; NL
    // digits cover the largest |x| of this token (int32 arithmetic while
    // NL <= 4, int64 beyond)
    int NL = 1;
    if (a.NR > 0 && (int)blockIdx.x < a.NR) {
        float mx = 0.f;
        for (int c = tid; c < H; c += nthr) mx = fmaxf(mx, fabsf(__half2float(xs[c])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(&sc[17]), __float_as_uint(mx));
        named_bar(1, nthr);
        {
            const double xmax = (double)__uint_as_float((unsigned)sc[17]) * 16777216.0;
            double cap = 127.0;                      // 127 * (256^NL - 1) / 255
            while (NL < kRouterMaxLimbs && xmax > cap) { NL++; cap = cap * 256.0 + 127.0; }
        }
        for (int c4 = tid; c4 < H / 4; c4 += nthr) {
            uint32_t packed[kRouterMaxLimbs];
#pragma unroll
            for (int dg = 0; dg < kRouterMaxLimbs; dg++) packed[dg] = 0;
#pragma unroll
            for (int t = 0; t < 4; t++) {
                const float xf = __half2float(xs[4 * c4 + t]) * 16777216.0f;   // exact
                if (NL <= 4) {
                    int X = __float2int_rn(xf);
#pragma unroll
                    for (int dg = 0; dg < 4; dg++) {
                        const int digit = ((X + 128) & 255) - 128;
                        packed[dg] |= (uint32_t)(digit & 255) << (8 * t);
                        X = (X - digit) >> 8;
                    }
                } else {
                    long long X = __float2ll_rn(xf);
#pragma unroll
                    for (int dg = 0; dg < kRouterMaxLimbs; dg++) {
                        const int digit = (int)((X + 128) & 255) - 128;
                        packed[dg] |= (uint32_t)(digit & 255) << (8 * t);
                        X = (X - digit) >> 8;
                    }
                }
            }
#pragma unroll
            for (int dg = 0; dg < kRouterMaxLimbs; dg++)
                if (dg < NL) reinterpret_cast<uint32_t*>(xl + dg * H)[c4] = packed[dg];
        }
        named_bar(1, nthr);
    }
    if (tid == 0) fused_trace(a, kTrProRouterLimbs);


    // ---- h limbs for the routed down rows: thread tid owns chunk tid + 256 j
    // of the routed intermediate (experts 0..k-1), loaded once every routed
    // gate/up item of the launch is done
    HLimbs dl[MAXD];
    int dq_off[MAXD], ds_off[MAXD];
    bool dvalid[MAXD];
    bool down_ready = false, sdown_ready = false;
    const int NCr = a.k * a.I / 32;                  // routed chunks
    const int NCs = a.Is / 32;                       // shared chunks
    // gate/up items of this CTA per class: the last of a class publishes
    const int q1 = a.NR + a.NSG, q2 = q1 + a.NRG;
    const int n_cls0 = count_mod(a.NR, q1, (int)blockIdx.x, (int)gridDim.x);
    const int n_cls1 = count_mod(q1, q2, (int)blockIdx.x, (int)gridDim.x);
    // this launch's tag of the shared down words: unique per (sync block,
    // epoch), so a word left by an earlier launch never matches
    const unsigned long long tag =
        (unsigned long long)(unsigned)((ep + 1) * 8 + (unsigned long long)a.sync_id) << 32;
    unsigned cnt_r = 0, cnt_gu = 0, cnt_g = 0, cnt_d = 0;
    int n_done = 0;
    bool first = true;

    int stage = 0;
    uint32_t phase = 0;
    // ---- router items first: a CTA's router items are its first items, and
    // the routing they lead to is the critical path of the launch
    bool aborted = false;
    const int n_router = (int)blockIdx.x < a.NR ? (a.NR - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    for (int ri = 0; ri < n_router; ri++) {
        if (!fused_wait_bar(&full[stage], phase, a.status, a.wait_ns)) { aborted = true; break; }
        const FusedDesc d = fused_read_desc(desc + stage);
        const uint32_t st_s = smem_u32(stages) + (uint32_t)stage * a.stage_bytes;
        if (first) {
            if (warp == 0 && lane == 0) fused_trace(a, kTrFirstItem);
            first = false;
        }
        if (warp == 0 && lane == 0) fused_trace_item(a, n_done, 1, d.type);
        {
            // -------- router rows: warp w -> row w / 4 of the item, quarter
            // w % 4 of its columns; exact partial sums meet in shared memory
            cnt_r++;
            const int row = warp >> 2, qt = warp & 3;
            // lane r holds row r's scale and bias for whichever warp turns
            // out to finish the item (the first item's were loaded at entry)
            double scale = 0.0, bias = 0.0;
            if (lane < d.rows) {
                if (ri == 0) {
                    scale = cs->rscale[lane];
                    bias = cs->rbias[lane];
                } else {
                    scale = (double)__half2float(a.rscale[kRouterRows * d.blk + lane]);
                    if (a.rbias) bias = (double)a.rbias[kRouterRows * d.blk + lane];
                }
            }
            if (row < d.rows) {
                int acc[kRouterMaxLimbs];
#pragma unroll
                for (int dg = 0; dg < kRouterMaxLimbs; dg++) acc[dg] = 0;
                const int nq = H / 64;                                    // 16-byte chunks per quarter
                const uint32_t wrow = st_s + (uint32_t)(row * H);
                const uint32_t xl_s = smem_u32(xl);
                for (int j = qt * nq + lane; j < (qt + 1) * nq; j += 32) {
                    const uint4 w4 = lds128(wrow + 16 * j);
#pragma unroll
                    for (int dg = 0; dg < kRouterMaxLimbs; dg++) {
                        if (dg < NL) {
                            const uint4 l4 = lds128(xl_s + (uint32_t)(dg * H) + 16 * j);
                            int s = acc[dg];
                            s = __dp4a((int)w4.x, (int)l4.x, s);
                            s = __dp4a((int)w4.y, (int)l4.y, s);
                            s = __dp4a((int)w4.z, (int)l4.z, s);
                            s = __dp4a((int)w4.w, (int)l4.w, s);
                            acc[dg] = s;
                        }
                    }
                }
                long long S = 0;
#pragma unroll
                for (int dg = 0; dg < kRouterMaxLimbs; dg++)
                    if (dg < NL) S += (long long)acc[dg] * (1ll << (8 * dg));
                S = warp_sum(S);
                if (lane == 0) atomicAdd(&cs->rsum[stage][row], (unsigned long long)S);
            }
            // the last of the eight warps turns the exact sums into logits
            // and publishes the item
            int old = 0;
            if (lane == 0) {
                fence_acq_rel_cta();
                old = atomicAdd(&cs->item_cnt[stage], 1);
            }
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old == kFusedConsumerWarps - 1) {
                fence_acq_rel_cta();
                if (lane < d.rows) {
                    const long long S = (long long)((volatile unsigned long long*)cs->rsum[stage])[lane];
                    const int er = kRouterRows * d.blk + lane;
                    double l = __ll2double_rn(S);
                    l = __dmul_rn(l, 0x1p-24);
                    l = __dmul_rn(l, scale);
                    if (a.rbias) l = __dadd_rn(l, bias);
                    a.logits[er] = l;
                    cs->rsum[stage][lane] = 0;
                }
                __syncwarp();
                unsigned long long rd = 0;
                if (lane == 0) {
                    cs->item_cnt[stage] = 0;
                    fence_acq_rel_gpu();
                    rd = atomicAdd(&a.sync->router_done, 1ull);
                    fused_trace(a, kTrRouterItem);
                }
                rd = __shfl_sync(0xffffffffu, rd, 0);
                if (rd == (ep + 1) * (unsigned long long)a.NR - 1) {
                    // this warp finished the launch's last router item
                    fence_acq_rel_gpu();
                    if (lane == 0) fused_trace(a, kTrTopkStart);
                    fused_topk_publish(a, ep, lane);
                    if (lane == 0) fused_trace(a, kTrTopk);
                }
            }
        }
        __syncwarp();
        if (warp == 0 && lane == 0) fused_trace_item(a, n_done, 2, d.type);
        n_done++;
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == a.n_stages) { stage = 0; phase ^= 1u; }
    }

    // ---- x limbs: one thread per 8-column word builds the shared table
    // (group max over the 8 words of its 64-column group by shuffles); lane
    // then owns chunks lane + 32 i of every row
    const int nch = H / 32;
    const uint32_t xs_s = smem_u32(xs);
    const uint32_t gl_s = smem_u32(glimb);
    if (a.NSG + a.NRG > 0) {          // every consumer thread reaches the barrier below
        for (int base = 0; base < H / 8; base += nthr) {
            const int wd = base + tid;
            const bool valid = wd < H / 8;
            float v[8];
            float m = 0.f, sx = 0.f;
            {
                const uint4 q = valid ? lds128(xs_s + 16 * wd) : make_uint4(0, 0, 0, 0);
                const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&qq[u]));
                    v[2 * u] = f.x;
                    v[2 * u + 1] = f.y;
                    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
                    sx += f.x + f.y;
                }
            }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            sx += __shfl_xor_sync(0xffffffffu, sx, 1);
            sx += __shfl_xor_sync(0xffffffffu, sx, 2);
            const int E = block_exp(m);
            uint32_t dg[6];
            word_digits24(v, E, dg);
            if (valid) {
                const int c = wd >> 2, j = wd & 3;
                uint32_t* dst = glimb + (size_t)c * kLimbWords;
                dst[j] = dg[0]; dst[4 + j] = dg[1]; dst[8 + j] = dg[2]; dst[12 + j] = dg[3];
                dst[16 + j] = dg[4]; dst[20 + j] = dg[5];
                if (j == 0) {
                    dst[24] = __float_as_uint(exp2_int(E - 23));
                    dst[25] = __float_as_uint(sx);
                }
            }
        }
        named_bar(1, nthr);
    }
    XLimbs gl[MAXC];
#pragma unroll
    for (int i = 0; i < MAXC; i++) {
        const int c = lane + 32 * i;
        const uint32_t src = gl_s + 4u * (uint32_t)((c < nch ? c : 0) * kLimbWords);
        const uint4 a0 = lds128(src), a1 = lds128(src + 16), a2 = lds128(src + 32),
                    a3 = lds128(src + 48), a4 = lds128(src + 64), a5 = lds128(src + 80);
        gl[i].d2e[0] = a0.x; gl[i].d2e[1] = a0.y; gl[i].d2e[2] = a0.z; gl[i].d2e[3] = a0.w;
        gl[i].d2o[0] = a1.x; gl[i].d2o[1] = a1.y; gl[i].d2o[2] = a1.z; gl[i].d2o[3] = a1.w;
        gl[i].b1e[0] = a2.x; gl[i].b1e[1] = a2.y; gl[i].b1e[2] = a2.z; gl[i].b1e[3] = a2.w;
        gl[i].b1o[0] = a3.x; gl[i].b1o[1] = a3.y; gl[i].b1o[2] = a3.z; gl[i].b1o[3] = a3.w;
        gl[i].b0e[0] = a4.x; gl[i].b0e[1] = a4.y; gl[i].b0e[2] = a4.z; gl[i].b0e[3] = a4.w;
        gl[i].b0o[0] = a5.x; gl[i].b0o[1] = a5.y; gl[i].b0o[2] = a5.z; gl[i].b0o[3] = a5.w;
        gl[i].fexp = __uint_as_float(lds32(src + 96));
        gl[i].sx = __uint_as_float(lds32(src + 100));
    }
    if (tid == 0) fused_trace(a, kTrProTable);
    fused_trace(a, kTrPrologue);

    // ---- gate/up and down items
    for (;;) {
        if (aborted || !fused_wait_bar(&full[stage], phase, a.status, a.wait_ns)) break;
        FusedDesc d = fused_read_desc(desc + stage);
        if (d.type < 0) break;
        const uint32_t st_s = smem_u32(stages) + (uint32_t)stage * a.stage_bytes;
        float* rs = red + (size_t)stage * kRedFloats;
        if (first) {
            if (warp == 0 && lane == 0) fused_trace(a, kTrFirstItem);
            first = false;
        }
        if (warp == 0 && lane == 0) fused_trace_item(a, n_done, 1, d.type);
        if (d.type == 1) {
            // -------- gate/up rows: warp w -> intermediate indices
            // 16*blk + 2w and + 2w + 1 (gate rows and up rows of both)
            cnt_gu++;
            if (d.e_slot < a.k) cnt_g++;
            const uint32_t qrow = H / 2, srow = H / 32;
            const uint32_t gq = st_s + 2 * warp * qrow;
            const uint32_t uq = st_s + 8u * H + 2 * warp * qrow;
            const uint32_t gs = st_s + 16u * H + 2 * warp * srow;
            const uint32_t us = gs + H / 2, gb = gs + H, ub = gs + 3 * H / 2;
            float v4[4] = {0.f, 0.f, 0.f, 0.f};         // gate0, gate1, up0, up1
#pragma unroll
            for (int i = 0; i < MAXC; i++) {
                const int c = lane + 32 * i;
                if (c < nch) {
                    const uint32_t grp2 = 2 * (c >> 1);
#pragma unroll
                    for (int r = 0; r < 2; r++) {
                        const uint4 qg = lds128(gq + r * qrow + 16 * c);
                        const uint4 qu = lds128(uq + r * qrow + 16 * c);
                        const float dg = chunk_dot_x(qg, gl[i]);
                        const float du = chunk_dot_x(qu, gl[i]);
                        v4[r] = fmaf(h2f_bits(lds16(gs + r * srow + grp2)) * gl[i].fexp, dg, v4[r]);
                        v4[r] = fmaf(h2f_bits(lds16(gb + r * srow + grp2)), gl[i].sx, v4[r]);
                        v4[2 + r] = fmaf(h2f_bits(lds16(us + r * srow + grp2)) * gl[i].fexp, du, v4[2 + r]);
                        v4[2 + r] = fmaf(h2f_bits(lds16(ub + r * srow + grp2)), gl[i].sx, v4[2 + r]);
                    }
                }
            }
            // lane l holds the total of v4[l / 8]: gate r at lanes 8r.., up r at 16 + 8r..
            const float tot = reduce_scatter<4>(v4, lane);
            const float up = __shfl_xor_sync(0xffffffffu, tot, 16);
            if (lane == 0 || lane == 8) {
                const float h = gelu_f(tot, a.gelu) * up * d.w;
                rs[2 * warp + (lane >> 3)] = h;
            }
            __syncwarp();
            // the last warp of the item packs its 16 intermediate values into
            // two 8-value limb words of the global h table
            int v = 0;
            if (lane == 0) {
                fence_acq_rel_cta();
                v = atomicAdd(&cs->item_cnt[stage], 1);
            }
            v = __shfl_sync(0xffffffffu, v, 0);
            if (v == kFusedConsumerWarps - 1) {
                fence_acq_rel_cta();
                const float hvv = lane < 16 ? ((volatile float*)rs)[lane] : 0.f;
                float m = fabsf(hvv), sx = hvv;
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    sx += __shfl_xor_sync(0xffffffffu, sx, o);
                }
                const int E = block_exp(m);
                const int X = to_fixed16(hvv, E);
                uint8_t* wb = reinterpret_cast<uint8_t*>(rs + 16);       // 2 words x 16 bytes
                if (lane < 16) {
                    const int word = lane >> 3, n = lane & 7;
                    const int kind = (n & 1) ? 4 : 0;                    // bytes: eh oh el ol
                    wb[16 * word + kind + (n >> 1)] = (uint8_t)((X >> 8) & 0xff);
                    wb[16 * word + 8 + kind + (n >> 1)] = (uint8_t)(X & 0xff);
                }
                __syncwarp();
                if (lane == 0 || lane == 8) {
                    const int word = lane >> 3;
                    const uint32_t* wv = reinterpret_cast<const uint32_t*>(wb + 16 * word);
                    const int koff = d.e_slot * a.I;                     // shared follows the k routed
                    const int wd = (koff + kGuRows * d.blk) / 8 + word;
                    uint32_t* dst = a.dlimb + (size_t)(wd >> 2) * kDLimbWords + (wd & 3);
                    dst[0] = wv[0];
                    dst[4] = wv[1];
                    dst[8] = wv[2];
                    dst[12] = wv[3];
                    dst[16] = __float_as_uint(exp2_int(E - 15));
                    dst[20] = __float_as_uint(sx);
                }
                __syncwarp();
                if (lane == 0) {
                    cs->item_cnt[stage] = 0;
                    fence_acq_rel_cta();
                    // the CTA's last item of its class publishes the class
                    const int cls = d.e_slot < a.k ? 1 : 0;
                    const int n_c = cls ? n_cls1 : n_cls0;
                    if (atomicAdd(&cs->gu_cls_done[cls], 1) + 1 == n_c) {
                        fence_acq_rel_gpu();
                        const unsigned long long old = atomicAdd(&a.sync->gu_done[cls], (unsigned long long)n_c);
                        // the CTA completing the shared class hands the shared h
                        // over to a later launch that holds its down rows
                        if (cls == 0 && a.shared_tag && a.NSD == 0 &&
                            old + (unsigned long long)n_c == (ep + 1) * (unsigned long long)a.NSG) {
                            fence_acq_rel_gpu();
                            st_release_u64(a.shared_tag, a.shared_seq);
                        }
                    }
                }
            }
        } else if (d.type == 3) {
            // -------- shared down rows: 32 rows of the shared expert; warp w
            // takes rows 4w..4w+3, lane l the 32-value chunks l, l + 32, ...
            // of the shared h, whose packed limbs come into shared memory by
            // one bulk copy once the launch's shared gate/up items are done
            if (!sdown_ready) {
                bool ok = true;
                if (warp == 0 && lane == 0) {
                    ok = a.NSG == 0 && a.shared_tag
                             ? fused_wait_ge(a.shared_tag, a.shared_seq, a.status, a.wait_ns)
                             : fused_wait_ge(&a.sync->gu_done[0], (ep + 1) * (unsigned long long)a.NSG, a.status,
                                             a.wait_ns);
                    if (ok) {
                        fence_proxy_async_global();
                        const uint32_t bytes = (uint32_t)NCs * kDLimbWords * 4;
                        mbar_arrive_expect_tx(hls_bar, bytes);
                        bulk_g2s(hls, a.dlimb + (size_t)NCr * kDLimbWords, bytes, hls_bar);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok || !fused_wait_bar(hls_bar, 0, a.status, a.wait_ns)) break;
                sdown_ready = true;
            }
            const uint32_t Is = (uint32_t)a.Is, hls_s = smem_u32(hls);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int c = lane; c < NCs; c += 32) {
                HLimbs L;
                const uint32_t src = hls_s + (uint32_t)c * (kDLimbWords * 4);
                const uint4 t0 = lds128(src), t1 = lds128(src + 16), t2 = lds128(src + 32),
                            t3 = lds128(src + 48), t4 = lds128(src + 64), t5 = lds128(src + 80);
                L.eh[0] = t0.x; L.eh[1] = t0.y; L.eh[2] = t0.z; L.eh[3] = t0.w;
                L.oh[0] = t1.x; L.oh[1] = t1.y; L.oh[2] = t1.z; L.oh[3] = t1.w;
                L.el[0] = t2.x; L.el[1] = t2.y; L.el[2] = t2.z; L.el[3] = t2.w;
                L.ol[0] = t3.x; L.ol[1] = t3.y; L.ol[2] = t3.z; L.ol[3] = t3.w;
                L.fexp[0] = __uint_as_float(t4.x); L.fexp[1] = __uint_as_float(t4.y);
                L.fexp[2] = __uint_as_float(t4.z); L.fexp[3] = __uint_as_float(t4.w);
                L.sx = __uint_as_float(t5.x) + __uint_as_float(t5.y) + __uint_as_float(t5.z) +
                       __uint_as_float(t5.w);
                const uint32_t g2 = 2u * (uint32_t)(c >> 1);
#pragma unroll
                for (int r = 0; r < 4; r++) {
                    const int ir = 4 * warp + r;                      // row of the item
                    const uint32_t tb = st_s + (uint32_t)(ir >> 4) * 9u * Is;
                    const uint32_t j = (uint32_t)(ir & 15);
                    const uint4 q = lds128(tb + j * (Is / 2) + 16u * (uint32_t)c);
                    const float dd = chunk_dot_h(q, L);
                    const uint16_t sv = lds16(tb + 8u * Is + j * (Is / 32) + g2);
                    const uint16_t bv = lds16(tb + 8u * Is + Is / 2 + j * (Is / 32) + g2);
                    acc[r] = fmaf(h2f_bits(sv), dd, acc[r]);
                    acc[r] = fmaf(h2f_bits(bv), L.sx, acc[r]);
                }
            }
            // lane l holds the total of row l / 8 of this warp
            const float tot = reduce_scatter<4>(acc, lane);
            if ((lane & 7) == 0)
                st_relaxed_u64(a.ysh + kSdRows * d.blk + 4 * warp + (lane >> 3),
                               tag | __float_as_uint(tot));
        } else {
            // -------- routed down rows + combine: 16 rows of the k routed
            // experts (routing weights are folded into h), then + shared
            cnt_d++;
            if (!down_ready) {
                // warp 0 waits for every routed gate/up item of the launch,
                // then copies their packed h into shared memory with one bulk
                // copy; every warp waits for that copy
                bool ok = true;
                if (warp == 0 && lane == 0) {
                    ok = fused_wait_ge(&a.sync->gu_done[1], (ep + 1) * (unsigned long long)a.NRG, a.status, a.wait_ns);
                    if (ok) {
                        fused_trace(a, kTrDownReady);
                        fence_proxy_async_global();
                        const uint32_t bytes = (uint32_t)NCr * kDLimbWords * 4;
                        mbar_arrive_expect_tx(hl_bar, bytes);
                        bulk_g2s(hl, a.dlimb, bytes, hl_bar);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok || !fused_wait_bar(hl_bar, 0, a.status, a.wait_ns)) break;
                const uint32_t hl_s = smem_u32(hl);
                const int cpe = a.I / 32;                            // chunks per expert
#pragma unroll
                for (int j = 0; j < MAXD; j++) {
                    const int L = tid + 256 * j;
                    const bool valid = L < NCr;
                    const int e = valid ? L / cpe : 0;
                    const int ce = valid ? L - e * cpe : 0;
                    uint4 t[6];
                    const uint32_t src = hl_s + (uint32_t)(valid ? L : 0) * (kDLimbWords * 4);
#pragma unroll
                    for (int u = 0; u < 6; u++) t[u] = valid ? lds128(src + 16 * u) : make_uint4(0, 0, 0, 0);
                    dl[j].eh[0] = t[0].x; dl[j].eh[1] = t[0].y; dl[j].eh[2] = t[0].z; dl[j].eh[3] = t[0].w;
                    dl[j].oh[0] = t[1].x; dl[j].oh[1] = t[1].y; dl[j].oh[2] = t[1].z; dl[j].oh[3] = t[1].w;
                    dl[j].el[0] = t[2].x; dl[j].el[1] = t[2].y; dl[j].el[2] = t[2].z; dl[j].el[3] = t[2].w;
                    dl[j].ol[0] = t[3].x; dl[j].ol[1] = t[3].y; dl[j].ol[2] = t[3].z; dl[j].ol[3] = t[3].w;
                    dl[j].fexp[0] = __uint_as_float(t[4].x); dl[j].fexp[1] = __uint_as_float(t[4].y);
                    dl[j].fexp[2] = __uint_as_float(t[4].z); dl[j].fexp[3] = __uint_as_float(t[4].w);
                    dl[j].sx = valid ? __uint_as_float(t[5].x) + __uint_as_float(t[5].y) +
                                       __uint_as_float(t[5].z) + __uint_as_float(t[5].w)
                                     : 0.f;
                    // expert e's down tile sits at e * 9 I in the stage
                    dq_off[j] = e * 9 * a.I + 16 * ce;
                    ds_off[j] = e * 9 * a.I + 8 * a.I + 2 * (ce >> 1);
                    dvalid[j] = valid;
                }
                down_ready = true;
                if (tid == 0) fused_trace(a, kTrDownLimbs);
            }
            float acc[kRdRows];
#pragma unroll
            for (int r = 0; r < kRdRows; r++) acc[r] = 0.f;
            const int qrow = a.I / 2, srow = a.I / 32, bo = a.I / 2;    // biases follow the scales
#pragma unroll
            for (int j = 0; j < MAXD; j++) {
                if (dvalid[j]) {
#pragma unroll
                    for (int r = 0; r < kRdRows; r++) {
                        const uint4 q = lds128(st_s + dq_off[j] + r * qrow);
                        const float dd = chunk_dot_h(q, dl[j]);
                        const uint16_t sv = lds16(st_s + ds_off[j] + r * srow);
                        const uint16_t bv = lds16(st_s + ds_off[j] + bo + r * srow);
                        acc[r] = fmaf(h2f_bits(sv), dd, acc[r]);
                        acc[r] = fmaf(h2f_bits(bv), dl[j].sx, acc[r]);
                    }
                }
            }
            // lane l holds the total of row l / 2
            const float tot = reduce_scatter<kRdRows>(acc, lane);
            if ((lane & 1) == 0) rs[warp * kRdRows + (lane >> 1)] = tot;
            __syncwarp();
            int old = 0;
            if (lane == 0) {
                fence_acq_rel_cta();
                old = atomicAdd(&cs->item_cnt[stage], 1);
            }
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old == kFusedConsumerWarps - 1) {
                fence_acq_rel_cta();
                bool ok = true;
                if (lane < kRdRows) {
                    const int row = kRdRows * d.blk + lane;
                    // the shared expert's output for the row (written by a
                    // shared down item of lower index; bounded wait for its tag)
                    unsigned long long ws = ld_relaxed_u64(a.ysh + row);
                    if ((ws & ~0xffffffffull) != tag) {
                        const unsigned long long t0 = gtimer_ns();
                        for (unsigned it = 0; (ws & ~0xffffffffull) != tag; it++) {
                            __nanosleep(128);
                            ws = ld_relaxed_u64(a.ysh + row);
                            if ((it & 15) == 15 && (fused_aborted(a.status) || gtimer_ns() - t0 > a.wait_ns)) {
                                fused_fail(a.status);
                                ok = false;
                                break;
                            }
                        }
                    }
                    const volatile float* vr = rs;
                    float yv = __uint_as_float((unsigned)ws);
#pragma unroll
                    for (int w = 0; w < kFusedConsumerWarps; w++) yv += vr[w * kRdRows + lane];
                    if (ok) {
                        a.y[row] = yv;
                        if (a.h_out) {
                            const __half hr = d.item < kMaxDownItems
                                                  ? cs->h_rows[kRdRows * d.item + lane]
                                                  : __ushort_as_half(__ldcg((const unsigned short*)a.x_in + row));
                            a.h_out[row] = __float2half_rn(__half2float(hr) + yv);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) cs->item_cnt[stage] = 0;
                if (!__all_sync(0xffffffffu, ok)) break;
            }
        }
        __syncwarp();
        if (warp == 0 && lane == 0) fused_trace_item(a, n_done, 2, d.type);
        n_done++;
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == a.n_stages) { stage = 0; phase ^= 1u; }
    }
    if (warp == 0 && lane == 0 && a.trace) {
        fused_trace(a, kTrConsumerEnd);
        const unsigned cnt_s = cnt_gu - cnt_g;
        a.trace[(size_t)blockIdx.x * kTraceWords + kTrCounts] =
            (unsigned long long)cnt_r | ((unsigned long long)cnt_s << 16) |
            ((unsigned long long)cnt_g << 32) | ((unsigned long long)cnt_d << 48);
        unsigned smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        a.trace[(size_t)blockIdx.x * kTraceWords + kTrSm] = smid;
    }
}

// Shared memory besides the stage ring: x [H] fp16, router limbs [6][H],
// cross-warp sums [stages][kRedFloats], x limb table [H/32][20] words,
// packed routed h [NCr][24] and shared h [NCs][24] words, descriptors,
// barriers, producer and consumer scalars.
struct FusedSmemLayout {
    size_t xs, xl, red, glimb, hl, hls, desc, full, empty, hlbar, hlsbar, ps, cs, total;
    __host__ __device__ FusedSmemLayout(int H, int NCr, int NCs, int n_stages, int stage_bytes) {
        size_t off = (size_t)n_stages * stage_bytes;
        xs = off;     off += ((size_t)H * 2 + 127) / 128 * 128;
        xl = off;     off += ((size_t)kRouterMaxLimbs * H + 127) / 128 * 128;
        red = off;    off += (size_t)n_stages * kRedFloats * sizeof(float);
        glimb = off;  off += ((size_t)(H / 32) * kLimbWords * 4 + 15) / 16 * 16;
        hl = off;     off += (size_t)NCr * kDLimbWords * 4;
        hls = off;    off += (size_t)NCs * kDLimbWords * 4;
        desc = off;   off += (size_t)n_stages * sizeof(FusedDesc);
        full = off;   off += (size_t)n_stages * 8;
        empty = off;  off += (size_t)n_stages * 8;
        hlbar = off;  off += 8;
        hlsbar = off; off += 8;
        ps = off;     off += (sizeof(ProducerShared) + 15) / 16 * 16;
        cs = off;     off += (sizeof(ConsumerShared) + 15) / 16 * 16;
        total = off;
    }
};

template <int MAXC, int MAXD>
__global__ void __launch_bounds__(kFusedThreads, 1) k_moe_layer_fused(const FusedArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const FusedSmemLayout lay(a.H, a.k * a.I / 32, a.Is / 32, a.n_stages, a.stage_bytes);
    uint8_t* stages = smem;
    __half* xs = reinterpret_cast<__half*>(smem + lay.xs);
    int8_t* xl = reinterpret_cast<int8_t*>(smem + lay.xl);
    float* red = reinterpret_cast<float*>(smem + lay.red);
    uint32_t* glimb = reinterpret_cast<uint32_t*>(smem + lay.glimb);
    FusedDesc* desc = reinterpret_cast<FusedDesc*>(smem + lay.desc);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.full);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + lay.empty);
    uint8_t* hl = smem + lay.hl;
    uint64_t* hl_bar = reinterpret_cast<uint64_t*>(smem + lay.hlbar);
    uint8_t* hls = smem + lay.hls;
    uint64_t* hls_bar = reinterpret_cast<uint64_t*>(smem + lay.hlsbar);
    ProducerShared* ps = reinterpret_cast<ProducerShared*>(smem + lay.ps);
    ConsumerShared* cs = reinterpret_cast<ConsumerShared*>(smem + lay.cs);

    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.n_stages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kFusedConsumerWarps);
            cs->item_cnt[s] = 0;
            for (int r = 0; r < kRouterRows; r++) cs->rsum[s][r] = 0;
        }
        mbar_init(hl_bar, 1);
        mbar_init(hls_bar, 1);
        cs->down_flag = 0;
        cs->gu_cls_done[0] = cs->gu_cls_done[1] = 0;
        cs->ep1 = 0;
        fence_mbar_init();
    }
    fused_trace(a, kTrEntry);
    __syncthreads();
    if (warp == kFusedConsumerWarps) {
        fused_producer(a, stages, desc, full, empty,
                       reinterpret_cast<volatile unsigned long long*>(&cs->ep1), ps,
                       threadIdx.x & 31);
        return;
    }
    fused_consumers<MAXC, MAXD>(a, stages, desc, full, empty, xs, xl, red, glimb, hl, hl_bar, hls,
                                hls_bar, cs);
}

// Shared memory bytes besides the stage ring.
__host__ inline size_t fused_fixed_smem(int H, int NCr, int NCs, int n_stages) {
    return FusedSmemLayout(H, NCr, NCs, n_stages, 0).total;
}

}  // namespace moeq4
