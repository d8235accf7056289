// moeq4_api.cu -- the C ABI of libmoeq4.so (declared in include/moeq4.h).
//
// Host side: argument checks, workspace, stream/event plumbing and launches.
// Every arithmetic step of the path runs in the kernels included below.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "ffn_tc.cuh"
#include "ep.cuh"
#include "ffn_simple.cuh"
#include "grouped.cuh"
#include "layer_fused.cuh"
#include "misc.cuh"
#include "router.cuh"

using namespace moeq4;

// ------------------------------------------------------------ errors --
static thread_local std::string g_err;

static int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

#define CK(call)                                                                   \
    do {                                                                           \
        cudaError_t e_ = (call);                                                   \
        if (e_ != cudaSuccess)                                                     \
            return fail(MOE_ERR_CUDA, "%s: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                        __FILE__, __LINE__);                                       \
    } while (0)

#define CKL() CK(cudaGetLastError())

#define TRY(expr)                 \
    do {                          \
        int rc_ = (expr);         \
        if (rc_ != MOE_OK) return rc_; \
    } while (0)

static inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
static inline bool aligned4(const void* p) { return ((uintptr_t)p & 3u) == 0; }

// ------------------------------------------------------------ context --
struct StackKey {
    std::vector<MoeLayer> layers;
    moe_half* h = nullptr;
    float* y_last = nullptr;
};

struct moe_ctx {
    MoeConfig cfg{};
    int maxT = 0;
    int device = 0;
    int maxI = 0;
    // device workspace (one allocation)
    uint8_t* ws = nullptr;
    double* logits = nullptr;
    int* router_done = nullptr;
    int32_t* idx = nullptr;
    float* w = nullptr;
    MoeFfnPair* pairs = nullptr;
    float* h_ws = nullptr;
    float* y_pairs = nullptr;
    __half* x_norm = nullptr;
    int32_t* slot_of = nullptr;
    int* cursor = nullptr;
    __half* h_cur = nullptr;
    float* y_cur = nullptr;
    // mapped pinned host memory for the streaming miss list
    int32_t* miss_host = nullptr;    // [maxT*k*2 + 4]; last words hold n_miss
    int32_t* miss_dev = nullptr;
    int32_t* miss_list_d = nullptr;  // [maxT*k*2] miss list in device memory (device-initiated fill)
    int32_t* n_miss_d = nullptr;
    int32_t* n_miss_host = nullptr;
    int32_t* n_miss_dev = nullptr;
    cudaEvent_t ev_lookup = nullptr, ev_copy = nullptr, ev_ffn = nullptr;
    int32_t* plan_host = nullptr;    // mapped pinned: a streaming chunk's batch plan (k_lfu_chunk)
    int32_t* plan_dev = nullptr;
    int32_t* batch_of = nullptr;     // [maxT * k] batch of every routed pair of a streaming chunk
    cudaStream_t cap_stream = nullptr;
    // stack graph
    cudaGraphExec_t stack_exec = nullptr;
    StackKey stack_key;
    // host-side fault injection (tests): fail the Nth blob copy before issue;
    // leave out the Nth shared-expert launch of a streaming layer
    long fail_copy_at = -1;
    long copies_seen = 0;
    long withhold_shared_at = -1;
    long shared_launches = 0;
    unsigned long long wait_ns = kWaitNs;  // bound of every device wait of the fused kernel
    unsigned long long* shared_tag = nullptr;   // hand-off word of split streaming layers
    unsigned long long stream_seq = 0;          // streaming layer calls so far
    // fused single-token layer kernel
    FusedSync* fsync = nullptr;        // [4 modes][2 parities]
    int* status = nullptr;             // device status word (bounded waits)
    __half* h_alt = nullptr;           // ping-pong residual buffer
    int fparity[4] = {0, 0, 0, 0};
    int n_sms = 0;
    bool fused_ok = false;
    bool grouped_ok = false;           // multi-token steps grouped by expert
    bool mma_ok = false;               // tensor-core kernels usable for this shape
    bool router_batch_ok = false;      // the batched router fits shared memory
    int mma_min_tok = 0;               // bucket size from which they run (0: never)
    __nv_bfloat16* h_pl = nullptr;     // [2][maxT * (k + 1)][maxI] h as bf16 hi / lo planes
    float* h_sum = nullptr;            // [maxT * (k + 1)][hsum_stride] group sums of h
    int hsum_stride = 0;               // maxI / 64 rounded up to 4 floats (16-byte rows)
    int xg_stride = 0;                 // H / 64 rounded up to 4 floats
    __half* xs = nullptr;              // [maxT * (k + 1)][H] x rows: tokens, then pairs by bucket
    float* xg_sum = nullptr;           // [maxT * (k + 1)][xg_stride] their group sums
    int* e_off = nullptr;              // [E + 1] pairs per expert (prefix)
    int* plist = nullptr;              // [maxT * k] pair indices grouped by expert
    uint32_t* dlimb = nullptr;         // packed intermediate of the fused kernel
    unsigned long long* ysh = nullptr; // tagged shared-expert down output [H]
    int f_stages = 0, f_stage_bytes = 0;
    int f_regs = 0, f_max_threads = 0;
    unsigned long long* trace = nullptr;   // [n_sms * 16] phase stamps
    bool tracing = false;
    size_t f_smem = 0;
    void (*f_kernel)(const FusedArgs) = nullptr;
};

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Raises a kernel's dynamic shared-memory limit to at least `bytes`.  The
// attribute belongs to the function and holds for the whole process, so it is
// never lowered: a context created later for a smaller shape must not shrink
// the limit under a larger context that is still in use.
static std::mutex g_smem_attr_mu;

template <typename F>
static cudaError_t raise_smem(F* fn, size_t bytes) {
    std::lock_guard<std::mutex> lock(g_smem_attr_mu);
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) return e;
    if ((size_t)fa.maxDynamicSharedSizeBytes >= bytes) return cudaSuccess;
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

static int check_cfg(const MoeConfig* c) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
    if (c->hidden <= 0 || c->hidden % MOE_GROUP || c->inter <= 0 || c->inter % MOE_GROUP ||
        c->inter_shared <= 0 || c->inter_shared % MOE_GROUP)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "hidden/inter/inter_shared must be positive multiples of 64 (%d, %d, %d)",
                    c->hidden, c->inter, c->inter_shared);
    if (c->hidden > 16384 || c->inter > 16384 || c->inter_shared > 16384)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "hidden/inter above 16384");
    if (c->top_k < 1 || c->top_k > MOE_MAX_TOPK || c->n_experts < c->top_k ||
        c->n_experts > MOE_MAX_EXPERTS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "need 1 <= top_k <= 8, top_k <= n_experts <= 256");
    if (c->n_slots <= c->top_k || c->n_slots > MOE_MAX_SLOTS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "need top_k < n_slots <= 32");
    if ((c->renorm != 0 && c->renorm != 1) || (c->gelu != MOE_GELU_TANH && c->gelu != MOE_GELU_ERF))
        return fail(MOE_ERR_INVALID_ARG, "renorm must be 0/1 and gelu a MOE_GELU_* value");
    if (!(c->rms_eps >= 0.0)) return fail(MOE_ERR_INVALID_ARG, "rms_eps must be >= 0");
    return MOE_OK;
}

extern "C" const char* moe_last_error(void) { return g_err.c_str(); }

void moeq4_set_error(const char* msg) { g_err = msg; }

// storage tier (store.cu)
size_t moeq4_store_blob(const moe_store* st);
int moeq4_store_fill(moe_store* st, int layer, const int32_t* experts, const int32_t* slot, int n,
                     uint8_t* slots, cudaStream_t copy, cudaEvent_t copy_done);

extern "C" size_t moe_blob_bytes(int hidden, int inter) {
    if (hidden <= 0 || inter <= 0 || hidden % MOE_GROUP || inter % MOE_GROUP) return 0;
    return BlobLayout(hidden, inter).bytes;
}

extern "C" int moe_ctx_destroy(moe_ctx* c) {
    if (!c) return MOE_OK;
    cudaSetDevice(c->device);
    cudaDeviceSynchronize();
    if (c->stack_exec) cudaGraphExecDestroy(c->stack_exec);
    if (c->ev_lookup) cudaEventDestroy(c->ev_lookup);
    if (c->ev_copy) cudaEventDestroy(c->ev_copy);
    if (c->ev_ffn) cudaEventDestroy(c->ev_ffn);
    if (c->plan_host) cudaFreeHost(c->plan_host);
    if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
    if (c->miss_host) cudaFreeHost(c->miss_host);
    if (c->ws) cudaFree(c->ws);
    delete c;
    return MOE_OK;
}

// Shared memory of the grouped kernels: the expert tile plus kGrpTokens rows
// of activations (fp32).
static size_t grouped_smem_gu(int H) { return (size_t)18 * H + (size_t)kGrpTokens * H * 4; }
static size_t grouped_smem_dn(int Ie) { return (size_t)9 * Ie + (size_t)kGrpTokens * Ie * 4; }

// cuTensorMapEncodeTiled from the driver (null when unavailable).
static PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map over the codes of tiled expert blobs: dims {row bytes, rows per
// tile, tiles, experts}; one copy takes 64 bytes (128 columns) of 128 rows
// (box_tiles tiles), 64-byte swizzle.
static bool encode_codes(CUtensorMap* m, const void* base, int row_bytes, int rows_per_tile,
                         size_t tile_stride, int tiles, size_t expert_stride, int experts, int box_tiles) {
    const cuuint64_t dims[4] = {(cuuint64_t)row_bytes, (cuuint64_t)rows_per_tile, (cuuint64_t)tiles,
                                (cuuint64_t)experts};
    const cuuint64_t strides[3] = {(cuuint64_t)row_bytes, (cuuint64_t)tile_stride, (cuuint64_t)expert_stride};
    const cuuint32_t box[4] = {64u, (cuuint32_t)rows_per_tile, (cuuint32_t)box_tiles, 1u};
    const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
    return tmap_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box,
                          es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over 16-bit rows: dims {cols, rows, planes}; one copy takes
// 64 columns x box_rows rows of every plane, 128-byte swizzle.
static bool encode_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int cols, int rows,
                        int planes, int box_rows) {
    const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)planes};
    const cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)cols * 2 * rows};
    const cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, (cuuint32_t)planes};
    const cuuint32_t es[3] = {1u, 1u, 1u};
    return tmap_encoder()(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Enables the grouped multi-token path when its tiles fit shared memory.
static cudaError_t setup_grouped(moe_ctx* c) {
    const MoeConfig& g = c->cfg;
    int optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c->device);
    if (e != cudaSuccess) return e;
    const size_t gu = grouped_smem_gu(g.hidden);
    const size_t dn = grouped_smem_dn(c->maxI);
    c->grouped_ok = gu <= (size_t)optin && dn <= (size_t)optin;
    if (!c->grouped_ok) return cudaSuccess;
    e = raise_smem(k_gateup_grouped<false>, (int)gu);
    if (e == cudaSuccess)
        e = raise_smem(k_gateup_grouped<true>, (int)gu);
    if (e == cudaSuccess)
        e = raise_smem(k_down_grouped<false>, (int)dn);
    if (e == cudaSuccess)
        e = raise_smem(k_down_grouped<true>, (int)dn);
    if (e != cudaSuccess) return e;
    // tensor-core kernels: items of 4 gate/up tiles (64 indices) or 128 down rows
    const size_t tc_gu = tc_smem_bytes<false>(g.hidden, c->xg_stride);
    const size_t tc_dn = tc_smem_bytes<true>(c->maxI, c->hsum_stride);
    if (!tmap_encoder() || tc_gu > (size_t)optin || tc_dn > (size_t)optin || g.hidden % kMmaRows ||
        g.inter % 64 || g.inter_shared % 64)
        return cudaSuccess;
    e = raise_smem(k_ffn_tc<false>, (size_t)tc_gu);
    if (e == cudaSuccess)
        e = raise_smem(k_ffn_tc<true>, (size_t)tc_dn);
    if (e != cudaSuccess) return e;
    c->mma_ok = true;
    c->mma_min_tok = kMmaDefaultMinTokens;
    return cudaSuccess;
}

// Chooses the fused kernel variant and its shared-memory ring for cfg.
static cudaError_t setup_fused(moe_ctx* c) {
    const MoeConfig& g = c->cfg;
    int dev = c->device, optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&c->n_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    const int nch = g.hidden / 32;
    const int maxc = (nch + 31) / 32;
    const int NCr = g.top_k * g.inter / 32, NCs = g.inter_shared / 32;
    const int maxd = (NCr + 255) / 256;
    // a stage holds one gate/up tile (18 H bytes), two shared down tiles
    // (18 Is) or one down tile of each routed expert (9 I k)
    size_t stage = (size_t)18 * g.hidden;
    if ((size_t)18 * g.inter_shared > stage) stage = (size_t)18 * g.inter_shared;
    if ((size_t)9 * g.inter * g.top_k > stage) stage = (size_t)9 * g.inter * g.top_k;
    stage = (stage + 127) / 128 * 128;
    int ns = 0;
    for (int n = kFusedMaxStages; n >= 2 && ns == 0; n--)
        if ((size_t)n * stage + fused_fixed_smem(g.hidden, NCr, NCs, n) <= (size_t)optin) ns = n;
    c->fused_ok = g.hidden <= 4096 && maxc >= 1 && maxc <= 4 && maxd >= 1 && maxd <= 2 &&
                  ns >= 2 && stage < (1u << 20) && c->n_sms > 0;
    if (!c->fused_ok) return cudaSuccess;
    typedef void (*KFn)(const FusedArgs);
    static const KFn table[4][2] = {
        {k_moe_layer_fused<1, 1>, k_moe_layer_fused<1, 2>},
        {k_moe_layer_fused<2, 1>, k_moe_layer_fused<2, 2>},
        {k_moe_layer_fused<3, 1>, k_moe_layer_fused<3, 2>},
        {k_moe_layer_fused<4, 1>, k_moe_layer_fused<4, 2>}};
    c->f_kernel = table[maxc - 1][maxd - 1];
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, c->f_kernel);
    if (e != cudaSuccess) return e;
    c->f_regs = fa.numRegs;
    c->f_max_threads = fa.maxThreadsPerBlock;
    if (fa.maxThreadsPerBlock < kFusedThreads) {    // registers would not fit: use the direct kernels
        c->fused_ok = false;
        return cudaSuccess;
    }
    c->f_stages = ns;
    c->f_stage_bytes = (int)stage;
    c->f_smem = (size_t)ns * stage + fused_fixed_smem(g.hidden, NCr, NCs, ns);
    return raise_smem(c->f_kernel, (int)c->f_smem);
}

extern "C" int moe_ctx_create(const MoeConfig* cfg, int max_tokens, moe_ctx** out) {
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    TRY(check_cfg(cfg));
    if (max_tokens < 1 || max_tokens > 65535)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "max_tokens must be 1..65535");
    moe_ctx* c = new moe_ctx();
    c->cfg = *cfg;
    c->maxT = max_tokens;
    c->maxI = cfg->inter > cfg->inter_shared ? cfg->inter : cfg->inter_shared;
    cudaGetDevice(&c->device);
    const size_t T = max_tokens, E = cfg->n_experts, k = cfg->top_k, H = cfg->hidden;
    const size_t P = T * (k + 1);
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
    size_t o_logits = take(T * E * sizeof(double));
    size_t o_done = take(T * sizeof(int));
    size_t o_idx = take(T * k * sizeof(int32_t));
    size_t o_w = take(T * k * sizeof(float));
    size_t o_pairs = take(P * sizeof(MoeFfnPair));
    size_t o_h = take(P * (size_t)c->maxI * sizeof(float));
    size_t o_y = take(P * H * sizeof(float));
    size_t o_xn = take(T * H * sizeof(__half));
    size_t o_slot = take(T * k * sizeof(int32_t));
    size_t o_batch = take(T * k * sizeof(int32_t));
    size_t o_cur = take(sizeof(int));
    size_t o_hcur = take(H * sizeof(__half));
    size_t o_ycur = take(H * sizeof(float));
    size_t o_fsync = take(8 * sizeof(FusedSync));
    size_t o_status = take(sizeof(int));
    size_t o_missd = take((T * k * 2 + 4) * sizeof(int32_t));
    size_t o_stag = take(sizeof(unsigned long long));
    size_t o_halt = take(H * sizeof(__half));
    size_t o_dlimb = take((k * (size_t)cfg->inter + cfg->inter_shared) / 32 * kDLimbWords * 4);
    size_t o_ysh = take(H * sizeof(unsigned long long));
    // buckets are experts, or cache slots for a streaming chunk
    size_t o_eoff = take(((E > MOE_MAX_SLOTS ? E : MOE_MAX_SLOTS) + 1) * sizeof(int));
    size_t o_plist = take(T * k * sizeof(int));
    size_t o_hpl = take(2 * P * (size_t)c->maxI * sizeof(__nv_bfloat16));   // h hi / lo planes
    size_t o_xs = take(P * H * sizeof(__half));                              // x rows, bucket order
    c->xg_stride = (int)((H / 64 + 3) / 4 * 4);
    c->hsum_stride = (c->maxI / 64 + 3) / 4 * 4;
    size_t o_xgsum = take(P * (size_t)c->xg_stride * sizeof(float));         // their group sums
    size_t o_hsum = take(P * (size_t)c->hsum_stride * sizeof(float));        // h group sums
    int n_sms_dev = 0;
    cudaDeviceGetAttribute(&n_sms_dev, cudaDevAttrMultiProcessorCount, c->device);
    size_t o_trace = take((size_t)(n_sms_dev > 0 ? n_sms_dev : 1) * kTraceWords * sizeof(unsigned long long));
    int rc = MOE_OK;
    cudaError_t e = cudaMalloc(&c->ws, off);
    if (e == cudaSuccess) e = cudaMemset(c->ws, 0, off);
    if (e == cudaSuccess) {
        c->logits = (double*)(c->ws + o_logits);
        c->router_done = (int*)(c->ws + o_done);
        c->idx = (int32_t*)(c->ws + o_idx);
        c->w = (float*)(c->ws + o_w);
        c->pairs = (MoeFfnPair*)(c->ws + o_pairs);
        c->e_off = (int*)(c->ws + o_eoff);
        c->plist = (int*)(c->ws + o_plist);
        c->h_pl = (__nv_bfloat16*)(c->ws + o_hpl);
        c->xs = (__half*)(c->ws + o_xs);
        c->xg_sum = (float*)(c->ws + o_xgsum);
        c->h_sum = (float*)(c->ws + o_hsum);
        c->h_ws = (float*)(c->ws + o_h);
        c->y_pairs = (float*)(c->ws + o_y);
        c->x_norm = (__half*)(c->ws + o_xn);
        c->slot_of = (int32_t*)(c->ws + o_slot);
        c->batch_of = (int32_t*)(c->ws + o_batch);
        c->cursor = (int*)(c->ws + o_cur);
        c->h_cur = (__half*)(c->ws + o_hcur);
        c->y_cur = (float*)(c->ws + o_ycur);
        c->fsync = (FusedSync*)(c->ws + o_fsync);
        c->status = (int*)(c->ws + o_status);
        c->miss_list_d = (int32_t*)(c->ws + o_missd);
        c->n_miss_d = c->miss_list_d + T * k * 2;
        c->shared_tag = (unsigned long long*)(c->ws + o_stag);
        c->h_alt = (__half*)(c->ws + o_halt);
        c->dlimb = (uint32_t*)(c->ws + o_dlimb);
        c->ysh = (unsigned long long*)(c->ws + o_ysh);
        c->trace = (unsigned long long*)(c->ws + o_trace);
        size_t nm = T * k * 2 + 4;
        e = cudaHostAlloc((void**)&c->miss_host, nm * sizeof(int32_t), cudaHostAllocMapped);
    }
    if (e == cudaSuccess) e = cudaHostGetDevicePointer((void**)&c->miss_dev, c->miss_host, 0);
    if (e == cudaSuccess) {
        c->n_miss_host = c->miss_host + T * k * 2;
        c->n_miss_dev = c->miss_dev + T * k * 2;
        e = cudaEventCreateWithFlags(&c->ev_lookup, cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_copy, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_ffn, cudaEventDisableTiming);
    if (e == cudaSuccess)
        e = cudaHostAlloc((void**)&c->plan_host, (4 * E + 8) * sizeof(int32_t), cudaHostAllocMapped);
    if (e == cudaSuccess) e = cudaHostGetDevicePointer((void**)&c->plan_dev, c->plan_host, 0);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking);
    const int smem_router = (int)(H * sizeof(long long));
    if (e == cudaSuccess)
        e = raise_smem(k_router, smem_router);
    if (e == cudaSuccess) {
        int optin = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c->device);
        const size_t rb = router_batch_smem(2, (int)H, (int)E);
        if (e == cudaSuccess && rb <= (size_t)optin) {
            e = raise_smem(k_router_batch<2>, (int)rb);
            c->router_batch_ok = e == cudaSuccess;
        }
    }
    if (e == cudaSuccess)
        e = raise_smem(k_ffn_gateup_simple, (int)(H * sizeof(float)));
    if (e == cudaSuccess)
        e = raise_smem(k_ffn_down_simple, (int)(c->maxI * sizeof(float)));
    if (e == cudaSuccess) e = setup_grouped(c);
    if (e == cudaSuccess) e = setup_fused(c);
    if (e != cudaSuccess) {
        rc = fail(MOE_ERR_CUDA, "moe_ctx_create: %s", cudaGetErrorString(e));
        moe_ctx_destroy(c);
        return rc;
    }
    if (const char* f = getenv("MOEQ4_FAIL_COPY_AT")) c->fail_copy_at = atol(f);
    if (const char* f = getenv("MOEQ4_WITHHOLD_SHARED_AT")) c->withhold_shared_at = atol(f);
    *out = c;
    return MOE_OK;
}

// ------------------------------------------------------------- launches --
static int launch_router(moe_ctx* c, const int8_t* Wr, const moe_half* sc, const float* bias,
                         const __half* x, int T, int32_t* idx, float* w, double* logits,
                         cudaStream_t s) {
    const MoeConfig& g = c->cfg;
    double* lg = logits ? logits : c->logits;
    if (T >= kRouterBatchMinTokens && c->router_batch_ok) {
        // many tokens: digits once per token, the router matrix once per CTA
        // expert blocks per token pair: as many as keep the grid within one
        // CTA per SM (each block forms its pair's digits)
        const int pairs = (T + 1) / 2, nmax = (g.n_experts + kRouterBatchExperts - 1) / kRouterBatchExperts;
        const int nb = std::max(1, std::min(nmax, c->n_sms / pairs));
        const int eper = (g.n_experts + nb * kRouterBatchExperts - 1) / (nb * kRouterBatchExperts) *
                         kRouterBatchExperts;
        const dim3 grid(pairs, (g.n_experts + eper - 1) / eper);
        k_router_batch<2><<<grid, kRouterBatchThreads, router_batch_smem(2, g.hidden, g.n_experts), s>>>(
            Wr, reinterpret_cast<const __half*>(sc), bias, x, T, g.n_experts, g.hidden, g.top_k,
            g.renorm, eper, lg, c->router_done, idx, w);
        CKL();
        return MOE_OK;
    }
    dim3 grid((g.n_experts + kRouterWarps - 1) / kRouterWarps, T);
    k_router<<<grid, 256, g.hidden * sizeof(long long), s>>>(
        Wr, reinterpret_cast<const __half*>(sc), bias, x, g.n_experts, g.hidden, g.top_k,
        g.renorm, lg, c->router_done, idx, w);
    CKL();
    return MOE_OK;
}

static int launch_ffn(moe_ctx* c, const MoeFfnPair* pairs, int n, const __half* x, int T,
                      float* h_ws, float* y, cudaStream_t s) {
    const MoeConfig& g = c->cfg;
    dim3 g1((c->maxI + 7) / 8, n);
    k_ffn_gateup_simple<<<g1, 256, g.hidden * sizeof(float), s>>>(
        pairs, x, T, g.hidden, g.inter, g.inter_shared, g.gelu, h_ws, c->maxI);
    CKL();
    dim3 g2(g.hidden / 8, n);
    k_ffn_down_simple<<<g2, 256, c->maxI * sizeof(float), s>>>(pairs, h_ws, c->maxI, g.hidden,
                                                               g.inter, g.inter_shared, y);
    CKL();
    return MOE_OK;
}

static int launch_combine(moe_ctx* c, const float* y_routed, const float* y_shared,
                          const float* w, int T, float* y, __half* residual, cudaStream_t s) {
    const MoeConfig& g = c->cfg;
    dim3 grid((g.hidden + 255) / 256, T);
    k_combine<<<grid, 256, 0, s>>>(y_routed, (size_t)g.top_k * g.hidden, y_shared, g.hidden, w,
                                   g.top_k, g.hidden, y, residual);
    CKL();
    return MOE_OK;
}

// One token through one layer with the fused kernel.  `mode` selects the
// work classes of this launch (kModeFull for a resident layer; streaming
// splits it into router / shared / routed+down launches).  Routed blobs are
// experts + sel[j] * stride with sel = the routing indices, or the cache
// slots when `sel_slots` is given.
static int launch_fused(moe_ctx* c, const MoeLayer* L, const __half* x_in, __half* h_out,
                        __half* x_norm_out, float* y, int32_t* idx_out, float* w_out,
                        int prenorm, cudaStream_t s, int mode = kModeFull,
                        const void* experts = nullptr, const int32_t* sel_slots = nullptr,
                        unsigned long long shared_seq = 0) {
    const MoeConfig& g = c->cfg;
    const int mi = mode == kModeFull ? 0 : mode == kModeRouter ? 1 : mode == kModeShared ? 2 : 3;
    FusedArgs a{};
    a.Wr = L->router_w;
    a.rscale = reinterpret_cast<const __half*>(L->router_scale);
    a.rbias = L->router_bias;
    a.shared = static_cast<const uint8_t*>(L->shared_blob);
    a.experts = static_cast<const uint8_t*>(experts ? experts : L->experts);
    a.stride = BlobLayout(g.hidden, g.inter).bytes;
    a.sel_src = sel_slots ? sel_slots : c->idx;
    a.x_in = x_in;
    a.h_out = h_out;
    a.x_norm_out = x_norm_out;
    a.y = y;
    a.idx_ws = c->idx;
    a.w_ws = c->w;
    a.idx_out = idx_out;
    a.w_out = w_out;
    a.logits = c->logits;
    a.dlimb = c->dlimb;
    a.ysh = c->ysh;
    a.sync_id = 2 * mi + c->fparity[mi];
    a.sync = c->fsync + a.sync_id;
    c->fparity[mi] ^= 1;
    a.status = c->status;
    a.trace = c->tracing ? c->trace : nullptr;
    a.wait_ns = c->wait_ns;
    a.shared_tag = shared_seq ? c->shared_tag : nullptr;
    a.shared_seq = shared_seq;
    a.eps = g.rms_eps;
    a.H = g.hidden; a.E = g.n_experts; a.k = g.top_k; a.I = g.inter; a.Is = g.inter_shared;
    a.gelu = g.gelu; a.renorm = g.renorm; a.prenorm = prenorm;
    a.n_stages = c->f_stages; a.stage_bytes = c->f_stage_bytes;
    a.NR = (mode & kModeRouter) ? (g.n_experts + kRouterRows - 1) / kRouterRows : 0;
    a.NSG = (mode & kModeShared) ? g.inter_shared / kGuRows : 0;
    a.NRG = (mode & kModeRouted) ? g.top_k * (g.inter / kGuRows) : 0;
    a.NSD = (mode & kModeDown) ? g.hidden / kSdRows : 0;
    a.NRD = (mode & kModeDown) ? g.hidden / kRdRows : 0;
    a.NTOT = a.NR + a.NSG + a.NSD + a.NRG + a.NRD;
    cudaLaunchConfig_t lc{};
    lc.gridDim = dim3(c->n_sms);
    lc.blockDim = dim3(kFusedThreads);
    lc.dynamicSmemBytes = c->f_smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    CK(cudaLaunchKernelEx(&lc, c->f_kernel, a));
    return MOE_OK;
}

// ------------------------------------------------------------- exports --
extern "C" int moe_router_topk(moe_ctx* c, const int8_t* Wr, const moe_half* row_scale,
                               const float* bias, const moe_half* x, int T, int32_t* topk_idx,
                               float* topk_w, double* logits, moe_stream_t stream) {
    if (!c || !Wr || !row_scale || !x || !topk_idx || !topk_w)
        return fail(MOE_ERR_INVALID_ARG, "moe_router_topk: NULL argument");
    if (T < 1 || T > c->maxT) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T=%d outside 1..%d", T, c->maxT);
    if (!aligned16(Wr) || !aligned16(row_scale) || !aligned16(x) || !aligned4(topk_idx) ||
        !aligned4(topk_w) || (bias && !aligned4(bias)) || (logits && !aligned16(logits)))
        return fail(MOE_ERR_ALIGNMENT, "moe_router_topk: misaligned pointer");
    return launch_router(c, Wr, row_scale, bias, reinterpret_cast<const __half*>(x), T, topk_idx,
                         topk_w, logits, stream);
}

extern "C" int moe_expert_ffn_q4(moe_ctx* c, const MoeFfnPair* pairs, int n_pairs,
                                 const moe_half* x, int T, float* y, moe_stream_t stream) {
    if (!c || !pairs || !x || !y) return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn_q4: NULL argument");
    if (n_pairs < 1 || n_pairs > c->maxT * (c->cfg.top_k + 1))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_pairs=%d outside 1..%d", n_pairs,
                    c->maxT * (c->cfg.top_k + 1));
    if (T < 1) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T must be >= 1");
    if (!aligned16(pairs) || !aligned16(x) || !aligned16(y))
        return fail(MOE_ERR_ALIGNMENT, "moe_expert_ffn_q4: pointers must be 16-byte aligned");
    return launch_ffn(c, pairs, n_pairs, reinterpret_cast<const __half*>(x), T, c->h_ws, y,
                      stream);
}

extern "C" int moe_combine(moe_ctx* c, const float* y_routed, const float* y_shared,
                           const float* topk_w, int T, float* y_out, moe_half* residual,
                           moe_stream_t stream) {
    if (!c || !y_routed || !y_shared || !topk_w || !y_out)
        return fail(MOE_ERR_INVALID_ARG, "moe_combine: NULL argument");
    if (T < 1 || T > 65535) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T=%d outside 1..65535", T);
    if (!aligned16(y_routed) || !aligned16(y_shared) || !aligned4(topk_w) || !aligned16(y_out) ||
        (residual && !aligned16(residual)))
        return fail(MOE_ERR_ALIGNMENT, "moe_combine: misaligned pointer");
    return launch_combine(c, y_routed, y_shared, topk_w, T, y_out,
                          reinterpret_cast<__half*>(residual), stream);
}

static int ffn_grouped(moe_ctx* c, const uint8_t* ex, int E, const uint8_t* sh, const __half* xin,
                       const int32_t* idx, int T, int k, cudaStream_t s, const int32_t* sel = nullptr,
                       int sel_val = 0, bool routed = true);

extern "C" int moe_ep_dispatch(moe_ctx* c, const int32_t* topk_idx, int T, int n_ranks,
                               const moe_half* x, moe_half* send_x, int32_t* send_expert,
                               int32_t* send_order, int32_t* send_counts, moe_stream_t stream) {
    if (!c || !topk_idx || !x || !send_x || !send_expert || !send_order || !send_counts)
        return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: NULL argument");
    const MoeConfig& g = c->cfg;
    if (T < 1 || T > c->maxT) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T=%d outside 1..%d", T, c->maxT);
    if (n_ranks < 1 || n_ranks > 32 || g.n_experts % n_ranks)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_ranks=%d must divide n_experts=%d (at most 32)",
                    n_ranks, g.n_experts);
    if (!aligned4(topk_idx) || !aligned16(x) || !aligned16(send_x) || !aligned4(send_expert) ||
        !aligned4(send_order) || !aligned4(send_counts))
        return fail(MOE_ERR_ALIGNMENT, "moe_ep_dispatch: misaligned pointer");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int P = T * g.top_k, epr = g.n_experts / n_ranks;
    k_ep_plan<<<1, 32 * n_ranks, 0, s>>>(topk_idx, P, g.n_experts, epr, n_ranks, send_counts, send_order,
                                          c->status);
    CKL();
    k_ep_gather<<<(P + 7) / 8, 256, 0, s>>>(reinterpret_cast<const __half*>(x), topk_idx, send_order, P,
                                             g.top_k, g.hidden, epr, reinterpret_cast<__half*>(send_x),
                                             send_expert);
    CKL();
    return MOE_OK;
}

extern "C" int moe_ffn_rows(moe_ctx* c, const void* experts, int n_experts, const int32_t* expert_of_row,
                            int R, const moe_half* x_rows, float* y_rows, moe_stream_t stream) {
    if (!c || !experts || !expert_of_row || !x_rows || !y_rows)
        return fail(MOE_ERR_INVALID_ARG, "moe_ffn_rows: NULL argument");
    const MoeConfig& g = c->cfg;
    if (n_experts < 1 || n_experts > g.n_experts)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_experts=%d outside 1..%d", n_experts, g.n_experts);
    // the rows take the place of R tokens with one pair each: 2 R workspace rows
    const int rmax = std::min(c->maxT * g.top_k, c->maxT * (g.top_k + 1) / 2);
    if (R < 0 || R > rmax)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "R=%d outside 0..%d (the context's max_tokens holds "
                    "min(max_tokens * top_k, max_tokens * (top_k + 1) / 2) rows)", R, rmax);
    if (!c->grouped_ok)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_ffn_rows needs the grouped kernels for this shape");
    if (!aligned16(experts) || !aligned4(expert_of_row) || !aligned16(x_rows) || !aligned16(y_rows))
        return fail(MOE_ERR_ALIGNMENT, "moe_ffn_rows: misaligned pointer");
    if (R == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // each row is its own token choosing one expert: rows T + q of the pair outputs
    TRY(ffn_grouped(c, static_cast<const uint8_t*>(experts), n_experts, nullptr,
                    reinterpret_cast<const __half*>(x_rows), expert_of_row, R, 1, s));
    CK(cudaMemcpyAsync(y_rows, c->y_pairs + (size_t)R * g.hidden, (size_t)R * g.hidden * sizeof(float),
                       cudaMemcpyDeviceToDevice, s));
    return MOE_OK;
}

extern "C" int moe_shared_ffn(moe_ctx* c, const void* shared_blob, const moe_half* x, int T, float* y,
                              moe_stream_t stream) {
    if (!c || !shared_blob || !x || !y) return fail(MOE_ERR_INVALID_ARG, "moe_shared_ffn: NULL argument");
    if (T < 1 || T > c->maxT) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T=%d outside 1..%d", T, c->maxT);
    if (!c->grouped_ok)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_shared_ffn needs the grouped kernels for this shape");
    if (!aligned16(shared_blob) || !aligned16(x) || !aligned16(y))
        return fail(MOE_ERR_ALIGNMENT, "moe_shared_ffn: pointers must be 16-byte aligned");
    const MoeConfig& g = c->cfg;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint8_t* sh = static_cast<const uint8_t*>(shared_blob);
    // the shared expert alone: no pair is grouped (the routing argument is
    // only read, never used)
    TRY(ffn_grouped(c, sh, 1, sh, reinterpret_cast<const __half*>(x), c->idx, T, g.top_k, s, nullptr, 0,
                    false));
    CK(cudaMemcpyAsync(y, c->y_pairs, (size_t)T * g.hidden * sizeof(float), cudaMemcpyDeviceToDevice, s));
    return MOE_OK;
}

extern "C" int moe_ep_unpermute(moe_ctx* c, const float* y_sorted, const int32_t* send_order, int n,
                                float* y_pairs, moe_stream_t stream) {
    if (!c || !y_sorted || !send_order || !y_pairs)
        return fail(MOE_ERR_INVALID_ARG, "moe_ep_unpermute: NULL argument");
    if (n < 0 || n > c->maxT * c->cfg.top_k)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n=%d outside 0..%d", n, c->maxT * c->cfg.top_k);
    if (!aligned16(y_sorted) || !aligned4(send_order) || !aligned16(y_pairs))
        return fail(MOE_ERR_ALIGNMENT, "moe_ep_unpermute: misaligned pointer");
    if (n == 0) return MOE_OK;
    k_ep_unpermute<<<(n + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(y_sorted, send_order, n,
                                                                                 c->cfg.hidden, y_pairs);
    CKL();
    return MOE_OK;
}

extern "C" int moe_lfu_init(moe_ctx* c, MoeLfuTable* table, int n_slots, moe_stream_t stream) {
    if (!c || !table) return fail(MOE_ERR_INVALID_ARG, "moe_lfu_init: NULL argument");
    if (n_slots <= c->cfg.top_k || n_slots > MOE_MAX_SLOTS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "need top_k < n_slots <= 32 (got %d)", n_slots);
    if (!aligned16(table)) return fail(MOE_ERR_ALIGNMENT, "table must be 16-byte aligned");
    k_lfu_init<<<1, 32, 0, stream>>>(table, n_slots);
    CKL();
    return MOE_OK;
}

extern "C" int moe_cache_lookup_lfu(moe_ctx* c, MoeLfuTable* table, const int32_t* topk_idx,
                                    int T, int32_t* slot_of, int32_t* miss_list, int32_t* n_miss,
                                    moe_stream_t stream) {
    if (!c || !table || !topk_idx || !slot_of || !miss_list || !n_miss)
        return fail(MOE_ERR_INVALID_ARG, "moe_cache_lookup_lfu: NULL argument");
    if (T < 1 || T > 65535) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T=%d outside 1..65535", T);
    if (!aligned16(table) || !aligned4(topk_idx) || !aligned4(slot_of) || !aligned4(miss_list) ||
        !aligned4(n_miss))
        return fail(MOE_ERR_ALIGNMENT, "moe_cache_lookup_lfu: misaligned pointer");
    k_lfu_lookup<<<1, 32, 0, stream>>>(table, topk_idx, T, c->cfg.top_k, slot_of, miss_list, n_miss);
    CKL();
    return MOE_OK;
}

// Multi-token FFNs of all experts resident (T >= 1 tokens, k pairs each,
// pair q = t * k + j choosing idx[q] < E): outputs in c->y_pairs, row t for
// the shared expert (when sh is given) and row T + q for pair q.  Each expert
// is read once for all of its tokens.  sel (device, optional): only the pairs
// with sel[q] == sel_val (a batch of cache slots); routed = false: the shared
// expert alone.
static int ffn_grouped(moe_ctx* c, const uint8_t* ex, int E, const uint8_t* sh, const __half* xin,
                       const int32_t* idx, int T, int k, cudaStream_t s, const int32_t* sel,
                       int sel_val, bool routed) {
    {
        const MoeConfig& g = c->cfg;
        const int H = g.hidden;
        const size_t stride = BlobLayout(H, g.inter).bytes;
        const int I = g.inter, Is = g.inter_shared;
        const bool with_shared = sh != nullptr;
        if (!with_shared) sh = ex;                    // shared-expert maps: encoded, never read
        // In steps of at least kMmaMinStep tokens, routed buckets of tau or more
        // pairs and the shared expert (T >= tau) run on the tensor cores
        // (tau = 0: none); the rest on the CUDA-core grouped kernels.
        const int tau = c->mma_ok ? c->mma_min_tok : 0;
        const bool tc = tau > 0 && T >= kMmaMinStep;
        const bool tc_shared = with_shared && tc && T >= tau;
        const int cap = tc ? tau : 0x7fffffff;
        const int P = T * (k + 1), hs = c->maxI;
        __nv_bfloat16 *hh = c->h_pl, *hl = c->h_pl + (size_t)P * hs;
        if (!routed) sel_val = -1;                    // no pair is grouped
        k_group_pairs<<<1, 1024, 0, s>>>(idx, T * k, E, c->e_off, c->plist, routed ? sel : idx, sel_val);
        CKL();
        CUtensorMap m_cgr, m_cgs, m_cdr, m_cds, m_x[3], m_h[3];
        TcArgs ta{};
        if (tc) {
            // x rows in bucket order (tokens first) with their group sums; this call's tensor maps
            k_gather_x<<<dim3((H + 2047) / 2048, P < 65535 ? P : 65535), 256, 0, s>>>(
                xin, H, T, k, P, c->plist, c->xs, c->xg_sum, c->xg_stride,
                (sel || !routed) ? c->e_off + E : nullptr);
            CKL();
            const BlobLayout Lr(H, I), Ls(H, Is);
            const size_t sb = Ls.bytes;
            bool enc = encode_codes(&m_cgr, ex, H / 2, 32, Lr.gu_tile, I / 16, stride, E, 4) &&
                       encode_codes(&m_cgs, sh, H / 2, 32, Ls.gu_tile, Is / 16, sb, 1, 4) &&
                       encode_codes(&m_cdr, ex + Lr.dn_base, I / 2, 16, Lr.dn_tile, H / 16, stride, E, 8) &&
                       encode_codes(&m_cds, sh + Ls.dn_base, Is / 2, 16, Ls.dn_tile, H / 16, sb, 1, 8);
            for (int b = 0; b < 3 && enc; b++)
                enc = encode_rows(&m_x[b], c->xs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, H, P, 1, 16 << b) &&
                      encode_rows(&m_h[b], hh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hs, P, 2, 16 << b);
            if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed");
            ta.H = H; ta.T = T; ta.k = k; ta.E = E; ta.gelu = g.gelu;
            ta.Ir = I; ta.Is = Is; ta.min_tok = routed ? tau : 0x7fffffff; ta.do_shared = tc_shared ? 1 : 0;
            ta.e_off = c->e_off; ta.list = c->plist;
            ta.h_hi = hh; ta.h_lo = hl; ta.h_sum = c->h_sum; ta.hs = hs; ta.hsum_stride = c->hsum_stride;
            ta.y_pairs = c->y_pairs; ta.status = c->status;
        }
        const int chunks = (T + kGrpChunk - 1) / kGrpChunk;
        // with a threshold of one pair every routed bucket is on the tensor cores
        const bool grp_routed = routed && !(tc && tau <= 1);
        if (grp_routed) {
            k_gateup_grouped<false><<<dim3(I / 16, E), kGrpThreads, grouped_smem_gu(H), s>>>(
                ex, stride, sh, H, I, xin, T, k, c->e_off, c->plist, cap, g.gelu, c->h_ws, c->maxI);
            CKL();
        }
        if (with_shared && !tc_shared) {
            k_gateup_grouped<true><<<dim3(Is / 16, 1, chunks), kGrpThreads, grouped_smem_gu(H), s>>>(
                ex, stride, sh, H, Is, xin, T, k, c->e_off, c->plist, cap, g.gelu, c->h_ws, c->maxI);
            CKL();
        }
        if (tc) {
            TcArgs gu = ta;
            gu.b_sum = c->xg_sum;
            gu.bs_stride = c->xg_stride;
            gu.kmax = H;
            k_ffn_tc<false><<<c->n_sms, kTcThreads, tc_smem_bytes<false>(H, c->xg_stride), s>>>(
                m_cgr, m_cgs, m_x[0], m_x[1], m_x[2], ex, stride, sh, gu);
            CKL();
        }
        if (grp_routed) {
            k_down_grouped<false><<<dim3(H / 16, E), kGrpThreads, grouped_smem_dn(I), s>>>(
                ex, stride, sh, H, I, T, c->e_off, c->plist, cap, c->h_ws, c->maxI, c->y_pairs);
            CKL();
        }
        if (with_shared && !tc_shared) {
            k_down_grouped<true><<<dim3(H / 16, 1, chunks), kGrpThreads, grouped_smem_dn(Is), s>>>(
                ex, stride, sh, H, Is, T, c->e_off, c->plist, cap, c->h_ws, c->maxI, c->y_pairs);
            CKL();
        }
        if (tc) {
            TcArgs dn = ta;
            dn.b_sum = c->h_sum;
            dn.bs_stride = c->hsum_stride;
            dn.kmax = c->maxI;
            k_ffn_tc<true><<<c->n_sms, kTcThreads, tc_smem_bytes<true>(c->maxI, c->hsum_stride), s>>>(
                m_cdr, m_cds, m_h[0], m_h[1], m_h[2], ex, stride, sh, dn);
            CKL();
        }
    }
    return MOE_OK;
}

// Resident layer body on one stream (also used inside the stack capture).
static int layer_resident(moe_ctx* c, const MoeLayer* L, __half* x, int T, const MoeLayerOut* o,
                          int flags, cudaStream_t s) {
    const MoeConfig& g = c->cfg;
    const int k = g.top_k, H = g.hidden;
    if (T == 1 && c->fused_ok) {
        const bool pre = (flags & MOE_PRENORM) != 0;
        TRY(launch_fused(c, L, x, pre ? c->h_alt : nullptr,
                         reinterpret_cast<__half*>(o->x_norm), o->y, o->topk_idx, o->topk_w,
                         pre ? 1 : 0, s));
        if (pre) {
            k_copy_rows<<<1, 256, 0, s>>>(c->h_alt, x, H);
            CKL();
        }
        return MOE_OK;
    }
    const __half* xin = x;
    __half* xn = o->x_norm ? reinterpret_cast<__half*>(o->x_norm) : c->x_norm;
    if (flags & MOE_PRENORM) {
        k_rmsnorm<<<T, 256, 0, s>>>(x, xn, H, g.rms_eps);
        CKL();
        xin = xn;
    }
    int32_t* idx = o->topk_idx ? o->topk_idx : c->idx;
    float* w = o->topk_w ? o->topk_w : c->w;
    TRY(launch_router(c, L->router_w, L->router_scale, L->router_bias, xin, T, idx, w, nullptr, s));
    const size_t stride = BlobLayout(H, g.inter).bytes;
    const int P = T * (k + 1);
    if (c->grouped_ok) {
        // each expert read once for all of its tokens
        TRY(ffn_grouped(c, static_cast<const uint8_t*>(L->experts), g.n_experts,
                        static_cast<const uint8_t*>(L->shared_blob), xin, idx, T, k, s));
    } else {
        k_build_pairs<<<(P + 127) / 128, 128, 0, s>>>(L->shared_blob, g.inter_shared,
                                                      static_cast<const uint8_t*>(L->experts), stride,
                                                      idx, g.inter, T, k, c->pairs);
        CKL();
        TRY(launch_ffn(c, c->pairs, P, xin, T, c->h_ws, c->y_pairs, s));
    }
    TRY(launch_combine(c, c->y_pairs + (size_t)T * H, c->y_pairs, w, T, o->y,
                       (flags & MOE_PRENORM) ? x : nullptr, s));
    return MOE_OK;
}

// Issues one cudaMemcpyAsync per missing blob on the copy stream (after the
// host has waited for the miss list); marks the table invalid on failure.
static int issue_fills(moe_ctx* c, const MoeLayer* L, cudaStream_t s, cudaStream_t cs) {
    const size_t stride = BlobLayout(c->cfg.hidden, c->cfg.inter).bytes;
    CK(cudaEventSynchronize(c->ev_lookup));
    const int nm = *(volatile int32_t*)c->n_miss_host;
    if (nm < 0) return fail(MOE_ERR_CACHE_STATE, "LFU table is invalid (an earlier fill failed)");
    const uint8_t* store = static_cast<const uint8_t*>(L->host_store);
    uint8_t* slots = static_cast<uint8_t*>(L->slots);
    if (L->store && !L->host_store) {
        // storage tier: parallel pread into staging, then one copy per blob
        std::vector<int32_t> ex(nm), sl(nm);
        for (int i = 0; i < nm; i++) { ex[i] = c->miss_host[2 * i]; sl[i] = c->miss_host[2 * i + 1]; }
        const int rc = moeq4_store_fill(const_cast<moe_store*>(L->store), L->store_layer, ex.data(), sl.data(),
                                        nm, slots, cs, c->ev_copy);
        if (rc != MOE_OK) {
            k_lfu_invalidate<<<1, 1, 0, s>>>(L->lfu);
            return rc;
        }
        CK(cudaStreamWaitEvent(s, c->ev_copy, 0));
        return MOE_OK;
    }
    for (int i = 0; i < nm; i++) {
        const int e = c->miss_host[2 * i], slot = c->miss_host[2 * i + 1];
        cudaError_t err = cudaSuccess;
        if (c->fail_copy_at >= 0 && c->copies_seen == c->fail_copy_at) err = cudaErrorInvalidValue;
        c->copies_seen++;
        if (err == cudaSuccess)
            err = cudaMemcpyAsync(slots + (size_t)slot * stride, store + (size_t)e * stride, stride,
                                  cudaMemcpyHostToDevice, cs);
        if (err != cudaSuccess) {
            k_lfu_invalidate<<<1, 1, 0, s>>>(L->lfu);
            return fail(MOE_ERR_CACHE_STATE, "fill of expert %d into slot %d failed: %s; table "
                        "marked invalid", e, slot, cudaGetErrorString(err));
        }
    }
    CK(cudaEventRecord(c->ev_copy, cs));
    CK(cudaStreamWaitEvent(s, c->ev_copy, 0));
    return MOE_OK;
}

// Streaming layer with the fused kernel: router launch, cache lookup, shared
// branch launch overlapping the fills, then routed + down launch reading the
// slots.  Same arithmetic as the resident fused launch, so identical output.
// The fills are either issued by the host (one cudaMemcpyAsync per missing
// blob, after one host wait for the miss list) or, with MOE_DEVICE_FILL, by a
// gather kernel on the copy stream that reads the miss list in device memory
// and pulls the blobs from pinned host memory: no host wait at all.
static int layer_streaming_fused(moe_ctx* c, const MoeLayer* L, __half* x, const MoeLayerOut* o,
                                 int flags, cudaStream_t s, cudaStream_t cs) {
    const MoeConfig& g = c->cfg;
    const int pre = (flags & MOE_PRENORM) ? 1 : 0;
    const bool dev_fill = (flags & MOE_DEVICE_FILL) != 0;
    int32_t* slot_of = o->slot_of ? o->slot_of : c->slot_of;
    const void* dstore = nullptr;
    if (dev_fill) {
        void* p = nullptr;
        if (cudaHostGetDevicePointer(&p, const_cast<void*>(L->host_store), 0) != cudaSuccess || !p) {
            cudaGetLastError();
            return fail(MOE_ERR_INVALID_ARG, "MOE_DEVICE_FILL needs host_store in pinned host memory "
                                             "that the device can address");
        }
        dstore = p;
    }
    TRY(launch_fused(c, L, x, nullptr, reinterpret_cast<__half*>(o->x_norm), nullptr, o->topk_idx,
                     o->topk_w, pre, s, kModeRouter));
    if (dev_fill)
        k_lfu_lookup<<<1, 32, 0, s>>>(L->lfu, c->idx, 1, g.top_k, slot_of, c->miss_list_d, c->n_miss_d,
                                      c->status);
    else
        k_lfu_lookup<<<1, 32, 0, s>>>(L->lfu, c->idx, 1, g.top_k, slot_of, c->miss_dev, c->n_miss_dev);
    CKL();
    CK(cudaEventRecord(c->ev_lookup, s));
    // the shared launch hands its h to the routed launch through a tagged word
    // (this call's sequence number); host fault injection can leave the shared
    // launch out, so that the routed launch's bounded wait for it runs out
    const unsigned long long seq = ++c->stream_seq;
    const bool withhold = c->withhold_shared_at >= 0 && c->shared_launches == c->withhold_shared_at;
    c->shared_launches++;
    if (!withhold)
        TRY(launch_fused(c, L, x, nullptr, nullptr, nullptr, nullptr, nullptr, pre, s, kModeShared,
                         nullptr, nullptr, seq));
    if (dev_fill) {
        const size_t stride = BlobLayout(g.hidden, g.inter).bytes;
        CK(cudaStreamWaitEvent(cs, c->ev_lookup, 0));
        k_fill_from_host<<<dim3(kFillParts, g.top_k), kFillThreads, 0, cs>>>(
            static_cast<const uint8_t*>(dstore), static_cast<uint8_t*>(L->slots), stride, c->miss_list_d,
            c->n_miss_d, g.n_experts, MOE_MAX_SLOTS);
        CKL();
        CK(cudaEventRecord(c->ev_copy, cs));
        CK(cudaStreamWaitEvent(s, c->ev_copy, 0));
    } else {
        TRY(issue_fills(c, L, s, cs));
    }
    TRY(launch_fused(c, L, x, pre ? c->h_alt : nullptr, nullptr, o->y, nullptr, nullptr, pre, s,
                     kModeRouted | kModeDown, L->slots, slot_of, seq));
    if (pre) {
        k_copy_rows<<<1, 256, 0, s>>>(c->h_alt, x, g.hidden);
        CKL();
    }
    return MOE_OK;
}

// Streaming chunk of T > 1 tokens (chunked prefill: [LH] 04 "Chunked
// Prefill" -- one expert fetched into the cache serves every row of the chunk
// that uses it).  Router for all T tokens, then one cache lookup of the whole
// chunk (k_lfu_chunk): the chunk's distinct experts are served in batches that
// fit the slots, each expert copied at most once.  The shared expert runs for
// all T tokens while the host reads the batch plan (one host wait per chunk).
// Per batch: one copy per missing blob (host-issued, or the device gather with
// MOE_DEVICE_FILL), issued after the previous batch's kernels, which may still
// read the slots they overwrite; then the CUDA-core grouped kernels serve the
// batch's pairs with the cache slots as the buckets.  Combine and residual for
// all T tokens at the end.
static int layer_streaming_chunk(moe_ctx* c, const MoeLayer* L, __half* x, int T, const MoeLayerOut* o,
                                 int flags, cudaStream_t s, cudaStream_t cs) {
    const MoeConfig& g = c->cfg;
    const int k = g.top_k, H = g.hidden, I = g.inter, E = g.n_experts;
    const bool dev_fill = (flags & MOE_DEVICE_FILL) != 0;
    const size_t stride = BlobLayout(H, I).bytes;
    const __half* xin = x;
    __half* xn = o->x_norm ? reinterpret_cast<__half*>(o->x_norm) : c->x_norm;
    if (flags & MOE_PRENORM) {
        k_rmsnorm<<<T, 256, 0, s>>>(x, xn, H, g.rms_eps);
        CKL();
        xin = xn;
    }
    int32_t* idx = o->topk_idx ? o->topk_idx : c->idx;
    float* w = o->topk_w ? o->topk_w : c->w;
    int32_t* slot_of = o->slot_of ? o->slot_of : c->slot_of;
    const void* dstore = nullptr;
    if (dev_fill) {
        void* p = nullptr;
        if (cudaHostGetDevicePointer(&p, const_cast<void*>(L->host_store), 0) != cudaSuccess || !p) {
            cudaGetLastError();
            return fail(MOE_ERR_INVALID_ARG, "MOE_DEVICE_FILL needs host_store in pinned host memory "
                                             "that the device can address");
        }
        dstore = p;
    }
    TRY(launch_router(c, L->router_w, L->router_scale, L->router_bias, xin, T, idx, w, nullptr, s));
    k_lfu_chunk<<<1, 32, 0, s>>>(L->lfu, idx, T, k, E, slot_of, c->batch_of, c->plan_dev, c->status);
    CKL();
    CK(cudaEventRecord(c->ev_lookup, s));
    // the shared expert for every token of the chunk (the kernels of a
    // resident step: tensor cores from two tokens), while the host reads the
    // plan and the first batch's misses are filled
    const uint8_t* sh = static_cast<const uint8_t*>(L->shared_blob);
    uint8_t* slots = static_cast<uint8_t*>(L->slots);
    const uint8_t* store = static_cast<const uint8_t*>(L->host_store);
    TRY(ffn_grouped(c, slots, MOE_MAX_SLOTS, sh, xin, slot_of, T, k, s, nullptr, 0, false));
    CK(cudaEventSynchronize(c->ev_lookup));
    const int max_b = E + 1;
    const int nb = *(volatile int32_t*)c->plan_host;
    if (nb < 0) return fail(MOE_ERR_CACHE_STATE, "LFU table is invalid (an earlier fill failed)");
    const int32_t* off = c->plan_host + 1;
    const int32_t* pairs = c->plan_host + 1 + (max_b + 1) + max_b;
    for (int b = 0; b < nb; b++) {
        const int n = off[b + 1] - off[b];
        // batch b's copies may overwrite slots the previous batch still reads
        CK(cudaStreamWaitEvent(cs, b > 0 ? c->ev_ffn : c->ev_lookup, 0));
        if (n > 0) {
            if (dev_fill) {
                k_fill_from_host<<<dim3(kFillParts, n), kFillThreads, 0, cs>>>(
                    static_cast<const uint8_t*>(dstore), slots, stride, c->plan_dev + (pairs - c->plan_host) + 2 * off[b],
                    c->plan_dev + 1 + (max_b + 1) + b, E, MOE_MAX_SLOTS);
                CKL();
            } else if (L->store && !L->host_store) {
                std::vector<int32_t> ex(n), sl(n);
                for (int m = 0; m < n; m++) { ex[m] = pairs[2 * (off[b] + m)]; sl[m] = pairs[2 * (off[b] + m) + 1]; }
                const int rc = moeq4_store_fill(const_cast<moe_store*>(L->store), L->store_layer, ex.data(),
                                                sl.data(), n, slots, cs, c->ev_copy);
                if (rc != MOE_OK) {
                    k_lfu_invalidate<<<1, 1, 0, s>>>(L->lfu);
                    return rc;
                }
            } else {
                for (int m = off[b]; m < off[b + 1]; m++) {
                    const int e = pairs[2 * m], sl = pairs[2 * m + 1];
                    cudaError_t err = cudaSuccess;
                    if (c->fail_copy_at >= 0 && c->copies_seen == c->fail_copy_at) err = cudaErrorInvalidValue;
                    c->copies_seen++;
                    if (err == cudaSuccess)
                        err = cudaMemcpyAsync(slots + (size_t)sl * stride, store + (size_t)e * stride, stride,
                                              cudaMemcpyHostToDevice, cs);
                    if (err != cudaSuccess) {
                        k_lfu_invalidate<<<1, 1, 0, s>>>(L->lfu);
                        return fail(MOE_ERR_CACHE_STATE, "fill of expert %d into slot %d failed: %s; table "
                                    "marked invalid", e, sl, cudaGetErrorString(err));
                    }
                }
            }
            CK(cudaEventRecord(c->ev_copy, cs));
            CK(cudaStreamWaitEvent(s, c->ev_copy, 0));
        }
        // the batch's routed pairs grouped by cache slot, through the kernels
        // of a resident step (each expert's bucket is whole within its batch)
        TRY(ffn_grouped(c, slots, MOE_MAX_SLOTS, nullptr, xin, slot_of, T, k, s, c->batch_of, b, true));
        CK(cudaEventRecord(c->ev_ffn, s));
    }
    TRY(launch_combine(c, c->y_pairs + (size_t)T * H, c->y_pairs, w, T, o->y,
                       (flags & MOE_PRENORM) ? x : nullptr, s));
    return MOE_OK;
}

static int layer_streaming(moe_ctx* c, const MoeLayer* L, __half* x, const MoeLayerOut* o,
                           int flags, cudaStream_t s, cudaStream_t cs) {
    if (c->fused_ok) return layer_streaming_fused(c, L, x, o, flags, s, cs);
    const MoeConfig& g = c->cfg;
    const int k = g.top_k, H = g.hidden, T = 1;
    const __half* xin = x;
    __half* xn = o->x_norm ? reinterpret_cast<__half*>(o->x_norm) : c->x_norm;
    if (flags & MOE_PRENORM) {
        k_rmsnorm<<<T, 256, 0, s>>>(x, xn, H, g.rms_eps);
        CKL();
        xin = xn;
    }
    int32_t* idx = o->topk_idx ? o->topk_idx : c->idx;
    float* w = o->topk_w ? o->topk_w : c->w;
    int32_t* slot_of = o->slot_of ? o->slot_of : c->slot_of;
    TRY(launch_router(c, L->router_w, L->router_scale, L->router_bias, xin, T, idx, w, nullptr, s));
    k_lfu_lookup<<<1, 32, 0, s>>>(L->lfu, idx, T, k, slot_of, c->miss_dev, c->n_miss_dev);
    CKL();
    CK(cudaEventRecord(c->ev_lookup, s));
    const size_t stride = BlobLayout(H, g.inter).bytes;
    k_build_pairs<<<1, 128, 0, s>>>(L->shared_blob, g.inter_shared,
                                    static_cast<const uint8_t*>(L->slots), stride, slot_of,
                                    g.inter, T, k, c->pairs);
    CKL();
    // shared branch computes while the misses are fetched
    TRY(launch_ffn(c, c->pairs, T, xin, T, c->h_ws, c->y_pairs, s));
    TRY(issue_fills(c, L, s, cs));
    TRY(launch_ffn(c, c->pairs + T, T * k, xin, T, c->h_ws + (size_t)T * c->maxI,
                   c->y_pairs + (size_t)T * H, s));
    TRY(launch_combine(c, c->y_pairs + (size_t)T * H, c->y_pairs, w, T, o->y,
                       (flags & MOE_PRENORM) ? x : nullptr, s));
    return MOE_OK;
}

extern "C" int moe_layer_decode(moe_ctx* c, const MoeLayer* L, moe_half* x, int T,
                                const MoeLayerOut* o, int flags, moe_stream_t main,
                                moe_stream_t copy) {
    if (!c || !L || !x || !o || !o->y) return fail(MOE_ERR_INVALID_ARG, "moe_layer_decode: NULL argument");
    if (flags & ~(MOE_PRENORM | MOE_DEVICE_FILL)) return fail(MOE_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
    if (T < 1 || T > c->maxT) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T=%d outside 1..%d", T, c->maxT);
    if (!L->router_w || !L->router_scale || !L->shared_blob)
        return fail(MOE_ERR_INVALID_ARG, "layer needs router_w, router_scale and shared_blob");
    const void* ptrs[] = {L->router_w, L->router_scale, L->shared_blob, x, o->y};
    for (const void* p : ptrs)
        if (!aligned16(p)) return fail(MOE_ERR_ALIGNMENT, "moe_layer_decode: pointers must be 16-byte aligned");
    if ((L->router_bias && !aligned4(L->router_bias)) || (o->topk_idx && !aligned4(o->topk_idx)) ||
        (o->topk_w && !aligned4(o->topk_w)) || (o->slot_of && !aligned4(o->slot_of)) ||
        (o->x_norm && !aligned16(o->x_norm)))
        return fail(MOE_ERR_ALIGNMENT, "moe_layer_decode: pointers must be 16-byte aligned");
    if (L->experts) {
        if (!aligned16(L->experts)) return fail(MOE_ERR_ALIGNMENT, "experts must be 16-byte aligned");
        return layer_resident(c, L, reinterpret_cast<__half*>(x), T, o, flags, main);
    }
    if ((!L->host_store && !L->store) || !L->slots || !L->lfu || !copy)
        return fail(MOE_ERR_INVALID_ARG, "streaming mode needs host_store or store, slots, lfu and a copy stream");
    if (L->store && !L->host_store && (flags & MOE_DEVICE_FILL))
        return fail(MOE_ERR_INVALID_ARG, "MOE_DEVICE_FILL reads host_store; a store is read by the host");
    if (L->store && !L->host_store && moeq4_store_blob(L->store) != BlobLayout(c->cfg.hidden, c->cfg.inter).bytes)
        return fail(MOE_ERR_INVALID_ARG, "the store's blob size does not match the layer shape");
    if (T > 1 && !c->grouped_ok)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "streaming chunks need the grouped kernels, whose tiles "
                    "do not fit this shape");
    if (!aligned16(L->slots) || !aligned16(L->lfu) || (L->host_store && !aligned16(L->host_store)))
        return fail(MOE_ERR_ALIGNMENT, "moe_layer_decode: pointers must be 16-byte aligned");
    if (T > 1) return layer_streaming_chunk(c, L, reinterpret_cast<__half*>(x), T, o, flags, main, copy);
    return layer_streaming(c, L, reinterpret_cast<__half*>(x), o, flags, main, copy);
}

extern "C" int moe_set_mma_min_tokens(moe_ctx* c, int min_tokens) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "moe_set_mma_min_tokens: NULL context");
    if (min_tokens < 0) return fail(MOE_ERR_INVALID_ARG, "moe_set_mma_min_tokens: %d < 0", min_tokens);
    if (min_tokens > 0 && !c->mma_ok)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "tensor-core kernels unavailable for this shape");
    c->mma_min_tok = min_tokens;
    return MOE_OK;
}

extern "C" int moe_ctx_check(moe_ctx* c, moe_stream_t stream) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "moe_ctx_check: NULL context");
    CK(cudaStreamSynchronize(stream));
    int st = 0;
    CK(cudaMemcpy(&st, c->status, sizeof(int), cudaMemcpyDeviceToHost));
    if (st == 0) return MOE_OK;
    // a bounded wait gave up: clear the status and the launch counters so the
    // context can be used again
    CK(cudaMemset(c->status, 0, sizeof(int)));
    CK(cudaMemset(c->fsync, 0, 8 * sizeof(FusedSync)));
    // epochs restart, so tagged words of earlier launches must not survive
    CK(cudaMemset(c->ysh, 0, (size_t)c->cfg.hidden * sizeof(unsigned long long)));
    CK(cudaMemset(c->shared_tag, 0, sizeof(unsigned long long)));
    for (int m = 0; m < 4; m++) c->fparity[m] = 0;
    return fail(st, st == MOE_ERR_TIMEOUT ? "a bounded device wait gave up; counters reset"
                                          : "a device-side cache lookup found the LFU table invalid");
}

extern "C" int moe_ctx_info(moe_ctx* c, char* buf, int len) {
    if (!c || !buf || len < 1) return fail(MOE_ERR_INVALID_ARG, "moe_ctx_info: bad argument");
    int n = snprintf(buf, (size_t)len,
                     "single-token path: %s; sms %d; stages %d x %d B; smem %zu B; "
                     "registers %d; max threads %d (needs %d); wait bound %llu ns",
                     c->fused_ok ? "fused" : "direct kernels", c->n_sms, c->f_stages,
                     c->f_stage_bytes, c->f_smem, c->f_regs, c->f_max_threads, kFusedThreads,
                     c->wait_ns);
    return n < 0 ? fail(MOE_ERR_INVALID_ARG, "moe_ctx_info: format") : MOE_OK;
}

extern "C" int moe_set_wait_ns(moe_ctx* c, unsigned long long ns) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "moe_set_wait_ns: NULL context");
    if (ns < 1000ull || ns > 60000000000ull)
        return fail(MOE_ERR_INVALID_ARG, "moe_set_wait_ns: %llu ns outside 1 us .. 60 s", ns);
    c->wait_ns = ns;
    return MOE_OK;
}

extern "C" int moe_ctx_trace(moe_ctx* c, int enable, unsigned long long* host_out,
                             int max_words) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "moe_ctx_trace: NULL context");
    const int words = c->n_sms * kTraceWords;
    int n = 0;
    if (host_out) {
        CK(cudaDeviceSynchronize());
        n = max_words < words ? max_words : words;
        if (n > 0) CK(cudaMemcpy(host_out, c->trace, (size_t)n * 8, cudaMemcpyDeviceToHost));
    }
    if (enable >= 0) {
        if (enable && !c->tracing) CK(cudaMemset(c->trace, 0, (size_t)words * 8));
        c->tracing = enable != 0;
    }
    return n;
}

static bool same_key(const StackKey& k, const MoeLayer* layers, int n, moe_half* h, float* y) {
    if ((int)k.layers.size() != n || k.h != h || k.y_last != y) return false;
    return memcmp(k.layers.data(), layers, sizeof(MoeLayer) * n) == 0;
}

extern "C" int moe_stack_decode(moe_ctx* c, const MoeLayer* layers, int n_layers, moe_half* h,
                                int T, float* y_last, moe_stream_t stream) {
    if (!c || !layers || !h) return fail(MOE_ERR_INVALID_ARG, "moe_stack_decode: NULL argument");
    if (n_layers < 1 || T < 1) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_layers and T must be >= 1");
    if (!aligned16(h) || (y_last && !aligned16(y_last)))
        return fail(MOE_ERR_ALIGNMENT, "moe_stack_decode: pointers must be 16-byte aligned");
    for (int l = 0; l < n_layers; l++) {
        const MoeLayer& L = layers[l];
        if (!L.router_w || !L.router_scale || !L.shared_blob || !L.experts)
            return fail(MOE_ERR_INVALID_ARG, "layer %d is not a resident layer", l);
        if (!aligned16(L.router_w) || !aligned16(L.router_scale) || !aligned16(L.shared_blob) ||
            !aligned16(L.experts) || (L.router_bias && !aligned4(L.router_bias)))
            return fail(MOE_ERR_ALIGNMENT, "layer %d: pointers must be 16-byte aligned", l);
    }
    const int H = c->cfg.hidden;
    if (!c->stack_exec || !same_key(c->stack_key, layers, n_layers, h, y_last)) {
        if (c->stack_exec) { cudaGraphExecDestroy(c->stack_exec); c->stack_exec = nullptr; }
        cudaStream_t cs = c->cap_stream;
        CK(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal));
        int rc = MOE_OK;
        k_copy_half_row<<<1, 256, 0, cs>>>(reinterpret_cast<__half*>(h), c->h_cur, c->cursor, H, 1);
        MoeLayerOut o{};
        o.y = c->y_cur;
        __half* cur = c->h_cur;
        for (int l = 0; l < n_layers && rc == MOE_OK; l++) {
            if (c->fused_ok) {
                __half* nxt = cur == c->h_cur ? c->h_alt : c->h_cur;
                rc = launch_fused(c, &layers[l], cur, nxt, nullptr, c->y_cur, nullptr, nullptr, 1, cs);
                cur = nxt;
            } else {
                rc = layer_resident(c, &layers[l], c->h_cur, 1, &o, MOE_PRENORM, cs);
            }
        }
        if (rc == MOE_OK)
            k_store_token<<<1, 256, 0, cs>>>(cur, c->y_cur, reinterpret_cast<__half*>(h), y_last,
                                             c->cursor, H);
        cudaGraph_t graph = nullptr;
        cudaError_t e = cudaStreamEndCapture(cs, &graph);
        if (rc != MOE_OK) { if (graph) cudaGraphDestroy(graph); return rc; }
        if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "stack capture: %s", cudaGetErrorString(e));
        e = cudaGraphInstantiate(&c->stack_exec, graph, 0);
        cudaGraphDestroy(graph);
        if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "stack instantiate: %s", cudaGetErrorString(e));
        c->stack_key.layers.assign(layers, layers + n_layers);
        c->stack_key.h = h;
        c->stack_key.y_last = y_last;
    }
    CK(cudaMemsetAsync(c->cursor, 0, sizeof(int), stream));
    for (int t = 0; t < T; t++) CK(cudaGraphLaunch(c->stack_exec, stream));
    return MOE_OK;
}

// ------------------------------------------------- router, no allocation --
// moe_router_topk_noalloc: the router above without a context.  Its scratch
// (the fp64 logits of every token and one completion counter per token) lives
// in this file-scope device array, which every GPU that loads the library
// holds until the process exits.  In host code the name is only a stand-in
// for the symbol; the device address comes from cudaGetSymbolAddress.
constexpr int kNoAllocMaxLogits = 8192;                  // T * n_experts
constexpr int kNoAllocMaxTokens = 256;
constexpr int kNoAllocMaxHidden = 6144;                  // x*2^24 as int64 in 48 KiB
constexpr size_t kNoAllocCounterOff = (size_t)kNoAllocMaxLogits * sizeof(double);
constexpr size_t kNoAllocScratchBytes = kNoAllocCounterOff + kNoAllocMaxTokens * sizeof(int);
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_router_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void* g_noalloc_dev_ptr[kNoAllocMaxDevices];      // per device ordinal

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and remembered, together with the
// router kernel's shared-memory limit.  A cudaDeviceReset unloads the module
// and invalidates the remembered address: the entry point must not be used
// after one.
static int noalloc_scratch(unsigned char** out) {
    int dev = -1;
    CK(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_router_topk_noalloc: device %d above %d", dev,
                    kNoAllocMaxDevices - 1);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_dev_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_router_scratch);
        if (e != cudaSuccess || !p)
            return fail(MOE_ERR_CUDA, "moe_router_topk_noalloc: cudaGetSymbolAddress: %s",
                        cudaGetErrorString(e));
        // k_router takes hidden * 8 bytes of dynamic shared memory; allow the
        // largest hidden this entry point accepts, whatever contexts exist
        const cudaError_t ea = raise_smem(k_router, (size_t)kNoAllocMaxHidden * sizeof(long long));
        if (ea != cudaSuccess)
            return fail(MOE_ERR_CUDA, "moe_router_topk_noalloc: shared-memory limit: %s",
                        cudaGetErrorString(ea));
        g_noalloc_dev_ptr[dev] = p;
    }
    *out = static_cast<unsigned char*>(g_noalloc_dev_ptr[dev]);
    return MOE_OK;
}

extern "C" int moe_router_topk_noalloc(int n_experts, int hidden, int top_k, int renorm,
                                       const int8_t* Wr, const moe_half* row_scale,
                                       const float* bias, const moe_half* x, int T,
                                       int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
    if (!Wr || !row_scale || !x || !topk_idx || !topk_w)
        return fail(MOE_ERR_INVALID_ARG, "moe_router_topk_noalloc: NULL argument");
    if (top_k < 1 || top_k > MOE_MAX_TOPK || n_experts < top_k || n_experts > MOE_MAX_EXPERTS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "moe_router_topk_noalloc: need 1 <= top_k <= 8, top_k <= n_experts <= 256");
    if (hidden <= 0 || hidden % MOE_GROUP || hidden > kNoAllocMaxHidden)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "moe_router_topk_noalloc: hidden=%d must be a positive multiple of 64 <= %d",
                    hidden, kNoAllocMaxHidden);
    if (renorm != 0 && renorm != 1)
        return fail(MOE_ERR_INVALID_ARG, "moe_router_topk_noalloc: renorm must be 0 or 1");
    if (T < 1) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_router_topk_noalloc: T must be >= 1");
    if (T > kNoAllocMaxTokens || (long long)T * n_experts > kNoAllocMaxLogits)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "moe_router_topk_noalloc: T=%d with n_experts=%d exceeds the static scratch "
                    "(T <= %d and T * n_experts <= %d)",
                    T, n_experts, kNoAllocMaxTokens, kNoAllocMaxLogits);
    if (!aligned16(Wr) || !aligned16(row_scale) || !aligned16(x) || !aligned4(topk_idx) ||
        !aligned4(topk_w) || (bias && !aligned4(bias)))
        return fail(MOE_ERR_ALIGNMENT, "moe_router_topk_noalloc: misaligned pointer");
    unsigned char* scratch = nullptr;
    TRY(noalloc_scratch(&scratch));
    double* logits = reinterpret_cast<double*>(scratch);
    int* done = reinterpret_cast<int*>(scratch + kNoAllocCounterOff);
    // the array keeps the previous call's contents: the counters start at 0
    CK(cudaMemsetAsync(done, 0, (size_t)T * sizeof(int), stream));
    dim3 grid((n_experts + kRouterWarps - 1) / kRouterWarps, T);
    k_router<<<grid, 256, (size_t)hidden * sizeof(long long), stream>>>(
        Wr, reinterpret_cast<const __half*>(row_scale), bias, reinterpret_cast<const __half*>(x),
        n_experts, hidden, top_k, renorm, logits, done, topk_idx, topk_w);
    CKL();
    return MOE_OK;
}
