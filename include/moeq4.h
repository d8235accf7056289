/*
 * moeq4.h -- C ABI of libmoeq4.so, the B200 (sm_100a) MoE decode hot path.
 *
 * Per token and layer the path is: an 8-bit router picks the top 8 of 128
 * routed experts; one shared expert and the 8 routed experts (4-bit affine
 * weights) each run a gated FFN; the outputs are combined with the router
 * weights; in streaming mode the missing experts are fetched into a 16-slot
 * LFU cache per layer while the shared branch computes.
 *
 * Sources (web pages on the TurboFieldfare engine):
 *  [LH] "Gemma 4 26B : Comment faire tourner un LLM en 2 Go de RAM",
 *       section 04 "Implementation technique", parts "Le pipeline de
 *       traitement" and "Concurrence pour masquer la latence".
 *  [DS] daily.steinslab.io TurboFieldfare article, sections "L'atout cache
 *       des modeles MoE" and "Trois optimisations cles" (items 1 and 3).
 *  [RM] "TurboFieldfare execute Mac Gemma 4 26B dans 2 Go, mais la vitesse du
 *       SSD devient le compromis", sections "Mac Gemma 4 26B tient en
 *       memoire ..." and "L'affirmation des 2 Go ...".
 *  [DT] "Een model met 26 miljard parameters uitvoeren in twee gigabyte
 *       geheugen op een gewone Mac", section "Wat is de belangrijkste
 *       architectuurtruuc".
 *
 * Conventions for every entry point:
 *  - Every call returns an int status (MOE_OK or a negative MOE_ERR_*);
 *    moe_last_error() returns a message for the calling thread's last error.
 *  - Pointers marked "device" are CUDA device pointers on the current device;
 *    "host" pointers are ordinary or pinned host memory as stated.
 *  - The caller owns all buffers and streams.  The library allocates only in
 *    moe_ctx_create (workspace, events, mapped host buffers) and frees them in
 *    moe_ctx_destroy; no entry point allocates on the hot path.
 *  - Calls are asynchronous on the given stream, except where a host wait is
 *    stated.  One context serves one stream order at a time: calls on the
 *    same context must not overlap on the GPU (they share its workspace).
 *  - Weight, blob, activation and output-row pointers must be 16-byte
 *    aligned; int32/fp32 index and weight arrays (topk_idx, topk_w, slot_of,
 *    miss_list, n_miss, router bias) need 4 bytes.  Sizes must satisfy the
 *    limits of moe_ctx_create.  A violation returns an error and launches
 *    nothing.
 *  - fp16 values travel as their IEEE binary16 bit patterns (moe_half).
 */
#ifndef MOEQ4_H
#define MOEQ4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_half;                 /* IEEE binary16 bits */
typedef struct CUstream_st *moe_stream_t;  /* same handle as cudaStream_t */

enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,      /* null pointer, bad count, bad flag */
    MOE_ERR_ALIGNMENT = -2,        /* a pointer is misaligned */
    MOE_ERR_UNSUPPORTED_SHAPE = -3,/* sizes outside the supported limits */
    MOE_ERR_CUDA = -4,             /* a CUDA runtime call failed */
    MOE_ERR_TIMEOUT = -5,          /* a bounded device wait gave up */
    MOE_ERR_CACHE_STATE = -6       /* LFU table invalid or fill failed */
};

enum { MOE_GELU_TANH = 0, MOE_GELU_ERF = 1 };

/* Limits checked by every entry point. */
enum {
    MOE_MAX_TOPK = 8,
    MOE_MAX_EXPERTS = 256,
    MOE_MAX_SLOTS = 32,
    MOE_GROUP = 64
};

/* Layer shape and switches.  hidden, inter and inter_shared are multiples of
 * 64 (one quantisation group); top_k <= 8; n_experts <= 256;
 * top_k < n_slots <= 32. */
typedef struct {
    int32_t hidden;        /* H  (2816 for the Gemma-like layer) */
    int32_t n_experts;     /* E  routed experts (128) */
    int32_t top_k;         /* k  experts per token (8) [DS], [LH] */
    int32_t inter;         /* I  routed-expert intermediate (704) */
    int32_t inter_shared;  /* Is shared-expert intermediate (2112) */
    int32_t n_slots;       /* S  LFU slots per layer (16) [DS], [RM] */
    int32_t renorm;        /* 1: routing weights renormalised over top-k */
    int32_t gelu;          /* MOE_GELU_TANH or MOE_GELU_ERF */
    double rms_eps;        /* RMSNorm epsilon (1e-6) */
} MoeConfig;

typedef struct moe_ctx moe_ctx;

/* Creates a context for cfg on the current CUDA device, sized for up to
 * max_tokens tokens per call.  Allocates its workspace, a mapped pinned host
 * buffer for the streaming miss list, events and a device status word.
 * Returns MOE_ERR_UNSUPPORTED_SHAPE when cfg breaks the limits above. */
int moe_ctx_create(const MoeConfig *cfg, int max_tokens, moe_ctx **out);

/* Synchronises the device and frees everything moe_ctx_create allocated.
 * A null ctx is accepted. */
int moe_ctx_destroy(moe_ctx *ctx);

/* Synchronises `stream` and reports whether any kernel of this context gave
 * up a bounded device wait since the last check (MOE_ERR_TIMEOUT, with the
 * context's counters reset so that it can be used again) or MOE_OK. */
int moe_ctx_check(moe_ctx *ctx, moe_stream_t stream);

/* One line describing the context: which kernels serve single-token layers
 * (the fused layer kernel, or the direct kernels when the shape or the device
 * does not fit it), its shared-memory ring and register use.  Writes at most
 * len bytes (NUL-terminated) into buf (host). */
int moe_ctx_info(moe_ctx *ctx, char *buf, int len);

/* Bound of every device wait of this context's fused layer kernel, in
 * nanoseconds (default 2e9).  When a wait runs out the kernel records
 * MOE_ERR_TIMEOUT and leaves; moe_ctx_check reports it.  Host call, no device
 * work.  Returns MOE_ERR_INVALID_ARG outside 1e3 .. 6e10 ns. */
int moe_set_wait_ns(moe_ctx *ctx, unsigned long long ns);

/* Multi-token steps with all experts resident group the (token, expert)
 * pairs by expert ("Gemma 4 26B : Comment faire tourner un LLM en 2 Go de
 * RAM", section 04 "Chunked Prefill": one expert applied to many rows).  In a
 * step of two or more tokens, an expert whose bucket holds min_tokens or more
 * pairs, and the shared expert once T >= min_tokens, run on the tensor cores
 * (tcgen05; the 4-bit codes and fp16 x are exact operands, h enters as two
 * bf16 planes; fp32 accumulation, one accumulator per 64-column group folded
 * with its scale and bias); the other buckets run on the CUDA-core grouped
 * kernels (a single token takes the fused layer kernel).  min_tokens = 0 keeps every
 * bucket on the CUDA cores.  The default is 1 where the shape allows the
 * tensor-core kernels (hidden a multiple of 128, the staging buffers within
 * shared memory), else 0.  Host call, no device work.  Returns
 * MOE_ERR_INVALID_ARG for min_tokens < 0 and MOE_ERR_UNSUPPORTED_SHAPE for
 * min_tokens > 0 on a shape or device without the tensor-core kernels (the
 * setting is then left unchanged). */
int moe_set_mma_min_tokens(moe_ctx *ctx, int min_tokens);

/* Tracing of the single-token layer kernel.  enable = 1 makes later launches
 * record, per CTA, 160 words: globaltimer stamps (ns) of kernel entry, end of
 * the input prologue, first item, routing known, down phase ready, consumer
 * end, producer end, top-k published; word 8 counts router / shared /
 * routed / down items in 16-bit fields; word 9 is the SM id; words 10-18
 * router item done, top-k start and steps, prologue steps; words 32.. hold,
 * for the CTA's first 42 items, three stamps each (copies issued, data
 * ready, item done): time in the low 56 bits, item type + 1 in bits 56-59.  enable = 0
 * stops recording, -1 leaves it as is.  When host_out is not NULL the device
 * is synchronised and up to max_words words of the last recorded launch are
 * copied; returns the number of words copied (>= 0) or an error. */
int moe_ctx_trace(moe_ctx *ctx, int enable, unsigned long long *host_out, int max_words);

/* Message for the calling thread's most recent error ("" if none). */
const char *moe_last_error(void);

/* ------------------------------------------------------------ formats --
 * Expert blob (one contiguous, 16-byte aligned buffer per expert; a blob is
 * the unit of one cache fill), stored as tiles so that each unit of work of
 * the kernels is one contiguous read.  The gate/up matrix has 2*inter rows
 * (gate rows 0..inter-1, up rows inter..2*inter-1) of hidden columns; the
 * down matrix has hidden rows of inter columns.
 *   inter/16 gate/up tiles, 18*hidden bytes each; tile t holds intermediate
 *   indices 16t..16t+15:
 *     [gate codes u32 [16][hidden/8]] [up codes u32 [16][hidden/8]]
 *     [gate scales fp16 [16][hidden/64]] [up scales fp16 [16][hidden/64]]
 *     [gate biases fp16 [16][hidden/64]] [up biases fp16 [16][hidden/64]]
 *   then hidden/16 down tiles, 9*inter bytes each; tile t holds output rows
 *   16t..16t+15:
 *     [codes u32 [16][inter/8]] [scales fp16 [16][inter/64]]
 *     [biases fp16 [16][inter/64]]
 * Weight (row r, column c) = scale[r][c/64] * code + bias[r][c/64] with
 * code = (word[r][c/8] >> 4*(c%8)) & 15: "MLX affine" 4-bit weights
 * ([RM] "L'affirmation des 2 Go ..."; [DS] "Trois optimisations cles" 1).
 * Router: int8 W[n_experts][hidden] with one fp16 scale per expert row
 * (8-bit router: [LH] pipeline step 1; [DS] item 1).
 */

/* Size in bytes of one expert blob with the given hidden/intermediate: the
 * unit an expert cache fill copies ([DS] "Trois optimisations cles" item 3;
 * [DT] "Wat is de belangrijkste architectuurtruuc": only the selected
 * experts' weights are brought in).  Returns 0 when hidden or inter is not a
 * positive multiple of 64. */
size_t moe_blob_bytes(int hidden, int inter);

/* ---------------------------------------------------------- router ----
 * [LH] pipeline step 1, [DS] "L'atout cache des modeles MoE": for each of T
 * tokens, logit_e = scale_e * sum_c W[e][c] * x[c] (+ bias_e), with the dot
 * product of int8 weights and fp16 activations formed exactly in integer
 * arithmetic and the epilogue in fp64; top_k experts by descending logit,
 * ties to the lower index; weights = softmax over all E logits, then
 * renormalised over the top_k when cfg.renorm.
 *   Wr        device int8 [E][H]
 *   row_scale device fp16 [E]
 *   bias      device fp32 [E] or NULL
 *   x         device fp16 [T][H]
 *   topk_idx  device int32 [T][k]   (descending logit order)
 *   topk_w    device fp32  [T][k]
 *   logits    device fp64  [T][E] or NULL
 * T must be 1..max_tokens. */
int moe_router_topk(moe_ctx *ctx, const int8_t *Wr, const moe_half *row_scale,
                    const float *bias, const moe_half *x, int T,
                    int32_t *topk_idx, float *topk_w, double *logits,
                    moe_stream_t stream);

/* ------------------------------------------- router, no allocation ----
 * The router above (same arithmetic, same outputs) for callers that cannot
 * allocate device memory: code running under another runtime's allocator or
 * a fixed device-memory budget, where cudaMalloc would bypass the owner's
 * accounting, and latency-bound loops where cudaMalloc/cudaFree would stall
 * on their implicit device synchronisation.  It takes no moe_ctx (creating
 * one allocates a workspace) and itself calls no cudaMalloc, cudaFree or
 * other allocating routine.  The pages describe no such entry point.
 *   n_experts, hidden, top_k, renorm  as in MoeConfig
 *   Wr, row_scale, bias, x, topk_idx, topk_w  as for moe_router_topk
 *   (the logits are not returned).
 * Scratch: the logits and per-token counters live in one static device
 * array of 66,560 bytes that every GPU loading this library holds until
 * exit.  Limits: T <= 256, T * n_experts <= 8192, hidden a multiple of 64
 * and <= 6144; larger requests return MOE_ERR_UNSUPPORTED_SHAPE before any
 * CUDA call.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  The address is remembered for the life of
 * the process: after a cudaDeviceReset this entry point must not be called.
 * Every call on a device shares the one array: calls whose executions overlap
 * on the GPU (other streams, other host threads) race on it and must be
 * serialised by the caller. */
int moe_router_topk_noalloc(int n_experts, int hidden, int top_k, int renorm,
                            const int8_t *Wr, const moe_half *row_scale,
                            const float *bias, const moe_half *x, int T,
                            int32_t *topk_idx, float *topk_w,
                            moe_stream_t stream);

/* ----------------------------------------------------- expert FFN ----
 * The expert feed-forward block on 4-bit "MLX affine" weights ([RM]
 * "L'affirmation des 2 Go ...": routed and shared experts stored as 4-bit
 * affine groups; [DT] "Wat is de belangrijkste architectuurtruuc": each
 * token runs the shared expert and its selected experts).
 * Grouped expert FFN over n_pairs (expert, token) pairs: for pair p,
 *   g = Wg x, u = Wu x, h = GELU(g) * u, y[p] = Wd h,
 * with x = row pairs[p].token of x, weights dequantised from the pair's
 * blob, fp32 accumulation.  The GELU form is cfg.gelu.
 *   pairs  device MoeFfnPair [n_pairs]; blob 16-byte aligned, inter equal
 *          to cfg.inter or cfg.inter_shared, 0 <= token < T
 *   x      device fp16 [T][H]
 *   y      device fp32 [n_pairs][H]
 * n_pairs must be 1..max_tokens*(top_k+1). */
typedef struct {
    const void *blob;   /* device expert blob */
    int32_t inter;      /* its intermediate size */
    int32_t token;      /* row of x */
} MoeFfnPair;

int moe_expert_ffn_q4(moe_ctx *ctx, const MoeFfnPair *pairs, int n_pairs,
                      const moe_half *x, int T, float *y, moe_stream_t stream);

/* ------------------------------------------------- expert parallel ----
 * Experts partitioned over n_ranks ranks (rank r owns experts
 * r * E / n_ranks .. (r + 1) * E / n_ranks - 1); each rank routes its own
 * tokens and sends every (token, expert) pair to the expert's owner, which
 * applies the expert and sends the row back.  The pages run one process on
 * one machine; this is the B200 scale-out reading of their per-expert FFN
 * step ([LH] 04 pipeline steps 2-3, one expert applied to the rows routed to
 * it).  The host exchanges the rows between the calls (two all-to-alls).
 *
 * moe_ep_dispatch: the T * top_k pairs of topk_idx (device int32 [T][k])
 * sorted by destination rank, pairs in index order within a destination:
 *   send_counts  device int32 [n_ranks]: pairs for each rank;
 *   send_order   device int32 [T * k]: pair index q = t * k + j per position;
 *   send_x       device fp16 [T * k][H]: x[q / k] per position (x [T][H]);
 *   send_expert  device int32 [T * k]: the expert's index at its owner.
 * n_ranks must divide n_experts (at most 32).  An expert index outside
 * [0, n_experts) is not sent and moe_ctx_check reports MOE_ERR_INVALID_ARG. */
int moe_ep_dispatch(moe_ctx *ctx, const int32_t *topk_idx, int T, int n_ranks,
                    const moe_half *x, moe_half *send_x, int32_t *send_expert,
                    int32_t *send_order, int32_t *send_counts, moe_stream_t stream);

/* moe_ffn_rows: R rows, row r through expert expert_of_row[r] of the
 * n_experts blobs at `experts` (device, blob stride moe_blob_bytes(H, I)):
 * y_rows[r] = down(GELU(gate x_r) * up x_r), the grouped / tensor-core
 * kernels of the multi-token path with each row its own token.
 *   expert_of_row device int32 [R]; x_rows device fp16 [R][H];
 *   y_rows device fp32 [R][H].
 * R must be 0..min(max_tokens * top_k, max_tokens * (top_k + 1) / 2) (each
 * row takes a token's and a pair's place in the context's workspace; R = 0
 * does nothing); larger R returns MOE_ERR_UNSUPPORTED_SHAPE. */
int moe_ffn_rows(moe_ctx *ctx, const void *experts, int n_experts, const int32_t *expert_of_row,
                 int R, const moe_half *x_rows, float *y_rows, moe_stream_t stream);

/* moe_shared_ffn: the shared expert, which every token runs next to its
 * routed experts ([LH] 04 pipeline: the shared expert is always computed;
 * [RM] "L'affirmation des 2 Go ..."), applied to T token rows:
 * y[t] = down(GELU(gate x_t) * up x_t) with the shared blob (device, layout
 * of moe_blob_bytes(H, inter_shared)), through the kernels of a resident
 * multi-token step (the tensor cores from two tokens, else the CUDA-core
 * grouped kernels).  x device fp16 [T][H], y device fp32 [T][H]; T must be
 * 1..max_tokens. */
int moe_shared_ffn(moe_ctx *ctx, const void *shared_blob, const moe_half *x, int T, float *y,
                   moe_stream_t stream);

/* moe_ep_unpermute: rows returned in send order back to pair order,
 * y_pairs[send_order[p]] = y_sorted[p] for p < n (device fp32 rows of H). */
int moe_ep_unpermute(moe_ctx *ctx, const float *y_sorted, const int32_t *send_order, int n,
                     float *y_pairs, moe_stream_t stream);

/* --------------------------------------------------------- combine ----
 * [LH] "Concurrence pour masquer la latence", [RM] "L'affirmation des 2 Go
 * ...": the shared and routed outputs combine,
 *   y_out[t] = y_shared[t] + sum_j topk_w[t][j] * y_routed[t][j]
 * summed in j order in fp32.  When residual is not NULL,
 *   residual[t][c] = fp16(float(residual[t][c]) + y_out[t][c]).
 *   y_routed device fp32 [T][k][H]; y_shared device fp32 [T][H];
 *   topk_w device fp32 [T][k]; y_out device fp32 [T][H];
 *   residual device fp16 [T][H] or NULL. */
int moe_combine(moe_ctx *ctx, const float *y_routed, const float *y_shared,
                const float *topk_w, int T, float *y_out, moe_half *residual,
                moe_stream_t stream);

/* ------------------------------------------------------- LFU cache ----
 * One layer's expert cache of n_slots slots ([DS] "Trois optimisations
 * cles" item 3; [RM] "Mac Gemma 4 26B tient en memoire ..."), kept in device
 * memory.  For each token in order:
 *  (i)  its experts in ascending id order: a resident expert is a hit and its
 *       count grows by one;
 *  (ii) each missing expert in ascending id order takes the lowest empty
 *       slot, else the slot not used by this token with the lowest count,
 *       ties to the oldest insertion; it starts with count 1 and the next
 *       insertion number.  A count does not survive eviction.
 * Only the missing experts are fetched ([LH] pipeline step 3). */
typedef struct {
    int32_t expert[MOE_MAX_SLOTS];  /* resident expert, -1 when empty */
    int64_t count[MOE_MAX_SLOTS];   /* uses since insertion */
    int64_t seq[MOE_MAX_SLOTS];     /* insertion number */
    int64_t counter;                /* last insertion number */
    int64_t hits;                   /* running totals */
    int64_t misses;
    int32_t n_slots;
    int32_t valid;                  /* 0 after a failed fill */
} MoeLfuTable;

/* Resets a device table to n_slots empty slots (top_k < n_slots <= 32). */
int moe_lfu_init(moe_ctx *ctx, MoeLfuTable *table, int n_slots,
                 moe_stream_t stream);

/* Looks up T tokens' experts in order, updating the table.
 *   table     device MoeLfuTable (valid)
 *   topk_idx  device int32 [T][k]
 *   slot_of   device int32 [T][k]: slot holding topk_idx[t][j] afterwards
 *   miss_list device-visible int32 [T*k][2]: (expert, slot) per fill, in
 *             fill order; may be mapped pinned host memory
 *   n_miss    device-visible int32 [1]: number of fills, or -1 when the
 *             table is invalid (nothing changed).
 * When T > 1 a slot filled for token t may be evicted again by a later token
 * of the same call; callers that fill after the call use T = 1. */
int moe_cache_lookup_lfu(moe_ctx *ctx, MoeLfuTable *table,
                         const int32_t *topk_idx, int T, int32_t *slot_of,
                         int32_t *miss_list, int32_t *n_miss,
                         moe_stream_t stream);

/* -------------------------------------------------------- full layer ----
 * One MoE layer for T tokens of one call ([LH] pipeline steps 1-4 and
 * "Concurrence pour masquer la latence"; [RM] "L'affirmation des 2 Go ...";
 * [DT] "Wat is de belangrijkste architectuurtruuc").
 *
 * Resident mode (layer->experts != NULL): router, grouped FFN of the shared
 * and the routed experts, combine; all on `main`, no host wait.
 *
 * Streaming mode (layer->experts == NULL; host_store, slots, lfu set), T = 1:
 * router and cache lookup on `main`, then the shared-expert FFN on `main`
 * while the host waits for the miss list and issues one cudaMemcpyAsync per
 * missing blob on `copy`; `main` waits for the copies, runs the routed FFN
 * from the slots and combines.  The call returns after the copies are
 * issued (one host wait per call).  If issuing a copy fails the table is
 * marked invalid and MOE_ERR_CACHE_STATE is returned.  The shared-expert part
 * hands its intermediate to the routed part through a tagged word that the
 * routed part waits for (bounded), so a missing shared part ends in
 * MOE_ERR_TIMEOUT from moe_ctx_check rather than in wrong output.
 *
 * Streaming mode, 1 < T <= max_tokens (chunked prefill, [LH] 04 "Chunked
 * Prefill": one expert fetched serves every row of the chunk that uses it):
 * router for the T tokens, then one LFU lookup of the whole chunk.  The
 * chunk's distinct experts are served in batches that fit the slots: hits
 * first (count += their uses in the chunk, slot pinned to batch 0), then each
 * missing expert in ascending id takes the lowest empty slot, else the
 * unpinned slot with the lowest count (ties to the oldest insertion), and a
 * new batch starts, with no slot pinned, when every slot is pinned; a
 * newcomer's count is its uses; hits and misses count distinct experts.  Each
 * expert is copied at most once per chunk.  The shared expert runs for all T
 * tokens while the host reads the batch plan (one host wait per call, in both
 * fill modes); then per batch the missing blobs are copied (after the
 * previous batch's kernels) and the grouped kernels serve the batch's
 * (token, choice) pairs from the slots; combine at the end.  slot_of receives
 * the slot each pair was served from.  With T = 1 this rule is the per-token
 * rule above.
 *
 * flags & MOE_PRENORM: `x` is the fp16 residual stream h; the layer input is
 * RMSNorm(h) (unit weight, eps = cfg.rms_eps, exact sum of squares, result
 * rounded to fp16) and afterwards h <- fp16(h + y) in place.
 *
 * flags & MOE_DEVICE_FILL (streaming mode): the misses are filled by the GPU
 * instead of the host ([LH] pipeline steps 3-4, with the read moved from the
 * host to the device): the cache lookup writes the miss list to device
 * memory, and a gather kernel on `copy` reads it and copies each missing blob
 * from host_store (which must be pinned host memory the device can address)
 * into its slot, while `main` runs the shared expert.  The call then makes no
 * host wait and returns as soon as the work is queued; it can be captured in
 * a CUDA graph.  A table made invalid by an earlier failed host fill makes
 * the layer compute with slot 0 and moe_ctx_check report MOE_ERR_CACHE_STATE.
 */
enum { MOE_PRENORM = 1, MOE_DEVICE_FILL = 2 };

typedef struct moe_store moe_store;    /* expert file reader (below) */

typedef struct {
    const int8_t *router_w;       /* device int8 [E][H] */
    const moe_half *router_scale; /* device fp16 [E] */
    const float *router_bias;     /* device fp32 [E] or NULL */
    const void *shared_blob;      /* device blob (inter_shared) */
    const void *experts;          /* resident: device [E] blobs, contiguous */
    const void *host_store;       /* streaming: pinned host [E] blobs */
    void *slots;                  /* streaming: device [n_slots] blobs */
    MoeLfuTable *lfu;             /* streaming: device table */
    const moe_store *store;       /* streaming without host_store: misses read
                                     from this expert file (storage tier) */
    int32_t store_layer;          /* the layer's index in the store */
    int32_t reserved;             /* zero */
} MoeLayer;

typedef struct {
    float *y;              /* device fp32 [T][H]: MoE output, required */
    int32_t *topk_idx;     /* device int32 [T][k] or NULL */
    float *topk_w;         /* device fp32 [T][k] or NULL */
    int32_t *slot_of;      /* device int32 [T][k] or NULL (streaming) */
    moe_half *x_norm;      /* device fp16 [T][H] or NULL (MOE_PRENORM) */
} MoeLayerOut;

int moe_layer_decode(moe_ctx *ctx, const MoeLayer *layer, moe_half *x, int T,
                     const MoeLayerOut *out, int flags, moe_stream_t main,
                     moe_stream_t copy);

/* ------------------------------------------------------- expert store ----
 * The storage tier of the cache ([DS] "Trois optimisations clés" items 2-3:
 * experts streamed from the SSD and read ahead with parallel pread; [LH] 04
 * "Le pipeline de traitement" steps 3-4: only the missing experts are read).
 *
 * File format: n_layers x n_experts expert blobs (each moe_blob_bytes of the
 * layer shape), layer-major; each blob is padded to moe_store_stride(blob)
 * bytes (the next multiple of 4096), so blob (l, e) starts at byte
 * (l * n_experts + e) * stride.  The padding keeps every read aligned to 4
 * KiB, so the store opens the file with O_DIRECT (no page cache) where the
 * file system accepts it, else with buffered reads.
 *
 * A streaming MoeLayer with host_store == NULL and store set reads its misses
 * from the file: after the cache lookup the host reads the missing blobs with
 * n_threads threads (each pread of at most 1 MiB) into the store's pinned
 * staging buffers (n_staging blobs, allocated by moe_store_open; page-aligned
 * host memory when no GPU is present), then copies each into its slot on the
 * copy stream, while the shared expert computes.  MOE_DEVICE_FILL is refused
 * with a store (the device cannot read the file).  A failed read marks the
 * table invalid and returns MOE_ERR_CACHE_STATE.  One store serves one
 * caller thread at a time. */
size_t moe_store_stride(size_t blob_bytes);

/* Opens path for n_layers x n_experts blobs of blob_bytes (a multiple of 16);
 * starts n_threads reader threads (1..256) and allocates n_staging staging
 * blobs (1..4096).  MOE_ERR_INVALID_ARG when the file is missing or shorter
 * than the format needs; the caller closes the store. */
int moe_store_open(const char *path, int n_layers, int n_experts, size_t blob_bytes,
                   int n_threads, int n_staging, moe_store **out);

/* Stops the threads, closes the file and frees the staging.  NULL accepted. */
int moe_store_close(moe_store *store);

/* Reads blobs (layer, experts[i]) for i < n into host buffers dst[i] (any
 * host memory, blob_bytes each), n_staging at a time in parallel. */
int moe_store_read(moe_store *store, int layer, const int32_t *experts, int n,
                   void *const *dst);

/* Totals since open: bytes of blobs read, seconds spent reading (wall
 * clock of the read calls), and whether reads bypass the page cache. */
int moe_store_stats(const moe_store *store, unsigned long long *bytes,
                    double *seconds, int *direct);

/* ------------------------------------------------------------- stack ----
 * Decodes T tokens one after another through n_layers resident layers
 * (each token: for every layer, x = RMSNorm(h), y = MoE(x), h <- fp16(h+y)),
 * the per-layer flow repeated over the layers and then per token ([RM]
 * "L'affirmation des 2 Go ...").  The token loop runs as a captured CUDA
 * graph replayed once per token; the first call for a given set of layers
 * captures it.
 *   layers  host array [n_layers] of resident MoeLayer
 *   h       device fp16 [T][H], updated in place
 *   y_last  device fp32 [T][H] or NULL: MoE output of the last layer */
int moe_stack_decode(moe_ctx *ctx, const MoeLayer *layers, int n_layers,
                     moe_half *h, int T, float *y_last, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOEQ4_H */
