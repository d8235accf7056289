/*
 * moe_oracle.c -- plain CPU oracle for the MoE decode hot path.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code, header,
 * table or helper with the CUDA library; nothing in the product path may call
 * it.  Everything here is scalar, one weight at a time, accumulated in fp64,
 * so that a reader can check it against the method by eye.
 *
 * Sources (web pages on the TurboFieldfare engine):
 *  [LH] "Gemma 4 26B : Comment faire tourner un LLM en 2 Go de RAM",
 *       section 04 "Implementation technique" (pipeline: 8-bit router, top 8
 *       experts, 16-slot cache, misses fetched, shared branch computed
 *       meanwhile, outputs combined).
 *  [DS] daily.steinslab.io TurboFieldfare article, sections "L'atout cache
 *       des modeles MoE" (router activates the 8 most relevant of 128
 *       experts) and "Trois optimisations cles" (1: 4-bit weights, 8-bit
 *       router; 3: 16 cache slots per layer managed by LFU).
 *  [RM] "TurboFieldfare execute Mac Gemma 4 26B dans 2 Go ...", section
 *       "Mac Gemma 4 26B tient en memoire ..." (eight routed experts plus one
 *       shared expert used for every token) and section "L'affirmation des
 *       2 Go ..." (MLX affine 4-bit weights, 8-bit router, per-layer flow).
 *
 * Storage format fixed by this library (the pages name "MLX affine 4-bit"
 * but print no layout): group of 64 weights along a row, one fp16 scale and
 * one fp16 bias per group, w = scale*q + bias, q in 0..15, eight 4-bit codes
 * per uint32 with the lowest nibble holding the lowest column.  The router is
 * int8 with one fp16 scale per expert row.
 *
 * Parity status: every function below is pinned by tests in tests/
 * (hand-built groups, brute-force dense matrices, closed forms, hand-written
 * LFU traces, an independent naive LFU simulator); none is "parity
 * unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define GROUP 64

/* ------------------------------------------------------------------ fp16 */

/* IEEE binary16 bits -> double (exact). */
double oracle_half_to_double(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);              /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 0x400), e - 25); /* (1024+m) * 2^(e-15-10) */
    return sign ? -v : v;
}

/* double -> IEEE binary16, round to nearest, ties to even. */
uint16_t oracle_double_to_half(double v)
{
    if (isnan(v))
        return 0x7e00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a >= 65520.0)                 /* midpoint 65504..65536 ties up to inf */
        return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {        /* subnormal range, quantum 2^-24 */
        double r = nearbyint(a * 16777216.0);
        return sign | (uint16_t)r;    /* r == 1024 is the smallest normal */
    }
    int e;
    frexp(a, &e);                     /* a in [2^(e-1), 2^e) */
    double r = nearbyint(ldexp(a, 11 - e)); /* in [1024, 2048] */
    int E = e - 1 + 15;
    if (r == 2048.0) {
        r = 1024.0;
        E += 1;
    }
    if (E >= 31)
        return sign | 0x7c00;
    return sign | (uint16_t)(E << 10) | (uint16_t)((int)r - 1024);
}

/* ------------------------------------------------------------ dequantise */

/* One weight of a q4 matrix with K columns, row r, column c:
 * code = nibble (c mod 8) of word c/8 (lowest nibble first), group c/64,
 * w = scale*code + bias.  The result is exact in fp64. */
double oracle_dequant(const uint32_t *q, const uint16_t *scale,
                      const uint16_t *bias, int K, int r, int c)
{
    uint32_t word = q[(size_t)r * (size_t)(K / 8) + (size_t)(c / 8)];
    int code = (int)((word >> (4 * (c % 8))) & 0xFu);
    size_t g = (size_t)r * (size_t)(K / GROUP) + (size_t)(c / GROUP);
    double s = oracle_half_to_double(scale[g]);
    double b = oracle_half_to_double(bias[g]);
    return s * (double)code + b;
}

/* ---------------------------------------------------------- expert blob */

/* Tiled expert blob with hidden H and intermediate I (the storage order is
 * this library's own choice; the pages print none):
 *   I/16 gate/up tiles of 18 H bytes, tile t holding intermediate indices
 *   16t..16t+15: gate codes [16][H/8] u32, up codes [16][H/8] u32, gate
 *   scales [16][H/64] fp16, up scales, gate biases, up biases;
 *   then H/16 down tiles of 9 I bytes, tile t holding output rows
 *   16t..16t+15: codes [16][I/8] u32, scales [16][I/64] fp16, biases.
 * The gate/up matrix has 2I rows (gate rows 0..I-1, up rows I..2I-1). */
size_t oracle_blob_bytes(int H, int I)
{
    return (size_t)(I / 16) * 18 * (size_t)H + (size_t)(H / 16) * 9 * (size_t)I;
}

/* Byte offsets of row r's codes, scales and biases: off[0..2]. */
void oracle_gu_row(int H, int I, int r, size_t off[3])
{
    int up = r >= I;
    int i = up ? r - I : r;
    size_t tile = (size_t)(i / 16) * 18 * (size_t)H;
    size_t row = (size_t)(16 * up + i % 16);        /* row within the tile */
    off[0] = tile + row * (size_t)(H / 2);
    off[1] = tile + 16 * (size_t)H + row * (size_t)(H / 32);
    off[2] = tile + 17 * (size_t)H + row * (size_t)(H / 32);
}

void oracle_dn_row(int H, int I, int r, size_t off[3])
{
    size_t tile = (size_t)(I / 16) * 18 * (size_t)H + (size_t)(r / 16) * 9 * (size_t)I;
    size_t row = (size_t)(r % 16);
    off[0] = tile + row * (size_t)(I / 2);                 /* 16 rows of codes: 8 I bytes */
    off[1] = tile + 8 * (size_t)I + row * (size_t)(I / 32);
    off[2] = tile + 8 * (size_t)I + (size_t)(I / 2) + row * (size_t)(I / 32);
}

/* Weight (row r, column c) of the gate/up (dn = 0, K = H) or down (dn = 1,
 * K = I) matrix of a blob. */
static double blob_weight(const uint8_t *blob, int H, int I, int dn, int r, int c)
{
    size_t off[3];
    if (dn)
        oracle_dn_row(H, I, r, off);
    else
        oracle_gu_row(H, I, r, off);
    return oracle_dequant((const uint32_t *)(blob + off[0]), (const uint16_t *)(blob + off[1]),
                          (const uint16_t *)(blob + off[2]), dn ? I : H, 0, c);
}

/* ----------------------------------------------------------------- GELU */

/* variant 0: tanh form 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)));
 * variant 1: erf form 0.5 g (1 + erf(g / sqrt 2)). */
double oracle_gelu(double g, int variant)
{
    if (variant == 1)
        return 0.5 * g * (1.0 + erf(g / sqrt(2.0)));
    double k = sqrt(2.0 / M_PI);
    return 0.5 * g * (1.0 + tanh(k * (g + 0.044715 * g * g * g)));
}

/* ---------------------------------------------------------------- FFN */

/* One expert FFN on an fp64 input x[H]:
 *   gate_i = sum_c Wg[i,c] x_c, up_i = sum_c Wu[i,c] x_c,
 *   h_i = GELU(gate_i) * up_i,
 *   y_r = sum_i Wd[r,i] h_i.
 * h_out (length I) may be NULL. */
void oracle_expert_ffn(const uint8_t *blob, int H, int I, int gelu,
                       const double *x, double *h_out, double *y)
{
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
#pragma omp parallel for schedule(static)
    for (int i = 0; i < I; i++) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; c++) {
            g += blob_weight(blob, H, I, 0, i, c) * x[c];
            u += blob_weight(blob, H, I, 0, I + i, c) * x[c];
        }
        h[i] = oracle_gelu(g, gelu) * u;
    }
#pragma omp parallel for schedule(static)
    for (int r = 0; r < H; r++) {
        double acc = 0.0;
        for (int i = 0; i < I; i++)
            acc += blob_weight(blob, H, I, 1, r, i) * h[i];
        y[r] = acc;
    }
    if (h_out)
        memcpy(h_out, h, sizeof(double) * (size_t)I);
    free(h);
}

/* -------------------------------------------------------------- router */

/* logit_e = scale_e * sum_c W[e,c] x_c (+ bias_e).
 * The dot product of int8 weights with fp16 activations is formed exactly:
 * every finite fp16 value times 2^24 is an integer below 2^40, so the sum of
 * H products fits in int64.  It is then rounded once to fp64, scaled by 2^-24
 * (exact), multiplied by the fp16 row scale and, if present, added to the
 * fp32 bias, each step one IEEE round-to-nearest operation. */
void oracle_router_logits(const int8_t *W, const uint16_t *scale,
                          const float *bias, const uint16_t *x, int E, int H,
                          double *logits)
{
    for (int e = 0; e < E; e++) {
        int64_t S = 0;
        for (int c = 0; c < H; c++) {
            int64_t X = (int64_t)(oracle_half_to_double(x[c]) * 16777216.0);
            S += (int64_t)W[(size_t)e * (size_t)H + (size_t)c] * X;
        }
        double l = (double)S;
        l = l * 0x1p-24;
        l = l * oracle_half_to_double(scale[e]);
        if (bias)
            l = l + (double)bias[e];
        logits[e] = l;
    }
}

/* Top-k: the k largest logits, largest first; equal logits are ordered by
 * the lower expert index first. */
void oracle_topk(const double *logits, int E, int k, int32_t *idx)
{
    char *taken = (char *)calloc((size_t)E, 1);
    for (int j = 0; j < k; j++) {
        int best = -1;
        for (int e = 0; e < E; e++) {
            if (taken[e])
                continue;
            if (best < 0 || logits[e] > logits[best])
                best = e;
        }
        taken[best] = 1;
        idx[j] = best;
    }
    free(taken);
}

/* Softmax over all E logits. */
void oracle_softmax(const double *logits, int E, double *p)
{
    double m = logits[0];
    for (int e = 1; e < E; e++)
        if (logits[e] > m)
            m = logits[e];
    double z = 0.0;
    for (int e = 0; e < E; e++) {
        p[e] = exp(logits[e] - m);
        z += p[e];
    }
    for (int e = 0; e < E; e++)
        p[e] = p[e] / z;
}

/* Routing weights of the selected experts: the softmax probability of each
 * selected expert, renormalised over the k selected when renorm != 0. */
void oracle_topk_weights(const double *p, const int32_t *idx, int k,
                         int renorm, double *w)
{
    double z = 0.0;
    for (int j = 0; j < k; j++)
        z += p[idx[j]];
    for (int j = 0; j < k; j++)
        w[j] = renorm ? p[idx[j]] / z : p[idx[j]];
}

/* ------------------------------------------------------------ combine */

/* The shared and routed branch outputs combine with the routing weights:
 *   y = y_shared + sum_j w_j y_routed[j]   (fp64). */
void oracle_combine(const double *y_shared, const double *y_routed,
                    const double *w, int k, int H, double *y)
{
    for (int c = 0; c < H; c++) {
        double acc = y_shared[c];
        for (int j = 0; j < k; j++)
            acc += w[j] * y_routed[(size_t)j * (size_t)H + (size_t)c];
        y[c] = acc;
    }
}

/* ---------------------------------------------------------- MoE layer */

/* One token through one MoE layer:
 *   logits, top-k, weights (router);
 *   y = FFN_shared(x) + sum_j w_j FFN_{idx_j}(x)   (combine).
 * Routed expert e's blob is expert_base + e * blob_stride.
 * y_shared and y_routed ([k][H]) may be NULL. */
void oracle_moe_layer(int H, int E, int k, int I, int Is, int gelu, int renorm,
                      const int8_t *Wr, const uint16_t *rscale,
                      const float *rbias, const uint8_t *shared_blob,
                      const uint8_t *expert_base, size_t blob_stride,
                      const uint16_t *x16, int32_t *idx, double *w,
                      double *logits, double *y, double *y_shared,
                      double *y_routed)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)H);
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    for (int c = 0; c < H; c++)
        x[c] = oracle_half_to_double(x16[c]);

    oracle_router_logits(Wr, rscale, rbias, x16, E, H, logits);
    oracle_topk(logits, E, k, idx);
    oracle_softmax(logits, E, p);
    oracle_topk_weights(p, idx, k, renorm, w);

    double *ys = (double *)malloc(sizeof(double) * (size_t)H);
    double *yr = (double *)malloc(sizeof(double) * (size_t)H * (size_t)k);
    oracle_expert_ffn(shared_blob, H, Is, gelu, x, NULL, ys);
    for (int j = 0; j < k; j++)
        oracle_expert_ffn(expert_base + (size_t)idx[j] * blob_stride, H, I,
                          gelu, x, NULL, yr + (size_t)j * (size_t)H);
    oracle_combine(ys, yr, w, k, H, y);
    if (y_shared)
        memcpy(y_shared, ys, sizeof(double) * (size_t)H);
    if (y_routed)
        memcpy(y_routed, yr, sizeof(double) * (size_t)H * (size_t)k);
    free(x);
    free(p);
    free(ys);
    free(yr);
}

/* ------------------------------------------------------------- RMSNorm */

/* x_c = fp16( h_c / sqrt(mean(h^2) + eps) ), unit weight.
 * The sum of squares is formed exactly (fp16 * 2^24 is an integer below
 * 2^40, its square below 2^80, accumulated in 128 bits) and rounded once to
 * fp64; mean = sum / H, r = 1 / sqrt(mean + eps), x_c = fp16(h_c * r), each
 * step one IEEE round-to-nearest operation. */
void oracle_rmsnorm(const uint16_t *h, int H, double eps, uint16_t *x)
{
    unsigned __int128 ss = 0;
    for (int c = 0; c < H; c++) {
        int64_t X = (int64_t)(oracle_half_to_double(h[c]) * 16777216.0);
        __int128 sq = (__int128)X * (__int128)X;
        ss += (unsigned __int128)sq;
    }
    double s = (double)ss;
    s = s * 0x1p-48;
    double ms = s / (double)H;
    double r = 1.0 / sqrt(ms + eps);
    for (int c = 0; c < H; c++)
        x[c] = oracle_double_to_half(oracle_half_to_double(h[c]) * r);
}

/* Residual update of the fp16 stream: h_c <- fp16(h_c + y_c). */
void oracle_residual_add(uint16_t *h, const double *y, int H)
{
    for (int c = 0; c < H; c++)
        h[c] = oracle_double_to_half(oracle_half_to_double(h[c]) + y[c]);
}

/* ----------------------------------------------------------------- LFU */

/* One token's lookup in one layer's LFU cache of S slots.
 * State per slot: expert (-1 when empty), use count, insertion sequence
 * number; *seq_counter is the layer's last sequence number.
 *  (i)  the token's experts in ascending id order: a resident expert is a
 *       hit and its count grows by one;
 *  (ii) then each missing expert in ascending id order: the lowest-index
 *       empty slot if any, else, among the slots this token does not use,
 *       the lowest count, ties to the oldest insertion; the newcomer starts
 *       with count 1 and the next sequence number.
 * slot_of[j] is the slot of idx[j]; the misses are listed in insertion order.
 * Returns 0, or -1 when no victim exists (S <= k) or an expert repeats. */
int oracle_lfu_token(int S, int32_t *slot_expert, int64_t *slot_count,
                     int64_t *slot_seq, int64_t *seq_counter,
                     const int32_t *idx, int k, int32_t *slot_of,
                     int32_t *miss_expert, int32_t *miss_slot,
                     int32_t *n_miss, int64_t *hits, int64_t *misses)
{
    int32_t order[64];
    char used[256];
    char is_hit[64];
    if (k < 1 || k > 64 || S < 1 || S > 256)
        return -1;
    memset(is_hit, 0, sizeof(is_hit));
    memset(used, 0, sizeof(used));
    /* insertion sort of positions by expert id */
    for (int j = 0; j < k; j++)
        order[j] = j;
    for (int a = 1; a < k; a++) {
        int32_t t = order[a];
        int b = a - 1;
        while (b >= 0 && idx[order[b]] > idx[t]) {
            order[b + 1] = order[b];
            b--;
        }
        order[b + 1] = t;
    }
    for (int a = 1; a < k; a++)
        if (idx[order[a]] == idx[order[a - 1]])
            return -1;

    for (int a = 0; a < k; a++) {
        int j = order[a];
        for (int s = 0; s < S; s++) {
            if (slot_expert[s] == idx[j]) {
                slot_count[s] += 1;
                used[s] = 1;
                slot_of[j] = s;
                is_hit[j] = 1;
                *hits += 1;
                break;
            }
        }
    }
    *n_miss = 0;
    for (int a = 0; a < k; a++) {
        int j = order[a];
        if (is_hit[j])
            continue;
        int victim = -1;
        for (int s = 0; s < S; s++)
            if (slot_expert[s] < 0) {
                victim = s;
                break;
            }
        if (victim < 0) {
            for (int s = 0; s < S; s++) {
                if (used[s])
                    continue;
                if (victim < 0 || slot_count[s] < slot_count[victim] ||
                    (slot_count[s] == slot_count[victim] &&
                     slot_seq[s] < slot_seq[victim]))
                    victim = s;
            }
        }
        if (victim < 0)
            return -1;
        *seq_counter += 1;
        slot_expert[victim] = idx[j];
        slot_count[victim] = 1;
        slot_seq[victim] = *seq_counter;
        used[victim] = 1;
        slot_of[j] = victim;
        miss_expert[*n_miss] = idx[j];
        miss_slot[*n_miss] = victim;
        *n_miss += 1;
        *misses += 1;
    }
    return 0;
}

/* A chunk of n_tok tokens (chunked prefill, [LH] 04 "Chunked Prefill": one
 * expert fetched from storage serves every row of the chunk that uses it) in
 * one layer's LFU cache.  The pages fix no rule for a chunk; this applies the
 * per-token rule above to the chunk's distinct experts, each weighted by its
 * uses, and serves them in batches that fit the slots, so that each expert is
 * copied at most once per chunk:
 *  (i)   the distinct experts in ascending id order: a resident expert is a
 *        hit, its count grows by its number of (token, choice) pairs in the
 *        chunk, and its slot is pinned to batch 0;
 *  (ii)  then each missing expert in ascending id order takes the lowest-index
 *        empty slot if any, else, among the slots not pinned by the current
 *        batch, the lowest count, ties to the oldest insertion; when every
 *        slot is pinned, the current batch is complete (its pairs are served
 *        from the slots), the next batch starts and no slot is pinned; the
 *        newcomer's count is its number of uses and it takes the next
 *        sequence number;
 *  (iii) hits and misses count distinct experts (a miss is one copy).
 * With one token per chunk (k < S) there is one batch and this is exactly
 * oracle_lfu_token.  idx is [n_tok][k]; slot_of[q] and batch_of[q] are the
 * slot and batch of pair q = t * k + j; the misses (batch, expert, slot) are
 * listed in insertion order; *n_batch is the number of batches.  Returns 0,
 * or -1 when an expert repeats within a token or the sizes are out of range. */
int oracle_lfu_chunk(int S, int32_t *slot_expert, int64_t *slot_count,
                     int64_t *slot_seq, int64_t *seq_counter,
                     const int32_t *idx, int n_tok, int k, int32_t *slot_of,
                     int32_t *batch_of, int32_t *miss_batch, int32_t *miss_expert,
                     int32_t *miss_slot, int32_t *n_miss, int32_t *n_batch,
                     int64_t *hits, int64_t *misses)
{
    enum { kMaxDistinct = 4096 };
    static int32_t ex[kMaxDistinct], slot_ex[kMaxDistinct], batch_ex[kMaxDistinct];
    static int64_t uses[kMaxDistinct];
    char pinned[256];
    int nu = 0;
    if (k < 1 || k > 64 || S < 1 || S > 256 || S <= k || n_tok < 1)
        return -1;
    for (int t = 0; t < n_tok; t++)
        for (int a = 0; a < k; a++)
            for (int b = a + 1; b < k; b++)
                if (idx[t * k + a] == idx[t * k + b])
                    return -1;
    /* distinct experts of the chunk and their uses, ascending */
    for (int q = 0; q < n_tok * k; q++) {
        int32_t e = idx[q];
        int i = 0;
        while (i < nu && ex[i] < e)
            i++;
        if (i < nu && ex[i] == e) {
            uses[i] += 1;
            continue;
        }
        if (nu == kMaxDistinct)
            return -1;
        for (int m = nu; m > i; m--) {
            ex[m] = ex[m - 1];
            uses[m] = uses[m - 1];
        }
        ex[i] = e;
        uses[i] = 1;
        nu++;
    }
    memset(pinned, 0, sizeof(pinned));
    for (int i = 0; i < nu; i++) {
        slot_ex[i] = -1;
        batch_ex[i] = 0;
        for (int s = 0; s < S; s++)
            if (slot_expert[s] == ex[i]) {
                slot_count[s] += uses[i];
                pinned[s] = 1;
                slot_ex[i] = s;
                *hits += 1;
                break;
            }
    }
    int batch = 0;
    *n_miss = 0;
    for (int i = 0; i < nu; i++) {
        if (slot_ex[i] >= 0)
            continue;
        int victim = -1;
        for (int pass = 0; pass < 2 && victim < 0; pass++) {
            if (pass == 1) {             /* every slot pinned: next batch */
                batch += 1;
                memset(pinned, 0, sizeof(pinned));
            }
            for (int s = 0; s < S; s++)
                if (slot_expert[s] < 0) {
                    victim = s;
                    break;
                }
            if (victim < 0)
                for (int s = 0; s < S; s++) {
                    if (pinned[s])
                        continue;
                    if (victim < 0 || slot_count[s] < slot_count[victim] ||
                        (slot_count[s] == slot_count[victim] &&
                         slot_seq[s] < slot_seq[victim]))
                        victim = s;
                }
        }
        *seq_counter += 1;
        slot_expert[victim] = ex[i];
        slot_count[victim] = uses[i];
        slot_seq[victim] = *seq_counter;
        pinned[victim] = 1;
        slot_ex[i] = victim;
        batch_ex[i] = batch;
        miss_batch[*n_miss] = batch;
        miss_expert[*n_miss] = ex[i];
        miss_slot[*n_miss] = victim;
        *n_miss += 1;
        *misses += 1;
    }
    *n_batch = batch + 1;
    for (int q = 0; q < n_tok * k; q++) {
        int i = 0;
        while (ex[i] != idx[q])
            i++;
        slot_of[q] = slot_ex[i];
        batch_of[q] = batch_ex[i];
    }
    return 0;
}

/* ------------------------------------------------------------ threads */

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
