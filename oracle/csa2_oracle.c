/*
 * CSA2 CPU oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, obviously correct CPU statement of what the Compressed
 * Sparse Attention 2 (CSA2) decode/prefill hot path computes.  Only the
 * test suite, the smoke check of __graft_entry__ and the CPU-baseline /
 * reference legs of bench.py may load this library.  The CUDA library
 * (libcsa2) never links, loads or calls it, and the two share no source,
 * header, table or constant.
 *
 * Sources (page title, section):
 *  [P1] "Why Is DeepSeek V4.1 Flash So Fast?", sections 3 (CSA2), 4 (the
 *       indexer, Top-K) and 5 (Full / Reindex / Reuse layers).
 *  [P2] "DeepSeek-V4.1-Flash" (visual explainer), sections "Sharing the
 *       cache across layers" and "Fast memory, persistent storage and
 *       recomputation" (FP4 main cache entries).
 *  [P3] "Inference-Efficient LLMs: How Sparse Compute and Compressed Memory
 *       Work", sections 3 (sliding-window state), 4 (CSA2 modes) and 6 (FP4
 *       KV cache with per-group scaling; SWA kept at higher precision).
 * The pages print no formula for any of these steps; every reading taken
 * where they are silent (E2M1 with 16-element groups and fp32 scales, the
 * amax/6 scale rule, the head-summed int8 score, the tie rule, the causal
 * rule, the joint softmax) is listed with its reason in the design notes
 * and restated at the function that uses it.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * -ffp-contract=off makes every fp32 multiply and add below round on its
 * own (no fused multiply-add), which the index score definition requires.
 *
 * Parity: every function here is pinned by CPU tests against facts that do
 * not come from this file (the E2M1 value table of the OCP MX format,
 * brute-force nearest rounding, exact integer arithmetic, hand-worked
 * rounding examples, dense attention from a library routine, the worked
 * cache-size example of [P2]).  Nothing here is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENOMEM 2
#define ORC_ERANGE 3

int orc_topk_row(const float *scores, int64_t V, int32_t k, int32_t *idx_out);

/* ------------------------------------------------------------------------ */
/* FP4 (E2M1) storage of the main cache entries, per-group scaling.         */
/* [P2] "Fast memory, persistent storage and recomputation"; [P3] section 6.*/
/* ------------------------------------------------------------------------ */

/* Value of a 4-bit E2M1 code from its bit fields (OCP Microscaling format):
 * bit 3 sign, bits 2..1 exponent with bias 1, bit 0 mantissa; exponent 0 is
 * subnormal (0.5 * mantissa); no infinities or NaNs. */
float orc_e2m1_value(uint32_t code)
{
    uint32_t sign = (code >> 3) & 1u;
    uint32_t expo = (code >> 1) & 3u;
    uint32_t mant = code & 1u;
    double mag;
    if (expo == 0)
        mag = 0.5 * (double)mant;
    else
        mag = ldexp(1.0 + 0.5 * (double)mant, (int)expo - 1);
    return (float)(sign ? -mag : mag);
}

/* Magnitude code (0..7) of y >= 0: the nearest E2M1 magnitude; on an exact
 * midpoint the code whose mantissa bit is 0 (round half to even); values
 * above the largest magnitude (6) saturate to it. */
uint32_t orc_e2m1_round_mag(float y)
{
    if (y >= orc_e2m1_value(7))
        return 7; /* saturate: the nearest magnitude of anything above 6 is 6 */
    uint32_t best = 0;
    double best_err = fabs((double)y - (double)orc_e2m1_value(0));
    for (uint32_t c = 1; c < 8; ++c) {
        double err = fabs((double)y - (double)orc_e2m1_value(c));
        if (err < best_err || (err == best_err && (c & 1u) == 0u)) {
            best = c;
            best_err = err;
        }
    }
    return best;
}

/* Pack rows of D fp32 values into E2M1 codes with one fp32 scale per group
 * of 16 consecutive elements.
 *   scale s = amax / 6 (fp32 divide), amax = largest |x| of the group;
 *   code    = sign | round_mag(|x / s|) (fp32 divide), sign bit only on a
 *             non-zero magnitude; a group with s == 0 stores all-zero codes;
 *   layout  = element 2i in the low nibble of byte i of its row.
 * codes is [rows, D/2], scales is [rows, D/16].  Inputs must be finite. */
int orc_pack_fp4(const float *src, int64_t rows, int32_t D, uint8_t *codes, float *scales)
{
    if (!src || !codes || !scales || rows < 0 || D <= 0 || D % 16 != 0)
        return ORC_EINVAL;
    const int32_t G = D / 16;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t g = 0; g < G; ++g) {
            const float *x = src + r * D + (int64_t)g * 16;
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i)
                if (fabsf(x[i]) > amax)
                    amax = fabsf(x[i]);
            float s = amax / 6.0f;
            scales[r * G + g] = s;
            for (int i = 0; i < 16; ++i) {
                uint32_t c = 0;
                if (s > 0.0f) {
                    float y = x[i] / s;
                    uint32_t mag = orc_e2m1_round_mag(fabsf(y));
                    c = mag;
                    if (mag != 0 && x[i] < 0.0f)
                        c |= 8u;
                }
                uint8_t *byte = codes + r * (D / 2) + (int64_t)g * 8 + i / 2;
                if (i % 2 == 0)
                    *byte = (uint8_t)((*byte & 0xF0u) | c);
                else
                    *byte = (uint8_t)((*byte & 0x0Fu) | (c << 4));
            }
        }
    }
    return ORC_OK;
}

/* Dequantise: e[r, i] = value(code[r, i]) * scale[r, i / 16], one fp32
 * multiply.  out is [rows, D]. */
int orc_unpack_fp4(const uint8_t *codes, const float *scales, int64_t rows, int32_t D, float *out)
{
    if (!codes || !scales || !out || rows < 0 || D <= 0 || D % 16 != 0)
        return ORC_EINVAL;
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t i = 0; i < D; ++i) {
            uint8_t byte = codes[r * (D / 2) + i / 2];
            uint32_t c = (i % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
            float s = scales[r * (D / 16) + i / 16];
            out[r * D + i] = orc_e2m1_value(c) * s;
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Entry append: the per-token write side of the cache.                     */
/* [P2] "Fast memory, persistent storage and recomputation": the main cache */
/* entries are stored in a 4-bit floating-point format; [P3] section 6: FP4 */
/* with per-group scaling.  Reading: when a decode token completes a        */
/* compressed entry, that entry (its D values as the compressor produced    */
/* them) is packed with the rule of orc_pack_fp4 into row pos[b] of its     */
/* sequence's store, and its int8 index key is written into the same row of */
/* the store's index keys; a sequence with pos[b] < 0 appends nothing.      */
/* src [B, D] fp32, key [B, d_I] int8, pos [B]; codes [B, N, D/2], scales   */
/* [B, N, D/16], k_idx [B, N, d_I] are updated in place.  A position >= N   */
/* is an error: nothing is written and ORC_ERANGE is returned.              */
/* ------------------------------------------------------------------------ */
int orc_append_entry(const float *src, const int8_t *key, const int64_t *pos, int32_t B, int32_t D,
                     int32_t d_I, int64_t N, uint8_t *codes, float *scales, int8_t *k_idx)
{
    if (!src || !key || !pos || !codes || !scales || !k_idx || B < 0 || D <= 0 || D % 16 != 0 ||
        d_I <= 0 || N < 0)
        return ORC_EINVAL;
    for (int32_t b = 0; b < B; ++b)
        if (pos[b] >= N)
            return ORC_ERANGE;
    for (int32_t b = 0; b < B; ++b) {
        const int64_t n = pos[b];
        if (n < 0)
            continue;
        const int64_t row = (int64_t)b * N + n;
        int rc = orc_pack_fp4(src + (int64_t)b * D, 1, D, codes + row * (D / 2),
                              scales + row * (D / 16));
        if (rc != ORC_OK)
            return rc;
        for (int32_t i = 0; i < d_I; ++i)
            k_idx[row * d_I + i] = key[(int64_t)b * d_I + i];
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Indexer: a cheap relevance score of every compressed entry.              */
/* [P1] section 4 ("The indexer"): index heads score the compressed         */
/* positions before the expensive attention.  Reading: per head h an exact  */
/* int8 dot product of the head's query with the entry's int8 index key,    */
/* then the heads are summed with fp32 weights, left to right, each        */
/* multiply and add rounded to fp32 on its own; no activation, no scaling.  */
/* ------------------------------------------------------------------------ */

/* q: [H_I, d_I] int8, w: [H_I] fp32, keys: [N, d_I] int8 -> out[N] fp32. */
void orc_index_score_row(const int8_t *q, const float *w, const int8_t *keys, int32_t H_I,
                         int32_t d_I, int64_t N, float *out)
{
    for (int64_t n = 0; n < N; ++n) {
        const int8_t *key = keys + n * d_I;
        float acc = 0.0f;
        for (int32_t h = 0; h < H_I; ++h) {
            int32_t dot = 0;
            for (int32_t i = 0; i < d_I; ++i)
                dot += (int32_t)q[h * d_I + i] * (int32_t)key[i];
            float term = w[h] * (float)dot;
            acc = acc + term;
        }
        out[n] = acc + 0.0f; /* a -0 sum is stored as +0 */
    }
}

/* ------------------------------------------------------------------------ */
/* FP4 index keys.  [P3] section 6: V4 already used FP4 for parts of its    */
/* attention indexing machinery.  Readings (the pages give no format for    */
/* them): an index key is stored as E2M1 elements with one shared power-of- */
/* two scale per block of 32 consecutive elements, the scale kept as an     */
/* 8-bit biased exponent (the OCP Microscaling MXFP4 block format), so a    */
/* d_I = 64 key takes 32 code bytes + 2 exponent bytes instead of 64 int8   */
/* bytes.  Packing follows that format's conversion: shared exponent        */
/* s = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent), clamped to    */
/* [-127, 127] and stored as s + 127; each element is x / 2^s rounded to    */
/* the nearest E2M1 value (ties to even, saturating at 6; zero magnitude is */
/* code 0); an all-zero block stores exponent byte 0 and zero codes.        */
/* ------------------------------------------------------------------------ */

/* 2^e as an fp32 value (exact for -149 <= e <= 127). */
static float orc_pow2f(int e)
{
    return ldexpf(1.0f, e);
}

/* src [rows, d] fp32 -> codes [rows, d/2] (element 2i in the low nibble of
 * byte i), exps [rows, d/32] (biased exponents).  d % 32 == 0. */
int orc_pack_mxfp4(const float *src, int64_t rows, int32_t d, uint8_t *codes, uint8_t *exps)
{
    if (!src || !codes || !exps || rows < 0 || d <= 0 || d % 32 != 0)
        return ORC_EINVAL;
    const int32_t nb = d / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t g = 0; g < nb; ++g) {
            const float *x = src + r * d + (int64_t)g * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i)
                if (fabsf(x[i]) > amax)
                    amax = fabsf(x[i]);
            uint8_t *cb = codes + r * (d / 2) + (int64_t)g * 16;
            if (amax == 0.0f) {
                exps[r * nb + g] = 0;
                memset(cb, 0, 16);
                continue;
            }
            int ex;
            frexp((double)amax, &ex); /* amax = m * 2^ex, 0.5 <= m < 1 */
            int s = (ex - 1) - 2;
            if (s < -127)
                s = -127;
            if (s > 127)
                s = 127;
            exps[r * nb + g] = (uint8_t)(s + 127);
            const float X = orc_pow2f(s);
            for (int i = 0; i < 32; ++i) {
                float y = x[i] / X;
                uint32_t mag = orc_e2m1_round_mag(fabsf(y));
                uint32_t c = mag;
                if (mag != 0 && x[i] < 0.0f)
                    c |= 8u;
                uint8_t *byte = cb + i / 2;
                if (i % 2 == 0)
                    *byte = (uint8_t)((*byte & 0xF0u) | c);
                else
                    *byte = (uint8_t)((*byte & 0x0Fu) | (c << 4));
            }
        }
    }
    return ORC_OK;
}

/* out[r, i] = E2M1(code[r, i]) * 2^(exps[r, i/32] - 127), one fp32 multiply. */
int orc_unpack_mxfp4(const uint8_t *codes, const uint8_t *exps, int64_t rows, int32_t d,
                     float *out)
{
    if (!codes || !exps || !out || rows < 0 || d <= 0 || d % 32 != 0)
        return ORC_EINVAL;
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t i = 0; i < d; ++i) {
            uint8_t byte = codes[r * (d / 2) + i / 2];
            uint32_t c = (i % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
            out[r * d + i] = orc_e2m1_value(c) * orc_pow2f((int)exps[r * (d / 32) + i / 32] - 127);
        }
    return ORC_OK;
}

/* Index score over FP4 keys.  Reading: per head h and key block g the exact
 * integer idot = sum_{i in g} q[h,i] * (2 * E2M1(code_i)) (twice the E2M1
 * value is an integer in {0, +-1, +-2, +-3, +-4, +-6, +-8, +-12}); the
 * head's dot product is the fp32 sum over blocks in ascending order of
 * (float)idot * 2^(exp_g - 128) (each multiply and add rounded on its own;
 * the -128 is the exponent bias 127 plus the factor 2 above); the heads are
 * then summed with their weights exactly as for int8 keys.
 * q: [H_I, d_I] int8, w: [H_I], codes: [N, d_I/2], exps: [N, d_I/32] -> out[N]. */
void orc_index_score_fp4k_row(const int8_t *q, const float *w, const uint8_t *codes,
                              const uint8_t *exps, int32_t H_I, int32_t d_I, int64_t N, float *out)
{
    const int32_t nb = d_I / 32;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *cb = codes + n * (d_I / 2);
        float acc = 0.0f;
        for (int32_t h = 0; h < H_I; ++h) {
            float dot = 0.0f;
            for (int32_t g = 0; g < nb; ++g) {
                int32_t idot = 0;
                for (int32_t i = 32 * g; i < 32 * g + 32; ++i) {
                    uint8_t byte = cb[i / 2];
                    uint32_t c = (i % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
                    int32_t v2 = (int32_t)(2.0f * orc_e2m1_value(c)); /* exact small integer */
                    idot += (int32_t)q[h * d_I + i] * v2;
                }
                float term = (float)idot * orc_pow2f((int)exps[n * nb + g] - 128);
                dot = dot + term;
            }
            float t = w[h] * dot;
            acc = acc + t;
        }
        out[n] = acc + 0.0f;
    }
}

/* Index scores + top-k over FP4 keys for all rows of a decode batch (one
 * query per sequence, every entry visible).  q_idx [B,H_I,d_I], w [B,H_I],
 * codes [B,N,d_I/2], exps [B,N,d_I/32]; idx_out [B, topk]; scores_out NULL
 * or [B, N]. */
int orc_index_topk_fp4k(const int8_t *q_idx, const float *w, const uint8_t *codes,
                        const uint8_t *exps, int32_t B, int32_t H_I, int32_t d_I, int64_t N,
                        int32_t topk, int32_t *idx_out, float *scores_out)
{
    if (!q_idx || !w || (N > 0 && (!codes || !exps)) || !idx_out || B < 0 || H_I <= 0 ||
        d_I <= 0 || d_I % 32 != 0 || N < 0 || topk <= 0)
        return ORC_EINVAL;
    float *row = (float *)malloc((size_t)(N > 0 ? N : 1) * sizeof(float));
    if (!row)
        return ORC_ENOMEM;
    int rc = ORC_OK;
    for (int32_t b = 0; b < B && rc == ORC_OK; ++b) {
        orc_index_score_fp4k_row(q_idx + (int64_t)b * H_I * d_I, w + (int64_t)b * H_I,
                                 codes + (int64_t)b * N * (d_I / 2), exps + (int64_t)b * N * (d_I / 32),
                                 H_I, d_I, N, row);
        if (scores_out)
            memcpy(scores_out + (int64_t)b * N, row, (size_t)N * sizeof(float));
        rc = orc_topk_row(row, N, topk, idx_out + (int64_t)b * topk);
    }
    free(row);
    return rc;
}

/* Number of entries query t of a chunk may see.  Decode (n_prior < 0): all
 * N stored entries.  Prefill: the n_prior entries that precede the chunk,
 * plus chunk entry j once every token it compresses (ratio*j .. ratio*j +
 * ratio - 1, token positions relative to the chunk start) is at or before
 * t; capped at N. */
int64_t orc_visible_count(int64_t N, int64_t n_prior, int32_t ratio, int64_t t)
{
    if (n_prior < 0)
        return N;
    int64_t v = n_prior + (t + 1) / ratio;
    return v < N ? v : N;
}

/* ------------------------------------------------------------------------ */
/* Top-K selection.  [P1] sections 3-4: keep the Top-K highest-scoring     */
/* compressed positions.  Reading: ties go to the lower index; the kept     */
/* indices are written in ascending order; when fewer than K entries are    */
/* visible the rest of the row is -1.                                       */
/* ------------------------------------------------------------------------ */

typedef struct {
    float score;
    int64_t n;
} orc_cand;

static int orc_cand_cmp(const void *pa, const void *pb)
{
    const orc_cand *a = (const orc_cand *)pa, *b = (const orc_cand *)pb;
    if (a->score > b->score)
        return -1;
    if (a->score < b->score)
        return 1;
    return (a->n < b->n) ? -1 : (a->n > b->n) ? 1 : 0;
}

static int orc_i32_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a < b) ? -1 : (a > b) ? 1 : 0;
}

/* scores[0..V) are the visible scores; writes idx_out[0..k). */
int orc_topk_row(const float *scores, int64_t V, int32_t k, int32_t *idx_out)
{
    if (V < 0 || k <= 0)
        return ORC_EINVAL;
    orc_cand *c = (orc_cand *)malloc((size_t)(V > 0 ? V : 1) * sizeof(orc_cand));
    if (!c)
        return ORC_ENOMEM;
    for (int64_t n = 0; n < V; ++n) {
        c[n].score = scores[n];
        c[n].n = n;
    }
    qsort(c, (size_t)V, sizeof(orc_cand), orc_cand_cmp);
    int64_t m = V < k ? V : k;
    for (int64_t i = 0; i < m; ++i)
        idx_out[i] = (int32_t)c[i].n;
    qsort(idx_out, (size_t)m, sizeof(int32_t), orc_i32_cmp);
    for (int64_t i = m; i < k; ++i)
        idx_out[i] = -1;
    free(c);
    return ORC_OK;
}

/* Index scores + top-k for chosen query rows.
 * q_idx [B,T,H_I,d_I] int8, w [B,T,H_I] fp32, k_idx [B,N,d_I] int8.
 * rows: flattened (b*T + t) row ids, or NULL for all B*T rows (then nrows
 * must be B*T).  idx_out [nrows, topk]; scores_out NULL or [nrows, N] with
 * -inf at the entries the row may not see. */
int orc_index_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B, int32_t T,
                   int32_t H_I, int32_t d_I, int64_t N, int64_t n_prior, int32_t ratio, int32_t topk,
                   const int64_t *rows, int64_t nrows, int32_t *idx_out, float *scores_out)
{
    if (!q_idx || !w || (!k_idx && N > 0) || !idx_out || B < 0 || T < 0 || H_I <= 0 || d_I <= 0 ||
        N < 0 || topk <= 0 || (n_prior >= 0 && ratio <= 0))
        return ORC_EINVAL;
    if (!rows && nrows != (int64_t)B * T)
        return ORC_EINVAL;
    float *row_scores = (float *)malloc((size_t)(N > 0 ? N : 1) * sizeof(float));
    if (!row_scores)
        return ORC_ENOMEM;
    int rc = ORC_OK;
    for (int64_t i = 0; i < nrows && rc == ORC_OK; ++i) {
        int64_t r = rows ? rows[i] : i;
        if (r < 0 || r >= (int64_t)B * T) {
            rc = ORC_ERANGE;
            break;
        }
        int64_t b = r / T, t = r % T;
        orc_index_score_row(q_idx + r * H_I * d_I, w + r * H_I, k_idx + b * N * d_I, H_I, d_I, N,
                            row_scores);
        int64_t V = orc_visible_count(N, n_prior, ratio, t);
        if (scores_out) {
            for (int64_t n = 0; n < N; ++n)
                scores_out[i * N + n] = (n < V) ? row_scores[n] : -INFINITY;
        }
        rc = orc_topk_row(row_scores, V, topk, idx_out + i * topk);
    }
    free(row_scores);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Sparse attention over the selected entries plus the local window.       */
/* [P1] section 3: a 128-token sliding window plus the indexer-selected    */
/* compressed positions; [P3] section 3: local keys and values are         */
/* layer-specific; [P3] section 6: the window stays at higher precision.   */
/* Readings: one softmax over selected entries and window together, scale   */
/* sm_scale (1/sqrt(D) by default); a global entry is used as both key and  */
/* value (MQA: one entry serves every head); window keys and values are     */
/* separate bf16 rows; query t of a chunk uses window rows t .. t+W-1 of a  */
/* [W-1+T, D] buffer (row t+W-1 is token t itself); an index of -1 is       */
/* padding and is skipped; with nothing to attend to, out = 0, lse = -inf.  */
/* Everything after dequantisation is computed in double.                  */
/* ------------------------------------------------------------------------ */

static double orc_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* q [B,T,H,D] bf16 bits; codes [B,N,D/2]; scales [B,N,D/16];
 * idx [B,T,topk] int32; win_k/win_v [B,W-1+T,D] bf16 bits (unused if W==0).
 * rows: flattened (b*T+t) ids or NULL (nrows = B*T).
 * out [nrows,H,D] double; lse [nrows,H] double. */
int orc_sparse_attn(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
                    const uint16_t *win_k, const uint16_t *win_v, int32_t B, int32_t T, int32_t H,
                    int32_t D, int64_t N, int32_t topk, int32_t W, float sm_scale,
                    const int64_t *rows, int64_t nrows, double *out, double *lse)
{
    if (!q || !out || !lse || B < 0 || T < 0 || H <= 0 || D <= 0 || D % 16 != 0 || N < 0 ||
        topk < 0 || W < 0 || (topk > 0 && !idx) || (W > 0 && (!win_k || !win_v)))
        return ORC_EINVAL;
    if (!rows && nrows != (int64_t)B * T)
        return ORC_EINVAL;
    const int64_t nkeys_max = (int64_t)topk + W;
    double *keys = (double *)malloc((size_t)(nkeys_max > 0 ? nkeys_max : 1) * D * sizeof(double));
    double *vals = (double *)malloc((size_t)(nkeys_max > 0 ? nkeys_max : 1) * D * sizeof(double));
    double *z = (double *)malloc((size_t)(nkeys_max > 0 ? nkeys_max : 1) * sizeof(double));
    float *ent = (float *)malloc((size_t)D * sizeof(float));
    if (!keys || !vals || !z || !ent) {
        free(keys);
        free(vals);
        free(z);
        free(ent);
        return ORC_ENOMEM;
    }
    int rc = ORC_OK;
    const int64_t win_rows = (int64_t)W - 1 + T;
    for (int64_t i = 0; i < nrows && rc == ORC_OK; ++i) {
        int64_t r = rows ? rows[i] : i;
        if (r < 0 || r >= (int64_t)B * T) {
            rc = ORC_ERANGE;
            break;
        }
        int64_t b = r / T, t = r % T;
        /* Gather the key/value list of this query. */
        int64_t nk = 0;
        for (int32_t j = 0; j < topk; ++j) {
            int32_t n = idx[r * topk + j];
            if (n < 0)
                continue;
            if ((int64_t)n >= N) {
                rc = ORC_ERANGE;
                break;
            }
            orc_unpack_fp4(codes + (b * N + n) * (D / 2), scales + (b * N + n) * (D / 16), 1, D, ent);
            for (int32_t d = 0; d < D; ++d) {
                keys[nk * D + d] = (double)ent[d];
                vals[nk * D + d] = (double)ent[d];
            }
            ++nk;
        }
        if (rc != ORC_OK)
            break;
        for (int32_t j = 0; j < W; ++j) {
            int64_t row = b * win_rows + t + j;
            for (int32_t d = 0; d < D; ++d) {
                keys[nk * D + d] = orc_bf16_to_double(win_k[row * D + d]);
                vals[nk * D + d] = orc_bf16_to_double(win_v[row * D + d]);
            }
            ++nk;
        }
        for (int32_t h = 0; h < H; ++h) {
            const uint16_t *qh = q + (r * H + h) * D;
            double *o = out + (i * H + h) * D;
            if (nk == 0) {
                for (int32_t d = 0; d < D; ++d)
                    o[d] = 0.0;
                lse[i * H + h] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int64_t j = 0; j < nk; ++j) {
                double dot = 0.0;
                for (int32_t d = 0; d < D; ++d)
                    dot += orc_bf16_to_double(qh[d]) * keys[j * D + d];
                z[j] = (double)sm_scale * dot;
                if (z[j] > m)
                    m = z[j];
            }
            double l = 0.0;
            for (int32_t d = 0; d < D; ++d)
                o[d] = 0.0;
            for (int64_t j = 0; j < nk; ++j) {
                double p = exp(z[j] - m);
                l += p;
                for (int32_t d = 0; d < D; ++d)
                    o[d] += p * vals[j * D + d];
            }
            for (int32_t d = 0; d < D; ++d)
                o[d] /= l;
            lse[i * H + h] = m + log(l);
        }
    }
    free(keys);
    free(vals);
    free(z);
    free(ent);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Cross-layer sharing: the per-layer mode table.                           */
/* [P1] section 5 and [P2] "Sharing the cache across layers": Full layers  */
/* own their entries and selection; Reindex layers share another layer's    */
/* entries and select afresh; Reuse layers share both.                      */
/* modes is [L][3] = {mode, kv_src, idx_src} with mode 0 Full, 1 Reindex,  */
/* 2 Reuse.  A table is valid when: a Full layer names itself for both;     */
/* a Reindex layer names an earlier Full layer as kv_src and itself as      */
/* idx_src; a Reuse layer names an earlier Full or Reindex layer as idx_src */
/* and that layer's kv_src as its own kv_src.                               */
/* ------------------------------------------------------------------------ */

int orc_validate_modes(const int32_t *modes, int32_t L)
{
    if (!modes || L <= 0)
        return ORC_EINVAL;
    for (int32_t l = 0; l < L; ++l) {
        int32_t mode = modes[3 * l], kv = modes[3 * l + 1], ix = modes[3 * l + 2];
        if (mode == 0) {
            if (kv != l || ix != l)
                return ORC_EINVAL;
        } else if (mode == 1) {
            if (kv < 0 || kv >= l || modes[3 * kv] != 0 || ix != l)
                return ORC_EINVAL;
        } else if (mode == 2) {
            if (ix < 0 || ix >= l || modes[3 * ix] == 2 || kv != modes[3 * ix + 1])
                return ORC_EINVAL;
        } else {
            return ORC_EINVAL;
        }
    }
    return ORC_OK;
}

/* The cache-size checklist of [P2] "Several mechanisms in one release":
 * entries x numbers per entry x stored layer copies x bits per number,
 * in bytes.  Stored layer copies = layers that keep their own entries
 * (Full layers); every other layer points at one of them. */
int orc_group_cache_bytes(const int32_t *modes, int32_t L, int64_t entries,
                          int64_t numbers_per_entry, int64_t bits_per_number, uint64_t *bytes_out)
{
    if (!bytes_out || entries < 0 || numbers_per_entry < 0 || bits_per_number <= 0)
        return ORC_EINVAL;
    int rc = orc_validate_modes(modes, L);
    if (rc != ORC_OK)
        return rc;
    uint64_t copies = 0;
    for (int32_t l = 0; l < L; ++l)
        if (modes[3 * l] == 0)
            ++copies;
    uint64_t bits = (uint64_t)entries * (uint64_t)numbers_per_entry * copies * (uint64_t)bits_per_number;
    *bytes_out = bits / 8u;
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Hierarchical sparse indexing.  [P3] section 5 ("Hierarchical Sparse      */
/* Indexing"): an earlier Full layer searches broadly and keeps a candidate */
/* pool -- the example keeps 2,048 blocks of eight positions, 16,384        */
/* candidates -- and later Reindex layers search only within that pool.    */
/* Readings (the pages give no formula):                                    */
/*  - a block is `block` consecutive compressed positions, block j covering */
/*    [j*block, (j+1)*block); the last block holds only visible positions;  */
/*  - a block's score is the largest of the Full layer's index scores over  */
/*    its visible positions; blocks are ranked by that score, ties to the   */
/*    lower block index, and the best n_blocks are kept (all of them when   */
/*    fewer are visible);                                                   */
/*  - the pool lists the kept blocks' positions in ascending order;         */
/*  - a Reindex layer scores only the pool's positions with its own index   */
/*    query (same score as above) and keeps their top-k with the same tie   */
/*    rule, ascending output and -1 padding.                                */
/* ------------------------------------------------------------------------ */

typedef struct {
    float score;
    int64_t j;
} orc_block;

static int orc_block_cmp(const void *pa, const void *pb)
{
    const orc_block *a = (const orc_block *)pa, *b = (const orc_block *)pb;
    if (a->score > b->score)
        return -1;
    if (a->score < b->score)
        return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j) ? 1 : 0;
}

/* scores[0..V): a Full layer's visible index scores.  Writes the pool to
 * pool_out[0..n_blocks*block) (-1 after its *pool_len entries). */
int orc_block_pool(const float *scores, int64_t V, int32_t block, int32_t n_blocks,
                   int32_t *pool_out, int64_t *pool_len)
{
    if (!pool_out || !pool_len || V < 0 || block <= 0 || n_blocks <= 0 || (V > 0 && !scores))
        return ORC_EINVAL;
    const int64_t nb = (V + block - 1) / block;
    orc_block *b = (orc_block *)malloc((size_t)(nb > 0 ? nb : 1) * sizeof(orc_block));
    unsigned char *kept = (unsigned char *)calloc((size_t)(nb > 0 ? nb : 1), 1);
    if (!b || !kept) {
        free(b);
        free(kept);
        return ORC_ENOMEM;
    }
    for (int64_t j = 0; j < nb; ++j) {
        const int64_t n0 = j * block, n1 = (n0 + block < V) ? n0 + block : V;
        float best = scores[n0];
        for (int64_t n = n0 + 1; n < n1; ++n)
            if (scores[n] > best)
                best = scores[n];
        b[j].score = best;
        b[j].j = j;
    }
    qsort(b, (size_t)nb, sizeof(orc_block), orc_block_cmp);
    const int64_t m = nb < n_blocks ? nb : n_blocks;
    for (int64_t i = 0; i < m; ++i)
        kept[b[i].j] = 1;
    int64_t len = 0;
    for (int64_t n = 0; n < V; ++n)
        if (kept[n / block])
            pool_out[len++] = (int32_t)n;
    for (int64_t i = len; i < (int64_t)n_blocks * block; ++i)
        pool_out[i] = -1;
    *pool_len = len;
    free(b);
    free(kept);
    return ORC_OK;
}

/* Top-k of one query row over a pool of positions.  q: [H_I, d_I] int8,
 * w: [H_I], keys: [N, d_I] int8, pool[0..pool_len) ascending positions
 * (each < N).  idx_out[0..k): kept positions, ascending, -1 padded. */
int orc_pool_topk(const int8_t *q, const float *w, const int8_t *keys, int32_t H_I, int32_t d_I,
                  int64_t N, const int32_t *pool, int64_t pool_len, int32_t k, int32_t *idx_out)
{
    if (!q || !w || !keys || !idx_out || H_I <= 0 || d_I <= 0 || N < 0 || pool_len < 0 ||
        k <= 0 || (pool_len > 0 && !pool))
        return ORC_EINVAL;
    orc_cand *c = (orc_cand *)malloc((size_t)(pool_len > 0 ? pool_len : 1) * sizeof(orc_cand));
    if (!c)
        return ORC_ENOMEM;
    for (int64_t i = 0; i < pool_len; ++i) {
        if (pool[i] < 0 || pool[i] >= N) {
            free(c);
            return ORC_ERANGE;
        }
        orc_index_score_row(q, w, keys + (int64_t)pool[i] * d_I, H_I, d_I, 1, &c[i].score);
        c[i].n = pool[i];
    }
    qsort(c, (size_t)pool_len, sizeof(orc_cand), orc_cand_cmp);
    const int64_t m = pool_len < k ? pool_len : k;
    for (int64_t i = 0; i < m; ++i)
        idx_out[i] = (int32_t)c[i].n;
    qsort(idx_out, (size_t)m, sizeof(int32_t), orc_i32_cmp);
    for (int64_t i = m; i < k; ++i)
        idx_out[i] = -1;
    free(c);
    return ORC_OK;
}
