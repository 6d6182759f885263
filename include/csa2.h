/*
 * csa2.h -- C ABI of the CSA2 (Compressed Sparse Attention 2) hot path for
 * NVIDIA B200 (sm_100a).  Library: libcsa2.so.
 *
 * What the path computes, per layer and query token (sources are web pages
 * on DeepSeek-V4.1-Flash, cited by title and section):
 *   1. an indexer scores every visible compressed global cache entry
 *      ("Why Is DeepSeek V4.1 Flash So Fast?", section 4, "The indexer");
 *   2. the Top-K best entries are kept (same page, sections 3-4);
 *   3. the kept entries, stored as FP4 with per-group scaling ("DeepSeek-
 *      V4.1-Flash" visual explainer, section "Fast memory, persistent
 *      storage and recomputation"; "Inference-Efficient LLMs", section 6),
 *      are gathered and dequantised;
 *   4. softmax attention runs over them together with the layer's own
 *      128-token sliding window kept at higher precision (bf16)
 *      ("Why Is DeepSeek V4.1 Flash So Fast?", section 3; "Inference-
 *      Efficient LLMs", sections 3 and 6);
 *   5. layers run in Full, Reindex or Reuse mode ("DeepSeek-V4.1-Flash",
 *      section "Sharing the cache across layers"; "Why Is DeepSeek V4.1
 *      Flash So Fast?", section 5).
 *
 * The pages fix no formula, size or format detail for any step; the
 * readings this library takes are stated at each call below.
 *
 * Conventions for every call:
 *  - Pointers named as device pointers must point to device (or managed)
 *    memory of the current CUDA device; host pointers are named as such.
 *    All arrays are dense, row-major, and device arrays are 16-byte
 *    aligned.  The caller owns every buffer; the library allocates no
 *    device memory.  Scratch ("workspace") is passed in by the caller; its
 *    size comes from the matching *_workspace_size query.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call only enqueues work on `stream` and returns; nothing synchronises
 *    except csa2_get_device_status.
 *  - bf16 arrays are passed as uint16_t bit patterns.
 *  - Errors are returned, never raised: arguments are validated on the
 *    host before anything is enqueued, and an invalid call enqueues
 *    nothing.  CSA2_ERR_CUDA means a launch failed; the CUDA error is then
 *    also left for cudaGetLastError.  Indices that point outside the entry
 *    store are skipped on the device and recorded in a device status word
 *    that csa2_get_device_status reports.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum csa2_status {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, bad mode table */
    CSA2_ERR_UNSUPPORTED = 2,   /* valid request outside the compiled shape set */
    CSA2_ERR_CUDA = 3,          /* a CUDA launch or query failed */
    CSA2_ERR_WORKSPACE = 4,     /* workspace missing or smaller than the query says */
    CSA2_ERR_DEVICE_STATUS = 5  /* a kernel recorded a bad index (see csa2_get_device_status) */
} csa2_status;

/* Layer modes ("DeepSeek-V4.1-Flash", section "Sharing the cache across
 * layers"): Full computes its own entries and its own selection; Reindex
 * shares another layer's entries and makes a fresh selection; Reuse shares
 * both.  Every layer keeps its own queries and its own local window. */
typedef enum csa2_mode {
    CSA2_FULL = 0,
    CSA2_REINDEX = 1,
    CSA2_REUSE = 2,
    /* A Reindex layer that searches only the candidate pool its kv_src Full
     * layer kept ("Inference-Efficient LLMs", section 5: later Reindex layers
     * search within the pool an earlier Full layer narrowed the context to;
     * the pool rule is that of csa2_index_pool, the selection that of
     * csa2_pool_topk).  Table rules as for CSA2_REINDEX; decode rows only;
     * the pool shape comes from csa2_dims.pool_block / pool_blocks. */
    CSA2_REINDEX_POOL = 3
} csa2_mode;

/* One row of the per-layer mode table.  kv_src: the layer whose entry store
 * (FP4 codes, scales, int8 index keys) this layer reads; idx_src: the layer
 * whose selection it uses.  Valid tables: Full names itself twice; Reindex
 * names an earlier Full layer as kv_src and itself as idx_src; Reuse names
 * an earlier Full or Reindex layer as idx_src and that layer's kv_src as
 * its own kv_src. */
typedef struct csa2_layer_mode {
    int32_t mode;
    int32_t kv_src;
    int32_t idx_src;
} csa2_layer_mode;

/* Human-readable name of a status code (static string, never NULL). */
const char *csa2_status_string(int32_t status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int32_t csa2_version(void);

/* ---------------------------------------------------------------------- */
/* FP4 entry store                                                         */
/* ---------------------------------------------------------------------- */

/* Pack fp32 entries into FP4 E2M1 codes with one fp32 scale per 16
 * consecutive elements ("FP4 representation with per-group scaling":
 * "Inference-Efficient LLMs", section 6; the E2M1 element format and the
 * group of 16 are this library's reading).  Per group: s = amax / 6 (IEEE
 * fp32 divide, amax = largest |x|); each element's code is the E2M1 value
 * nearest to x / s (fp32 divide), ties to the even code, saturating at 6;
 * a zero magnitude is stored as code 0 (never negative zero); a group with
 * s == 0 stores all-zero codes.  Element 2i goes in the low nibble of byte i.
 *   src    device, fp32 [rows, D], finite values
 *   codes  device, uint8 [rows, D/2]   (output)
 *   scales device, fp32 [rows, D/16]   (output)
 *   D % 16 == 0, D > 0; rows >= 0 (rows == 0 enqueues nothing). */
csa2_status csa2_pack_fp4(const float *src, int64_t rows, int32_t D, uint8_t *codes,
                          float *scales, void *stream);

/* Entry append: the per-token write side of the cache.  When a decode
 * token completes a compressed entry, the entry is stored in FP4 ("DeepSeek-
 * V4.1-Flash" visual explainer, section "Fast memory, persistent storage and
 * recomputation"; "Inference-Efficient LLMs", section 6: FP4 with per-group
 * scaling) in the next row of its sequence's store, with its int8 index key
 * beside it.  For each sequence b with pos[b] >= 0: src[b] is packed with
 * the rule of csa2_pack_fp4 into row pos[b] of codes/scales, and key[b] is
 * copied into row pos[b] of k_idx; a sequence with pos[b] < 0 appends
 * nothing.  A position >= N is skipped and recorded in the device status
 * word (bit 0).  The entry values and the key come from the model (the
 * compressor and the indexer's key projection), which this library does
 * not hold.
 *   src    device, fp32 [B, D]      (16-byte aligned)
 *   key    device, int8 [B, d_I]    (16-byte aligned)
 *   pos    device, int64 [B]
 *   codes  device, uint8 [B, N, D/2]   (updated)
 *   scales device, fp32 [B, N, D/16]   (updated)
 *   k_idx  device, int8 [B, N, d_I]    (updated)
 *   D % 16 == 0, d_I % 16 == 0. */
csa2_status csa2_append_entry(const float *src, const int8_t *key, const int64_t *pos, int32_t B,
                              int32_t D, int32_t d_I, int64_t N, uint8_t *codes, float *scales,
                              int8_t *k_idx, void *stream);

/* Dequantise: out[r, i] = E2M1(code[r, i]) * scale[r, i / 16] (one fp32
 * multiply).  codes device uint8 [rows, D/2]; scales device fp32 [rows,
 * D/16]; out device fp32 [rows, D]. */
csa2_status csa2_unpack_fp4(const uint8_t *codes, const float *scales, int64_t rows, int32_t D,
                            float *out, void *stream);

/* ---------------------------------------------------------------------- */
/* Indexer score + Top-K                                                   */
/* ---------------------------------------------------------------------- */

/* Workspace bytes csa2_index_topk needs for these sizes (0 on invalid
 * sizes). */
size_t csa2_index_topk_workspace_size(int32_t B, int32_t T, int32_t H_I, int32_t d_I, int64_t N,
                                      int32_t topk);

/* Indexer scores and Top-K selection ("Why Is DeepSeek V4.1 Flash So
 * Fast?", section 4: a cheap relevance search over all compressed
 * positions, then the Top-K go on to attention).
 * Score of entry n for query (b, t), this library's reading:
 *   dot_h    = sum_i q_idx[b,t,h,i] * k_idx[b,n,i]   (exact int32)
 *   score    = (((0 + w[b,t,0]*dot_0) + w[b,t,1]*dot_1) + ...) + 0
 * each fp32 product and sum rounded on its own (no fused multiply-add).
 * Visibility: decode (n_prior < 0) sees all N entries; a prefill chunk
 * (n_prior >= 0) query t sees n < min(N, n_prior + (t + 1) / ratio), i.e.
 * chunk entry j once all `ratio` tokens it compresses are at or before t.
 * Selection: the min(topk, visible) visible entries with the largest score,
 * ties to the lower index, written in ascending index order; the rest of
 * the row is -1.
 *   q_idx     device, int8 [B, T, H_I, d_I]
 *   w         device, fp32 [B, T, H_I]
 *   k_idx     device, int8 [B, N, d_I]  (the entry store's index keys)
 *   idx_out   device, int32 [B, T, topk]           (output)
 *   score_out device, fp32 [B, T, N] or NULL       (optional output: the
 *             score of every entry, -inf where the query may not see it)
 *   ws        device workspace of ws_bytes >= csa2_index_topk_workspace_size
 * Supported: d_I in {16, 32, 64, 128}, H_I in {1, 2, 4, 8}, H_I * d_I <= 512,
 * 1 <= topk <= 65536, N < 2^31, ratio >= 1 when n_prior >= 0. */
csa2_status csa2_index_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                            int32_t T, int32_t H_I, int32_t d_I, int64_t N, int64_t n_prior,
                            int32_t ratio, int32_t topk, int32_t *idx_out, float *score_out,
                            void *ws, size_t ws_bytes, void *stream);

/* Same computation and results as csa2_index_topk, for callers that cannot
 * allocate device memory: e.g. a host runtime that owns all device memory
 * through its own allocator and hands extensions no workspace, or a serving
 * loop that must not allocate after start-up because an allocation there
 * could fail or stall at the wrong moment.  The pages describe no such call;
 * it has no counterpart there.
 * Scratch comes from a fixed 16 MiB array inside the library (held on every
 * GPU that loads the library until the process exits); this call allocates
 * nothing itself.  Sizes whose scratch would exceed it
 * (csa2_index_topk_workspace_size(...) > 16 MiB) return CSA2_ERR_UNSUPPORTED
 * before anything is enqueued.  The first call on a device looks up the
 * array's device address (in the device's primary context, the one the
 * CUDA runtime uses; calls made under another context of the same device
 * are not supported) and sets kernel attributes; make that first call
 * before any stream capture.  All calls share the one array and leave their
 * contents in it (the parts that must start at zero are cleared by each
 * call), so calls that overlap on the GPU -- on different streams, or from
 * several host threads -- race and corrupt each other's results: serialise
 * them.  Keep the kernel timing trace off (its default).  Arguments as for
 * csa2_index_topk, without ws / ws_bytes. */
csa2_status csa2_index_topk_noalloc(const int8_t *q_idx, const float *w, const int8_t *k_idx,
                                    int32_t B, int32_t T, int32_t H_I, int32_t d_I, int64_t N,
                                    int64_t n_prior, int32_t ratio, int32_t topk,
                                    int32_t *idx_out, float *score_out, void *stream);

/* ---------------------------------------------------------------------- */
/* FP4 index keys                                                          */
/* ---------------------------------------------------------------------- */

/* "Inference-Efficient LLMs", section 6: V4 already used FP4 for parts of
 * its attention indexing machinery.  This library's reading for the index
 * keys: E2M1 elements with one power-of-two scale per block of 32 elements,
 * stored as an 8-bit biased exponent (the OCP Microscaling MXFP4 block
 * format), so a key of d_I elements takes d_I/2 + d_I/32 bytes (34 for
 * d_I = 64, against 64 as int8).  Per block: s = floor(log2(amax)) - 2,
 * clamped to [-127, 127], exponent byte s + 127; each element's code is the
 * E2M1 value nearest to x / 2^s (IEEE divide, ties to the even code,
 * saturating at 6; zero magnitude is code 0); an all-zero block stores
 * exponent byte 0 and zero codes; element 2i is the low nibble of byte i.
 *   src   device, fp32 [rows, d_I]
 *   codes device, uint8 [rows, d_I/2]   (output, 16-byte aligned)
 *   exps  device, uint8 [rows, d_I/32]  (output)
 *   d_I % 32 == 0. */
csa2_status csa2_pack_index_keys_fp4(const float *src, int64_t rows, int32_t d_I,
                                     uint8_t *codes, uint8_t *exps, void *stream);

/* Workspace bytes for csa2_index_topk_fp4k (0 on unsupported sizes). */
size_t csa2_index_topk_fp4k_workspace_size(int32_t B, int32_t H_I, int32_t d_I, int64_t N,
                                           int32_t topk);

/* Index score + Top-K over FP4 keys, decode rows (one query per sequence,
 * every entry visible).  Score of entry n (this library's reading): per
 * head h and key block g the exact integer idot = sum over the block of
 * q_idx[b,h,i] * (2 * E2M1(code_i)); the head's dot is the fp32 sum over the
 * blocks in ascending order of idot * 2^(exp_g - 128) (each multiply and add
 * rounded on its own); the heads are combined with their weights exactly as
 * in csa2_index_topk.  Selection as in csa2_index_topk.
 *   q_idx   device, int8 [B, H_I, d_I];  w device, fp32 [B, H_I]
 *   k_codes device, uint8 [B, N, d_I/2]; k_exps device, uint8 [B, N, d_I/32]
 *   idx_out device, int32 [B, topk]   (output)
 *   ws      device workspace of ws_bytes >= csa2_index_topk_fp4k_workspace_size
 * Supported: d_I in {32, 64}, H_I == 4, N % 16 == 0, N >= 1, topk <= 65536. */
csa2_status csa2_index_topk_fp4k(const int8_t *q_idx, const float *w, const uint8_t *k_codes,
                                 const uint8_t *k_exps, int32_t B, int32_t H_I, int32_t d_I,
                                 int64_t N, int32_t topk, int32_t *idx_out, void *ws,
                                 size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------- */
/* Hierarchical indexer: a Full layer's candidate pool, a Reindex layer's  */
/* top-k within it                                                         */
/* ---------------------------------------------------------------------- */

/* "Inference-Efficient LLMs: How Sparse Compute and Compressed Memory
 * Work", section 5 ("Hierarchical Sparse Indexing"): an earlier Full layer
 * searches the whole context and keeps a candidate pool (the example: 2,048
 * blocks of eight positions, 16,384 candidates); later Reindex layers
 * search only within that pool.  This library's reading: block j covers
 * positions [j*block, (j+1)*block) (the last block only those < N); a
 * block's score is the largest index score (as in csa2_index_topk) among
 * its positions; the best n_blocks blocks are kept, ties to the lower block;
 * the pool lists their positions ascending.  Decode shape: one query per
 * sequence. */

/* Workspace bytes for csa2_index_pool (0 on invalid or unsupported sizes). */
size_t csa2_index_pool_workspace_size(int32_t B, int32_t H_I, int32_t d_I, int64_t N,
                                      int32_t block, int32_t n_blocks);

/* The pool of each sequence's Full-layer query.
 *   q_idx    device, int8 [B, H_I, d_I]
 *   w        device, fp32 [B, H_I]
 *   k_idx    device, int8 [B, N, d_I]   (16-byte aligned)
 *   pool_out device, int32 [B, n_blocks * block]   (output) the kept
 *            positions ascending, then -1 (fewer when fewer blocks exist, or
 *            when the last block is partial)
 *   ws       device workspace of ws_bytes >= csa2_index_pool_workspace_size
 * Supported: the index shapes of csa2_index_topk, 1 <= block <= 64,
 * n_blocks * block <= 65536, B <= 65535. */
csa2_status csa2_index_pool(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                            int32_t H_I, int32_t d_I, int64_t N, int32_t block, int32_t n_blocks,
                            int32_t *pool_out, void *ws, size_t ws_bytes, void *stream);

/* Workspace bytes for csa2_pool_topk (0 on invalid or unsupported sizes). */
size_t csa2_pool_topk_workspace_size(int32_t B, int32_t P, int32_t topk);

/* Top-k of each sequence's (Reindex-layer) query within its pool: the
 * index score of every pool position, then the min(topk, positions) best,
 * ties to the lower position, ascending, then -1.
 *   q_idx, w, k_idx as for csa2_index_pool (the Reindex layer's query, the
 *            store's index keys)
 *   pool     device, int32 [B, P]: positions ascending, then -1 entries (as
 *            written by csa2_index_pool); an entry >= N counts as -1 and is
 *            recorded in the device status word (bad index)
 *   idx_out  device, int32 [B, topk]   (output)
 *   ws       device workspace of ws_bytes >= csa2_pool_topk_workspace_size
 * Supported: the index shapes of csa2_index_topk, P <= 65536,
 * 1 <= topk <= 65536, B <= 65535. */
csa2_status csa2_pool_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                           int32_t H_I, int32_t d_I, int64_t N, const int32_t *pool, int32_t P,
                           int32_t topk, int32_t *idx_out, void *ws, size_t ws_bytes,
                           void *stream);

/* ---------------------------------------------------------------------- */
/* Sparse attention over the selected entries + the local window           */
/* ---------------------------------------------------------------------- */

/* Workspace bytes for csa2_sparse_attn_decode / _prefill.  The current
 * kernels merge their partial softmax states on chip and need none (0);
 * ws may then be NULL. */
size_t csa2_sparse_attn_workspace_size(int32_t B, int32_t T, int32_t H, int32_t D, int32_t topk,
                                       int32_t W);

/* Decode attention ("Why Is DeepSeek V4.1 Flash So Fast?", section 3: the
 * selected compressed positions plus a 128-token sliding window).  Per
 * head h of sequence b, this library's reading: one softmax over the
 * logits sm_scale * <q[b,h], key> of every selected entry (key = the
 * dequantised entry, which is also its value: one entry serves all heads)
 * and every window row (key win_k, value win_v); out = sum p * value,
 * lse = natural log of sum exp(logit).  Index -1 is padding and skipped;
 * an index >= N is skipped and recorded in the device status word.  With
 * nothing to attend to, out = 0 and lse = -inf.  fp32 accumulation.
 *   q       device, bf16 [B, H, D]
 *   codes   device, uint8 [B, N, D/2]; scales device, fp32 [B, N, D/16]
 *   idx     device, int32 [B, topk]
 *   win_k, win_v  device, bf16 [B, W, D]; row W-1 is the current token
 *           (may be NULL when W == 0)
 *   out     device, fp32 [B, H, D] (output); lse device, fp32 [B, H] or NULL
 * Supported: D in {64, 128}, 1 <= H <= 128, 0 <= topk <= 65536,
 * 0 <= W <= 4096. */
csa2_status csa2_sparse_attn_decode(const uint16_t *q, const uint8_t *codes, const float *scales,
                                    const int32_t *idx, const uint16_t *win_k,
                                    const uint16_t *win_v, int32_t B, int32_t H, int32_t D,
                                    int64_t N, int32_t topk, int32_t W, float sm_scale, float *out,
                                    float *lse, void *ws, size_t ws_bytes, void *stream);

/* Prefill (chunk) attention: as decode, for T query tokens per sequence.
 *   q       device, bf16 [B, T, H, D]
 *   idx     device, int32 [B, T, topk]  (e.g. from csa2_index_topk with
 *           n_prior >= 0)
 *   win_k, win_v device, bf16 [B, W-1+T, D]; query t reads rows t .. t+W-1
 *           (row t+W-1 is token t itself)
 *   out     device, fp32 [B, T, H, D]; lse device, fp32 [B, T, H] or NULL */
csa2_status csa2_sparse_attn_prefill(const uint16_t *q, const uint8_t *codes, const float *scales,
                                     const int32_t *idx, const uint16_t *win_k,
                                     const uint16_t *win_v, int32_t B, int32_t T, int32_t H,
                                     int32_t D, int64_t N, int32_t topk, int32_t W,
                                     float sm_scale, float *out, float *lse, void *ws,
                                     size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------- */
/* Cross-layer groups                                                      */
/* ---------------------------------------------------------------------- */

/* Shapes shared by every layer of a group. */
typedef struct csa2_dims {
    int32_t B, T, H, D;      /* batch, query tokens per sequence, heads, entry dim */
    int64_t N;               /* stored entries per sequence */
    int32_t H_I, d_I;        /* indexer heads and dim */
    int32_t topk, W;         /* selected entries, window length */
    int64_t n_prior;         /* -1: decode; >= 0: prefill chunk after n_prior entries */
    int32_t ratio;           /* tokens per entry (prefill visibility) */
    float sm_scale;          /* softmax scale (1/sqrt(D) by convention) */
    int32_t pool_block;      /* pool layers: positions per block (1..64), else 0 */
    int32_t pool_blocks;     /* pool layers: blocks kept (pool_block*pool_blocks <= 65536) */
} csa2_dims;

/* Per-layer device pointers (shapes as in the calls above).  q, q_idx, w,
 * win_k, win_v, out, lse are the layer's own.  codes, scales, k_idx are
 * read only for a layer that is some layer's kv_src (a Full layer).  idx
 * [B, T, topk] is written for Full and Reindex layers; a Reuse layer's idx
 * is ignored (it reads its idx_src layer's buffer). */
typedef struct csa2_layer_io {
    const uint16_t *q;
    const int8_t *q_idx;
    const float *w;
    const uint16_t *win_k;
    const uint16_t *win_v;
    const uint8_t *codes;
    const float *scales;
    const int8_t *k_idx;
    int32_t *idx;
    float *out;
    float *lse;
    /* Optional, read for a Full layer's store: index keys in FP4 (see
     * csa2_pack_index_keys_fp4) instead of int8 -- k_idx then points at the
     * FP4 codes [B, N, d_I/2] and k_exps at the block exponents [B, N,
     * d_I/32].  NULL: int8 keys.  Layers over FP4 keys need the decode shape
     * of csa2_index_topk_fp4k. */
    const uint8_t *k_exps;
    /* Optional, Full layers with int8 keys: this step's entry append
     * (csa2_append_entry) into the layer's own store before its index scan,
     * so a completed entry is visible to the same step's query.  app_src fp32
     * [B, D], app_key int8 [B, d_I], app_pos int64 [B] (device); NULL app_pos
     * = no append.  With app_pos set, the layer's codes, scales and k_idx
     * are written. */
    const float *app_src;
    const int8_t *app_key;
    const int64_t *app_pos;
    /* A Full layer that is the kv_src of a CSA2_REINDEX_POOL layer writes its
     * candidate pool here: int32 [B, pool_blocks * pool_block], positions
     * ascending then -1 (csa2_index_pool's layout), from the same scan as its
     * own selection; the pool layer reads it from its kv_src's entry. */
    int32_t *pool;
} csa2_layer_io;

/* CSA2_OK when the table follows the rules of csa2_layer_mode. */
csa2_status csa2_validate_modes(const csa2_layer_mode *modes, int32_t L);

/* The visual explainer's cache checklist ("DeepSeek-V4.1-Flash", section
 * "Several mechanisms in one release"): entries x numbers per entry x
 * stored layer copies x bits per number, in bytes, where stored layer
 * copies = the table's Full layers.  modes is a host array of L rows. */
csa2_status csa2_group_cache_bytes(const csa2_layer_mode *modes, int32_t L, int64_t entries,
                                   int64_t numbers_per_entry, int64_t bits_per_number,
                                   uint64_t *bytes_out);

/* Workspace bytes for csa2_layer_group_run and csa2_layer_run. */
size_t csa2_layer_group_workspace_size(const csa2_dims *dims);

/* Run only layer `layer` (0 <= layer < L) of the table, exactly as
 * csa2_layer_group_run runs it (the table is validated whole; `layer`'s
 * sources must already hold their outputs when it reads them). */
csa2_status csa2_layer_run(const csa2_layer_mode *modes, const csa2_layer_io *io, int32_t L,
                           int32_t layer, const csa2_dims *dims, void *ws, size_t ws_bytes,
                           void *stream);

/* Run L layers in table order on one stream: Full and Reindex layers run
 * the index + Top-K step over their kv_src store's index keys with their
 * own index query; Reuse layers take idx_src's selection; then every layer
 * runs attention (decode when dims->T == 1 and n_prior < 0, else prefill)
 * over its kv_src store with its own queries and window.
 *   modes host array [L]; io host array [L] of device pointers; dims host.
 * The table is validated before anything is enqueued. */
csa2_status csa2_layer_group_run(const csa2_layer_mode *modes, const csa2_layer_io *io, int32_t L,
                                 const csa2_dims *dims, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------- */
/* Staging copies                                                          */
/* ---------------------------------------------------------------------- */

/* One copy of csa2_stage_copies: `rows` rows of `row_bytes` bytes, row i
 * from src + i * src_stride to dst + i * dst_stride (byte strides).  src
 * and dst are each either memory of the current device or page-locked host
 * memory that the device addresses at the same pointer (cudaHostAlloc /
 * cudaMallocHost under unified addressing).  Pointers, row_bytes and both
 * strides are multiples of 16 bytes; dst_stride >= row_bytes when rows > 1;
 * src_stride >= 0. */
typedef struct csa2_copy2d {
    const void *src;
    void *dst;
    int64_t rows;
    int64_t row_bytes;
    int64_t src_stride;
    int64_t dst_stride;
} csa2_copy2d;

#define CSA2_MAX_STAGE_COPIES 16

/* Up to CSA2_MAX_STAGE_COPIES copies in one kernel launch on `stream`: a
 * decode step's inputs from pinned host buffers into their device buffers
 * (a window's new row straight into its slot), or its results back to the
 * host.  Every thread moves 16-byte pieces through the mapped host buffer
 * itself (host memory read uncached, written through), so all pieces are in
 * flight at once and a step pays about one round trip over the host link
 * instead of a copy-engine transfer per buffer.  The pages describe no such
 * call: it is the library's input/output path.  The copies run concurrently:
 * no destination may overlap another copy's source or destination.  The
 * host must leave a host source unchanged, and not read a host destination,
 * until the stream has passed the launch.
 *   copies  host array [n]; rows == 0 or row_bytes == 0 skips a copy.
 * Errors: CSA2_ERR_INVALID_ARG for n outside [0, CSA2_MAX_STAGE_COPIES], a
 * null pointer, misalignment, a negative size or stride, or memory the
 * device cannot address at that pointer (pageable host memory, another
 * device's memory; both ends of each range are checked); CSA2_ERR_CUDA when
 * a pointer query or the launch fails. */
csa2_status csa2_stage_copies(const csa2_copy2d *copies, int32_t n, void *stream);

/* ---------------------------------------------------------------------- */
/* Kernel timing trace                                                     */
/* ---------------------------------------------------------------------- */

/* Turn the kernel timing trace on (enable != 0; clears earlier records) or
 * off.  While on, every kernel the library launches is bracketed by a pair
 * of CUDA events recorded on the launch stream, so per-kernel device time
 * can be read back.  Host-side state, not thread-safe: enable, run and
 * read from one host thread.  At most 1<<16 records are kept. */
csa2_status csa2_trace_enable(int32_t enable);

/* Number of kernel launches recorded since the trace was enabled. */
int32_t csa2_trace_count(void);

/* Record i: *name receives the kernel's static name, *ms its device time
 * in milliseconds.  Waits for the record's stop event. */
csa2_status csa2_trace_get(int32_t i, const char **name, float *ms);

/* ---------------------------------------------------------------------- */
/* Device status                                                           */
/* ---------------------------------------------------------------------- */

/* Decode kernels.  Decode rows (one query per sequence, every entry
 * visible, no score output) are served either by two launches per layer --
 * the index scan (scores to the workspace) and one thread-block cluster per
 * query row for the top-k and the attention (CSA2_DECODE_SCAN_CLUSTER, the
 * default) -- or by one cooperative launch that keeps each CTA's scores in
 * shared memory and meets the other CTAs through global counters
 * (CSA2_DECODE_FUSED).  Both compute the same results bit for bit (indices)
 * and within the attention tolerance.  FP4 index keys and candidate pools
 * are served by both.  Process-wide; the environment variable
 * CSA2_DECODE_KERNEL=fused sets the initial choice.  Not synchronised with
 * calls in flight on other host threads. */
#define CSA2_DECODE_SCAN_CLUSTER 0
#define CSA2_DECODE_FUSED 1
csa2_status csa2_set_decode_kernel(int32_t kernel);
int32_t csa2_get_decode_kernel(void);

/* Self-test of the library's bounded waits (every wait on a pipeline
 * barrier, on another CTA's delivery or on another CTA's counter gives up
 * after a limit, records bit 1 in the device status word and lets the
 * kernel finish).  Launches one thread that waits, with a limit of
 * limit_cycles SM cycles (1 .. 2^32), on a barrier phase that never
 * completes and on a counter that nothing raises: afterwards
 * csa2_get_device_status reports bit 1 and the device keeps working.  The
 * pages describe no such call; it exists for tests. */
csa2_status csa2_wait_timeout_selftest(int64_t limit_cycles, void *stream);

/* Synchronise `stream`, then read and clear the current device's status
 * word.  *code_out (may be NULL) receives the raw word: 0 = clean, bit 0 =
 * an attention index >= N was skipped, bit 1 = a pipeline wait gave up
 * after its iteration limit.  Returns CSA2_ERR_DEVICE_STATUS when the word
 * was non-zero, CSA2_ERR_CUDA when the synchronisation failed. */
csa2_status csa2_get_device_status(void *stream, int32_t *code_out);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */
