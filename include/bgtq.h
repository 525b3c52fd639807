/*
 * bgtq.h -- C ABI of libbgtq: Block-GTQ / TQ-MSE packed-KV decode attention on B200.
 *
 * Sources of the operations (page title, passage):
 *  [BGTQ] "Block-GTQ: RoPE-Block Rate Allocation for KV-Cache Quantization", abstract:
 *         s2 RoPE 2-D frequency blocks carry the key precision; s3 label-free query-key
 *         energy score with codec-dependent rate penalties; s4 largest-marginal-gain
 *         allocation; s5 TQ-MSE instantiation, equal-rate blocks grouped, attention over
 *         packed caches without a decoded fp16 KV cache; s7 "K2V2" logical rates;
 *         s8 no fp16 sink or recent-token buffer.
 *  [TQ]   "TurboQuant: paper algorithm and vLLM engineering implementation" (pipeline
 *         diagram): input vector x (per-head K or V) -> random rotation -> per-coordinate
 *         MSE scalar quantisation with a few centroids; exercise 1: KV memory footprint;
 *         vLLM column, box "NC": norm correction of the distortion of the norm by the
 *         centroids (the "_nc" presets).
 *
 * Conventions for every call:
 *  - head_dim is 128; RoPE block j (0..63) is the coordinate pair {j, j+64}
 *    (rotate-half RoPE). Keys are passed AFTER RoPE.
 *  - All device buffers are allocated and owned by the caller. A layout owns only its
 *    host tables and, after bgtq_layout_upload, one device allocation of constants.
 *  - Device calls are asynchronous on the given stream (a cudaStream_t passed as void*;
 *    NULL = legacy default stream). They never allocate, never synchronise, and check
 *    every argument before launching; on error nothing is written.
 *  - A failing call returns a status and leaves a message for bgtq_last_error_string()
 *    (per host thread). No C++ exception crosses the ABI.
 *
 * Packed cache format (one (batch row, KV head) = capacity/64 consecutive tiles):
 *  tile of 64 tokens = [K codes | V codes | K norms | V norms]
 *   Both code areas are fragment-major: cut into per-lane bit strings (lane l = 4g + t of
 *   a 32-lane warp) that hold exactly the codes one lane turns into its tensor-core
 *   operands. Words are little-endian; bit n of a string is bit n%8 of its byte n/8.
 *   K codes:   64 x Kb bytes, Kb = 128*avg_k_bits/8. Packed key dimensions: K groups by
 *              descending rate; in a group, blocks ascending, coordinate j before j+64.
 *              Each group is cut into quads of 4 dimension pairs (8 dimensions); the
 *              group's last quad holds the remaining P = 1..3 pairs when its dimension
 *              count is not a multiple of 8. Quad blocks follow one another, 16*P*r bytes
 *              each. In a quad, lane i = g*P + e (g = 0..7, pair e = 0..P-1) holds for
 *              the tokens g + 8m (m = 0..7) the codes lo (dim 2e) and hi (dim 2e+1) as a
 *              16r-bit string: r = 1: bit m = lo, bit 8+m = hi; r = 2..4: field m of 2r
 *              bits at bit 2rm = lo | hi << r. The string sits at bit 16r*i of the block,
 *              except r = 3: bits 0..31 at bit 32i, bits 32..47 at bit 256P + 16i.
 *   V codes:   four 16-token chunks of 256*b_V bytes (tokens 16c..16c+15). Lane l = 4g+t
 *              holds 32 fields n = 4mt + k (mt = 0..7, k = 0..3): value dimension
 *              16g + 2mt + (k&1), tokens lo = 2t + 8(k>>1) and hi = lo + 1 of the chunk,
 *              as a 64*b_V-bit string: b_V = 1: word u = 0,1 has bit f = lo and bit
 *              16+f = hi of field 16u+f; b_V = 2..4: field n of 2b_V bits at bit 2b_V*n
 *              = lo | hi << b_V. The string sits at bit 64*b_V*l of the chunk, except
 *              b_V = 3, 4: bits 0..127 at bit 128l, the rest at bit 4096 + (64b_V-128)l.
 *   K norms:   n_kgroups x 64 fp32, group-major: the norm s of each token's group g
 *              (s = |x_g|; with BGTQ_LAYOUT_NORM_CORRECT s = |x_g| sqrt(d_g) / |c|, c the
 *              vector of the token's centroids in the group).
 *   V norms:   64 fp32, likewise.
 *   With BGTQ_LAYOUT_NORM_FP16 both norm areas hold fp16 (round to nearest even; a norm
 *   above 65504 is stored as 65504).
 *  tile_bytes = 64*(Kb + 16*b_V) + 64*nb*(n_kgroups + 1), nb = 4 (fp32 norms) or 2 (fp16).
 *  A token decodes to x_hat_g = (s / sqrt(d_g)) R_g^T c.
 *  A code c of a group with rate r stands for the Lloyd-Max centroid c of N(0,1) with 2^r
 *  levels (ascending); the coordinate it encodes is y = sqrt(d_g) * (R_g x_g)_i / |x_g|.
 */
#ifndef BGTQ_H
#define BGTQ_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BGTQ_OK = 0,
  BGTQ_ERR_INVALID = 1,     /* bad argument: null pointer, bad size, unsupported shape */
  BGTQ_ERR_INFEASIBLE = 2,  /* rate budget outside [n*min_rate, n*max_rate] */
  BGTQ_ERR_CAPACITY = 3,    /* capacity not a multiple of 64 or too small for the call */
  BGTQ_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  BGTQ_ERR_NOMEM = 5,       /* host or device allocation failed (layout calls only) */
  BGTQ_ERR_WORKSPACE = 6,   /* workspace pointer null or smaller than required */
  BGTQ_ERR_DEVICE = 7       /* layout not uploaded, or uploaded to another device */
} bgtq_status;

enum { BGTQ_F32 = 0, BGTQ_BF16 = 1, BGTQ_F16 = 2 };

#define BGTQ_HEAD_DIM 128
#define BGTQ_N_BLOCKS 64
#define BGTQ_TILE_TOKENS 64
#define BGTQ_MAX_GQA 32  /* query columns per KV head: (h_q / h_kv) x query tokens */
#define BGTQ_MAX_KGROUPS 4

/* Device status bits reported by bgtq_device_status. */
#define BGTQ_STATUS_ENCODE_OVERFLOW 1u  /* encode: seq_len + n_new > capacity; those tokens skipped */
#define BGTQ_STATUS_DECODE_CLAMPED 2u   /* decode: seq_len > capacity or > max_seq_len; clamped */
#define BGTQ_STATUS_TIMEOUT 4u          /* decode: a bulk copy did not complete within the kernel's bounded
                                           wait; that call's output is invalid */
#define BGTQ_STATUS_BAD_PAGE 8u        /* paged calls: a block-table entry outside the pool; the encode
                                          skips that token, the attention reads nothing for that tile */

typedef struct bgtq_layout bgtq_layout;

typedef struct {
  int head_dim;                       /* 128 */
  int n_blocks;                       /* 64 */
  int n_kgroups;                      /* number of distinct key rates, 1..4 */
  int group_rate[BGTQ_MAX_KGROUPS];   /* descending */
  int group_dim[BGTQ_MAX_KGROUPS];    /* d_g = 2 x blocks in the group */
  int v_rate;
  int k_record_bytes;                 /* Kb */
  int v_record_bytes;                 /* 16 * v_rate */
  int bytes_per_token;                /* Kb + 16 v_rate + norm_bytes (n_kgroups + 1) */
  int tile_tokens;                    /* 64 */
  int tile_bytes;
  unsigned long long seed;
  unsigned flags;                     /* BGTQ_LAYOUT_* options of bgtq_layout_create_ex */
  int norm_bytes;                     /* 4 (fp32 norms) or 2 (fp16) */
  int n_packed;                       /* stored key dimensions: 128 - 2 x (rate-0 blocks) */
} bgtq_layout_info;

/* Message of the last failing call on this host thread ("" if none). */
const char* bgtq_last_error_string(void);
/* ABI version: 200 (bgtq_layout_info gained flags, norm_bytes and n_packed; layout
 * options, rate-0 blocks, per-head scores and multi-token calls were added). */
int bgtq_version(void);

/* ---------------------------------------------------------------- host planning ---- */

/* Gaussian Lloyd-Max quantiser [TQ, "per-coordinate MSE scalar quantisation"]:
 * bits in 1..4; writes 2^bits ascending centroids, 2^bits - 1 thresholds (midpoints,
 * middle one exactly 0) and the per-coordinate MSE on N(0,1). Any output may be NULL. */
bgtq_status bgtq_lloyd_max(int bits, double* centroids, double* thresholds, double* mse);

/* Energy score per RoPE block [BGTQ s3]. q_cal [n_q, h_q, 128] and k_cal [n_k, h_kv, 128]
 * fp32 host arrays (post-RoPE is fine: RoPE rotates inside each block). score_out[64]:
 * sum over KV heads of (mean over calibration queries and that head's h_q/h_kv query
 * heads of |q_j|^2) x (mean over calibration keys of |k_j|^2). */
bgtq_status bgtq_block_energy(const float* q_cal, long long n_q, int h_q,
                              const float* k_cal, long long n_k, int h_kv, double* score_out);
/* The same energy score per KV head, for a rate allocation per KV head: score_out
 * [h_kv * 64], score_out[h * 64 + j] = the term of KV head h in bgtq_block_energy (whose
 * score is their sum). A per-head allocation gives each KV head its own layout; such
 * heads are cached and decoded together through a layout set (bgtq_layout_set_create,
 * below), or with one call per KV head (h_kv = 1). */
bgtq_status bgtq_block_energy_heads(const float* q_cal, long long n_q, int h_q,
                                    const float* k_cal, long long n_k, int h_kv, double* score_out);

/* Largest-marginal-gain rate allocation [BGTQ s4]. Rates start at min_rate; each step
 * adds one bit to the block with the largest score[j] * (D[b_j] - D[b_j + 1]) among
 * blocks below max_rate (ties: lowest j) until the rates sum to total_bits.
 * distortion: array indexed by rate (entries min_rate..max_rate used), or NULL for the
 * Gaussian Lloyd-Max MSE with D(0) = 1 (a rate-0 block is not stored and decodes to 0).
 * 0 <= min_rate <= max_rate <= 4, max_rate >= 1. BGTQ_ERR_INFEASIBLE if
 * total_bits is outside [n_blocks*min_rate, n_blocks*max_rate]. rates_out[n_blocks]. */
bgtq_status bgtq_allocate_rates(const double* score, int n_blocks, int min_rate, int max_rate,
                                long long total_bits, const double* distortion, int* rates_out);

/* Layout of one layer [BGTQ s5]: k_rates[64] in 0..4 summing to a multiple of 4 (so a K
 * record is whole bytes) with at least one block coded, v_rate in 1..4, seed of the
 * rotations. A rate-0 block is not stored: it joins no group and its two coordinates
 * decode to 0 (they take no part in the scores). Groups equal-rate blocks,
 * draws one seeded Haar rotation per K group (Philox4x32-10 stream = rate) and one for V
 * (stream 0), and builds the Lloyd-Max tables. Host only. */
bgtq_status bgtq_layout_create(const int* k_rates, int v_rate, unsigned long long seed,
                               bgtq_layout** out);
/* Layout options (bit flags of bgtq_layout_create_ex; 0 = the layout of bgtq_layout_create).
 * NORM_CORRECT [TQ, box "NC"]: the stored norm of a group is |x_g| sqrt(d_g) / |c| instead
 *   of |x_g|, so the decoded vector (s / sqrt(d_g)) R_g^T c has the norm of the input.
 *   The codes are unchanged; only the norm the encoder writes differs.
 * NORM_FP16: norms stored as fp16 (2 bytes per token and group instead of 4). */
#define BGTQ_LAYOUT_NORM_CORRECT 1u
#define BGTQ_LAYOUT_NORM_FP16 2u
/* bgtq_layout_create with options; BGTQ_ERR_INVALID for an unknown flag bit. */
bgtq_status bgtq_layout_create_ex(const int* k_rates, int v_rate, unsigned long long seed, unsigned flags,
                                  bgtq_layout** out);
void bgtq_layout_destroy(bgtq_layout* layout);
bgtq_status bgtq_layout_get_info(const bgtq_layout* layout, bgtq_layout_info* info);
/* Rotation of K group g (0..n_kgroups-1) or of V (g = n_kgroups), row-major d x d fp64,
 * y = R x. max_elems bounds the write. */
bgtq_status bgtq_layout_rotation(const bgtq_layout* layout, int group, double* out, long long max_elems);
/* packed_to_coord[128]: original coordinate of each packed key dimension. */
bgtq_status bgtq_layout_coords(const bgtq_layout* layout, int* packed_to_coord);

/* Resident bytes of a packed cache [TQ exercise 1]: batch x h_kv x ceil(tokens/64) tiles.
 * Returns -1 on bad arguments. */
long long bgtq_cache_bytes(const bgtq_layout* layout, int batch, int h_kv, long long tokens);

/* ---------------------------------------------------------------- device calls ----- */

/* Copies the layout's constants to `device` (one cudaMalloc, freed by destroy). Must
 * precede the device calls; not for use during stream capture. */
bgtq_status bgtq_layout_upload(bgtq_layout* layout, int device);

/* TQ-MSE encode and append [TQ pipeline; BGTQ s5]. k, v: [batch, n_new, h_kv, 128]
 * contiguous, dtype BGTQ_F32/BF16/F16, device memory. seq_lens_dev[batch] int32 device:
 * the position of token 0 of row b (not modified; the caller advances it). cache: device
 * buffer of bgtq_cache_bytes(layout, batch, h_kv, capacity) bytes. Tokens whose position
 * is >= capacity are skipped and set BGTQ_STATUS_ENCODE_OVERFLOW. Writes each token's
 * K record, V codes and norms; the rest of the cache is untouched. */
bgtq_status bgtq_encode_append(const bgtq_layout* layout, const void* k, const void* v, int dtype,
                               int batch, int n_new, int h_kv, const int* seq_lens_dev,
                               void* cache, long long capacity, void* stream);

/* Workspace bytes that bgtq_decode_attention needs for this shape on the current device
 * (split-K partials). 0 on bad arguments. */
size_t bgtq_workspace_bytes(const bgtq_layout* layout, int batch, int h_q, int h_kv,
                            long long max_seq_len);

/* Single-token decode attention over the packed cache [BGTQ s5, s8]. q [batch, h_q, 128]
 * (dtype as above, device; query head i uses KV head i / (h_q/h_kv)), cache as written by
 * bgtq_encode_append, seq_lens_dev[batch] int32 device = number of cached tokens of each
 * row (0 gives a zero output row), max_seq_len >= every seq_len (plans the split-K grid;
 * larger lengths are clamped and flagged), softmax_scale (e.g. 1/sqrt(128)).
 * out [batch, h_q, 128] fp32 device. workspace: device buffer of at least
 * bgtq_workspace_bytes(...). h_q/h_kv must be 1..32; a KV head's query heads are taken 8 at
 * a time (each group of 8 reads the head's cache once). */
bgtq_status bgtq_decode_attention(const bgtq_layout* layout, const void* q, int q_dtype,
                                  int batch, int h_q, int h_kv, const void* cache,
                                  const int* seq_lens_dev, long long capacity, long long max_seq_len,
                                  float softmax_scale, float* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* One decode step of one layer [TQ pipeline; BGTQ s5, s8]: appends n_new tokens per row,
 * then attends the query over the grown cache. The same results as bgtq_encode_append
 * (k_new, v_new, kv_dtype, n_new, seq_lens_dev) followed by bgtq_decode_attention over
 * seq_lens_dev[b] + n_new tokens, in one chain of three kernels: the encode and the
 * rotation of q share the first launch. seq_lens_dev[batch] int32 device = tokens cached
 * before the step (not modified; the caller advances it). max_seq_len >= every
 * seq_lens_dev[b] + n_new; workspace as for bgtq_decode_attention. n_new = 0 attends only. */
bgtq_status bgtq_decode_step(const bgtq_layout* layout, const void* k_new, const void* v_new,
                             int kv_dtype, int n_new, const void* q, int q_dtype, int batch, int h_q,
                             int h_kv, void* cache, const int* seq_lens_dev, long long capacity,
                             long long max_seq_len, float softmax_scale, float* out,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Attention logits over the packed cache [BGTQ s5]: scores[(b*h_q + i)*scores_ld + t] =
 * softmax_scale * q_i . k_hat_t for every cached token t < seq_lens_dev[b] (k_hat decoded
 * from the packed codes: sum over groups of |k_g|/sqrt(d_g) R_g^T c[codes]), fp32 device
 * memory owned by the caller; entries at t >= seq_lens_dev[b] are not written.
 * scores_ld >= max_seq_len. Other arguments and the workspace as for
 * bgtq_decode_attention. Computed with the same key path as the attention (for
 * diagnostics such as the logit error of a rate allocation). */
bgtq_status bgtq_decode_scores(const bgtq_layout* layout, const void* q, int q_dtype, int batch,
                               int h_q, int h_kv, const void* cache, const int* seq_lens_dev,
                               long long capacity, long long max_seq_len, float softmax_scale,
                               float* scores, long long scores_ld, void* workspace,
                               size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- split over token ranges */

/* Decode attention over one part of every row's tokens, for attention split over
 * disjoint token ranges (e.g. one range per GPU, each holding the packed cache of its
 * range), merged afterwards by bgtq_merge_partials. [BGTQ s5: attention over packed
 * caches; the split is the log-sum-exp bookkeeping of split attention, which reaches the
 * same result as attention over all tokens.] Arguments as bgtq_decode_attention (the
 * cache holds this part's tokens of each row, seq_lens_dev their count); instead of out,
 * partial [batch, h_q, 130] fp32 device receives per query head: m = the largest logit
 * in base-2 units (softmax_scale q.k_hat / ln 2), l = sum_t 2^(logit_t - m), and
 * o'[128] = sum_t 2^(logit_t - m) v'_t / l with v'_t = (|v_t| / sqrt(128)) c[vcodes_t]
 * the value in V's rotated space. A row with no token gives m = -inf, l = 0, o' = 0. */
bgtq_status bgtq_decode_attention_partial(const bgtq_layout* layout, const void* q, int q_dtype, int batch,
                                          int h_q, int h_kv, const void* cache, const int* seq_lens_dev,
                                          long long capacity, long long max_seq_len, float softmax_scale,
                                          float* partial, void* workspace, size_t workspace_bytes, void* stream);
/* Merges n_parts partial records of the same rows and heads over disjoint token ranges:
 * partials [n_parts, batch, h_q, 130] fp32 device (each part as written by
 * bgtq_decode_attention_partial), out [batch, h_q, 128] fp32 device = R_V^T of the
 * log-sum-exp merge (M = max m, w = l 2^(m - M), o' = sum w o' / sum w): the attention
 * output over the union of the parts' tokens. */
bgtq_status bgtq_merge_partials(const bgtq_layout* layout, const float* partials, int n_parts, int batch, int h_q,
                                float* out, void* stream);

/* ---------------------------------------------------------------- paged caches */

/* The calls above with a paged cache (sequences of different lengths share one pool,
 * e.g. in a serving engine). The pool holds num_pages pages of h_kv * tile_bytes bytes:
 * page p = the h_kv tiles (KV heads in order, each in the tile format above) of one
 * 64-token span of one batch row. block_table_dev[b * max_pages + i] (int32, device) is
 * the page of tokens 64 i .. 64 i + 63 of row b; a row holds at most max_pages * 64
 * tokens (its "capacity"). Entries outside [0, num_pages) set BGTQ_STATUS_BAD_PAGE (the
 * encode then skips the token, the attention leaves that tile out); the caller keeps
 * pages of different rows distinct. Results are the same as with a contiguous cache. */
long long bgtq_paged_pool_bytes(const bgtq_layout* layout, int h_kv, long long num_pages);
bgtq_status bgtq_encode_append_paged(const bgtq_layout* layout, const void* k, const void* v, int dtype,
                                     int batch, int n_new, int h_kv, const int* seq_lens_dev, void* pool,
                                     long long num_pages, const int* block_table_dev, long long max_pages,
                                     void* stream);
bgtq_status bgtq_decode_attention_paged(const bgtq_layout* layout, const void* q, int q_dtype, int batch,
                                        int h_q, int h_kv, const void* pool, long long num_pages,
                                        const int* block_table_dev, long long max_pages,
                                        const int* seq_lens_dev, long long max_seq_len,
                                        float softmax_scale, float* out, void* workspace,
                                        size_t workspace_bytes, void* stream);
bgtq_status bgtq_decode_step_paged(const bgtq_layout* layout, const void* k_new, const void* v_new,
                                   int kv_dtype, int n_new, const void* q, int q_dtype, int batch,
                                   int h_q, int h_kv, void* pool, long long num_pages,
                                   const int* block_table_dev, long long max_pages,
                                   const int* seq_lens_dev, long long max_seq_len, float softmax_scale,
                                   float* out, void* workspace, size_t workspace_bytes, void* stream);

/* Multi-token decode attention ([BGTQ s5]: attention over the packed cache; causal as in
 * autoregressive attention): n_q consecutive query tokens per row whose keys and values
 * are already in the cache, as its last n_q tokens. q [batch, n_q, h_q, 128] device
 * (q_dtype), out [batch, n_q, h_q, 128] fp32 device; query j of row b sits at position
 * seq_len_b - n_q + j and attends to tokens 0 .. seq_len_b - n_q + j (a row with
 * seq_len_b < n_q gives zeros for the queries that see no token). The query columns of
 * a KV head share a tensor-core tile, 8 at a time: (h_q / h_kv) * n_q must be <= 32
 * (BGTQ_ERR_INVALID otherwise; each tile of 8 columns reads the head's cache once). Workspace: bgtq_workspace_bytes(layout, batch,
 * h_q * n_q, h_kv, max_seq_len). n_q = 1 is bgtq_decode_attention. Other arguments,
 * ownership and errors as bgtq_decode_attention. */
bgtq_status bgtq_decode_attention_multi(const bgtq_layout* layout, const void* q, int q_dtype, int batch,
                                        int n_q, int h_q, int h_kv, const void* cache,
                                        const int* seq_lens_dev, long long capacity, long long max_seq_len,
                                        float softmax_scale, float* out, void* workspace,
                                        size_t workspace_bytes, void* stream);
/* Multi-token decode step (speculative verification, a prefill chunk): append n_new >= 1
 * tokens per row at seq_lens_dev[b] (k_new, v_new [batch, n_new, h_kv, 128]) and attend
 * with their own queries q [batch, n_new, h_q, 128], causal among them, in one kernel
 * chain; out [batch, n_new, h_q, 128] fp32. seq_lens_dev holds the lengths BEFORE the
 * call and is not modified. (h_q / h_kv) * n_new <= 32; workspace as
 * bgtq_decode_attention_multi with n_q = n_new. Errors as bgtq_decode_step. */
bgtq_status bgtq_decode_step_multi(const bgtq_layout* layout, const void* k_new, const void* v_new,
                                   int kv_dtype, int n_new, const void* q, int q_dtype, int batch, int h_q,
                                   int h_kv, void* cache, const int* seq_lens_dev, long long capacity,
                                   long long max_seq_len, float softmax_scale, float* out, void* workspace,
                                   size_t workspace_bytes, void* stream);
/* bgtq_decode_step_multi on a paged cache (pool, num_pages, block table as
 * bgtq_decode_step_paged). */
bgtq_status bgtq_decode_step_multi_paged(const bgtq_layout* layout, const void* k_new, const void* v_new,
                                         int kv_dtype, int n_new, const void* q, int q_dtype, int batch,
                                         int h_q, int h_kv, void* pool, long long num_pages,
                                         const int* block_table_dev, long long max_pages,
                                         const int* seq_lens_dev, long long max_seq_len,
                                         float softmax_scale, float* out, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- one layout per KV head */

/* [BGTQ s3-s5]: the rate allocation may be made per KV head (bgtq_block_energy_heads), each
 * head then coded with its own layout (its own groups, rotations and codebook tables). A
 * layout set holds the layouts of the h_kv heads of one attention layer, in head order,
 * so that one call encodes or decodes every head. The layouts must be uploaded to the
 * current device and share the value rate, the options (BGTQ_LAYOUT_*) and the seed (the
 * value rotation); BGTQ_ERR_INVALID otherwise. The set refers to the layouts' device
 * constants: destroy it before any of its layouts. */
typedef struct bgtq_layout_set bgtq_layout_set;
bgtq_status bgtq_layout_set_create(const bgtq_layout* const* layouts, int h_kv, bgtq_layout_set** out);
void bgtq_layout_set_destroy(bgtq_layout_set* set);
/* Bytes of one tile of every head in the set's cache: the largest tile of its layouts (a
 * head with a smaller tile leaves the rest of each tile unused). 0 for a null set. */
int bgtq_layout_set_tile_bytes(const bgtq_layout_set* set);
/* Bytes of a contiguous cache [batch][h_kv][capacity/64][tile] of the set (0 on bad
 * arguments: capacity must be a positive multiple of 64). */
size_t bgtq_layout_set_cache_bytes(const bgtq_layout_set* set, int batch, long long capacity);
/* bgtq_encode_append with KV head h coded by layout h of the set: k, v [batch, n_new,
 * h_kv, 128], h_kv = the set's size, cache of bgtq_layout_set_cache_bytes. Arguments,
 * ownership and errors otherwise as bgtq_encode_append; status bits go to the set
 * (bgtq_layout_set_status). */
bgtq_status bgtq_encode_append_heads(const bgtq_layout_set* set, const void* k, const void* v, int dtype,
                                     int batch, int n_new, const int* seq_lens_dev, void* cache,
                                     long long capacity, void* stream);
/* bgtq_decode_attention over a cache written by bgtq_encode_append_heads: one call for
 * every KV head (h_kv = the set's size; h_q a multiple of it). Workspace:
 * bgtq_workspace_bytes(any layout of the set, batch, h_q, h_kv, max_seq_len). Arguments,
 * ownership and errors otherwise as bgtq_decode_attention. */
bgtq_status bgtq_decode_attention_heads(const bgtq_layout_set* set, const void* q, int q_dtype, int batch,
                                        int h_q, const void* cache, const int* seq_lens_dev,
                                        long long capacity, long long max_seq_len, float softmax_scale,
                                        float* out, void* workspace, size_t workspace_bytes, void* stream);
/* bgtq_decode_attention_multi over a cache written by bgtq_encode_append_heads (n_q query
 * tokens per row, causal among them; h_kv = the set's size; workspace as
 * bgtq_decode_attention_multi). */
bgtq_status bgtq_decode_attention_multi_heads(const bgtq_layout_set* set, const void* q, int q_dtype,
                                              int batch, int n_q, int h_q, const void* cache,
                                              const int* seq_lens_dev, long long capacity,
                                              long long max_seq_len, float softmax_scale, float* out,
                                              void* workspace, size_t workspace_bytes, void* stream);
/* bgtq_decode_scores over a cache written by bgtq_encode_append_heads (h_kv = the set's
 * size). */
bgtq_status bgtq_decode_scores_heads(const bgtq_layout_set* set, const void* q, int q_dtype, int batch,
                                     int h_q, const void* cache, const int* seq_lens_dev, long long capacity,
                                     long long max_seq_len, float softmax_scale, float* scores,
                                     long long scores_ld, void* workspace, size_t workspace_bytes,
                                     void* stream);
/* bgtq_decode_step over a cache written by bgtq_encode_append_heads: appends n_new tokens
 * per row (k_new, v_new [batch, n_new, h_kv, 128], every KV head coded with its own layout)
 * and attends the query over the grown cache, in one kernel chain (h_kv = the set's size).
 * Arguments, ownership and errors otherwise as bgtq_decode_step. */
bgtq_status bgtq_decode_step_heads(const bgtq_layout_set* set, const void* k_new, const void* v_new,
                                   int kv_dtype, int n_new, const void* q, int q_dtype, int batch, int h_q,
                                   void* cache, const int* seq_lens_dev, long long capacity,
                                   long long max_seq_len, float softmax_scale, float* out, void* workspace,
                                   size_t workspace_bytes, void* stream);
/* bgtq_decode_step_multi over a cache written by bgtq_encode_append_heads: appends n_new
 * >= 1 tokens per row and attends each new token's own queries (q [batch][n_new][h_q][128],
 * out likewise, causal among the new tokens) over the grown cache, every KV head with its
 * own layout (h_kv = the set's size). Workspace: bgtq_workspace_bytes(any layout of the
 * set, batch, h_q * n_new, h_kv, max_seq_len). Errors as bgtq_decode_step_multi. */
bgtq_status bgtq_decode_step_multi_heads(const bgtq_layout_set* set, const void* k_new, const void* v_new,
                                         int kv_dtype, int n_new, const void* q, int q_dtype, int batch,
                                         int h_q, void* cache, const int* seq_lens_dev, long long capacity,
                                         long long max_seq_len, float softmax_scale, float* out,
                                         void* workspace, size_t workspace_bytes, void* stream);
/* Paged caches of a layout set: a page holds the h_kv tiles of one 64-token span of one
 * row at the set's tile stride (-1 on bad arguments); the encode and attention calls take
 * the pool and block table as bgtq_encode_append_paged / bgtq_decode_attention_paged. */
long long bgtq_layout_set_paged_pool_bytes(const bgtq_layout_set* set, long long num_pages);
bgtq_status bgtq_encode_append_paged_heads(const bgtq_layout_set* set, const void* k, const void* v, int dtype,
                                           int batch, int n_new, const int* seq_lens_dev, void* pool,
                                           long long num_pages, const int* block_table_dev, long long max_pages,
                                           void* stream);
bgtq_status bgtq_decode_attention_paged_heads(const bgtq_layout_set* set, const void* q, int q_dtype,
                                              int batch, int h_q, const void* pool, long long num_pages,
                                              const int* block_table_dev, long long max_pages,
                                              const int* seq_lens_dev, long long max_seq_len,
                                              float softmax_scale, float* out, void* workspace,
                                              size_t workspace_bytes, void* stream);
/* bgtq_decode_step_heads over a paged cache of the set (pool and block table as
 * bgtq_decode_step_paged). */
bgtq_status bgtq_decode_step_paged_heads(const bgtq_layout_set* set, const void* k_new, const void* v_new,
                                         int kv_dtype, int n_new, const void* q, int q_dtype, int batch,
                                         int h_q, void* pool, long long num_pages, const int* block_table_dev,
                                         long long max_pages, const int* seq_lens_dev, long long max_seq_len,
                                         float softmax_scale, float* out, void* workspace,
                                         size_t workspace_bytes, void* stream);
/* The set's status bits (BGTQ_STATUS_*), as bgtq_device_status. */
bgtq_status bgtq_layout_set_status(const bgtq_layout_set* set, unsigned* flags, int clear);

/* ---------------------------------------------------------------- no-allocation variant */

/* The pages have no counterpart to this call: it is a library convenience.
 * bgtq_decode_attention without the workspace argument, for callers that cannot call
 * cudaMalloc (an inference server that gives all device memory to its own pool at
 * start-up, a plugin whose framework forbids allocation inside its execute callback,
 * a fixed and audited memory budget). The split-K scratch is one file-scope device array
 * of BGTQ_NOALLOC_SCRATCH_BYTES (8 MiB), held on every GPU that loads the library until
 * exit; shapes whose scratch would exceed it return BGTQ_ERR_WORKSPACE with a message.
 * Nothing is allocated. The first call on a device looks up the array's device address
 * (once per device, that device current): make it before any stream capture. All calls
 * share the array, so calls whose kernels overlap on the GPU race and give wrong
 * results; serialise them (one stream). Arguments and results as bgtq_decode_attention. */
#define BGTQ_NOALLOC_SCRATCH_BYTES (8u << 20)
bgtq_status bgtq_decode_attention_noalloc(const bgtq_layout* layout, const void* q, int q_dtype,
                                          int batch, int h_q, int h_kv, const void* cache,
                                          const int* seq_lens_dev, long long capacity,
                                          long long max_seq_len, float softmax_scale, float* out,
                                          void* stream);
/* BGTQ_NOALLOC_SCRATCH_BYTES, as compiled into the library. */
size_t bgtq_noalloc_scratch_capacity(void);

/* Reads (synchronously) the layout's device status bits; clears them if clear != 0. */
bgtq_status bgtq_device_status(const bgtq_layout* layout, unsigned* flags, int clear);

#ifdef __cplusplus
}
#endif
#endif /* BGTQ_H */
