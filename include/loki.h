/*
 * loki.h -- C ABI of the B200 (sm_100a) implementation of Loki decode-time
 * sparse attention ("Loki: Low-Rank Keys for Efficient Sparse Attention").
 *
 * What the method computes (NeurIPS 2024 poster page of the paper, TL;DR and
 * "Visual Insights" Figure 1 caption; briefgpt.xyz abstract page):
 *   offline : a PCA basis P of each KV head's keys, from calibration keys;
 *   append  : every key enters the KV-cache rotated, K~ = K P;
 *   decode  : per (batch, query head), q~ = q P; approximate scores on the
 *             first d principal components, s_j = q~[:d] . K~_j[:d]; keep the
 *             k tokens with the largest s_j; exact softmax attention over
 *             those k tokens with their full D-dimensional rotated keys
 *             (q~ . K~_j = q . K_j because P is orthonormal) and values.
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers owned by the caller. The
 *     library never allocates, frees or synchronises; work is enqueued on
 *     `stream`, a cudaStream_t passed as an opaque pointer (NULL = the legacy
 *     default stream). Calls are asynchronous: device-side failures surface
 *     at the caller's next synchronisation.
 *   - Layouts are dense row-major with the last dimension contiguous:
 *       q, out            [B, H_q, D]
 *       K~ cache, V cache [B, H_kv, S_max, D]  (rows [0, S) valid)
 *       P                 [H_kv, D, D] fp32, P[h][i][c] = entry i of
 *                         principal component c (eigenvalue-descending)
 *       selected_idx      [B, H_q, k] int32, ascending token index
 *     Query head h reads KV head h / (H_q / H_kv) (grouped-query attention).
 *   - dt is the element type of q, caches, new keys/values and out.
 *   - Device pointers must be 16-byte aligned; workspaces 256-byte aligned.
 *   - Arguments are checked on the host before anything is enqueued; on any
 *     error nothing is launched and a loki_status other than LOKI_OK is
 *     returned. loki_last_error() then describes the failing argument.
 *   - D must be 128 or 96, the head sizes the Loki pages name (others return
 *     LOKI_ERR_UNSUPPORTED), and H_q / H_kv must be at most 8.
 *     loki_decode_attention_fused takes D = 128 only.
 *   - Entry points are thread-safe; calls on one stream are ordered.
 */
#ifndef LOKI_H
#define LOKI_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LOKI_API __attribute__((visibility("default")))
#else
#define LOKI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum loki_status {
    LOKI_OK = 0,
    LOKI_ERR_INVALID_ARG = 1,         /* null pointer, bad size, misaligned pointer */
    LOKI_ERR_UNSUPPORTED = 2,         /* valid but not implemented (e.g. D = 64) */
    LOKI_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the *_workspace_size() figure */
    LOKI_ERR_CUDA = 4                 /* a CUDA runtime call or launch failed */
} loki_status;

typedef enum loki_dtype {
    LOKI_DTYPE_F32 = 0,
    LOKI_DTYPE_BF16 = 1
} loki_dtype;

/* Text for a status code (static storage). */
LOKI_API const char* loki_status_string(loki_status st);

/* Description of the last failure on the calling thread ("" if none). */
LOKI_API const char* loki_last_error(void);

/*
 * Kernel error word of the current device: 1 if a staged kernel's bounded
 * wait on an asynchronous copy gave up, 2 if a paged call met a block-table
 * entry outside the page pool (the results of the call are then invalid). Synchronous: copies 4 bytes from the device (waiting for prior
 * work); with reset != 0 the word is cleared afterwards.
 */
LOKI_API loki_status loki_device_error(int* code, int reset);

/* ------------------------------------------------------------------------ */
/* Offline calibration                                                      */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace loki_calibrate_pca needs. */
LOKI_API size_t loki_calibrate_workspace_size(int64_t N, int H_kv, int D);

/*
 * PCA of calibration keys, one basis per KV head. Poster page, "Visual
 * Insights" Figure 1 caption (offline PCA on calibration keys) and the
 * study.space summary (PCA reduces the key dimensionality).
 *   keys    [N, H_kv, D] of type dt, N >= 2
 *   P       out, [H_kv, D, D] fp32; column c = unit eigenvector of the
 *           centred covariance (divisor N - 1) with the c-th largest
 *           eigenvalue, sign chosen so its largest-magnitude entry (lowest
 *           index on a tie) is positive
 *   eigvals out, [H_kv, D] fp32 descending, or NULL
 * Covariance in fp64, eigen-decomposition by cyclic Jacobi in fp64.
 */
LOKI_API loki_status loki_calibrate_pca(const void* keys, loki_dtype dt, int64_t N, int H_kv, int D,
                               float* P, float* eigvals, void* ws, size_t ws_bytes,
                               void* stream);

/* ------------------------------------------------------------------------ */
/* KV-cache append                                                          */
/* ------------------------------------------------------------------------ */

/*
 * Append T new tokens per (batch, KV head): K~ = K_new P (fp32 accumulate,
 * rounded to dt, nearest-even) into K~ cache rows [pos, pos + T); V_new is
 * copied unchanged into the same rows of the V cache. The poster page's
 * "Loki's Computational Cost" section names this append as a step of every
 * decode iteration.
 *   K_new, V_new [B, H_kv, T, D] of type dt;  P [H_kv, D, D] fp32
 *   requires 0 <= pos and pos + T <= S_max
 */
LOKI_API loki_status loki_append_keys(const void* K_new, const void* V_new, const float* P,
                             void* Kt_cache, void* V_cache, int B, int H_kv, int T, int D,
                             int64_t S_max, int64_t pos, loki_dtype dt, void* stream);

/*
 * Same append, for caches that also keep a low-dimensional key plane:
 *   Kt_lo [B, H_kv, S_max, d_lo] (dt) receives the first d_lo rotated columns
 *   of each new key (a copy of K~[..., :d_lo]); d_lo * sizeof(dt) must be a
 *   multiple of 16 bytes. The plane lets the score scan read d_lo contiguous
 *   columns per token instead of d_lo columns out of every D-column row (a
 *   memory-layout choice of this library; the method itself is unchanged).
 */
LOKI_API loki_status loki_append_keys_plane(const void* K_new, const void* V_new, const float* P,
                                            void* Kt_cache, void* V_cache, void* Kt_lo, int d_lo,
                                            int B, int H_kv, int T, int D, int64_t S_max,
                                            int64_t pos, loki_dtype dt, void* stream);

/* ------------------------------------------------------------------------ */
/* Decode attention (the per-step hot path)                                 */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace loki_decode_attention needs (q~, scores, partials). */
LOKI_API size_t loki_decode_workspace_size(int B, int H_q, int H_kv, int64_t S, int D, int d, int64_t k);

/*
 * One Loki decode step over a cache holding S valid tokens (poster TL;DR and
 * Figure 1 caption; briefgpt.xyz abstract page).
 *   q [B, H_q, D] (dt); Kt_cache, V_cache [B, H_kv, S_max, D] (dt); P fp32
 *   1 <= d <= D, 1 <= k <= S <= S_max, S < 2^31
 *   scale   softmax scale of the final scores; <= 0 selects 1/sqrt(D)
 *   out     [B, H_q, D] (dt): softmax over the k selected tokens only
 *   selected_idx [B, H_q, k] int32: the k tokens with the largest
 *           low-dimensional score, ties to the lower index, ascending
 * Arithmetic: fp32 (q~, scores, softmax, accumulation) on dt inputs. When
 * d >= D / 2 (and d * sizeof(dt) is a multiple of 16 bytes), each selected
 * token's full-D score is its low-dimensional score (already computed for
 * the selection) plus the product over columns [d, D), so the gather reads
 * only those columns of its key row.
 */
LOKI_API loki_status loki_decode_attention(const void* q, const void* Kt_cache, const void* V_cache,
                                  const float* P, int B, int H_q, int H_kv, int64_t S,
                                  int64_t S_max, int D, int d, int64_t k, float scale,
                                  loki_dtype dt, void* out, int32_t* selected_idx, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * loki_decode_attention over a cache that also holds a low-dimensional key
 * plane Kt_lo [B, H_kv, S_max, d_lo] (filled by loki_append_keys_plane):
 * identical results; the score scan reads the plane. Requires d <= d_lo.
 * Same workspace size as loki_decode_attention.
 */
LOKI_API loki_status loki_decode_attention_plane(const void* q, const void* Kt_cache,
                                                 const void* V_cache, const void* Kt_lo, int d_lo,
                                                 const float* P, int B, int H_q, int H_kv,
                                                 int64_t S, int64_t S_max, int D, int d, int64_t k,
                                                 float scale, loki_dtype dt, void* out,
                                                 int32_t* selected_idx, void* ws, size_t ws_bytes,
                                                 void* stream);

/*
 * One decode step that first appends the step's new tokens: the poster page's
 * "Loki's Computational Cost" section names the per-step KV-cache append as a
 * limiting cost, so here it is folded into the step's first kernel instead of
 * running as a launch of its own.
 *   K_new, V_new [B, H_kv, T, D] (dt): the T new tokens of every (batch, KV
 *           head); their rotated keys K~ = K_new P (fp32 accumulate, rounded
 *           to dt, exactly as loki_append_keys) go to cache rows [pos, pos + T)
 *           of Kt_cache (and of the plane Kt_lo when it is not NULL: d_lo
 *           columns, as loki_append_keys_plane), their values to V_cache.
 *   Then the decode over S = pos + T cached tokens, as loki_decode_attention
 *   (Kt_lo == NULL) or loki_decode_attention_plane: same arguments, same
 *   results, same workspace size (loki_decode_workspace_size with S).
 * The query rotation and the key rotation run in one kernel; the score scan
 * starts streaming rows [0, pos) at once and waits for that kernel only
 * before reading the new rows. With a key plane and few (batch, KV head)
 * units (where loki_decode_attention_plane runs as one kernel) the step runs
 * the append's rotation and then that single decode kernel behind it.
 *   requires 1 <= T, 0 <= pos, pos + T <= S_max, 1 <= k <= pos + T
 */
LOKI_API loki_status loki_decode_step(const void* q, const void* K_new, const void* V_new,
                                      const float* P, void* Kt_cache, void* V_cache, void* Kt_lo,
                                      int d_lo, int B, int H_q, int H_kv, int T, int64_t pos,
                                      int64_t S_max, int D, int d, int64_t k, float scale,
                                      loki_dtype dt, void* out, int32_t* selected_idx, void* ws,
                                      size_t ws_bytes, void* stream);

/*
 * The same decode step as loki_decode_attention_plane in a single kernel:
 * one thread block per (batch, KV head) unit rotates the unit's queries,
 * scans its key plane, keeps the scores in on-chip shared memory, selects the
 * top k per query head and runs the sparse attention, so the scores and the
 * selection never make a round trip through device memory. No workspace.
 * Identical results (same selection rule, fp32 arithmetic). Limits:
 * D = 128; H_q / H_kv in {1, 2, 4, 8}; S <= 8192; d_lo * sizeof(dt) in
 * {16, 32, 64, 128} bytes; the unit's keys and selection must fit in shared
 * memory. Shapes outside them return LOKI_ERR_UNSUPPORTED before any launch;
 * other argument errors as loki_decode_attention_plane.
 */
LOKI_API loki_status loki_decode_attention_fused(const void* q, const void* Kt_cache,
                                                 const void* V_cache, const void* Kt_lo, int d_lo,
                                                 const float* P, int B, int H_q, int H_kv,
                                                 int64_t S, int64_t S_max, int D, int d, int64_t k,
                                                 float scale, loki_dtype dt, void* out,
                                                 int32_t* selected_idx, void* stream);

/*
 * loki_decode_attention without a workspace argument, for callers that cannot
 * allocate device memory (a plugin inside a framework that owns all device
 * allocations, a thread that must not call cudaMalloc/cudaFree because they
 * can synchronise the device). The paper has no counterpart: this is a
 * memory-management convenience of this library. Scratch comes from a
 * 32 MiB array built into the library (held on every GPU that loads it until
 * the process exits); a decode that needs more (loki_decode_workspace_size)
 * returns LOKI_ERR_UNSUPPORTED without launching anything. All calls share
 * the array, so calls that overlap on the GPU race. The first call on each
 * device looks up the array's address; make it before any stream capture.
 * Other arguments and results are those of loki_decode_attention.
 */
LOKI_API loki_status loki_decode_attention_noalloc(const void* q, const void* Kt_cache,
                                                   const void* V_cache, const float* P, int B,
                                                   int H_q, int H_kv, int64_t S, int64_t S_max,
                                                   int D, int d, int64_t k, float scale,
                                                   loki_dtype dt, void* out, int32_t* selected_idx,
                                                   void* stream);

/* Ragged batches over a paged KV-cache ------------------------------------- */
/*
 * The Loki pages evaluate one prompt length at a time and say nothing about
 * batches of sequences with their own lengths or about cache memory layout;
 * these entry points carry the same decode step (and append) to the paged
 * layout of serving engines. Every sequence b keeps its own length S_b, and
 * the selection keeps min(k, S_b) tokens (the plainest reading when a
 * sequence holds fewer than k).
 *
 * Page pool layout (all dt, 16-byte aligned, caller-owned):
 *   Kt_pages, V_pages  [n_pages, H_kv, page_size, D]    rotated keys, values
 *   Kt_lo_pages        [n_pages, H_kv, page_size, d_lo] low-dimensional key plane
 *   block_table        [B, max_pages] int32: sequence b's token j lives in page
 *                      block_table[b][j / page_size], row j % page_size
 * A contiguous cache [B, H_kv, S_max, D] is the case page_size = S_max,
 * max_pages = 1, block_table[b][0] = b. Limits: page_size * max_pages <=
 * 262144 tokens per sequence; n_pages * H_kv * page_size < 2^31 rows. Page
 * numbers outside [0, n_pages) are not followed: the token is skipped (the
 * decode) or not written (the append), and loki_device_error then reports 2.
 */

/* Bytes of workspace loki_decode_attention_paged needs. */
LOKI_API size_t loki_paged_decode_workspace_size(int B, int H_q, int H_kv, int page_size,
                                                 int max_pages, int D, int d, int64_t k);

/*
 * One decode step per sequence over its own S_b = seq_lens[b] cached tokens
 * (device array, int32; values are clamped to [0, page_size * max_pages]; a
 * sequence with S_b = 0 gives zeros and no selection). Otherwise as
 * loki_decode_attention_plane: same selection rule and arithmetic, over the
 * token indices j < S_b of each sequence.
 *   out          [B, H_q, D] (dt)
 *   selected_idx [B, H_q, k] int32: the min(k, S_b) selected token indices
 *                ascending, then -1
 * The scan reads the plane pages (d <= d_lo; plane rows of 16, 32, 64 or 128
 * bytes with (H_q / H_kv) * d_lo <= 64 elements), the attention the key and
 * value pages.
 */
LOKI_API loki_status loki_decode_attention_paged(const void* q, const void* Kt_pages,
                                                 const void* V_pages, const void* Kt_lo_pages,
                                                 int d_lo, const float* P,
                                                 const int32_t* block_table,
                                                 const int32_t* seq_lens, int B, int H_q, int H_kv,
                                                 int page_size, int max_pages, int64_t n_pages,
                                                 int D, int d, int64_t k, float scale,
                                                 loki_dtype dt, void* out, int32_t* selected_idx,
                                                 void* ws, size_t ws_bytes, void* stream);

/*
 * loki_append_keys into the page pool: the T new tokens of sequence b become
 * its tokens positions[b] + t (positions: device array, int32), their rotated
 * keys (and plane rows when Kt_lo_pages is not NULL) and values written into
 * the pages block_table names. Same arithmetic as loki_append_keys.
 *   K_new, V_new [B, H_kv, T, D] (dt)
 */
LOKI_API loki_status loki_append_keys_paged(const void* K_new, const void* V_new, const float* P,
                                            void* Kt_pages, void* V_pages, void* Kt_lo_pages,
                                            int d_lo, const int32_t* block_table,
                                            const int32_t* positions, int B, int H_kv, int T,
                                            int page_size, int max_pages, int64_t n_pages, int D,
                                            loki_dtype dt, void* stream);

/* Steps of loki_decode_attention, callable one by one ------------------- */

/* q_rot [B, H_q, D] fp32 = q P (query rotated into its KV head's basis). */
LOKI_API loki_status loki_project_query(const void* q, const float* P, int B, int H_q, int H_kv, int D,
                               loki_dtype dt, float* q_rot, void* stream);

/*
 * scores [B, H_q, S] fp32: s_j = sum_{i<d} q_rot[i] K~_j[i] for j < S. Only
 * the first d columns of each cached key are read; each KV head's rows are
 * read once for all of its query heads. Kt_cache rows hold D elements: the
 * rotated cache of heads of D = 128 or 96 (q_rot is then [B, H_q, D]), or a
 * low-dimensional key plane of 128-wide heads (any other D = d_lo, with
 * D * sizeof(dt) a multiple of 16 bytes; q_rot is [B, H_q, 128]); 1 <= d <= D.
 */
LOKI_API loki_status loki_score_lowdim(const float* q_rot, const void* Kt_cache, int B, int H_q, int H_kv,
                              int64_t S, int64_t S_max, int D, int d, loki_dtype dt,
                              float* scores, void* stream);

/* Bytes of workspace loki_topk needs (currently 0; reserved). */
LOKI_API size_t loki_topk_workspace_size(int64_t rows, int64_t S, int64_t k);

/*
 * Per row of `scores` [rows, S] fp32: the k indices of the largest values,
 * ties to the lower index, written ascending to selected_idx [rows, k].
 * -0.0 equals +0.0; NaN ranks below every number. 1 <= k <= S.
 */
LOKI_API loki_status loki_topk(const float* scores, int64_t rows, int64_t S, int64_t k,
                      int32_t* selected_idx, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace loki_sparse_attention needs (split-k partials). */
LOKI_API size_t loki_sparse_attention_workspace_size(int B, int H_q, int64_t k, int D);

/*
 * Exact attention over the selected tokens: a_j = scale q_rot . K~_j over all
 * D dimensions for j in selected_idx[b, h, :], softmax over those k, out =
 * sum p_j V_j. Indices outside [0, S) are skipped (they contribute nothing);
 * a row whose indices are all out of range yields zeros.
 */
LOKI_API loki_status loki_sparse_attention(const float* q_rot, const void* Kt_cache, const void* V_cache,
                                  const int32_t* selected_idx, int B, int H_q, int H_kv,
                                  int64_t S, int64_t S_max, int D, int64_t k, float scale,
                                  loki_dtype dt, void* out, void* ws, size_t ws_bytes,
                                  void* stream);

/* PCAAttn ------------------------------------------------------------------ */

/* Bytes of workspace loki_pca_attention needs (q~ and split-S partials). */
LOKI_API size_t loki_pca_attention_workspace_size(int B, int H_q, int H_kv, int64_t S, int D);

/*
 * PCAAttn, the variant of Loki the poster page evaluates in its "More on
 * tables" PCAAttn table: the softmax is taken directly over the
 * reduced-dimensional scores of all S cached tokens, with no top-k and no
 * full-dimensional rescoring:
 *   s_j = q~[:d] . K~_j[:d] (q~ = q P), p = softmax(scale * s) over j < S,
 *   out = sum_j p_j V_j.
 * The keys are read from the low-dimensional key plane Kt_lo [B, H_kv, S_max,
 * d_lo] (plane rows of 16, 32, 64 or 128 bytes, d <= d_lo), the values in
 * full. scale <= 0 selects 1/sqrt(D) (the reading: the same scale as the full
 * scores). Arithmetic: fp32.
 */
LOKI_API loki_status loki_pca_attention(const void* q, const void* Kt_lo, int d_lo,
                                        const void* V_cache, const float* P, int B, int H_q,
                                        int H_kv, int64_t S, int64_t S_max, int D, int d,
                                        float scale, loki_dtype dt, void* out, void* ws,
                                        size_t ws_bytes, void* stream);

/* Pre-rotary PCA ------------------------------------------------------------ */

/*
 * The pre-rotary variant the poster page compares with the post-rotary one
 * ("More on figures": the perplexity figure with pre- and post-rotary PCA
 * transforms, and the rank figure over pre- and post-rotary keys). The pages
 * give no mechanism; the reading taken here: the basis P is calibrated on
 * keys before the rotary position embedding, the token scores and the top-k
 * use the pre-rotary query and keys in that basis, and the exact attention
 * over the selected tokens uses the post-rotary query and keys, as the model
 * would without Loki:
 *   q~ = q_pre P, s_j = q~[:d] . K~pre_j[:d], I = top-k of s (ties to the
 *   lower index, ascending), a_j = scale q_post . K_j for j in I,
 *   out = softmax(a) V_I.
 * The caches: Kt_lo [B, H_kv, S_max, d_lo] holds the first d_lo columns of
 * the pre-rotary keys rotated by P (K_pre P, rounded once to dt); K_cache
 * [B, H_kv, S_max, D] holds the post-rotary keys as the model makes them (in
 * no PCA basis); V_cache the values. q_pre, q_post [B, H_q, D] of type dt.
 * Workspace: loki_decode_prerotary_workspace_size bytes. Other arguments,
 * limits and errors as loki_decode_attention_plane.
 */
LOKI_API size_t loki_decode_prerotary_workspace_size(int B, int H_q, int H_kv, int64_t S, int D,
                                                     int d, int64_t k);
LOKI_API loki_status loki_decode_attention_prerotary(
    const void* q_pre, const void* q_post, const void* K_cache, const void* V_cache,
    const void* Kt_lo, int d_lo, const float* P, int B, int H_q, int H_kv, int64_t S,
    int64_t S_max, int D, int d, int64_t k, float scale, loki_dtype dt, void* out,
    int32_t* selected_idx, void* ws, size_t ws_bytes, void* stream);

/*
 * The append of the pre-rotary variant: T new tokens per (batch, KV head) at
 * rows [pos, pos + T). The plane Kt_lo receives the first d_lo columns of
 * K_new_pre P (pre-rotary keys [B, H_kv, T, D], rounded once to dt); K_cache
 * receives K_new_post (the post-rotary keys) and V_cache V_new unchanged.
 * Two kernels on `stream`; errors as loki_append_keys_plane.
 */
LOKI_API loki_status loki_append_keys_prerotary(const void* K_new_pre, const void* K_new_post,
                                                const void* V_new, const float* P, void* K_cache,
                                                void* V_cache, void* Kt_lo, int d_lo, int B,
                                                int H_kv, int T, int D, int64_t S_max, int64_t pos,
                                                loki_dtype dt, void* stream);

/* ------------------------------------------------------------------------ */
/* Dense baseline                                                           */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace dense_decode_attention needs (split-S partials). */
LOKI_API size_t dense_decode_workspace_size(int B, int H_q, int H_kv, int64_t S, int D);

/*
 * Full decode attention over all S cached tokens, the baseline Loki is
 * compared with (poster page, "More on tables": full attention rows;
 * per-layer attention time figure under "More on figures"). q and K may be
 * both rotated or both unrotated: the scores are the same.
 *   q [B, H_q, D]; K_cache, V_cache [B, H_kv, S_max, D]; out [B, H_q, D]
 */
LOKI_API loki_status dense_decode_attention(const void* q, const void* K_cache, const void* V_cache,
                                   int B, int H_q, int H_kv, int64_t S, int64_t S_max, int D,
                                   float scale, loki_dtype dt, void* out, void* ws,
                                   size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LOKI_H */
