/*
 * misa.h -- C ABI of the MISA indexer library (libmisa.so, CUDA, sm_100a).
 *
 * The method is the one on "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
 * Inference" (gist.science/paper/2605.07363), "Technical Summary":
 *   - "Methodology: MISA", "Lightweight Block-Pooled Router": the prefix is cut into
 *     M = ceil(L/B) blocks of B keys, every block is summarised by the mean of its index keys,
 *     every indexer head gets one affinity aggregated over those pooled keys, and the h best of
 *     the H_I heads are routed;
 *   - "Methodology: MISA", "Sparse Token Scoring": only the routed heads score every prefix
 *     token and the top-k tokens by that reduced score are kept;
 *   - "Hierarchical Variant (MISA-dagger)": the routed pass keeps k' > k candidates that the
 *     dense indexer with all H_I heads re-scores, keeping the top-k;
 *   - "Problem Statement": the dense DSA indexer scores every prefix token with all H_I heads.
 * The pages do not write the formulas.  This library computes, for query t with prefix n_t:
 *   kbar_b  = mean of keys [bB, min((b+1)B, n_t))             (b < M_t = ceil(n_t/B))
 *   r_{t,j} = w_{t,j} * sum_{b < M_t} max(0, q_{t,j} . kbar_b)     (router score of head j)
 *   R_t     = the h heads with the largest r_{t,j}                 (ties to the lower head)
 *   I_{t,s} = sum_{j in R_t} w_{t,j} * max(0, q_{t,j} . k_s)       (s < n_t)
 *   F_{t,s} = sum_{j < H_I}  w_{t,j} * max(0, q_{t,j} . k_s)       (dense score)
 * No scale factor is applied.  Selections order by score descending; exact ties go to the lower
 * token index.  Scores are accumulated in fp32 (bf16 products are exact in fp32).
 *
 * Common conventions
 *   - Every pointer argument is device memory owned by the caller unless stated otherwise.
 *     Nothing is allocated inside the library; scratch comes from the caller's workspace
 *     (size from misa_workspace_bytes), which must be 256-byte aligned.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *     Arguments are validated on the host before any launch; on error nothing is launched.
 *   - Layouts are dense row-major.  q is [T, H_I, d], w is [T, H_I] (fp32), n is [T] (int32).
 *     The key cache of query t starts at k + t * k_seq_stride elements: k_seq_stride = 0 makes
 *     all queries share one cache (prefill), k_seq_stride = L*d gives one cache per query
 *     (batched decode).  Each cache holds L keys of d elements.
 *   - dtype is the element type of q and k (MISA_BF16 or MISA_F32).  d must be 128.
 *     H_I must be a multiple of 8 in [8, 128]; 1 <= h <= H_I.
 *   - Prefix lengths n_t are read on the device: values above L count as L, values below 1 give
 *     an empty prefix (no tokens selected; all router scores 0).
 *   - Index outputs hold min(topk, n_t) token indices followed by -1 padding.  The selected set
 *     is what the method defines (and identical from run to run); the order of the indices
 *     inside a row is not specified.
 *   - Errors: MISA_ERR_INVALID_ARG (null pointer, size out of range), MISA_ERR_UNSUPPORTED
 *     (d != 128, H_I not a multiple of 8, dtype, k' too large), MISA_ERR_WORKSPACE (workspace
 *     too small or misaligned), MISA_ERR_CUDA (a launch failed; cudaGetLastError's code is
 *     consumed).  Errors that arise on the device after a launch are reported by
 *     misa_device_check.
 */
#ifndef MISA_H_
#define MISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MISA_OK = 0,
  MISA_ERR_INVALID_ARG = 1,
  MISA_ERR_UNSUPPORTED = 2,
  MISA_ERR_WORKSPACE = 3,
  MISA_ERR_CUDA = 4,
  MISA_ERR_DEVICE_TIMEOUT = 5,
  MISA_ERR_BAD_INDEX = 6
} misa_status;

typedef enum { MISA_BF16 = 0, MISA_F32 = 1 } misa_dtype;

/* Operation codes for misa_workspace_bytes. */
typedef enum {
  MISA_OP_ROUTE = 0,
  MISA_OP_SCORE_TOPK = 1,
  MISA_OP_RERANK = 2,
  MISA_OP_DENSE_TOPK = 3,
  MISA_OP_TOPK_SELECT = 4,
  MISA_OP_BLOCK_FILTER = 5,
  MISA_OP_ROUTE_PAGED = 6,
  MISA_OP_SCORE_TOPK_PAGED = 7,
  MISA_OP_RERANK_PAGED = 8,
  MISA_OP_SCORE_TOPK_FUSED = 9,
  MISA_OP_HIER_FUSED = 10
} misa_op;

/* Largest k' accepted by misa_hier_rerank (its candidates are ranked in shared memory). */
#define MISA_MAX_KP 16384

/* Library version, major*10000 + minor*100 + patch. */
int misa_version(void);

/* Static text for a status code. */
const char* misa_status_str(int status);

/*
 * Workspace bytes needed by one call of `op` with these sizes (0 if it needs none).
 * Arguments an op does not use are ignored.  Sizes <= 0 give 0.  For MISA_OP_BLOCK_FILTER the
 * last argument carries m, the number of kept blocks (0 when m * B exceeds MISA_MAX_KP).
 */
size_t misa_workspace_bytes(int op, int T, int L, int H_I, int B, int h, int topk, int kp);

/*
 * Block mean-pool of key caches ("Lightweight Block-Pooled Router": mean-pooled indexing keys
 * over M = ceil(L/B) blocks).
 *   k      : n_seq caches of L keys [L, d] at stride k_seq_stride elements (dtype)
 *   kbar   : out, fp32, n_seq x [ceil(L/B), d] at stride kbar_seq_stride floats
 *   blocks [block_begin, block_end) of every cache are written (clamped to [0, ceil(L/B)));
 *   block b averages keys [bB, min((b+1)B, L)) (a partial last block over its valid keys).
 * The router and the block filter average the last block of every prefix from the keys
 * themselves, so a decode loop calls this with [b, b+1) once its prefix has moved past block b
 * (once every B steps), not for the block that holds the newest key.
 */
misa_status misa_pool_keys(const void* k, int64_t k_seq_stride, int n_seq, int L, int d, int B,
                           int dtype, float* kbar, int64_t kbar_seq_stride, int block_begin,
                           int block_end, void* stream);

/*
 * Block-pooled router and top-h head selection ("Lightweight Block-Pooled Router").
 *   kbar   : fp32 block means from misa_pool_keys; query t reads kbar + t*kbar_seq_stride
 *            (0 = shared).  Only blocks b < M_t - 1 are read from it; the last block of a prefix,
 *            keys [(M_t - 1) B, n_t) (full or partial), is averaged from k directly, so it may
 *            hold the newest keys without being pooled.
 *   heads  : out [T, h] int32, routed heads in descending router score (ties: lower head)
 *   r_opt  : out [T, H_I] fp32 router scores, or NULL
 *   ws     : workspace of misa_workspace_bytes(MISA_OP_ROUTE, T, L, H_I, B, h, 0, 0) bytes
 */
misa_status misa_route(const void* q, const float* w, const void* k, int64_t k_seq_stride,
                       const float* kbar, int64_t kbar_seq_stride, const int32_t* n, int T, int L,
                       int H_I, int d, int B, int h, int dtype, int32_t* heads, float* r_opt,
                       void* ws, size_t ws_bytes, void* stream);

/*
 * Routed-head token scores ("Sparse Token Scoring"): scores[t, s] = I_{t,s} for s < n_t.
 *   heads    : [T, h] routed heads (any order; NULL = all H_I heads, i.e. the dense score F)
 *   scores   : out fp32 [T, ld_scores], ld_scores >= L; entries s >= n_t are not written.
 *   select_ws, select_ws_bytes, select_topk : optional (NULL, 0, 0).  A workspace of
 *              misa_workspace_bytes(MISA_OP_TOPK_SELECT, T, L, ...) bytes in which the call also
 *              prepares a top-select_topk selection of these scores; pass the same workspace to
 *              misa_topk_select with ws_prepared = 1.  For fewer than 256 rows longer than
 *              16384 entries it builds a candidate list per query right after the scores: one
 *              CTA per row places the row's cut from a sample of its scores (256 evenly spaced
 *              runs of 8; the rank of the expected count above the select_topk-th score plus
 *              three standard deviations), then CTAs over chunks of 8192 scores append every
 *              score at or above it.  The selection ranks those entries and takes an exact pass
 *              over the score row whenever they cannot hold the answer (fewer than select_topk,
 *              or the list overflowed), so the result never depends on where the cut fell.
 *              Shorter rows, many rows and rows whose lists would not fit get no list and are
 *              selected from the scores.
 */
misa_status misa_token_scores(const void* q, const float* w, const void* k, int64_t k_seq_stride,
                              const int32_t* n, const int32_t* heads, int T, int L, int H_I, int d,
                              int h, int dtype, float* scores, int64_t ld_scores, int select_topk,
                              void* select_ws, size_t select_ws_bytes, void* stream);

/*
 * Top-k selection over per-query score rows ("Sparse Token Scoring": the final top-k tokens
 * are selected on the reduced scores).  scores [T, ld_scores] fp32, entries s < n_t are read.
 *   idx         : out [T, topk] int32, -1 padded
 *   score_opt   : out [T, topk] fp32 score of each selected token (0 for padding), or NULL
 *   ws          : misa_workspace_bytes(MISA_OP_TOPK_SELECT, T, L, ...) bytes
 *   ws_prepared : 1 if misa_token_scores already prepared ws for these scores and this topk
 * Scores must be finite.  Without ws_prepared the call first builds the candidate lists of long
 * rows itself (as misa_token_scores does); then one CTA per row selects, from its list or, for rows
 * without one, from a sampled cut and a pass over the row.  Both give the same set.
 */
misa_status misa_topk_select(const float* scores, int64_t ld_scores, const int32_t* n, int T,
                             int L, int topk, int32_t* idx, float* score_opt, void* ws,
                             size_t ws_bytes, int ws_prepared, void* stream);

/*
 * Routed scoring followed by top-k: misa_token_scores (preparing the selection) then
 * misa_topk_select.  With topk = k' this is the coarse stage of MISA-dagger ("Hierarchical
 * Variant": enlarged candidate set).
 *   scores_full_opt : [T, L] fp32 buffer that receives every score, or NULL (scores then live in
 *                     the workspace)
 *   ws : misa_workspace_bytes(MISA_OP_SCORE_TOPK, T, L, ...) bytes (with scores_full_opt given,
 *        misa_workspace_bytes(MISA_OP_TOPK_SELECT, T, L, ...) bytes suffice)
 */
misa_status misa_score_topk(const void* q, const float* w, const void* k, int64_t k_seq_stride,
                            const int32_t* n, const int32_t* heads, int T, int L, int H_I, int d,
                            int h, int topk, int dtype, int32_t* idx, float* score_opt,
                            float* scores_full_opt, void* ws, size_t ws_bytes, void* stream);

/*
 * MISA-dagger fine stage ("Hierarchical Variant (MISA-dagger)": the dense indexer with all H_I
 * heads re-scores only the k' candidates and keeps the final top-k).
 *   cand      : [T, kp] candidate token indices; entries < 0 or >= n_t are empty slots
 *   idx       : out [T, topk] the kept candidates, -1 padded
 *   score_opt : out [T, topk] their dense scores, or NULL
 *   ws        : misa_workspace_bytes(MISA_OP_RERANK, T, 0, H_I, 0, 0, topk, kp) bytes
 * Requires topk <= kp <= MISA_MAX_KP; duplicate candidates are the caller's error.
 */
misa_status misa_hier_rerank(const void* q, const float* w, const void* k, int64_t k_seq_stride,
                             const int32_t* n, const int32_t* cand, int T, int L, int H_I, int d,
                             int kp, int topk, int dtype, int32_t* idx, float* score_opt, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * Dense DSA indexer ("Problem Statement": every prefix token scored with all H_I heads, top-k
 * kept): top-k of F_{t,s} over s < n_t.  Outputs as misa_score_topk.
 *   ws : misa_workspace_bytes(MISA_OP_DENSE_TOPK, T, L, ...) bytes
 */
misa_status dsa_dense_topk(const void* q, const float* w, const void* k, int64_t k_seq_stride,
                           const int32_t* n, int T, int L, int H_I, int d, int topk, int dtype,
                           int32_t* idx, float* score_opt, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * Token-axis block filter composed with MISA ("HISA: Efficient Hierarchical Indexing for
 * Fine-Grained Sparse Attention", arXiv 2603.28458, abstract: a coarse stage scores pooled block
 * representatives and keeps candidate blocks, then the indexer scores only their tokens; "MISA",
 * "Problem Statement" and "Significance and Claims": token-axis and head-axis savings combine).
 * For query t with routed heads R_t (heads[t], from misa_route):
 *   S_{t,b} = sum_{j in R_t} w_{t,j} * max(0, q_{t,j} . kbar_b)     (b < M_t = ceil(n_t/B))
 * with kbar_b the router's block means (the last block, full or partial, averaged from k); the m
 * blocks with the largest S_{t,b} are kept (ties: lower block); their prefix tokens are scored
 * with I_{t,s} and the top-k of those is selected (ties: lower token).  m >= M_t gives exactly
 * misa_score_topk's selection; h = H_I gives the block filter on the dense indexer.
 *   kbar             : fp32 block means from misa_pool_keys, 16-byte aligned; query t reads
 *                      kbar + t*kbar_seq_stride (0 = shared; else a multiple of 4, >= M*d);
 *                      blocks b < M_t - 1 only, as misa_route
 *   heads            : [T, h] routed heads in [0, H_I) (other ids are never dereferenced, but
 *                      the results are then unspecified)
 *   m                : blocks kept per query, 1 <= m with m * B <= MISA_MAX_KP
 *   block_scores_opt : out [T, ld_block_scores] fp32 S_{t,b} for b < M_t (ld >= ceil(L/B)), or NULL
 *   blocks           : out [T, m] kept blocks, -1 padded (order unspecified)
 *   idx, score_opt   : out [T, topk] selected tokens (-1 padded when the kept blocks hold fewer
 *                      than topk prefix tokens) and their scores I, or NULL for score_opt
 *   ws               : misa_workspace_bytes(MISA_OP_BLOCK_FILTER, T, L, H_I, B, h, topk, m) bytes
 * Errors as above; m * B > MISA_MAX_KP gives MISA_ERR_UNSUPPORTED.
 */
misa_status misa_block_filter_topk(const void* q, const float* w, const void* k,
                                   int64_t k_seq_stride, const float* kbar,
                                   int64_t kbar_seq_stride, const int32_t* n,
                                   const int32_t* heads, int T, int L, int H_I, int d, int B, int h,
                                   int m, int topk, int dtype, float* block_scores_opt,
                                   int64_t ld_block_scores, int32_t* blocks, int32_t* idx,
                                   float* score_opt, void* ws, size_t ws_bytes, void* stream);

/*
 * Paged key caches.  Serving stores each sequence's keys in fixed-size pages of one pool shared by
 * all sequences (the pages call MISA a drop-in replacement for the DSA indexer, "Key
 * Contributions"; this is the layout such a replacement reads).  The *_paged calls compute exactly
 * what their contiguous counterparts compute on each sequence's logical cache:
 *   pool       : [num_pages, page_size, d] keys (dtype); num_pages * page_size < 2^31
 *   page_table : [T, max_pages] int32; logical key s of query t's sequence is row s % page_size of
 *                physical page page_table[t][s / page_size].  Entries for pages past a prefix are
 *                never read.  max_pages * page_size >= L (L: the longest prefix, as elsewhere).
 *   n          : [T] prefix lengths, as elsewhere.
 * A page id outside [0, num_pages) inside a prefix is never dereferenced: its keys read as zero
 * (pooling, router) or the token is left out of scoring; results are then unspecified.
 * kbar is one pooled cache per query ([T, ceil(L/B), d] at kbar_seq_stride >= ceil(L/B) * d), as
 * written by misa_pool_keys_paged.  Queries that share a sequence repeat its table row.
 */
/* misa_pool_keys through page tables (page_table rows are the n_seq sequences). */
misa_status misa_pool_keys_paged(const void* pool, int64_t num_pages, int page_size,
                                 const int32_t* page_table, int64_t max_pages, int n_seq, int L,
                                 int d, int B, int dtype, float* kbar, int64_t kbar_seq_stride,
                                 int block_begin, int block_end, void* stream);

/* misa_route on paged caches.
 *   ws : misa_workspace_bytes(MISA_OP_ROUTE_PAGED, T, L, H_I, B, h, 0, 0) bytes */
misa_status misa_route_paged(const void* q, const float* w, const void* pool, int64_t num_pages,
                             int page_size, const int32_t* page_table, int64_t max_pages,
                             const float* kbar, int64_t kbar_seq_stride, const int32_t* n, int T,
                             int L, int H_I, int d, int B, int h, int dtype, int32_t* heads,
                             float* r_opt, void* ws, size_t ws_bytes, void* stream);

/* misa_score_topk on paged caches (with topk = k', the MISA-dagger coarse stage).
 *   ws : misa_workspace_bytes(MISA_OP_SCORE_TOPK_PAGED, T, L, H_I, 0, h, topk, 0) bytes */
misa_status misa_score_topk_paged(const void* q, const float* w, const void* pool, int64_t num_pages,
                                  int page_size, const int32_t* page_table, int64_t max_pages,
                                  const int32_t* n, const int32_t* heads, int T, int L, int H_I,
                                  int d, int h, int topk, int dtype, int32_t* idx, float* score_opt,
                                  void* ws, size_t ws_bytes, void* stream);

/* misa_hier_rerank on paged caches.
 *   ws : misa_workspace_bytes(MISA_OP_RERANK_PAGED, T, 0, H_I, 0, 0, topk, kp) bytes */
misa_status misa_hier_rerank_paged(const void* q, const float* w, const void* pool, int64_t num_pages,
                                   int page_size, const int32_t* page_table, int64_t max_pages,
                                   const int32_t* n, const int32_t* cand, int T, int L, int H_I,
                                   int d, int kp, int topk, int dtype, int32_t* idx,
                                   float* score_opt, void* ws, size_t ws_bytes, void* stream);

/*
 * misa_score_topk for queries that share one bf16 key cache (chunked prefill), without writing
 * score rows ("Sparse Token Scoring": the top-k tokens by the routed score).  The tensor-core
 * scorer first scores every 32nd tile of 128 keys of each prefix; each query's cut is placed on that
 * sample (the expected number of sampled scores above the k-th, plus three standard deviations and
 * a margin); a second pass over every key appends only the scores at or above the cut to a list of
 * 4k entries per query, from which the top-k is selected.  A query whose list holds fewer than
 * min(k, n_t) entries or overflowed is redone exactly on the device by the unfused scorer and
 * selection, so the selected set is always misa_score_topk's.
 *   k  : one shared cache [L, d] (k_seq_stride 0), bf16 like q
 *   ws : misa_workspace_bytes(MISA_OP_SCORE_TOPK_FUSED, T, L, H_I, 0, h, topk, 0) bytes (it also
 *        holds score rows for the queries that are redone)
 * Requires 4 * topk <= 16384 (else MISA_ERR_UNSUPPORTED); other arguments and outputs as
 * misa_score_topk.
 */
misa_status misa_score_topk_fused(const void* q, const float* w, const void* k, const int32_t* n,
                                  const int32_t* heads, int T, int L, int H_I, int d, int h,
                                  int topk, int dtype, int32_t* idx, float* score_opt, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * MISA-dagger for decode batches with one key cache per query, without gathering the candidates
 * ("Hierarchical Variant (MISA-dagger)": the top-k' tokens by the routed score are re-scored with
 * all H_I heads and the top-k of that dense score is kept).  The result is misa_score_topk with
 * topk = k' followed by misa_hier_rerank on its candidates, up to the rounding of the dense scores
 * (a different summation on the tensor cores: near-ties at the k-th dense score may be ordered
 * differently).  For fewer than 256 queries longer than 16384 keys and h <= 8, the list cut's sample
 * of each prefix (256 evenly spaced runs of 8 keys) is scored first, each query's cut is placed on
 * it (the expected number of sampled scores above the k'-th, plus three standard deviations and a
 * margin), and one pass over the keys writes every routed score and keeps each token at or above
 * the cut with its dense score, computed from the key row the pass already holds; the top-k' of
 * those by the routed score and the top-k of them by the dense score are then selected.  A query
 * whose kept tokens are fewer than k' or overflow 16384 is answered exactly from its score row on
 * the device (the dense scores of its k' candidates computed there), so the selected set never
 * depends on the sample.  Other shapes take that exact way for every query.
 *   k         : per-query caches [T, L, d] (k_seq_stride >= L * d), bf16 like q
 *   heads     : [T, h] routed heads (misa_route)
 *   idx       : out [T, topk] the kept tokens (order not specified), -1 padded when n_t < topk
 *   score_opt : out [T, topk] their dense scores, or NULL
 *   ws        : misa_workspace_bytes(MISA_OP_HIER_FUSED, T, L, H_I, 0, h, topk, kp) bytes
 * Requires topk <= kp <= MISA_MAX_KP (else MISA_ERR_INVALID_ARG / MISA_ERR_UNSUPPORTED); a shared
 * cache (k_seq_stride 0) or fp32 inputs give MISA_ERR_UNSUPPORTED.
 */
misa_status misa_hier_topk_fused(const void* q, const float* w, const void* k, int64_t k_seq_stride,
                                 const int32_t* n, const int32_t* heads, int T, int L, int H_I, int d,
                                 int h, int kp, int topk, int dtype, int32_t* idx, float* score_opt,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * Device-side status of the calls made so far on the current device.  The tensor-core kernels
 * (scoring and routing queries that share one bf16 cache, and the re-rank of gathered candidates)
 * pipeline their copies and MMAs through shared-memory barriers; every wait on them is bounded
 * (about one second).  A wait that runs
 * out makes the kernel stop early, leaving its outputs incomplete, and records the event in a
 * per-device status word.  This call waits for all work on the device to finish
 * (cudaDeviceSynchronize), then reads and clears that word (and, in the bounds-checked build,
 * the counts of skipped out-of-range ids described below).
 *   returns MISA_OK, MISA_ERR_DEVICE_TIMEOUT (some call since the last check stopped early),
 *   MISA_ERR_BAD_INDEX (bounds-checked build: out-of-range ids were seen and skipped), or
 *   MISA_ERR_CUDA (the synchronisation or the read failed).
 */
misa_status misa_device_check(void);

/*
 * Bounds-checked build.  libmisa_checked.so (python -m long_context_sparse_mean_b200.build
 * --checked) is the same library compiled with MISA_CHECKED: every id that a kernel skips because
 * it lies outside its range is also counted on the device, by kind:
 *   out[0] routed head ids outside [0, H_I)            (scoring and block-filter calls)
 *   out[1] candidate token ids outside [0, n_t), other than the empty marker -1 (re-rank calls,
 *          paged or not; the header's "empty slot" rule still applies: they are skipped)
 *   out[2] page-table entries inside a prefix outside [0, num_pages) (paged calls; per key row
 *          read through the entry)
 * The counts are occurrences seen, not distinct ids.  In both builds such ids are never
 * dereferenced.  misa_device_check returns MISA_ERR_BAD_INDEX (after MISA_ERR_DEVICE_TIMEOUT,
 * which takes precedence) when any count is nonzero, and clears them.
 */
/* 1 for the bounds-checked build, 0 otherwise. */
int misa_checked_build(void);

/*
 * Waits for the device (cudaDeviceSynchronize), then writes the counts of skipped out-of-range
 * ids since the last read into out[3] (kinds as above; zeros in the normal build) and clears them.
 * Returns MISA_OK, MISA_ERR_INVALID_ARG (out is NULL) or MISA_ERR_CUDA.
 */
misa_status misa_bad_index_counts(unsigned int* out);

/*
 * Capacity, in floats, of the fixed scratch array used by misa_hier_rerank_static
 * (4 MiB per GPU that loads the library, held until the process exits).
 */
#define MISA_STATIC_RERANK_SCRATCH_FLOATS (1 << 20)

/*
 * misa_hier_rerank without a workspace argument, for callers that cannot allocate device
 * memory.  The pages have no counterpart to this call; it exists for the deployment side only.
 * Who needs it: a plugin that its host framework hands only input and output buffers (the
 * framework owns the device memory and offers the plugin no allocator), or a latency-critical
 * decode loop that must not risk an allocation failure, or the device synchronisation that
 * cudaMalloc / cudaFree can cause, in the middle of a step.
 * Same arguments, results and checks as misa_hier_rerank, minus ws and ws_bytes.  Its T * kp
 * floats of scratch live in one array compiled into the library (MISA_STATIC_RERANK_SCRATCH_FLOATS
 * floats per device); the call allocates nothing.
 *   - T * kp above MISA_STATIC_RERANK_SCRATCH_FLOATS: returns MISA_ERR_WORKSPACE, nothing launched.
 *   - All calls on a device share the array and it keeps the last call's contents; nothing in it
 *     needs to start at zero.  Calls that overlap on the GPU (unordered streams) race on it and
 *     give undefined results: order them on one stream or with events.
 *   - The first call on a device looks up the array's device address with that device current
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 */
misa_status misa_hier_rerank_static(const void* q, const float* w, const void* k,
                                    int64_t k_seq_stride, const int32_t* n, const int32_t* cand,
                                    int T, int L, int H_I, int d, int kp, int topk, int dtype,
                                    int32_t* idx, float* score_opt, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MISA_H_ */
