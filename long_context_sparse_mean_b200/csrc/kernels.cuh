// Internal launchers of the MISA indexer kernels (C++ linkage; the C ABI lives in capi.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "select.cuh"

namespace misa {

// Block mean-pool ("Lightweight Block-Pooled Router": mean-pooled index keys).
void launch_pool(DType dt, const void* k, int64_t k_seq_stride, int n_seq, int L, int B,
                 float* kbar, int64_t kbar_seq_stride, int b0, int b1, cudaStream_t s);

// Router: last-block means, per-chunk affinities, then sum, weight and top-h.
int route_chunks(int L, int B);  // chunks of kRouteTile blocks per query (upper bound)
// Blocks below kbar_blocks(n_t, B) are read from kbar, the last block of each prefix is averaged
// from the keys.  kbar_parts: [3][ceil(L/B)][128] bf16 scratch for the tensor-core router (shared
// cache).  pm_in: [T][128] means of each query's last block computed beforehand (paged caches), or
// nullptr to average them from k.
void launch_route(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                  const float* kbar, int64_t kbar_seq_stride, const int32_t* n, int T, int L,
                  int H_I, int B, int h, int32_t* heads, float* r_opt, float* pm, float* partial,
                  uint32_t* done, __nv_bfloat16* kbar_parts, const float* pm_in, cudaStream_t s);

// Router on the tensor cores for queries that share one bf16 cache and its pooled keys: per-tile
// sums over the blocks below kbar_blocks(n_t, B) into Sp [T][nch][H_I], then route_finish.  False (nothing launched) when
// the shapes do not suit it (H_I must divide 128).
constexpr int kRouteTcMinQueries = 64;
bool launch_route_tc(const void* q, const float* w, const void* k, const float* kbar, const int32_t* n, int T,
                     int L, int H_I, int B, int h, int32_t* heads, float* r_opt, __nv_bfloat16* kbar_parts,
                     float* Sp, int nch, cudaStream_t s);
void launch_kbar_split(const float* kbar, int M, __nv_bfloat16* parts, cudaStream_t s);
void launch_route_finish(const __nv_bfloat16* q, const float* w, const __nv_bfloat16* k, const int32_t* n, int T,
                         int L, int H_I, int B, int h, const float* Sp, int nch, int tile, int32_t* heads,
                         float* r_opt, cudaStream_t s);

// Candidate lists of a top-k over long score rows (select.cuh holds the sizes), built after the
// scores are written: list_cut_kernel places each row's cut from a sample of its scores (the row
// kernel's own sample and rank), list_sweep_kernel appends every entry at or above it with CTAs over
// chunks of 8192 scores; the per-row selection ranks the list's entries at or above the row's cut.
struct ListState {
  uint32_t* cnt;     // [T] entries appended (also past cap); kNoList: no list for this row
  uint32_t* cutkey;  // [T] the row's cut as an order key: every score at or above it is listed, and
                     // every list entry is at or above it (right after cnt)
  uint2* list;       // [T][stride] (order key, token); the first cap entries of a row are used
  int cap;
  int topk;
  // [T] n_t of a row the list could not answer (0 for the rows answered): the row is redone from
  // its scores (or, with no score rows behind the lists, by the caller)
  int32_t* redo = nullptr;
  int64_t stride = kListCap;
};
size_t list_state_bytes(int T, int cap = kListCap);
ListState list_state(void* ws, int T, int topk, int cap = kListCap);
// cnt = kNoList for every row (no lists).
void mark_no_lists(const ListState& l, int T, cudaStream_t s);
// Builds the candidate lists of score rows [T, ld] (entries s < min(n_t, L)) for fewer than 256
// rows longer than the list (per row: unless the sample cannot place the cut or the list is not
// expected to fit; those rows get kNoList): the cut from the row kernel's sample by one CTA per
// row, then list_sweep_kernel.  Otherwise marks every row as having none.  Returns whether the list
// kernels ran.  list_state gives rows of 256 or more queries a cap of 8192.
bool launch_list_build(const float* scores, int64_t ld, const int32_t* n, int T, int L, const ListState& l,
                       cudaStream_t s);
// One warp per row: the top-k of each row's list (exact, ties to the lower token); rows the list
// cannot answer get l.redo[t] = n_t and no output, the others l.redo[t] = 0.  hi (optional): per row
// the largest score of the sample that placed the cut, which bounds most of the list's entries
// and lets two passes over the list do (the general rounds otherwise).
void launch_list_select_warp(const int32_t* n, int T, int L, int topk, const ListState& l, int32_t* idx,
                             float* score_opt, cudaStream_t s, const float* hi = nullptr);

// MISA-dagger decode in one pass over the keys ("Hierarchical Variant (MISA-dagger)"), for one
// cache per query, h <= 8 and bf16: launch_scores_sample scores the list cut's sample of every row
// longer than the cap (kSampleRuns runs of kSampleRunLen tokens, into the score rows at those
// tokens), launch_list_cut places each row's cut on it (with topk = k'), launch_scores_dense_list
// writes every routed score and appends each token at or above the cut with its dense score over
// all H_I heads (computed from the key row the scorer already holds: nothing is gathered), and
// launch_hier_select takes per row the top-k' by the routed score, then the top-k of those by the
// dense score.
struct DenseList {
  uint2* list;          // [T][stride] (order key of the routed score, token)
  float* f;             // [T][stride] the dense score of the same token
  uint32_t* cnt;        // [T] entries appended (also past cap); kNoList: no list for this row
  const uint32_t* cut;  // [T] the row's cut as an order key
  int64_t stride;
  int cap;
};
constexpr size_t kDenseListMaxSmem = 110 * 1024;  // dynamic shared memory of the list scorer (2 CTAs per SM)
constexpr int kDenseListMaxRows = 255;            // lists pay off for a few rows (one CTA per row fills the GPU)
size_t dense_list_smem(int T, int H_I);
// False (nothing launched) unless h <= 8, per-query caches and T <= 8192.
bool launch_scores_sample(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n,
                          const int32_t* heads, int T, int L, int H_I, int h, int cap, float* out, int64_t ld,
                          cudaStream_t s);
// Rows whose cnt[t] is kNoList get their scores only.  False (nothing launched) as above, or when
// the shared memory would not fit.
bool launch_scores_dense_list(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n,
                              const int32_t* heads, int T, int L, int H_I, int h, float* out, int64_t ld,
                              const DenseList& dl, cudaStream_t s);
// The cut of list_cut_kernel alone (cnt[t] = 0 and cut[t], or cnt[t] = kNoList).
void launch_list_cut(const float* scores, int64_t ld, const int32_t* n, int T, int L, int topk, int cap,
                     uint32_t* lcnt, uint32_t* lcut, cudaStream_t s);
// One CTA per row (kp <= 16384): idx [T, topk] (score_opt: the dense scores) from the dense lists, or
// for a row they cannot answer, from its score row (exact top-k', dense scores of the candidates
// computed here).  ctok: [T][kp] scratch.
void launch_hier_select(const float* scores, int64_t ld, const int32_t* n, int T, int L, int kp, int topk,
                        const DenseList& dl, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                        int H_I, int32_t* ctok, int32_t* idx, float* score_opt, cudaStream_t s);

// Token scores with a head list (heads == nullptr: all H_I heads).  rows != nullptr gathers:
// position p of query t scores token rows[t*P + p] and writes out[t*ld + p].
void launch_scores(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                   const int32_t* n, const int32_t* heads, int T, int L, int H_I, int h,
                   const int32_t* rows, int P, float* out, int64_t ld, cudaStream_t s);

// Tensor-core scoring for queries sharing one bf16 key cache (k_seq_stride 0, no gather).  Returns
// false without launching when the inputs do not suit it (alignment, no TMA encoder).
bool launch_scores_tc(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads, int T,
                      int L, int H_I, int h, float* out, int64_t ld, cudaStream_t s);
// Dense scores of gathered candidates on the tensor cores (rerank_tc.cu): out[t, p] = F of token
// cand[t, p] (0 when outside [0, n_t)) for p < P, bf16 q and k.  False (nothing launched) when the
// inputs do not suit it (H_I a multiple of 16 in [16, 128], 16-byte aligned rows).
bool launch_rerank_tc(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n, int T,
                      int L, int H_I, const int32_t* cand, int P, float* out, int64_t ld, cudaStream_t s);
// Reads and clears the status word the tensor-core kernels set when a bounded wait runs out.
int read_and_clear_tc_status();
int read_and_clear_route_tc_status();
int read_and_clear_rerank_tc_status();
// Bounds-checked build: add each file's counts of skipped out-of-range ids to out[kBadIdKinds] and
// clear them (always true and nothing added in the normal build).
bool read_and_clear_bad_ids_score(unsigned int* out);
bool read_and_clear_bad_ids_paged(unsigned int* out);
bool read_and_clear_bad_ids_block_filter(unsigned int* out);
bool read_and_clear_bad_ids_rerank_tc(unsigned int* out);

// Top-k of each row of scores [T, ld]: positions p < n_t are tokens p (ids == nullptr, P unused),
// or positions p < P are tokens ids[t*P + p] (empty when outside [0, n_t); P <= 16384).  lst: the
// candidate lists launch_scores appended for these rows (or nullptr).  One CTA per row, no
// workspace.  Output order within a row is not specified.
void launch_topk_rows(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T,
                      int L, int topk, const ListState* lst, int32_t* idx, float* score_opt, cudaStream_t s,
                      const int32_t* only = nullptr);
// only (optional): rows with only[t] <= 0 are skipped and keep their outputs.

// The tensor-core scorer's other output modes (score_tc.cu), for queries sharing one bf16 cache:
// every tile_stride-th key tile of each prefix (tiles 0, S, 2S, ...), written packed (sampled tile i
// of row t goes to sample[t, 128 i .. 128 i + 127]); or no score row at all, every score at or above
// tau[t] appended as (order key, token) to query t's list (lists [T][cap], lcnt[t] counting every
// such score, also past cap).  False (nothing launched) when the inputs do not suit the kernel.
bool launch_scores_tc_sample(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads,
                             int T, int L, int H_I, int h, int tile_stride, float* sample, int64_t ld,
                             cudaStream_t s);
bool launch_scores_tc_compact(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads,
                              int T, int L, int H_I, int h, const float* tau, uint2* lists, uint32_t* lcnt, int cap,
                              cudaStream_t s);

// Routed scoring + top-k for queries sharing one bf16 cache without score rows (fused.cu): a sample
// pass over every kFusedStride-th key tile, a cut per query from its sample, the compact pass, the
// selection from the lists, and an exact redo of the queries whose list could not answer.
constexpr int kFusedStride = 32;
int fused_cap(int topk);                    // list entries per query (0: topk unsupported)
int64_t fused_sample_cols(int L);           // packed sample columns of a cache of L keys
size_t fused_ws_bytes(int T, int L, int topk);
// False (after launching part of it) when the tensor-core scorer cannot take these inputs; the
// caller then runs the unfused path on the same workspace's score rows.
bool launch_score_topk_fused(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads,
                             int T, int L, int H_I, int h, int topk, void* ws, int32_t* idx, float* score_opt,
                             float** rows_out, int64_t* ld_out, cudaStream_t s);

// Top-k of short candidate lists in shared memory (no workspace): values F[t, P], ids cand[t, P].
size_t topk_cand_smem(int P);
void launch_topk_cand(const float* F, const int32_t* cand, const int32_t* n, int T, int L, int P,
                      int topk, int32_t* idx, float* score_opt, cudaStream_t s);

// Token-axis block filter composed with MISA (block_filter.cu).  Block scores of every query with
// its routed heads: S[t, b] = sum_{j in heads[t]} w[t, j] * max(0, q[t, j] . kbar_b) for
// b < M_t = ceil(n_t / B), where blocks below kbar_blocks(n_t, B) come from kbar and the last block
// is averaged from k; Mt[t] receives M_t.  Entries b >= M_t are not written.
void launch_block_scores(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                         const float* kbar, int64_t kbar_seq_stride, const int32_t* n, const int32_t* heads, int T,
                         int L, int H_I, int B, int h, float* S, int64_t ldS, int32_t* Mt, cudaStream_t s);
// rows[t, a*B + i] = blocks[t, a]*B + i, or -1 for an empty slot or a token past the prefix.
void launch_expand_blocks(const int32_t* blocks, int m, const int32_t* n, int T, int L, int B, int32_t* rows,
                          cudaStream_t s);

// Paged key caches (paged.cu): pool [num_pages, page_size, 128], table [T][max_pages].
// rows[t, p] = physical pool row of logical token p (ids == nullptr) or ids[t, p] when it lies in
// [0, n_t) and its page is in range, else -1; n_phys[t] = num_pages * page_size.
void launch_paged_rows(const int32_t* table, int64_t max_pages, int64_t num_pages, int page_size, const int32_t* n,
                       int T, int L, const int32_t* ids, int P, int32_t* rows, int32_t* n_phys, cudaStream_t s);
// Block means of logical blocks [b0, b1) of every sequence (as launch_pool).
void launch_pool_paged(DType dt, const void* pool, int64_t num_pages, int page_size, const int32_t* table,
                       int64_t max_pages, int n_seq, int L, int B, float* kbar, int64_t kbar_seq_stride, int b0,
                       int b1, cudaStream_t s);
// pm[t] = mean of the last block of query t's prefix (full or partial; untouched for an empty prefix).
void launch_partial_mean_paged(DType dt, const void* pool, int64_t num_pages, int page_size, const int32_t* table,
                               int64_t max_pages, const int32_t* n, int T, int L, int B, float* pm, cudaStream_t s);

}  // namespace misa
