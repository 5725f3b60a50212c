// Internal launchers of the MISA indexer kernels (C++ linkage; the C ABI lives in capi.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace misa {

// Block mean-pool ("Lightweight Block-Pooled Router": mean-pooled index keys).
void launch_pool(DType dt, const void* k, int64_t k_seq_stride, int n_seq, int L, int B,
                 float* kbar, int64_t kbar_seq_stride, int b0, int b1, cudaStream_t s);

// Router: partial-block means, per-chunk affinities, then sum, weight and top-h.
int route_chunks(int L, int B);  // chunks of kRouteTile blocks per query (upper bound)
// kbar_parts: [3][ceil(L/B)][128] bf16 scratch for the tensor-core router (shared cache).
// pm_in: [T][128] means of each query's partial last block computed beforehand (paged caches),
// or nullptr to average them from k.
void launch_route(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                  const float* kbar, int64_t kbar_seq_stride, const int32_t* n, int T, int L,
                  int H_I, int B, int h, int32_t* heads, float* r_opt, float* pm, float* partial,
                  uint32_t* done, __nv_bfloat16* kbar_parts, const float* pm_in, cudaStream_t s);

// Router on the tensor cores for queries that share one bf16 cache and its pooled keys: per-tile
// sums over full blocks into Sp [T][nch][H_I], then route_finish.  False (nothing launched) when
// the shapes do not suit it (H_I must divide 128).
constexpr int kRouteTcMinQueries = 64;
bool launch_route_tc(const void* q, const float* w, const void* k, const float* kbar, const int32_t* n, int T,
                     int L, int H_I, int B, int h, int32_t* heads, float* r_opt, __nv_bfloat16* kbar_parts,
                     float* Sp, int nch, cudaStream_t s);
void launch_kbar_split(const float* kbar, int M, __nv_bfloat16* parts, cudaStream_t s);
void launch_route_finish(const __nv_bfloat16* q, const float* w, const __nv_bfloat16* k, const int32_t* n, int T,
                         int L, int H_I, int B, int h, const float* Sp, int nch, int tile, int32_t* heads,
                         float* r_opt, cudaStream_t s);

// Level-0 selection state the decode scoring kernel can build while it scores (select.cuh):
// hist [T][4096] and rec [T][8], both zeroed beforehand (topk_rows_prepare).
struct TopkFuse {
  uint32_t* hist;
  uint32_t* rec;
  int topk;
};

// Token scores with a head list (heads == nullptr: all H_I heads).  rows != nullptr gathers:
// position p of query t scores token rows[t*P + p] and writes out[t*ld + p].  Returns true if it
// also filled *fuse (only the persistent bf16 kernel does).
bool launch_scores(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                   const int32_t* n, const int32_t* heads, int T, int L, int H_I, int h,
                   const int32_t* rows, int P, float* out, int64_t ld, const TopkFuse* fuse, cudaStream_t s);

// Tensor-core scoring for queries sharing one bf16 key cache (k_seq_stride 0, no gather).  Returns
// false without launching when the inputs do not suit it (alignment, no TMA encoder).
bool launch_scores_tc(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads, int T,
                      int L, int H_I, int h, float* out, int64_t ld, cudaStream_t s);
// Reads and clears the status word the tensor-core kernels set when a bounded wait runs out.
int read_and_clear_tc_status();
int read_and_clear_route_tc_status();

// Top-k of each row of scores [T, ld]: positions p < n_t are tokens p (ids == nullptr, P unused),
// or positions p < P are tokens ids[t*P + p] (empty when outside [0, n_t)).  ws holds
// topk_rows_ws(T, P or L) bytes, 256-byte aligned; hist_ready: the scoring kernel already filled
// the level-0 state in ws (the partition/resolve kernels then select); otherwise one CTA per row
// selects.  Output order within a row is not specified.
size_t topk_rows_ws(int T, int P);
void topk_rows_prepare(void* ws, int T, cudaStream_t s);
TopkFuse topk_rows_fuse(void* ws, int T, int topk);
void launch_topk_rows(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T,
                      int L, int topk, void* ws, bool hist_ready, int32_t* idx, float* score_opt,
                      cudaStream_t s);
// Only the level-0 state (prepare + histogram pass), for scores written without it.
void launch_topk_level0(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T,
                        int L, int topk, void* ws, cudaStream_t s);

// Top-k of short candidate lists in shared memory (no workspace): values F[t, P], ids cand[t, P].
size_t topk_cand_smem(int P);
void launch_topk_cand(const float* F, const int32_t* cand, const int32_t* n, int T, int L, int P,
                      int topk, int32_t* idx, float* score_opt, cudaStream_t s);

// Token-axis block filter composed with MISA (block_filter.cu).  Block scores of every query with
// its routed heads: S[t, b] = sum_{j in heads[t]} w[t, j] * max(0, q[t, j] . kbar_b) for
// b < M_t = ceil(n_t / B), where full blocks come from kbar and a partial last block is averaged
// from k; Mt[t] receives M_t.  Entries b >= M_t are not written.
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
// pm[t] = mean of the partial last block of query t's prefix (untouched when n_t is a multiple of B).
void launch_partial_mean_paged(DType dt, const void* pool, int64_t num_pages, int page_size, const int32_t* table,
                               int64_t max_pages, const int32_t* n, int T, int L, int B, float* pm, cudaStream_t s);

}  // namespace misa
