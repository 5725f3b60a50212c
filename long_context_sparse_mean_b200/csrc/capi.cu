// C ABI of the MISA indexer library: argument checks, workspace layout, launch order.
// The declarations and their documentation are in include/misa.h.
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/misa.h"
#include "kernels.cuh"

using misa::DType;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) % kAlign) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Row stride of internal score buffers: L rounded up to 4 floats (16 bytes).
int64_t score_ld(int L) { return (L + 3) / 4 * 4; }

misa_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MISA_OK : MISA_ERR_CUDA;
}

misa_status check_common(const void* q, const float* w, const void* k, const int32_t* n, int T, int L,
                         int H_I, int d, int dtype, int64_t k_seq_stride) {
  if (T < 0 || L < 1 || k_seq_stride < 0) return MISA_ERR_INVALID_ARG;
  if (T > 0 && (!q || !w || !k || !n)) return MISA_ERR_INVALID_ARG;
  if (dtype != MISA_BF16 && dtype != MISA_F32) return MISA_ERR_UNSUPPORTED;
  if (d != misa::kD) return MISA_ERR_UNSUPPORTED;
  if (H_I < 8 || H_I > misa::kMaxHeads || H_I % 8 != 0) return MISA_ERR_UNSUPPORTED;
  if (k_seq_stride != 0 && k_seq_stride < (int64_t)L * d) return MISA_ERR_INVALID_ARG;
  return MISA_OK;
}

DType to_dtype(int dtype) { return dtype == MISA_F32 ? DType::F32 : DType::BF16; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

size_t route_ws(int T, int L, int H_I, int B) {
  if (T <= 0 || L <= 0 || H_I <= 0 || B <= 0) return 0;
  const size_t pm = align_up(sizeof(float) * (size_t)T * misa::kD);
  const size_t part = align_up(sizeof(float) * (size_t)T * misa::route_chunks(L, B) * H_I);
  const size_t done = align_up(sizeof(uint32_t) * (size_t)T);
  const size_t parts = align_up(sizeof(uint16_t) * 3 * (size_t)((L + B - 1) / B) * misa::kD);
  return pm + part + done + parts;
}

size_t scores_part(int T, int L) { return align_up(sizeof(float) * (size_t)T * score_ld(L)); }

// misa_topk_select / misa_token_scores' selection state: the candidate lists of the rows and their
// counts and cut keys (the per-row selection itself needs no workspace)
size_t select_bytes(int T, int P) {
  if (T <= 0 || P <= 0) return 0;
  return align_up(misa::list_state_bytes(T));
}

// misa_score_topk / dsa_dense_topk: [scores][selection]
size_t scores_ws(int T, int L) {
  if (T <= 0 || L <= 0) return 0;
  return scores_part(T, L) + select_bytes(T, L);
}

// misa_hier_rerank: [dense scores of the candidates][selection over the candidate lists]
size_t rerank_ws(int T, int kp) {
  if (T <= 0 || kp <= 0) return 0;
  return align_up(sizeof(float) * (size_t)T * kp) + select_bytes(T, kp);
}

// misa_block_filter_topk: [block scores][M_t per query][token ids of the kept blocks]
// [their scores][selection]
size_t block_filter_ws(int T, int L, int B, int m) {
  if (T <= 0 || L <= 0 || B <= 0 || m <= 0 || (int64_t)m * B > MISA_MAX_KP) return 0;
  const int M = (int)ceil_div(L, B);
  const int64_t P = (int64_t)m * B;
  return align_up(sizeof(float) * (size_t)T * score_ld(M)) + align_up(sizeof(int32_t) * (size_t)T) +
         2 * align_up(sizeof(float) * (size_t)T * P) + select_bytes(T, (int)std::max<int64_t>(M, P));
}

// Paged caches: [physical rows of the positions scored][n_phys] in front of each op's own layout.
size_t paged_rows_part(int T, int P) {
  return align_up(sizeof(int32_t) * (size_t)T * P) + align_up(sizeof(int32_t) * (size_t)T);
}

size_t route_paged_ws(int T, int L, int H_I, int B) {
  if (T <= 0 || L <= 0 || H_I <= 0 || B <= 0) return 0;
  return route_ws(T, L, H_I, B) + align_up(sizeof(float) * (size_t)T * misa::kD);
}

size_t score_topk_paged_ws(int T, int L) {
  if (T <= 0 || L <= 0) return 0;
  return paged_rows_part(T, L) + scores_ws(T, L);
}

size_t rerank_paged_ws(int T, int kp) {
  if (T <= 0 || kp <= 0) return 0;
  return paged_rows_part(T, kp) + rerank_ws(T, kp);
}

misa_status check_paged(const void* pool, int64_t num_pages, int page_size, const int32_t* page_table,
                        int64_t max_pages, int L, int T) {
  if (num_pages < 1 || page_size < 1 || max_pages < 1) return MISA_ERR_INVALID_ARG;
  if ((int64_t)L > max_pages * page_size) return MISA_ERR_INVALID_ARG;  // the table cannot cover L keys
  if (num_pages * (int64_t)page_size > INT32_MAX) return MISA_ERR_UNSUPPORTED;
  if (T > 0 && (!pool || !page_table)) return MISA_ERR_INVALID_ARG;
  return MISA_OK;
}

}  // namespace

extern "C" {

int misa_version(void) { return 100; }

const char* misa_status_str(int status) {
  switch (status) {
    case MISA_OK:
      return "ok";
    case MISA_ERR_INVALID_ARG:
      return "invalid argument";
    case MISA_ERR_UNSUPPORTED:
      return "unsupported configuration";
    case MISA_ERR_WORKSPACE:
      return "workspace too small or misaligned";
    case MISA_ERR_CUDA:
      return "CUDA launch failed";
    case MISA_ERR_DEVICE_TIMEOUT:
      return "a device-side wait ran out; outputs of some call are incomplete";
    case MISA_ERR_BAD_INDEX:
      return "out-of-range ids were seen and skipped (bounds-checked build)";
    default:
      return "unknown status";
  }
}

namespace {
bool read_bad_ids(unsigned int* out) {
  for (int i = 0; i < misa::kBadIdKinds; ++i) out[i] = 0;
  return misa::read_and_clear_bad_ids_score(out) && misa::read_and_clear_bad_ids_paged(out) &&
         misa::read_and_clear_bad_ids_block_filter(out) && misa::read_and_clear_bad_ids_rerank_tc(out);
}
}  // namespace

int misa_checked_build(void) {
#ifdef MISA_CHECKED
  return 1;
#else
  return 0;
#endif
}

misa_status misa_bad_index_counts(unsigned int* out) {
  if (!out) return MISA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MISA_ERR_CUDA;
  return read_bad_ids(out) ? MISA_OK : MISA_ERR_CUDA;
}

misa_status misa_device_check(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return MISA_ERR_CUDA;
  const int v = misa::read_and_clear_tc_status();
  const int u = misa::read_and_clear_route_tc_status();
  const int x = misa::read_and_clear_rerank_tc_status();
  unsigned int bad[misa::kBadIdKinds];
  if (v < 0 || u < 0 || x < 0 || !read_bad_ids(bad)) return MISA_ERR_CUDA;
  if (v || u || x) return MISA_ERR_DEVICE_TIMEOUT;
  return (bad[0] || bad[1] || bad[2]) ? MISA_ERR_BAD_INDEX : MISA_OK;
}

// misa_hier_topk_fused: [score rows][list counts][cuts][dense lists (entries, dense scores)]
// [candidates of the rows the lists cannot answer]
size_t hier_fused_ws(int T, int L, int kp) {
  if (T <= 0 || L <= 0 || kp <= 0) return 0;
  const size_t cap = misa::kListCap;
  return scores_part(T, L) + 2 * align_up(sizeof(uint32_t) * (size_t)T) + align_up(sizeof(uint2) * (size_t)T * cap) +
         align_up(sizeof(float) * (size_t)T * cap) + align_up(sizeof(int32_t) * (size_t)T * kp);
}

size_t misa_workspace_bytes(int op, int T, int L, int H_I, int B, int h, int topk, int kp) {
  (void)h;
  switch (op) {
    case MISA_OP_ROUTE:
      return route_ws(T, L, H_I, B);
    case MISA_OP_SCORE_TOPK:
    case MISA_OP_DENSE_TOPK:
      return scores_ws(T, L);
    case MISA_OP_RERANK:
      return rerank_ws(T, kp);
    case MISA_OP_TOPK_SELECT:
      return select_bytes(T, L);
    case MISA_OP_BLOCK_FILTER:
      return block_filter_ws(T, L, B, kp);
    case MISA_OP_ROUTE_PAGED:
      return route_paged_ws(T, L, H_I, B);
    case MISA_OP_SCORE_TOPK_PAGED:
      return score_topk_paged_ws(T, L);
    case MISA_OP_RERANK_PAGED:
      return rerank_paged_ws(T, kp);
    case MISA_OP_SCORE_TOPK_FUSED:
      return T > 0 && L > 0 && misa::fused_cap(topk) > 0 ? align_up(misa::fused_ws_bytes(T, L, topk)) : 0;
    case MISA_OP_HIER_FUSED:
      return hier_fused_ws(T, L, kp);
    default:
      return 0;
  }
}

misa_status misa_pool_keys(const void* k, int64_t k_seq_stride, int n_seq, int L, int d, int B, int dtype,
                           float* kbar, int64_t kbar_seq_stride, int block_begin, int block_end, void* stream) {
  if (n_seq < 0 || L < 1 || B < 1 || k_seq_stride < 0 || kbar_seq_stride < 0) return MISA_ERR_INVALID_ARG;
  if (dtype != MISA_BF16 && dtype != MISA_F32) return MISA_ERR_UNSUPPORTED;
  if (d != misa::kD) return MISA_ERR_UNSUPPORTED;
  const int M = (int)ceil_div(L, B);
  if (n_seq > 1 && (k_seq_stride < (int64_t)L * d || kbar_seq_stride < (int64_t)M * d)) return MISA_ERR_INVALID_ARG;
  const int b0 = block_begin < 0 ? 0 : block_begin;
  const int b1 = block_end > M ? M : block_end;
  if (n_seq == 0 || b1 <= b0) return MISA_OK;
  if (!k || !kbar) return MISA_ERR_INVALID_ARG;
  misa::launch_pool(to_dtype(dtype), k, k_seq_stride, n_seq, L, B, kbar, kbar_seq_stride, b0, b1,
                    as_stream(stream));
  return launch_status();
}

misa_status misa_route(const void* q, const float* w, const void* k, int64_t k_seq_stride, const float* kbar,
                       int64_t kbar_seq_stride, const int32_t* n, int T, int L, int H_I, int d, int B, int h,
                       int dtype, int32_t* heads, float* r_opt, void* ws, size_t ws_bytes, void* stream) {
  misa_status st = check_common(q, w, k, n, T, L, H_I, d, dtype, k_seq_stride);
  if (st != MISA_OK) return st;
  if (B < 1 || h < 1 || h > H_I || kbar_seq_stride < 0) return MISA_ERR_INVALID_ARG;
  if (T == 0) return MISA_OK;
  if (!kbar || !heads) return MISA_ERR_INVALID_ARG;
  const size_t need = route_ws(T, L, H_I, B);
  if (!ws || ws_bytes < need || !aligned(ws)) return MISA_ERR_WORKSPACE;
  char* p = static_cast<char*>(ws);
  float* pm = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * (size_t)T * misa::kD);
  float* partial = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * (size_t)T * misa::route_chunks(L, B) * H_I);
  uint32_t* done = reinterpret_cast<uint32_t*>(p);
  p += align_up(sizeof(uint32_t) * (size_t)T);
  __nv_bfloat16* parts = reinterpret_cast<__nv_bfloat16*>(p);
  misa::launch_route(to_dtype(dtype), q, w, k, k_seq_stride, kbar, kbar_seq_stride, n, T, L, H_I, B, h, heads,
                     r_opt, pm, partial, done, parts, nullptr, as_stream(stream));
  return launch_status();
}

misa_status misa_token_scores(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n,
                              const int32_t* heads, int T, int L, int H_I, int d, int h, int dtype, float* scores,
                              int64_t ld_scores, int select_topk, void* select_ws, size_t select_ws_bytes,
                              void* stream) {
  misa_status st = check_common(q, w, k, n, T, L, H_I, d, dtype, k_seq_stride);
  if (st != MISA_OK) return st;
  if (heads && (h < 1 || h > H_I)) return MISA_ERR_INVALID_ARG;
  if (ld_scores < L) return MISA_ERR_INVALID_ARG;
  if (select_ws && select_topk < 1) return MISA_ERR_INVALID_ARG;
  if (T == 0) return MISA_OK;
  if (!scores) return MISA_ERR_INVALID_ARG;
  if (select_ws && (select_ws_bytes < select_bytes(T, L) || !aligned(select_ws))) return MISA_ERR_WORKSPACE;
  const cudaStream_t s = as_stream(stream);
  const int m = heads ? h : H_I;
  misa::launch_scores(to_dtype(dtype), q, w, k, k_seq_stride, n, heads, T, L, H_I, m, nullptr, 0, scores, ld_scores,
                      s);
  if (select_ws) misa::launch_list_build(scores, ld_scores, n, T, L, misa::list_state(select_ws, T, select_topk), s);
  return launch_status();
}

misa_status misa_topk_select(const float* scores, int64_t ld_scores, const int32_t* n, int T, int L, int topk,
                             int32_t* idx, float* score_opt, void* ws, size_t ws_bytes, int ws_prepared,
                             void* stream) {
  if (T < 0 || L < 1 || topk < 1 || ld_scores < L) return MISA_ERR_INVALID_ARG;
  if (T == 0) return MISA_OK;
  if (!scores || !n || !idx) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < select_bytes(T, L) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  const misa::ListState lst = misa::list_state(ws, T, topk);
  const cudaStream_t s = as_stream(stream);
  if (!ws_prepared) misa::launch_list_build(scores, ld_scores, n, T, L, lst, s);
  misa::launch_topk_rows(scores, ld_scores, nullptr, 0, n, T, L, topk, &lst, idx, score_opt, s);
  return launch_status();
}

misa_status misa_score_topk(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n,
                            const int32_t* heads, int T, int L, int H_I, int d, int h, int topk, int dtype,
                            int32_t* idx, float* score_opt, float* scores_full_opt, void* ws, size_t ws_bytes,
                            void* stream) {
  misa_status st = check_common(q, w, k, n, T, L, H_I, d, dtype, k_seq_stride);
  if (st != MISA_OK) return st;
  if (!heads && T > 0) return MISA_ERR_INVALID_ARG;
  if (h < 1 || h > H_I || topk < 1) return MISA_ERR_INVALID_ARG;
  if (T == 0) return MISA_OK;
  if (!idx) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < (scores_full_opt ? select_bytes(T, L) : scores_ws(T, L)) || !aligned(ws))
    return MISA_ERR_WORKSPACE;
  char* p = static_cast<char*>(ws);
  float* buf = scores_full_opt;
  int64_t ld = L;
  if (!buf) {
    buf = reinterpret_cast<float*>(p);
    ld = score_ld(L);
    p += scores_part(T, L);
  }
  const cudaStream_t s = as_stream(stream);
  const misa::ListState lst = misa::list_state(p, T, topk);
  misa::launch_scores(to_dtype(dtype), q, w, k, k_seq_stride, n, heads, T, L, H_I, h, nullptr, 0, buf, ld, s);
  misa::launch_list_build(buf, ld, n, T, L, lst, s);
  misa::launch_topk_rows(buf, ld, nullptr, 0, n, T, L, topk, &lst, idx, score_opt, s);
  return launch_status();
}

misa_status misa_hier_rerank(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n,
                             const int32_t* cand, int T, int L, int H_I, int d, int kp, int topk, int dtype,
                             int32_t* idx, float* score_opt, void* ws, size_t ws_bytes, void* stream) {
  misa_status st = check_common(q, w, k, n, T, L, H_I, d, dtype, k_seq_stride);
  if (st != MISA_OK) return st;
  if (topk < 1 || kp < topk) return MISA_ERR_INVALID_ARG;
  if (kp > MISA_MAX_KP) return MISA_ERR_UNSUPPORTED;
  if (T == 0) return MISA_OK;
  if (!cand || !idx) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < rerank_ws(T, kp) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  float* F = static_cast<float*>(ws);
  misa::launch_scores(to_dtype(dtype), q, w, k, k_seq_stride, n, nullptr, T, L, H_I, H_I, cand, kp, F, kp,
                      as_stream(stream));
  misa::launch_topk_rows(F, kp, cand, kp, n, T, L, topk, nullptr, idx, score_opt, as_stream(stream));
  return launch_status();
}

misa_status dsa_dense_topk(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n,
                           int T, int L, int H_I, int d, int topk, int dtype, int32_t* idx, float* score_opt,
                           void* ws, size_t ws_bytes, void* stream) {
  misa_status st = check_common(q, w, k, n, T, L, H_I, d, dtype, k_seq_stride);
  if (st != MISA_OK) return st;
  if (topk < 1) return MISA_ERR_INVALID_ARG;
  if (T == 0) return MISA_OK;
  if (!idx) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < scores_ws(T, L) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  char* p = static_cast<char*>(ws);
  float* buf = reinterpret_cast<float*>(p);
  const int64_t ld = score_ld(L);
  const misa::ListState lst = misa::list_state(p + scores_part(T, L), T, topk);
  const cudaStream_t s = as_stream(stream);
  misa::launch_scores(to_dtype(dtype), q, w, k, k_seq_stride, n, nullptr, T, L, H_I, H_I, nullptr, 0, buf, ld, s);
  misa::launch_list_build(buf, ld, n, T, L, lst, s);
  misa::launch_topk_rows(buf, ld, nullptr, 0, n, T, L, topk, &lst, idx, score_opt, s);
  return launch_status();
}

misa_status misa_block_filter_topk(const void* q, const float* w, const void* k, int64_t k_seq_stride,
                                   const float* kbar, int64_t kbar_seq_stride, const int32_t* n,
                                   const int32_t* heads, int T, int L, int H_I, int d, int B, int h, int m,
                                   int topk, int dtype, float* block_scores_opt, int64_t ld_block_scores,
                                   int32_t* blocks, int32_t* idx, float* score_opt, void* ws, size_t ws_bytes,
                                   void* stream) {
  misa_status st = check_common(q, w, k, n, T, L, H_I, d, dtype, k_seq_stride);
  if (st != MISA_OK) return st;
  if (B < 1 || h < 1 || h > H_I || m < 1 || topk < 1 || kbar_seq_stride < 0) return MISA_ERR_INVALID_ARG;
  if ((int64_t)m * B > MISA_MAX_KP) return MISA_ERR_UNSUPPORTED;
  const int M = (int)ceil_div(L, B);
  if (kbar_seq_stride != 0 && (kbar_seq_stride < (int64_t)M * d || kbar_seq_stride % 4 != 0))
    return MISA_ERR_INVALID_ARG;
  if (block_scores_opt && ld_block_scores < M) return MISA_ERR_INVALID_ARG;
  if (T == 0) return MISA_OK;
  if (!kbar || !heads || !blocks || !idx || (reinterpret_cast<uintptr_t>(kbar) & 15) != 0)
    return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < block_filter_ws(T, L, B, m) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  const int P = m * B;
  char* p = static_cast<char*>(ws);
  float* S = block_scores_opt;
  int64_t ldS = ld_block_scores;
  if (!S) {
    S = reinterpret_cast<float*>(p);
    ldS = score_ld(M);
  }
  p += align_up(sizeof(float) * (size_t)T * score_ld(M));
  int32_t* Mt = reinterpret_cast<int32_t*>(p);
  p += align_up(sizeof(int32_t) * (size_t)T);
  int32_t* rows = reinterpret_cast<int32_t*>(p);
  p += align_up(sizeof(float) * (size_t)T * P);
  float* F = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * (size_t)T * P);
  const cudaStream_t s = as_stream(stream);
  misa::launch_block_scores(to_dtype(dtype), q, w, k, k_seq_stride, kbar, kbar_seq_stride, n, heads, T, L, H_I, B,
                            h, S, ldS, Mt, s);
  misa::launch_topk_rows(S, ldS, nullptr, 0, Mt, T, M, m, nullptr, blocks, nullptr, s);
  misa::launch_expand_blocks(blocks, m, n, T, L, B, rows, s);
  misa::launch_scores(to_dtype(dtype), q, w, k, k_seq_stride, n, heads, T, L, H_I, h, rows, P, F, P, s);
  misa::launch_topk_rows(F, P, rows, P, n, T, L, topk, nullptr, idx, score_opt, s);
  return launch_status();
}

misa_status misa_pool_keys_paged(const void* pool, int64_t num_pages, int page_size, const int32_t* page_table,
                                 int64_t max_pages, int n_seq, int L, int d, int B, int dtype, float* kbar,
                                 int64_t kbar_seq_stride, int block_begin, int block_end, void* stream) {
  if (n_seq < 0 || L < 1 || B < 1 || kbar_seq_stride < 0) return MISA_ERR_INVALID_ARG;
  if (dtype != MISA_BF16 && dtype != MISA_F32) return MISA_ERR_UNSUPPORTED;
  if (d != misa::kD) return MISA_ERR_UNSUPPORTED;
  misa_status st = check_paged(pool, num_pages, page_size, page_table, max_pages, L, n_seq);
  if (st != MISA_OK) return st;
  const int M = (int)ceil_div(L, B);
  if (n_seq > 1 && kbar_seq_stride < (int64_t)M * d) return MISA_ERR_INVALID_ARG;
  const int b0 = block_begin < 0 ? 0 : block_begin;
  const int b1 = block_end > M ? M : block_end;
  if (n_seq == 0 || b1 <= b0) return MISA_OK;
  if (!kbar) return MISA_ERR_INVALID_ARG;
  misa::launch_pool_paged(to_dtype(dtype), pool, num_pages, page_size, page_table, max_pages, n_seq, L, B, kbar,
                          kbar_seq_stride, b0, b1, as_stream(stream));
  return launch_status();
}

misa_status misa_route_paged(const void* q, const float* w, const void* pool, int64_t num_pages, int page_size,
                             const int32_t* page_table, int64_t max_pages, const float* kbar, int64_t kbar_seq_stride,
                             const int32_t* n, int T, int L, int H_I, int d, int B, int h, int dtype, int32_t* heads,
                             float* r_opt, void* ws, size_t ws_bytes, void* stream) {
  misa_status st = check_common(q, w, pool, n, T, L, H_I, d, dtype, 0);
  if (st != MISA_OK) return st;
  st = check_paged(pool, num_pages, page_size, page_table, max_pages, L, T);
  if (st != MISA_OK) return st;
  if (B < 1 || h < 1 || h > H_I) return MISA_ERR_INVALID_ARG;
  const int M = (int)ceil_div(L, B);
  if (T > 1 && kbar_seq_stride < (int64_t)M * d) return MISA_ERR_INVALID_ARG;  // one pooled cache per query
  if (T == 0) return MISA_OK;
  if (!kbar || !heads) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < route_paged_ws(T, L, H_I, B) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  char* p = static_cast<char*>(ws);
  float* pm = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * (size_t)T * misa::kD);
  float* partial = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * (size_t)T * misa::route_chunks(L, B) * H_I);
  uint32_t* done = reinterpret_cast<uint32_t*>(p);
  p += align_up(sizeof(uint32_t) * (size_t)T);
  __nv_bfloat16* parts = reinterpret_cast<__nv_bfloat16*>(p);
  p += align_up(sizeof(uint16_t) * 3 * (size_t)M * misa::kD);
  float* pm_in = reinterpret_cast<float*>(p);
  const cudaStream_t s = as_stream(stream);
  misa::launch_partial_mean_paged(to_dtype(dtype), pool, num_pages, page_size, page_table, max_pages, n, T, L, B,
                                  pm_in, s);
  misa::launch_route(to_dtype(dtype), q, w, pool, 0, kbar, kbar_seq_stride, n, T, L, H_I, B, h, heads, r_opt, pm,
                     partial, done, parts, pm_in, s);
  return launch_status();
}

misa_status misa_score_topk_paged(const void* q, const float* w, const void* pool, int64_t num_pages, int page_size,
                                  const int32_t* page_table, int64_t max_pages, const int32_t* n,
                                  const int32_t* heads, int T, int L, int H_I, int d, int h, int topk, int dtype,
                                  int32_t* idx, float* score_opt, void* ws, size_t ws_bytes, void* stream) {
  misa_status st = check_common(q, w, pool, n, T, L, H_I, d, dtype, 0);
  if (st != MISA_OK) return st;
  st = check_paged(pool, num_pages, page_size, page_table, max_pages, L, T);
  if (st != MISA_OK) return st;
  if (!heads && T > 0) return MISA_ERR_INVALID_ARG;
  if (h < 1 || h > H_I || topk < 1) return MISA_ERR_INVALID_ARG;
  if (T == 0) return MISA_OK;
  if (!idx) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < score_topk_paged_ws(T, L) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  char* p = static_cast<char*>(ws);
  int32_t* rows = reinterpret_cast<int32_t*>(p);
  p += align_up(sizeof(int32_t) * (size_t)T * L);
  int32_t* n_phys = reinterpret_cast<int32_t*>(p);
  p += align_up(sizeof(int32_t) * (size_t)T);
  float* buf = reinterpret_cast<float*>(p);
  const int64_t ld = score_ld(L);
  p += scores_part(T, L);
  const int pool_rows = (int)(num_pages * page_size);
  const cudaStream_t s = as_stream(stream);
  misa::launch_paged_rows(page_table, max_pages, num_pages, page_size, n, T, L, nullptr, L, rows, n_phys, s);
  misa::launch_scores(to_dtype(dtype), q, w, pool, 0, n_phys, heads, T, pool_rows, H_I, h, rows, L, buf, ld, s);
  const misa::ListState lst = misa::list_state(p, T, topk);
  misa::launch_list_build(buf, ld, n, T, L, lst, s);
  misa::launch_topk_rows(buf, ld, nullptr, 0, n, T, L, topk, &lst, idx, score_opt, s);
  return launch_status();
}

misa_status misa_hier_rerank_paged(const void* q, const float* w, const void* pool, int64_t num_pages, int page_size,
                                   const int32_t* page_table, int64_t max_pages, const int32_t* n,
                                   const int32_t* cand, int T, int L, int H_I, int d, int kp, int topk, int dtype,
                                   int32_t* idx, float* score_opt, void* ws, size_t ws_bytes, void* stream) {
  misa_status st = check_common(q, w, pool, n, T, L, H_I, d, dtype, 0);
  if (st != MISA_OK) return st;
  st = check_paged(pool, num_pages, page_size, page_table, max_pages, L, T);
  if (st != MISA_OK) return st;
  if (topk < 1 || kp < topk) return MISA_ERR_INVALID_ARG;
  if (kp > MISA_MAX_KP) return MISA_ERR_UNSUPPORTED;
  if (T == 0) return MISA_OK;
  if (!cand || !idx) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < rerank_paged_ws(T, kp) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  char* p = static_cast<char*>(ws);
  int32_t* rows = reinterpret_cast<int32_t*>(p);
  p += align_up(sizeof(int32_t) * (size_t)T * kp);
  int32_t* n_phys = reinterpret_cast<int32_t*>(p);
  p += align_up(sizeof(int32_t) * (size_t)T);
  float* F = reinterpret_cast<float*>(p);
  const int pool_rows = (int)(num_pages * page_size);
  const cudaStream_t s = as_stream(stream);
  misa::launch_paged_rows(page_table, max_pages, num_pages, page_size, n, T, L, cand, kp, rows, n_phys, s);
  misa::launch_scores(to_dtype(dtype), q, w, pool, 0, n_phys, nullptr, T, pool_rows, H_I, H_I, rows, kp, F, kp, s);
  misa::launch_topk_rows(F, kp, cand, kp, n, T, L, topk, nullptr, idx, score_opt, s);
  return launch_status();
}

misa_status misa_score_topk_fused(const void* q, const float* w, const void* k, const int32_t* n,
                                  const int32_t* heads, int T, int L, int H_I, int d, int h, int topk, int dtype,
                                  int32_t* idx, float* score_opt, void* ws, size_t ws_bytes, void* stream) {
  misa_status st = check_common(q, w, k, n, T, L, H_I, d, dtype, 0);
  if (st != MISA_OK) return st;
  if (!heads && T > 0) return MISA_ERR_INVALID_ARG;
  if (h < 1 || h > H_I || topk < 1) return MISA_ERR_INVALID_ARG;
  if (dtype != MISA_BF16 || misa::fused_cap(topk) == 0) return MISA_ERR_UNSUPPORTED;
  if (T == 0) return MISA_OK;
  if (!idx) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < misa::fused_ws_bytes(T, L, topk) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  const cudaStream_t s = as_stream(stream);
  float* rows = nullptr;
  int64_t ld = 0;
  if (!misa::launch_score_topk_fused(q, w, k, n, heads, T, L, H_I, h, topk, ws, idx, score_opt, &rows, &ld, s)) {
    // the tensor-core scorer cannot take these inputs: every query by the unfused path
    misa::launch_scores(misa::DType::BF16, q, w, k, 0, n, heads, T, L, H_I, h, nullptr, 0, rows, ld, s);
    misa::launch_topk_rows(rows, ld, nullptr, 0, n, T, L, topk, nullptr, idx, score_opt, s);
  }
  return launch_status();
}

misa_status misa_hier_topk_fused(const void* q, const float* w, const void* k, int64_t k_seq_stride,
                                 const int32_t* n, const int32_t* heads, int T, int L, int H_I, int d, int h, int kp,
                                 int topk, int dtype, int32_t* idx, float* score_opt, void* ws, size_t ws_bytes,
                                 void* stream) {
  misa_status st = check_common(q, w, k, n, T, L, H_I, d, dtype, k_seq_stride);
  if (st != MISA_OK) return st;
  if (!heads && T > 0) return MISA_ERR_INVALID_ARG;
  if (h < 1 || h > H_I || topk < 1 || kp < topk) return MISA_ERR_INVALID_ARG;
  if (kp > MISA_MAX_KP) return MISA_ERR_UNSUPPORTED;
  if (dtype != MISA_BF16 || k_seq_stride == 0) return MISA_ERR_UNSUPPORTED;
  if (T == 0) return MISA_OK;
  if (!idx) return MISA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < hier_fused_ws(T, L, kp) || !aligned(ws)) return MISA_ERR_WORKSPACE;
  const cudaStream_t s = as_stream(stream);
  const int64_t ld = score_ld(L);
  char* p = static_cast<char*>(ws);
  float* rows = reinterpret_cast<float*>(p);
  p += scores_part(T, L);
  misa::DenseList dl{};
  dl.cnt = reinterpret_cast<uint32_t*>(p);
  p += align_up(sizeof(uint32_t) * (size_t)T);
  uint32_t* cut = reinterpret_cast<uint32_t*>(p);
  dl.cut = cut;
  p += align_up(sizeof(uint32_t) * (size_t)T);
  dl.cap = misa::kListCap;
  dl.stride = misa::kListCap;
  dl.list = reinterpret_cast<uint2*>(p);
  p += align_up(sizeof(uint2) * (size_t)T * dl.cap);
  dl.f = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * (size_t)T * dl.cap);
  int32_t* ctok = reinterpret_cast<int32_t*>(p);
  // lists for a few long rows (many rows fill the GPU with one CTA per row already); the scorer's
  // shared memory must fit two CTAs per SM
  const bool lists = T <= misa::kDenseListMaxRows && L > dl.cap && h <= 8 &&
                     misa::dense_list_smem(T, H_I) <= misa::kDenseListMaxSmem;
  if (lists) {
    misa::launch_scores_sample(q, w, k, k_seq_stride, n, heads, T, L, H_I, h, dl.cap, rows, ld, s);
    misa::launch_list_cut(rows, ld, n, T, L, kp, dl.cap, dl.cnt, cut, s);
    misa::launch_scores_dense_list(q, w, k, k_seq_stride, n, heads, T, L, H_I, h, rows, ld, dl, s);
  } else {
    cudaMemsetAsync(dl.cnt, 0xff, sizeof(uint32_t) * (size_t)T, s);  // kNoList: every row from its score row
    misa::launch_scores(misa::DType::BF16, q, w, k, k_seq_stride, n, heads, T, L, H_I, h, nullptr, 0, rows, ld, s);
  }
  misa::launch_hier_select(rows, ld, n, T, L, kp, topk, dl, q, w, k, k_seq_stride, H_I, ctok, idx, score_opt, s);
  return launch_status();
}

}  // extern "C"
