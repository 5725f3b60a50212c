// Routed scoring + top-k for queries that share one key cache (chunked prefill), without score
// rows, exact.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", "Methodology: MISA",
// "Sparse Token Scoring": the top-k tokens of each query by its routed score I_{t,s}.  The unfused
// path writes every score row (4 bytes per scored pair) and reads it back to select; here:
//   1. the tensor-core scorer scores every kFusedStride-th key tile of each prefix (the sample,
//      1/32 of the work), written packed;
//   2. fused_cut_kernel places each query's cut from its sample, one warp per query: the lower
//      edge of the narrow bin (rounds of 1024 bins over the key range) holding the sample entry
//      whose rank is the expected sample count above the k-th score plus three standard
//      deviations and a margin; prefixes of at most cap keys take every key;
//   3. the scorer runs over every key tile in compact mode: each score at or above its query's cut
//      is appended as (order key, token) to the query's list of cap = 4k entries, no score row;
//   4. one warp per query selects from its list (list_select_warp_kernel): the list's scores lie
//      mostly between the cut and the sample's largest score, so one pass bins them linearly and a
//      second writes the selection, ranking only the k-th entry's bin;
//   5. a query whose list holds fewer than min(k, n_t) entries or lost some past cap is redone
//      exactly: the rows scorer and the per-row top-k, restricted to those queries (both launches
//      find nothing to do when every list answered).
// Whenever a list holds at least min(k, n_t) entries and lost none, it holds every score at or
// above the k-th, so the selection is the unfused one.
#include <cuda_runtime.h>
#include <math.h>

#include "kernels.cuh"
#include "warp_select.cuh"

namespace misa {

namespace {

size_t al(size_t x) { return (x + 255) / 256 * 256; }

// One warp per query: cut[t] (and the list's cut key) from the packed sample row of query t, the
// lower edge of the narrow bin holding the sample entry of the given rank (warp_sample_cut).
__global__ void __launch_bounds__(32 * kSelWarps, 3) fused_cut_kernel(const int32_t* __restrict__ n, int L, int T,
                                                                   int topk, int cap,
                                                                   const float* __restrict__ sample,
                                                                   int64_t ld_sample, float* __restrict__ tau,
                                                                   uint32_t* __restrict__ cutkey,
                                                                   float* __restrict__ shi) {
  __shared__ uint32_t hist[kSelWarps][kWarpBinWords];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelWarps + warp;
  if (t >= T) return;  // uniform across the warp
  const int nt = clamp_len(n[t], L);
  if (nt <= cap) {  // the list takes every key
    if (lane == 0) {
      tau[t] = -INFINITY;
      cutkey[t] = 0u;
    }
    return;
  }
  // keys of the prefix inside sampled tiles: full tiles 0, S, 2S, ... and the partial tile when sampled
  const int full = nt / 128, rem = nt % 128;
  const int ns = (full + kFusedStride - 1) / kFusedStride * 128 + ((rem > 0 && full % kFusedStride == 0) ? rem : 0);
  const float mean = (float)topk * (float)ns / (float)nt;
  const uint32_t rank = (uint32_t)(mean + 3.f * sqrtf(mean) + 8.f);
  if (rank > (uint32_t)ns) {  // the sample cannot place the cut: no list, the query is redone
    if (lane == 0) {
      tau[t] = INFINITY;
      cutkey[t] = 0xffffffffu;
    }
    return;
  }
  const float* st = sample + (int64_t)t * ld_sample;
  uint32_t smax;
  const uint32_t cut =
      warp_sample_cut(ns, [&](int i) { return order_key(__ldg(st + i)); }, rank, hist[warp], &smax);
  if (lane == 0) {
    tau[t] = key_to_float(cut);
    cutkey[t] = cut;
    shi[t] = key_to_float(smax);
  }
}

struct FusedWs {
  ListState lst;
  float* tau;      // [T]
  float* shi;      // [T] the sample's largest score
  float* sample;   // [T][fused_sample_cols(L)]
  int64_t ld_sample;
  float* rows;     // [T][ld] score rows of redone queries
  int64_t ld;
};

FusedWs carve(void* ws, int T, int L, int topk) {
  char* p = static_cast<char*>(ws);
  FusedWs f;
  const int cap = fused_cap(topk);
  f.lst = list_state(p, T, topk, cap);
  p += list_state_bytes(T, cap);
  f.tau = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * (size_t)T);
  f.shi = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * (size_t)T);
  f.ld_sample = fused_sample_cols(L);
  f.sample = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * (size_t)T * f.ld_sample);
  f.ld = (L + 3) / 4 * 4;
  f.rows = reinterpret_cast<float*>(p);
  return f;
}

}  // namespace

int fused_cap(int topk) {
  const int64_t cap = 4 * (int64_t)topk;
  return topk >= 1 && cap <= kListCap ? (int)cap : 0;
}

int64_t fused_sample_cols(int L) {
  const int64_t tiles = (L + 127) / 128;
  return (tiles + kFusedStride - 1) / kFusedStride * 128;
}

size_t fused_ws_bytes(int T, int L, int topk) {
  if (T <= 0 || L <= 0 || fused_cap(topk) == 0) return 0;
  const int64_t ld = (L + 3) / 4 * 4;
  return list_state_bytes(T, fused_cap(topk)) + 2 * al(sizeof(float) * (size_t)T) +
         al(sizeof(float) * (size_t)T * fused_sample_cols(L)) + al(sizeof(float) * (size_t)T * ld);
}

bool launch_score_topk_fused(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads,
                             int T, int L, int H_I, int h, int topk, void* ws, int32_t* idx, float* score_opt,
                             float** rows_out, int64_t* ld_out, cudaStream_t s) {
  const FusedWs f = carve(ws, T, L, topk);
  *rows_out = f.rows;
  *ld_out = f.ld;
  if (T <= 0) return true;
  cudaMemsetAsync(f.lst.cnt, 0, sizeof(uint32_t) * 2 * (size_t)T, s);  // counts and cut keys
  if (!launch_scores_tc_sample(q, w, k, n, heads, T, L, H_I, h, kFusedStride, f.sample, f.ld_sample, s)) return false;
  fused_cut_kernel<<<(T + kSelWarps - 1) / kSelWarps, 32 * kSelWarps, 0, s>>>(n, L, T, topk, f.lst.cap, f.sample,
                                                                              f.ld_sample, f.tau, f.lst.cutkey, f.shi);
  if (!launch_scores_tc_compact(q, w, k, n, heads, T, L, H_I, h, f.tau, f.lst.list, f.lst.cnt, f.lst.cap, s))
    return false;
  launch_list_select_warp(n, T, L, topk, f.lst, idx, score_opt, s, f.shi);
  // exact redo of the queries whose list could not answer: rows and selection restricted to them
  if (!launch_scores_tc(q, w, k, f.lst.redo, heads, T, L, H_I, h, f.rows, f.ld, s)) return false;
  launch_topk_rows(f.rows, f.ld, nullptr, 0, f.lst.redo, T, L, topk, nullptr, idx, score_opt, s, f.lst.redo);
  return true;
}

}  // namespace misa
