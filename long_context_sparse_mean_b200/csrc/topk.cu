// Top-k selection.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", Technical Summary,
// "Methodology: MISA", "Sparse Token Scoring": the final top-k tokens are selected on the reduced
// scores; "Hierarchical Variant (MISA-dagger)": the k' candidates are narrowed to the top-k by
// their dense scores.  Rule: score descending, exact ties to the lower token id (select.cuh).
//
// Rows of scores (one per query; a position p is token p, or token ids[p] for candidate lists)
// are selected by a radix cascade over the order keys, every pass reading the rows from L2 with
// wide loads, 4096 positions per CTA:
//   1. level-0 pass: 4096-bucket histogram of key bits 31..20 per row; the last CTA of a row to
//      finish (a counter per row) finds the bucket holding the k-th key and how many keys above it
//      are taken;
//   2. level-1 pass: histogram of bits 19..8 of the keys in that bucket; again the last CTA of the
//      row fixes the 24-bit boundary prefix;
//   3. partition: keys above the boundary are written out directly (slots reserved with one atomic
//      per CTA), keys on the boundary prefix go to a short (key, id) list;
//   4. resolve: one CTA per row ranks that list on the last 8 key bits and, for exact ties, on the
//      token id, in shared memory (straight from global memory if the list is too long).
// Clustered scores put about half of a 131072-key row in one level-0 bucket, which is why the
// cascade has two histogram levels before the partition.  The selected set is exact; its order in
// the output is not specified.
// select_small_kernel ranks a short candidate list entirely in one CTA's shared memory; it needs
// no workspace (used by the entry point without allocation).
#include "kernels.cuh"
#include "select.cuh"

namespace misa {

namespace {

constexpr int kPassThreads = 256;
constexpr int kPassItems = 16;                         // positions per thread
constexpr int kPassChunk = kPassThreads * kPassItems;  // positions per CTA
constexpr int kResolveThreads = 256;
constexpr int kResolveSmemItems = 8192;  // boundary pairs ranked in shared memory
constexpr int kSmallThreads = 1024;
constexpr int kRec = 8;  // words of per-row state

// Per-row state rec[t][kRec]:
//   0: level-0 CTAs finished   1: level-1 CTAs finished
//   2: level-0 prefix (bits 31..20)   3: keys still needed inside the level-0 bucket
//   4: 24-bit boundary prefix (bits 31..8)   5: keys still needed on the boundary prefix
//   6: slots filled by keys above the boundary   7: boundary pairs written

__device__ __forceinline__ int padded(int e) { return e + (e >> 5); }

// The row positions handled by one thread of a pass CTA: 4 groups of 4 consecutive positions.
struct RowSlice {
  const float* row;
  const int32_t* ids;  // null: token = position
  int s1, nt;
  bool vec;
  __device__ int pos(int base, int item) const {
    return base + 4 * ((int)threadIdx.x + (item >> 2) * kPassThreads) + (item & 3);
  }
  __device__ void load(int base, float (&v)[kPassItems], uint32_t (&key)[kPassItems], bool (&ok)[kPassItems]) const {
#pragma unroll
    for (int j = 0; j < kPassItems / 4; ++j) {
      const int s = pos(base, 4 * j);
      if (vec && s + 3 < s1) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(row + s));
        v[4 * j] = x.x;
        v[4 * j + 1] = x.y;
        v[4 * j + 2] = x.z;
        v[4 * j + 3] = x.w;
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[4 * j + i] = s + i < s1 ? __ldcg(row + s + i) : 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < kPassItems; ++i) {
      const int s = pos(base, i);
      bool in = s < s1;
      if (in && ids) {
        const int32_t id = __ldcg(ids + s);
        in = id >= 0 && id < nt;
      }
      key[i] = order_key(v[i]);
      ok[i] = in && key[i] != 0u;
    }
  }
  __device__ int32_t token(int p) const { return ids ? ids[p] : p; }
};

// Histogram pass of level LVL (0: bits 31..20 of all keys; 1: bits 19..8 of the keys in the
// level-0 bucket); the row's last CTA turns the histogram into a boundary.
template <int LVL>
__global__ void __launch_bounds__(kPassThreads) hist_pass_kernel(const float* __restrict__ scores, int64_t ld,
                                                                 const int32_t* __restrict__ ids, int P,
                                                                 const int32_t* __restrict__ n, int L, int topk,
                                                                 uint32_t* __restrict__ hist, uint32_t* __restrict__ rec) {
  __shared__ uint32_t h[kHistBins];
  __shared__ uint32_t scratch[35];
  __shared__ int last;
  const int t = blockIdx.y;
  const int nt = clamp_len(n[t], L);
  const int npos = ids ? P : nt;
  if (!ids && npos <= topk) return;  // the whole prefix is selected
  const int nchunks = (npos + kPassChunk - 1) / kPassChunk;
  const int base = blockIdx.x * kPassChunk;
  if (base >= npos) return;
  uint32_t* rt = rec + (int64_t)t * kRec;
  uint32_t* ht = hist + (int64_t)t * kHistBins;
  for (int b = threadIdx.x; b < kHistBins; b += kPassThreads) h[b] = 0;
  const RowSlice rs{scores + (int64_t)t * ld, ids ? ids + (int64_t)t * P : nullptr, min(base + kPassChunk, npos), nt,
                    (ld % 4) == 0};
  float v[kPassItems];
  uint32_t key[kPassItems];
  bool ok[kPassItems];
  rs.load(base, v, key, ok);
  const uint32_t top0 = LVL == 1 ? (__ldcg(rt + 2) >> 20) : 0u;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kPassItems; ++i) {
    const bool in = ok[i] && (LVL == 0 || (key[i] >> 20) == top0);
    hist_add(h, LVL == 0 ? key[i] >> 20 : (key[i] >> 8) & 4095u, in);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kHistBins; b += kPassThreads)
    if (h[b]) atomicAdd(ht + b, h[b]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(rt + LVL, 1u) == (uint32_t)(nchunks - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int b = threadIdx.x; b < kHistBins; b += kPassThreads) h[b] = __ldcg(ht + b);
  __syncthreads();
  if (LVL == 0) {
    // with a candidate list fewer than k keys may be valid: then all of them are taken
    uint32_t local = 0;
    for (int b = threadIdx.x; b < kHistBins; b += kPassThreads) local += h[b];
    uint32_t total;
    block_exclusive_scan(local, scratch, &total);
    const uint32_t need = min((uint32_t)topk, total);
    const Bucket bk = block_bucket_bits(h, kHistBins, 20, 0u, need, scratch);
    if (threadIdx.x == 0) {
      rt[2] = need ? bk.prefix : 0xffffffffu;
      rt[3] = need ? bk.need : 0u;
    }
  } else {
    const uint32_t need = __ldcg(rt + 3);
    const Bucket bk = block_bucket_bits(h, kHistBins, 8, __ldcg(rt + 2), need, scratch);
    if (threadIdx.x == 0) {
      rt[4] = need ? bk.prefix : 0xffffffffu;
      rt[5] = need ? bk.need : 0u;
    }
  }
}

__global__ void __launch_bounds__(kPassThreads) partition_kernel(const float* __restrict__ scores, int64_t ld,
                                                                 const int32_t* __restrict__ ids, int P,
                                                                 const int32_t* __restrict__ n, int L, int topk,
                                                                 uint32_t* __restrict__ rec, uint2* __restrict__ pairs,
                                                                 int64_t pairs_ld, int32_t* __restrict__ idx,
                                                                 float* __restrict__ score_opt) {
  __shared__ uint32_t scratch[35];
  __shared__ uint32_t basev[2];
  const int t = blockIdx.y;
  const int nt = clamp_len(n[t], L);
  const int npos = ids ? P : nt;
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  const float* row = scores + (int64_t)t * ld;
  if (!ids && npos <= topk) {  // every prefix token is selected; this CTA writes its share of the slots
    const int per = (topk + gridDim.x - 1) / gridDim.x;
    for (int a = blockIdx.x * per + threadIdx.x; a < min(topk, (int)(blockIdx.x + 1) * per); a += kPassThreads) {
      oi[a] = a < nt ? a : -1;
      if (ov) ov[a] = a < nt ? row[a] : 0.f;
    }
    return;
  }
  const int base = blockIdx.x * kPassChunk;
  if (base >= npos) return;
  uint32_t* rt = rec + (int64_t)t * kRec;
  const uint32_t b24 = __ldcg(rt + 4);
  const bool none = b24 == 0xffffffffu;  // no valid key at all
  const uint32_t prefix = b24 >> 8;
  const RowSlice rs{row, ids ? ids + (int64_t)t * P : nullptr, min(base + kPassChunk, npos), nt, (ld % 4) == 0};
  float v[kPassItems];
  uint32_t key[kPassItems];
  bool ok[kPassItems];
  rs.load(base, v, key, ok);
  uint32_t gtm = 0, eqm = 0;
#pragma unroll
  for (int i = 0; i < kPassItems; ++i) {
    gtm |= (uint32_t)(!none && ok[i] && (key[i] >> 8) > prefix) << i;
    eqm |= (uint32_t)(!none && ok[i] && (key[i] >> 8) == prefix) << i;
  }
  uint32_t tg, te;
  uint32_t pg = block_exclusive_scan(__popc(gtm), scratch, &tg);
  uint32_t pe = block_exclusive_scan(__popc(eqm), scratch, &te);
  if (threadIdx.x == 0) {
    basev[0] = tg ? atomicAdd(rt + 6, tg) : 0u;
    basev[1] = te ? atomicAdd(rt + 7, te) : 0u;
  }
  __syncthreads();
  pg += basev[0];
  pe += basev[1];
  uint2* pt = pairs + (int64_t)t * pairs_ld;
#pragma unroll
  for (int i = 0; i < kPassItems; ++i) {
    const int p = rs.pos(base, i);
    if ((gtm >> i) & 1u) {
      if (pg < (uint32_t)topk) {
        oi[pg] = rs.token(p);
        if (ov) ov[pg] = v[i];
      }
      ++pg;
    }
    if ((eqm >> i) & 1u) {
      if (pe < (uint32_t)pairs_ld) pt[pe] = make_uint2(key[i], (uint32_t)rs.token(p));
      ++pe;
    }
  }
}

struct PairList {
  const uint2* p;
  __device__ uint32_t key(int i) const { return p[i].x; }
  __device__ uint32_t id(int i) const { return p[i].y; }
};

// One CTA per row: slots [n_out, n_out + need) come from the boundary pairs; the rest of the row
// after the selection is padded with -1.
__global__ void __launch_bounds__(kResolveThreads) resolve_kernel(const int32_t* __restrict__ n, int L, bool lists,
                                                                  int topk, const uint32_t* __restrict__ rec,
                                                                  const uint2* __restrict__ pairs, int64_t pairs_ld,
                                                                  int32_t* __restrict__ idx,
                                                                  float* __restrict__ score_opt) {
  extern __shared__ uint2 list[];  // [kResolveSmemItems]
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scratch[35];
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  if (!lists && nt <= topk) return;
  const uint32_t* rt = rec + (int64_t)t * kRec;
  const uint32_t n_out = min(__ldcg(rt + 6), (uint32_t)topk);
  const int c = (int)min(__ldcg(rt + 7), (uint32_t)pairs_ld);
  const uint32_t need = min(__ldcg(rt + 5), (uint32_t)c);
  const uint32_t prefix = __ldcg(rt + 4);
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  const uint2* pt = pairs + (int64_t)t * pairs_ld;
  const uint32_t kk = min((uint32_t)topk, n_out + need);
  if ((uint32_t)c <= need) {
    for (int i = threadIdx.x; i < c; i += kResolveThreads)
      if (n_out + i < (uint32_t)topk) {
        oi[n_out + i] = (int32_t)pt[i].y;
        if (ov) ov[n_out + i] = key_to_float(pt[i].x);
      }
  } else if (c <= kResolveSmemItems) {
    for (int i = threadIdx.x; i < c; i += kResolveThreads) list[i] = pt[i];
    __syncthreads();
    const PairList acc{list};
    const SelectResult r = radix_select_items(acc, c, need, 2, prefix, 0xffffff00u, hist, scratch);
    write_selection(acc, c, r, false, oi + n_out, ov ? ov + n_out : nullptr, need, scratch);
  } else {
    const PairList acc{pt};
    const SelectResult r = radix_select_items(acc, c, need, 2, prefix, 0xffffff00u, hist, scratch);
    write_selection(acc, c, r, false, oi + n_out, ov ? ov + n_out : nullptr, need, scratch);
  }
  for (int a = (int)kk + threadIdx.x; a < topk; a += kResolveThreads) {
    oi[a] = -1;
    if (ov) ov[a] = 0.f;
  }
}

struct SmemItems {
  const uint32_t* keys;
  const uint32_t* ids;
  __device__ uint32_t key(int i) const { return keys[padded(i)]; }
  __device__ uint32_t id(int i) const { return ids[padded(i)]; }
};

// Top-k of candidate lists in one CTA: values F[t, P], ids cand[t, P] (ids outside [0, n_t) are
// empty).
__global__ void __launch_bounds__(kSmallThreads) select_small_kernel(const float* __restrict__ F,
                                                                     const int32_t* __restrict__ cand,
                                                                     const int32_t* __restrict__ n, int L, int P,
                                                                     int topk, int32_t* __restrict__ idx,
                                                                     float* __restrict__ score_opt) {
  extern __shared__ uint32_t sm[];
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scratch[35];
  uint32_t* keys = sm;
  uint32_t* ids = sm + padded(P) + 1;
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const float* ft = F + (int64_t)t * P;
  const int32_t* ctp = cand + (int64_t)t * P;
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  uint32_t mine = 0;
  for (int i = threadIdx.x; i < P; i += kSmallThreads) {
    const int32_t id = ctp[i];
    const bool ok = id >= 0 && id < nt;
    keys[padded(i)] = ok ? order_key(ft[i]) : 0u;
    ids[padded(i)] = ok ? (uint32_t)id : 0u;
    mine += ok;
  }
  uint32_t nvalid;
  block_exclusive_scan(mine, scratch, &nvalid);
  const uint32_t kk = min((uint32_t)topk, nvalid);
  const SmemItems acc{keys, ids};
  if (kk == nvalid) {
    write_selection(acc, P, SelectResult{}, true, oi, ov, kk, scratch);
  } else {
    const SelectResult r = radix_select_items(acc, P, kk, 0, 0u, 0u, hist, scratch);
    write_selection(acc, P, r, false, oi, ov, kk, scratch);
  }
  for (int a = (int)kk + threadIdx.x; a < topk; a += kSmallThreads) {
    oi[a] = -1;
    if (ov) ov[a] = 0.f;
  }
}

}  // namespace

// Workspace of one selection: hist0 [T][4096], hist1 [T][4096], rec [T][8], pairs [T][P] (uint2).
size_t topk_rows_ws(int T, int P) {
  return sizeof(uint32_t) * (2 * (size_t)kHistBins + kRec) * (size_t)T + sizeof(uint2) * (size_t)T * P;
}

void launch_topk_rows(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T, int L,
                      int topk, void* ws, int32_t* idx, float* score_opt, cudaStream_t s) {
  if (T <= 0) return;
  const int npos = ids ? P : L;
  uint32_t* hist0 = static_cast<uint32_t*>(ws);
  uint32_t* hist1 = hist0 + (size_t)kHistBins * T;
  uint32_t* rec = hist1 + (size_t)kHistBins * T;
  uint2* pairs = reinterpret_cast<uint2*>(rec + (size_t)kRec * T);  // 8-byte aligned: even word count
  cudaMemsetAsync(ws, 0, sizeof(uint32_t) * (2 * (size_t)kHistBins + kRec) * (size_t)T, s);
  const dim3 grid((npos + kPassChunk - 1) / kPassChunk, T);
  hist_pass_kernel<0><<<grid, kPassThreads, 0, s>>>(scores, ld, ids, P, n, L, topk, hist0, rec);
  hist_pass_kernel<1><<<grid, kPassThreads, 0, s>>>(scores, ld, ids, P, n, L, topk, hist1, rec);
  partition_kernel<<<grid, kPassThreads, 0, s>>>(scores, ld, ids, P, n, L, topk, rec, pairs, npos, idx, score_opt);
  const size_t smem = sizeof(uint2) * (size_t)kResolveSmemItems;
  cudaFuncSetAttribute(resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  resolve_kernel<<<T, kResolveThreads, smem, s>>>(n, L, ids != nullptr, topk, rec, pairs, npos, idx, score_opt);
}

size_t topk_cand_smem(int P) { return sizeof(uint32_t) * 2 * (size_t)(P + P / 32 + 2); }

void launch_topk_cand(const float* F, const int32_t* cand, const int32_t* n, int T, int L, int P, int topk,
                      int32_t* idx, float* score_opt, cudaStream_t s) {
  if (T <= 0) return;
  const size_t smem = topk_cand_smem(P);
  cudaFuncSetAttribute(select_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  select_small_kernel<<<T, kSmallThreads, smem, s>>>(F, cand, n, L, P, topk, idx, score_opt);
}

}  // namespace misa
