// Top-k selection.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", Technical Summary,
// "Methodology: MISA", "Sparse Token Scoring": the final top-k tokens are selected on the reduced
// scores; "Hierarchical Variant (MISA-dagger)": the k' candidates are narrowed to the top-k by
// their dense scores.  Rule: score descending, exact ties to the lower token id (select.cuh).
//
// Rows of scores (one per query; a position p is token p, or token ids[p] for candidate lists).
// Two ways, both exact; the selected set's order in the output is not specified:
//   * one CTA per row (row_topk_kernel, the default): a sampled cut, one pass that gathers the
//     entries at or above it into shared memory, a selection there; an exact path for rows the
//     sample cannot place (described with the kernel below);
//   * after a level-0 histogram (4096 buckets of key bits 31..20 per row, and the bucket holding
//     the k-th key) that the decode scoring kernel builds while it writes the scores (the CTA that
//     finishes a row's last tile finds the bucket), or that hist_pass_kernel builds in a pass
//     over the rows with the same last-CTA rule:
//       partition: keys above the bucket are written out directly (slots reserved with one atomic
//       per CTA), the bucket's keys go to a (key, id) list;
//       resolve: one CTA per row ranks that list on the remaining 20 key bits and, for exact ties,
//       on the token id, in shared memory (straight from global memory if the list is too long).
// select_small_kernel ranks a short candidate list entirely in one CTA's shared memory; it needs
// no workspace (used by the entry point without allocation).
#include "kernels.cuh"
#include "select.cuh"

namespace misa {

namespace {

constexpr int kPassThreads = 256;
constexpr int kRowItems = 16;   // positions per thread for score rows (4096 per CTA)
constexpr int kListItems = 4;   // for candidate lists (1024 per CTA: more CTAs on short lists)
constexpr int kResolveSmemItems = 24576;  // boundary pairs ranked in shared memory (192 KB)
constexpr int kSmallThreads = 1024;
constexpr int kRec = 8;  // words of per-row state
constexpr int kRowKernelMinRows = 256;  // from this many rows on, 2 row CTAs per SM
constexpr int kRowListLarge = 16384;    // list of the 1024-thread row kernel (128 KB)

// Per-row state rec[t][kRec] (kRec and the meaning of words 0, 2, 3 are shared with the scoring
// kernel that builds the histogram):
//   0: tiles or CTAs that have added to the histogram
//   2: level-0 boundary prefix (bits 31..20; 0xffffffff: no valid key)   3: keys needed from it
//   6: slots filled by keys above the boundary   7: boundary pairs written

__device__ __forceinline__ int padded(int e) { return e + (e >> 5); }

// The row positions handled by one thread of a pass CTA: ITEMS/4 groups of 4 consecutive positions.
template <int ITEMS>
struct RowSlice {
  static constexpr int kChunk = kPassThreads * ITEMS;
  const float* row;
  const int32_t* ids;  // null: token = position
  int s1, nt;
  bool vec;
  __device__ int pos(int base, int item) const {
    return base + 4 * ((int)threadIdx.x + (item >> 2) * kPassThreads) + (item & 3);
  }
  __device__ void load(int base, float (&v)[ITEMS], uint32_t (&key)[ITEMS], bool (&ok)[ITEMS]) const {
#pragma unroll
    for (int j = 0; j < ITEMS / 4; ++j) {
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
    for (int i = 0; i < ITEMS; ++i) {
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

// Level-0 histogram pass; the row's last CTA turns the histogram into the boundary.
template <int ITEMS>
__global__ void __launch_bounds__(kPassThreads) hist_pass_kernel(const float* __restrict__ scores, int64_t ld,
                                                                 const int32_t* __restrict__ ids, int P,
                                                                 const int32_t* __restrict__ n, int L, int topk,
                                                                 uint32_t* __restrict__ hist, uint32_t* __restrict__ rec) {
  __shared__ uint32_t h[kHistPadded];
  __shared__ uint32_t scratch[35];
  __shared__ int last;
  const int t = blockIdx.y;
  const int nt = clamp_len(n[t], L);
  const int npos = ids ? P : nt;
  if (!ids && npos <= topk) return;  // the whole prefix is selected
  constexpr int kChunk = RowSlice<ITEMS>::kChunk;
  const int nchunks = (npos + kChunk - 1) / kChunk;
  const int base = blockIdx.x * kChunk;
  if (base >= npos) return;
  uint32_t* rt = rec + (int64_t)t * kRec;
  uint32_t* ht = hist + (int64_t)t * kHistBins;
  for (int b = threadIdx.x; b < kHistPadded; b += kPassThreads) h[b] = 0;
  const RowSlice<ITEMS> rs{scores + (int64_t)t * ld, ids ? ids + (int64_t)t * P : nullptr, min(base + kChunk, npos),
                           nt, (ld % 4) == 0};
  float v[ITEMS];
  uint32_t key[ITEMS];
  bool ok[ITEMS];
  rs.load(base, v, key, ok);
  __syncthreads();
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) hist_add(h, (uint32_t)hpad((int)(key[i] >> 20)), ok[i]);
  __syncthreads();
  for (int b = threadIdx.x; b < kHistBins; b += kPassThreads)
    if (h[hpad(b)]) atomicAdd(ht + b, h[hpad(b)]);
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // cumulative: orders the whole CTA's adds before the count
    last = atomicAdd(rt, 1u) == (uint32_t)(nchunks - 1);
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  const Bucket bk = level0_boundary<kPassThreads>(ht, (uint32_t)topk, h, scratch);
  if (threadIdx.x == 0) {
    rt[2] = bk.prefix;
    rt[3] = bk.need;
  }
}

template <int ITEMS>
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
  constexpr int kChunk = RowSlice<ITEMS>::kChunk;
  const int base = blockIdx.x * kChunk;
  if (base >= npos) return;
  uint32_t* rt = rec + (int64_t)t * kRec;
  const uint32_t b0 = __ldcg(rt + 2);
  const bool none = b0 == 0xffffffffu;  // no valid key at all
  const uint32_t prefix = b0 >> 20;
  const RowSlice<ITEMS> rs{row, ids ? ids + (int64_t)t * P : nullptr, min(base + kChunk, npos), nt, (ld % 4) == 0};
  float v[ITEMS];
  uint32_t key[ITEMS];
  bool ok[ITEMS];
  rs.load(base, v, key, ok);
  uint32_t gtm = 0, eqm = 0;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    gtm |= (uint32_t)(!none && ok[i] && (key[i] >> 20) > prefix) << i;
    eqm |= (uint32_t)(!none && ok[i] && (key[i] >> 20) == prefix) << i;
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
  for (int i = 0; i < ITEMS; ++i) {
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
  __device__ float value(int i) const { return key_to_float(p[i].x); }
};

// One CTA per row: slots [n_out, n_out + need) come from the boundary pairs; the rest of the row
// after the selection is padded with -1.
template <int NT>
__global__ void __launch_bounds__(NT) resolve_kernel(const int32_t* __restrict__ n, int L, bool lists,
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
  const uint32_t need = min(__ldcg(rt + 3), (uint32_t)c);
  const uint32_t prefix = __ldcg(rt + 2);
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  const uint2* pt = pairs + (int64_t)t * pairs_ld;
  const uint32_t kk = min((uint32_t)topk, n_out + need);
  if ((uint32_t)c <= need) {
    for (int i = threadIdx.x; i < c; i += NT)
      if (n_out + i < (uint32_t)topk) {
        oi[n_out + i] = (int32_t)pt[i].y;
        if (ov) ov[n_out + i] = key_to_float(pt[i].x);
      }
  } else if (c <= kResolveSmemItems) {
#pragma unroll 8
    for (int i = threadIdx.x; i < c; i += NT) list[i] = pt[i];
    __syncthreads();
    const PairList acc{list};
    const SelectResult r = radix_select_items(acc, c, need, 1, prefix, 0xfff00000u, hist, scratch);
    write_selection(acc, c, r, false, oi + n_out, ov ? ov + n_out : nullptr, need, scratch);
  } else {
    const PairList acc{pt};
    const SelectResult r = radix_select_items(acc, c, need, 1, prefix, 0xfff00000u, hist, scratch);
    write_selection(acc, c, r, false, oi + n_out, ov ? ov + n_out : nullptr, need, scratch);
  }
  for (int a = (int)kk + threadIdx.x; a < topk; a += NT) {
    oi[a] = -1;
    if (ov) ov[a] = 0.f;
  }
}

// ---- one CTA per row ----------------------------------------------------------------------------
//
// Each row (a query's scores over its prefix, or over a list of candidate tokens) is read once by
// its CTA: 512 threads, 2 CTAs per SM and an 8192-entry list for many rows (prefill chunks);
// 1024 threads, 1 CTA per SM and a 16384-entry list for a few long rows (decode) and for
// candidate lists:
//   1. cut: rows longer than the list are sampled (256 evenly spaced runs of 8 scores, 2048
//      keys); a 4096-bin histogram over the sampled key range places the sample key whose rank
//      is the expected sample count above the k-th key plus three standard deviations and a
//      margin, and the lower edge of its bin is the threshold value; shorter rows take every
//      entry;
//   2. one pass appends (key, token) of every entry at or above the threshold to the list (a bit
//      mask per 16 entries a thread, one warp scan and one shared atomic per warp and step) and
//      tracks the smallest and largest key;
//   3. the list's keys are rewritten relative to the smallest so that they spread over the high
//      bits (same order); one 4096-bin histogram finds the bucket of the k-th key; keys above it
//      go straight to the output, the bucket's keys are ranked by one warp (when at most 32) or
//      on the remaining bits, and, for exact ties, on the token.
// Whenever the list holds at least k keys it holds every selected key, so the result is exact.
// Otherwise (fewer than k at or above the cut, or more than the list holds) a score row takes the
// exact path: full level-0 histogram of the row, keys above the boundary bucket written out, the
// bucket's keys ranked as above (from global memory if they overflow the list).  Candidate lists
// always fit the list.

constexpr int kRowSegments = 256;  // sample runs per long row
constexpr int kRowSegLen = 8;      // scores per run (one 32-byte sector)
constexpr int kSweepBatch = 8;     // float4 loads in flight per thread (exact path)

struct SmemPairs {
  const uint2* p;
  __device__ uint32_t key(int i) const { return p[i].x; }
  __device__ uint32_t id(int i) const { return p[i].y; }
  __device__ float value(int i) const { return key_to_float(p[i].x); }
};

// A shared-memory list whose keys were rewritten as 0x80000000 | ((key - lo) << sh): the same
// order, spread over the high bits.
struct ShiftedPairs {
  const uint2* p;
  uint32_t lo;
  int sh;
  __device__ uint32_t key(int i) const { return p[i].x; }
  __device__ uint32_t id(int i) const { return p[i].y; }
  __device__ float value(int i) const { return key_to_float(((p[i].x & 0x7fffffffu) >> sh) + lo); }
};

// The row in global memory restricted to one level-0 bucket (other keys read as absent).
struct RowBucket {
  const float* row;
  uint32_t prefix;
  __device__ uint32_t key(int i) const {
    const uint32_t k = order_key(__ldcg(row + i));
    return (k & 0xfff00000u) == prefix ? k : 0u;
  }
  __device__ uint32_t id(int i) const { return (uint32_t)i; }
  __device__ float value(int i) const { return __ldcg(row + i); }
};

// Slot for every lane whose `take` is set, counted by *cnt (one shared atomic per warp).
__device__ __forceinline__ uint32_t warp_slot(bool take, uint32_t* cnt) {
  const unsigned m = __ballot_sync(0xffffffffu, take);
  if (m == 0u) return 0u;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(m) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(cnt, (uint32_t)__popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  return base + (uint32_t)__popc(m & ((1u << lane) - 1u));
}

// Visits positions [0, nt) of a score row, four per step, with all lanes of every warp taking the
// same number of steps (f gets position, key and a validity flag).  Loads are issued kSweepBatch
// steps ahead of their use.  Used by the exact path only.
template <int NT, class F>
__device__ __forceinline__ void row_sweep(const float* row, int nt, bool vec, F&& f) {
  if (vec) {
    const int n4 = (nt + 3) / 4;
    const int steps = (n4 + NT - 1) / NT;
    for (int j0 = 0; j0 < steps; j0 += kSweepBatch) {
      float4 x[kSweepBatch];
#pragma unroll
      for (int u = 0; u < kSweepBatch; ++u) {
        const int i = (j0 + u) * NT + (int)threadIdx.x;
        x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (4 * i + 3 < nt) {
          x[u] = __ldcg(reinterpret_cast<const float4*>(row) + i);
        } else if (4 * i < nt) {
          x[u].x = __ldcg(row + 4 * i);
          if (4 * i + 1 < nt) x[u].y = __ldcg(row + 4 * i + 1);
          if (4 * i + 2 < nt) x[u].z = __ldcg(row + 4 * i + 2);
        }
      }
#pragma unroll
      for (int u = 0; u < kSweepBatch; ++u) {
        if (j0 + u >= steps) break;  // uniform across the block
        const int i = (j0 + u) * NT + (int)threadIdx.x;
        const float v[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int s = 4 * i + e;
          f(s, order_key(v[e]), s < nt);
        }
      }
    }
  } else {
    const int steps = (nt + NT - 1) / NT;
    for (int j = 0; j < steps; ++j) {
      const int s = j * NT + (int)threadIdx.x;
      const float v = s < nt ? __ldcg(row + s) : 0.f;
      f(s, order_key(v), s < nt);
    }
  }
}

// Appends (key, token) of every entry p < np whose score is >= thr to the list and folds the
// appended keys into mm[0] (min) and mm[1] (max).  The token is p, or ids[p] for candidate lists
// (entries whose id is outside [0, nt) are skipped).  A thread reads 16 entries (4 float4) a
// step, the next step's loads in flight while it handles the current one, and marks its
// candidates in a bit mask; one warp scan and one shared atomic per warp and step place them.
template <int NT>
__device__ __forceinline__ void collect_above(const float* row, const int32_t* ids, int np, int nt, bool vec,
                                              float thr, uint2* list, int cap, uint32_t* cnt, uint32_t* mm) {
  constexpr int U = 4;  // float4 per thread and step
  const int lane = threadIdx.x & 31;
  uint32_t lo = 0xffffffffu, hi = 0u;
  auto load = [&](int j0, float4 (&x)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = (j0 + u) * NT + (int)threadIdx.x;
      float v[4] = {NAN, NAN, NAN, NAN};  // NaN: never at or above the threshold
      if (vec && 4 * i + 3 < np) {
        const float4 f = __ldcg(reinterpret_cast<const float4*>(row) + i);
        v[0] = f.x;
        v[1] = f.y;
        v[2] = f.z;
        v[3] = f.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * i + e < np) v[e] = __ldcg(row + 4 * i + e);
      }
      if (ids) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int p = 4 * i + e;
          const int32_t id = p < np ? __ldcg(ids + p) : -1;
          if (id < 0 || id >= nt) v[e] = NAN;
        }
      }
      x[u] = make_float4(v[0], v[1], v[2], v[3]);
    }
  };
  const int steps = ((np + 3) / 4 + NT - 1) / NT;  // float4 groups a thread
  float4 cur[U], nxt[U];
  load(0, cur);
  for (int j0 = 0; j0 < steps; j0 += U) {
    if (j0 + U < steps) load(j0 + U, nxt);
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      m |= (uint32_t)(cur[u].x >= thr) << (4 * u);
      m |= (uint32_t)(cur[u].y >= thr) << (4 * u + 1);
      m |= (uint32_t)(cur[u].z >= thr) << (4 * u + 2);
      m |= (uint32_t)(cur[u].w >= thr) << (4 * u + 3);
    }
    const uint32_t c = (uint32_t)__popc(m);
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    uint32_t base = 0;
    if (lane == 31 && incl) base = atomicAdd(cnt, incl);
    base = __shfl_sync(0xffffffffu, base, 31);
    if (m) {
      uint32_t pos = base + incl - c;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int s0 = 4 * ((j0 + u) * NT + (int)threadIdx.x);
        const float v[4] = {cur[u].x, cur[u].y, cur[u].z, cur[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if ((m >> (4 * u + e)) & 1u) {
            const uint32_t k = order_key(v[e]);
            lo = min(lo, k);
            hi = max(hi, k);
            const uint32_t tok = ids ? (uint32_t)__ldcg(ids + s0 + e) : (uint32_t)(s0 + e);
            if (pos < (uint32_t)cap) list[pos] = make_uint2(k, tok);
            ++pos;
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) cur[u] = nxt[u];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0 && hi >= lo) {
    atomicMin(&mm[0], lo);
    atomicMax(&mm[1], hi);
  }
}

// Ranks n <= 32 entries of list (keys descending, then tokens ascending) in one warp and writes
// the first `need` to oi/ov at their rank.
template <class Acc>
__device__ __forceinline__ void warp_rank_write(const uint2* list, int n, uint32_t need, const Acc& acc, int32_t* oi,
                                                float* ov) {
  const int lane = threadIdx.x & 31;
  const bool mine = lane < n;
  const uint2 e = mine ? list[lane] : make_uint2(0u, 0xffffffffu);
  uint32_t rank = 0;
  for (int j = 0; j < n; ++j) {
    const uint32_t kj = __shfl_sync(0xffffffffu, e.x, j);
    const uint32_t ij = __shfl_sync(0xffffffffu, e.y, j);
    rank += (kj > e.x) || (kj == e.x && ij < e.y);
  }
  if (mine && rank < need) {
    oi[rank] = (int32_t)e.y;
    if (ov) ov[rank] = acc.value(lane);
  }
}

// Top `need` of the c list entries (c >= need), keys spread (ShiftedPairs, bit 31 set): written
// to oi/ov [0, need).  One histogram of key bits 30..19; keys above the boundary bucket go out
// directly, the bucket's entries move to the front of the list and are ranked (one warp when
// they are few).  hist: kHistBins words; ctr: 2 words; scratch: 35 words.
template <int NT, int LIST>
__device__ void select_list(uint2* list, int c, uint32_t need, uint32_t lo, int sh, uint32_t* hist, uint32_t* ctr,
                            uint32_t* scratch, int32_t* oi, float* ov) {
  const int tid = threadIdx.x;
  for (int b = tid; b < kHistBins; b += NT) hist[b] = 0;
  if (tid < 2) ctr[tid] = 0;
  __syncthreads();
  for (int i = tid; i < c; i += NT) hist_add(hist, (list[i].x >> 19) & 4095u, true);
  __syncthreads();
  const Bucket bk = block_bucket_bits(hist, kHistBins, 19, 0x80000000u, need, scratch);
  const uint32_t pb = bk.prefix >> 19;
  const ShiftedPairs acc{list, lo, sh};
  constexpr int kPer = LIST / NT;
  uint2 keep[kPer];
  int nk = 0;
  const int steps = (c + NT - 1) / NT;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (j >= steps) break;  // uniform
    const int i = j * NT + tid;
    const uint2 e = i < c ? list[i] : make_uint2(0u, 0u);
    const bool gt = i < c && (e.x >> 19) > pb;
    const uint32_t slot = warp_slot(gt, &ctr[0]);
    if (gt) {
      oi[slot] = (int32_t)e.y;
      if (ov) ov[slot] = acc.value(i);
    }
    const bool eq = i < c && (e.x >> 19) == pb;
    if (eq) keep[nk] = e;
    nk += eq;
  }
  __syncthreads();  // every entry read
  uint32_t total;
  const uint32_t off = block_exclusive_scan((uint32_t)nk, scratch, &total);
  for (int x = 0; x < kPer; ++x)
    if (x < nk) list[off + x] = keep[x];
  __syncthreads();
  const uint32_t n_gt = ctr[0];
  const uint32_t need2 = need - n_gt;
  if (total <= need2) {
    for (uint32_t i = tid; i < total; i += NT) {
      oi[n_gt + i] = (int32_t)list[i].y;
      if (ov) ov[n_gt + i] = acc.value((int)i);
    }
  } else if (total <= 32) {
    if (tid < 32) warp_rank_write(list, (int)total, need2, acc, oi + n_gt, ov ? ov + n_gt : nullptr);
  } else {
    const SelectResult r =
        radix_select_items(acc, (int)total, need2, 1, bk.prefix & 0xfff00000u, 0xfff00000u, hist, scratch);
    write_selection(acc, (int)total, r, false, oi + n_gt, ov ? ov + n_gt : nullptr, need2, scratch);
  }
}

// Rows of scores [T, ld]; ids == nullptr: entry p < n_t is token p; otherwise entry p < P is token
// ids[t P + p] (empty when outside [0, n_t)), and P <= LIST.
template <int NT, int LIST, int MINB>
__global__ void __launch_bounds__(NT, MINB) row_topk_kernel(const float* __restrict__ scores, int64_t ld,
                                                            const int32_t* __restrict__ ids_all, int P,
                                                            const int32_t* __restrict__ n, int L, int topk,
                                                            int32_t* __restrict__ idx, float* __restrict__ score_opt) {
  extern __shared__ uint2 list[];  // [LIST]
  __shared__ uint32_t hp[kHistPadded];
  __shared__ uint32_t scratch[35];
  __shared__ uint32_t cnt[2];
  __shared__ uint32_t mm[2];
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const float* row = scores + (int64_t)t * ld;
  const int32_t* ids = ids_all ? ids_all + (int64_t)t * P : nullptr;
  const int np = ids ? P : nt;  // entries of the row
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  const int tid = threadIdx.x;
  if (!ids && nt <= topk) {  // every prefix token is selected
    for (int a = tid; a < topk; a += NT) {
      oi[a] = a < nt ? a : -1;
      if (ov) ov[a] = a < nt ? row[a] : 0.f;
    }
    return;
  }
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  if (tid < 2) cnt[tid] = 0;
  if (tid == 0) {
    mm[0] = 0xffffffffu;
    mm[1] = 0u;
  }

  // ---- 1. the cut ----
  bool exact = false;
  float thr = -INFINITY;
  constexpr int ns = kRowSegments * kRowSegLen;
  // expected sample count above the k-th key, plus three standard deviations and a margin
  const float mean = (float)topk * (float)ns / (float)max(np, 1);
  const uint32_t rank = (uint32_t)(mean + 3.f * sqrtf(mean) + 8.f);
  if (np > LIST && rank > (uint32_t)ns) {
    exact = true;  // k close to n_t: the sample cannot place the cut
    __syncthreads();
  } else if (np > LIST) {
    const int seg = (np / kRowSegments) & ~(kRowSegLen - 1);  // >= 32 here
    constexpr int per = ns / NT;
    uint32_t sk[per];
    uint32_t slo = 0xffffffffu, shi = 0u;
#pragma unroll
    for (int u = 0; u < per; ++u) {
      const int i = u * NT + tid;
      sk[u] = order_key(__ldcg(row + (int64_t)(i / kRowSegLen) * seg + (i % kRowSegLen)));
      slo = min(slo, sk[u]);
      shi = max(shi, sk[u]);
    }
    for (int b = tid; b < kHistBins; b += NT) hp[b] = 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      slo = min(slo, __shfl_xor_sync(0xffffffffu, slo, o));
      shi = max(shi, __shfl_xor_sync(0xffffffffu, shi, o));
    }
    __syncthreads();  // mm initialised
    if ((tid & 31) == 0) {
      atomicMin(&mm[0], slo);
      atomicMax(&mm[1], shi);
    }
    __syncthreads();
    // 4096 bins over the sampled key range
    slo = mm[0];
    const uint32_t srange = mm[1] - slo;
    const int ssh = srange >= 4096u ? 32 - __clz(srange) - 12 : 0;
#pragma unroll
    for (int u = 0; u < per; ++u) hist_add(hp, (sk[u] - slo) >> ssh, true);
    __syncthreads();
    const Bucket cut = block_bucket_bits(hp, kHistBins, ssh, 0u, rank, scratch);
    // keys >= slo + cut.prefix are the scores >= this value
    thr = key_to_float(slo + cut.prefix);
    if (tid == 0) {
      mm[0] = 0xffffffffu;
      mm[1] = 0u;
    }
    __syncthreads();
  } else {
    __syncthreads();
  }

  // ---- 2-3. candidates and their selection ----
  if (!exact) {
    collect_above<NT>(row, ids, np, nt, vec, thr, list, LIST, &cnt[0], mm);
    __syncthreads();
    const uint32_t c = cnt[0];
    if (np <= LIST && c <= (uint32_t)topk) {  // every valid entry is selected
      for (uint32_t i = tid; i < (uint32_t)topk; i += NT) {
        oi[i] = i < c ? (int32_t)list[i].y : -1;
        if (ov) ov[i] = i < c ? key_to_float(list[i].x) : 0.f;
      }
      return;
    }
    if (c >= (uint32_t)topk && c <= (uint32_t)LIST) {
      const uint32_t lo = mm[0], range = mm[1] - mm[0];
      if (__clz(range) > 0) {
        const int sh = range ? __clz(range) - 1 : 31;
        for (uint32_t i = tid; i < c; i += NT) list[i].x = 0x80000000u | ((list[i].x - lo) << sh);
        __syncthreads();
        select_list<NT, LIST>(list, (int)c, (uint32_t)topk, lo, sh, hp, cnt, scratch, oi, ov);
      } else {  // the keys span more than half the key range: rank them as they are
        const SmemPairs acc{list};
        const SelectResult r = radix_select_items(acc, (int)c, (uint32_t)topk, 0, 0u, 0u, hp, scratch);
        write_selection(acc, (int)c, r, false, oi, ov, (uint32_t)topk, scratch);
      }
      return;  // c >= topk entries: every slot is filled
    }
    __syncthreads();
  }

  // ---- exact path (score rows only): full level-0 histogram, boundary bucket, rank the bucket ----
  uint32_t kk = 0;  // slots filled
  for (int b = tid; b < kHistPadded; b += NT) hp[b] = 0;
  if (tid < 2) cnt[tid] = 0;
  __syncthreads();
  row_sweep<NT>(row, nt, vec, [&](int s, uint32_t k, bool in) {
    (void)s;
    hist_add(hp, (uint32_t)hpad((int)(k >> 20)), in && k != 0u);
  });
  __syncthreads();
  uint32_t local = 0;
  for (int b = tid; b < kHistBins; b += NT) local += hp[hpad(b)];
  uint32_t total;
  block_exclusive_scan(local, scratch, &total);
  const uint32_t want = min((uint32_t)topk, total);
  if (want > 0) {
    const Bucket bk = bucket_search_padded(hp, want, scratch);
    const uint32_t pb = bk.prefix >> 20;
    // keys above the bucket straight to the output, the bucket's keys to the list
    row_sweep<NT>(row, nt, vec, [&](int s, uint32_t k, bool in) {
      const bool ok = in && k != 0u;
      const bool gt = ok && (k >> 20) > pb;
      const uint32_t slot = warp_slot(gt, &cnt[1]);
      if (gt && slot < (uint32_t)topk) {
        oi[slot] = s;
        if (ov) ov[slot] = key_to_float(k);
      }
      const bool eq = ok && (k >> 20) == pb;
      const uint32_t e = warp_slot(eq, &cnt[0]);
      if (eq && e < (uint32_t)LIST) list[e] = make_uint2(k, (uint32_t)s);
    });
    __syncthreads();
    const uint32_t n_gt = min(cnt[1], (uint32_t)topk);
    const uint32_t c = cnt[0];
    const uint32_t need = min(bk.need, want - n_gt);
    if (c <= (uint32_t)LIST) {
      const SmemPairs acc{list};
      if (c <= need) {
        for (uint32_t i = tid; i < c; i += NT) {
          oi[n_gt + i] = (int32_t)list[i].y;
          if (ov) ov[n_gt + i] = key_to_float(list[i].x);
        }
      } else {
        const SelectResult r = radix_select_items(acc, (int)c, need, 1, bk.prefix, 0xfff00000u, hp, scratch);
        write_selection(acc, (int)c, r, false, oi + n_gt, ov ? ov + n_gt : nullptr, need, scratch);
      }
    } else {
      const RowBucket acc{row, bk.prefix};
      const SelectResult r = radix_select_items(acc, nt, need, 1, bk.prefix, 0xfff00000u, hp, scratch);
      write_selection(acc, nt, r, false, oi + n_gt, ov ? ov + n_gt : nullptr, need, scratch);
    }
    kk = n_gt + need;
  }
  for (int a = (int)kk + tid; a < topk; a += NT) {
    oi[a] = -1;
    if (ov) ov[a] = 0.f;
  }
}

template <int NT, int LIST, int MINB>
void launch_row_topk(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T, int L,
                     int topk, int32_t* idx, float* score_opt, cudaStream_t s) {
  const size_t smem = sizeof(uint2) * (size_t)LIST;
  cudaFuncSetAttribute(row_topk_kernel<NT, LIST, MINB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  row_topk_kernel<NT, LIST, MINB><<<T, NT, smem, s>>>(scores, ld, ids, P, n, L, topk, idx, score_opt);
}

struct SmemItems {
  const uint32_t* keys;
  const uint32_t* ids;
  __device__ uint32_t key(int i) const { return keys[padded(i)]; }
  __device__ uint32_t id(int i) const { return ids[padded(i)]; }
  __device__ float value(int i) const { return key_to_float(keys[padded(i)]); }
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

// Workspace of one selection: hist [T][4096], rec [T][kRec], pairs [T][P] (uint2).
size_t topk_rows_ws(int T, int P) {
  return sizeof(uint32_t) * ((size_t)kHistBins + kRec) * (size_t)T + sizeof(uint2) * (size_t)T * P;
}

void topk_rows_prepare(void* ws, int T, cudaStream_t s) {
  if (T > 0) cudaMemsetAsync(ws, 0, sizeof(uint32_t) * ((size_t)kHistBins + kRec) * (size_t)T, s);
}

TopkFuse topk_rows_fuse(void* ws, int T, int topk) {
  uint32_t* hist = static_cast<uint32_t*>(ws);
  return TopkFuse{hist, hist + (size_t)kHistBins * T, topk};
}

void launch_topk_level0(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T, int L,
                        int topk, void* ws, cudaStream_t s) {
  if (T <= 0) return;
  const int npos = ids ? P : L;
  uint32_t* hist = static_cast<uint32_t*>(ws);
  uint32_t* rec = hist + (size_t)kHistBins * T;
  topk_rows_prepare(ws, T, s);
  if (ids) {
    constexpr int C = RowSlice<kListItems>::kChunk;
    hist_pass_kernel<kListItems><<<dim3((npos + C - 1) / C, T), kPassThreads, 0, s>>>(scores, ld, ids, P, n, L, topk,
                                                                                      hist, rec);
  } else {
    constexpr int C = RowSlice<kRowItems>::kChunk;
    hist_pass_kernel<kRowItems><<<dim3((npos + C - 1) / C, T), kPassThreads, 0, s>>>(scores, ld, ids, P, n, L, topk,
                                                                                     hist, rec);
  }
}

void launch_topk_rows(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T, int L,
                      int topk, void* ws, bool hist_ready, int32_t* idx, float* score_opt, cudaStream_t s) {
  if (T <= 0) return;
  if (!hist_ready) {  // one CTA per row
    if (ids) {
      if (P <= kRowListLarge) {
        launch_row_topk<1024, kRowListLarge, 1>(scores, ld, ids, P, n, T, L, topk, idx, score_opt, s);
        return;
      }
    } else if (T >= kRowKernelMinRows) {
      launch_row_topk<512, 8192, 2>(scores, ld, nullptr, 0, n, T, L, topk, idx, score_opt, s);
      return;
    } else {
      launch_row_topk<1024, kRowListLarge, 1>(scores, ld, nullptr, 0, n, T, L, topk, idx, score_opt, s);
      return;
    }
  }
  const int npos = ids ? P : L;
  uint32_t* hist = static_cast<uint32_t*>(ws);
  uint32_t* rec = hist + (size_t)kHistBins * T;
  uint2* pairs = reinterpret_cast<uint2*>(rec + (size_t)kRec * T);  // 8-byte aligned: even word count
  if (!hist_ready) launch_topk_level0(scores, ld, ids, P, n, T, L, topk, ws, s);
  const size_t smem = sizeof(uint2) * (size_t)kResolveSmemItems;
  if (ids) {
    constexpr int C = RowSlice<kListItems>::kChunk;
    partition_kernel<kListItems><<<dim3((npos + C - 1) / C, T), kPassThreads, 0, s>>>(
        scores, ld, ids, P, n, L, topk, rec, pairs, npos, idx, score_opt);
    cudaFuncSetAttribute(resolve_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    resolve_kernel<256><<<T, 256, smem, s>>>(n, L, true, topk, rec, pairs, npos, idx, score_opt);
  } else {
    constexpr int C = RowSlice<kRowItems>::kChunk;
    partition_kernel<kRowItems><<<dim3((npos + C - 1) / C, T), kPassThreads, 0, s>>>(
        scores, ld, ids, P, n, L, topk, rec, pairs, npos, idx, score_opt);
    cudaFuncSetAttribute(resolve_kernel<1024>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    resolve_kernel<1024><<<T, 1024, smem, s>>>(n, L, false, topk, rec, pairs, npos, idx, score_opt);
  }
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
