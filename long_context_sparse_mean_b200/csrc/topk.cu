// Top-k selection.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", Technical Summary,
// "Methodology: MISA", "Sparse Token Scoring": the final top-k tokens are selected on the reduced
// scores; "Hierarchical Variant (MISA-dagger)": the k' candidates are narrowed to the top-k by
// their dense scores.  Rule: score descending, exact ties to the lower token id (select.cuh).
//
// Rows of scores (one per query; a position p is token p, or token ids[p] for candidate lists),
// one CTA per row (row_topk_kernel), exact; the selected set's order in the output is not
// specified.  The candidates of a row (the entries that can still be selected) reach a list in
// shared memory in one of two ways:
//   * from the row: a sampled cut, then one pass that gathers the entries at or above it;
//   * from a candidate list built beforehand, copied in: for a few long rows, one CTA per row
//     places the row's cut from the same sample (list_cut_kernel) and CTAs over chunks of 8192
//     scores append the entries at or above it (list_sweep_kernel), so the pass over the row runs
//     on every SM instead of one per row.
// Candidate lists without score rows (the fused prefill scorer's) are ranked one warp per row
// (list_select_warp_kernel).
// The list is then ranked by rounds of 4096-bin histograms over what is left of its key range,
// which find the k-th key exactly; one pass writes the selection.  A row whose
// candidates cannot be trusted to hold the selection takes an exact path over the whole row.
// select_small_kernel ranks a short candidate list entirely in one CTA's shared memory; it needs
// no workspace (used by the entry point without allocation).
#include "kernels.cuh"
#include "mma_frag.cuh"
#include "select.cuh"
#include "warp_select.cuh"

namespace misa {

namespace {

constexpr int kSmallThreads = 1024;
constexpr int kRowKernelMinRows = 256;  // from this many rows on, 2 row CTAs per SM
constexpr int kRowListLarge = 16384;    // list of the 1024-thread row kernel (128 KB)
static_assert(kRowListLarge >= kListCap, "the decode candidate lists fit the row kernel's list");

__device__ __forceinline__ int padded(int e) { return e + (e >> 5); }

// ---- one CTA per row ----------------------------------------------------------------------------
//
// Each row (a query's scores over its prefix, or over a list of candidate tokens) is handled by
// one CTA: 512 threads, 2 CTAs per SM and an 8192-entry list for many rows (prefill chunks);
// 1024 threads, 1 CTA per SM and a 16384-entry list for a few long rows (decode), for candidate
// lists and for rows whose candidates the scoring kernel already gathered:
//   1. candidates: rows with a candidate list (list_cut_kernel and list_sweep_kernel, below: every
//      score at or above the row's cut key) copy the entries at or above the cut key in.  Otherwise rows longer than the
//      list are sampled (256 evenly spaced runs of 8 scores, 2048 keys) and a 4096-bin histogram
//      over the sampled key range places the sample key whose rank is the expected sample count
//      above the k-th key plus three standard deviations and a margin; the lower edge of its bin
//      is the threshold value (shorter rows take every entry), and one pass appends (key, token)
//      of every entry at or above it to the list (a bit mask per 16 entries a thread, one warp
//      scan and one shared atomic per warp and step), tracking the smallest and largest key;
//   2. selection (select_list_exact): rounds of 4096 bins over what is left of the list's key range
//      find the k-th key; exact ties there go to the lower tokens; one pass writes the selection.
// Whenever the list holds at least k keys and every entry at or above its cut, it holds every
// selected key, so the result is exact.  Otherwise (fewer than k at or above the cut, or more than
// the list holds) a score row takes the exact path: full level-0 histogram of the row, keys above
// the boundary bucket written out, the bucket's keys ranked (from global memory if they overflow
// the list).  Candidate lists always fit the list.

constexpr int kRowSegments = kSampleRuns;   // sample runs per long row
constexpr int kRowSegLen = kSampleRunLen;   // scores per run (one 32-byte sector)
constexpr int kSweepBatch = 8;              // float4 loads in flight per thread (exact path)

struct SmemPairs {
  const uint2* p;
  __device__ uint32_t key(int i) const { return p[i].x; }
  __device__ uint32_t id(int i) const { return p[i].y; }
  __device__ float value(int i) const { return key_to_float(p[i].x); }
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

// Appends (key, token p) of every entry p < np of a score row whose score is >= thr to the list and
// folds the appended keys into mm[0] (min) and mm[1] (max).  A thread reads 16 entries (4 float4) a
// step, the next step's loads in flight while it handles the current one, and marks its candidates
// in a bit mask; one warp scan and one shared atomic per warp and step place them.  The lanes then
// take their candidates one per round (lowest set bit, its value picked from the 16 by a select
// tree), as many rounds as the lane with the most candidates needs, which for a sampled cut is two
// or three instead of a pass over all 16 bits.
template <int NT>
__device__ __forceinline__ void collect_above(const float* row, int np, bool vec, float thr, uint2* list, int cap,
                                              uint32_t* cnt, uint32_t* mm) {
  constexpr int U = 4;  // float4 per thread and step
  const int lane = threadIdx.x & 31;
  uint32_t lo = 0xffffffffu, hi = 0u;
  auto load = [&](int j0, float4 (&x)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = (j0 + u) * NT + (int)threadIdx.x;
      if (vec && 4 * i + 3 < np) {
        x[u] = __ldcg(reinterpret_cast<const float4*>(row) + i);
      } else {
        float v[4] = {NAN, NAN, NAN, NAN};  // NaN: never at or above the threshold
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * i + e < np) v[e] = __ldcg(row + 4 * i + e);
        x[u] = make_float4(v[0], v[1], v[2], v[3]);
      }
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
    uint32_t pos = base + incl - c;
    const uint32_t rounds = __reduce_max_sync(0xffffffffu, c);
    for (uint32_t r = 0; r < rounds; ++r) {
      if (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1u;
        // entry b: float4 b >> 2, component b & 3
        const float4 q = (b & 8) ? ((b & 4) ? cur[3] : cur[2]) : ((b & 4) ? cur[1] : cur[0]);
        const float v = (b & 2) ? ((b & 1) ? q.w : q.z) : ((b & 1) ? q.y : q.x);
        const uint32_t k = order_key(v);
        lo = min(lo, k);
        hi = max(hi, k);
        const uint32_t tok = (uint32_t)(4 * ((j0 + (b >> 2)) * NT + (int)threadIdx.x) + (b & 3));
        if (pos < (uint32_t)cap) list[pos] = make_uint2(k, tok);
        ++pos;
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

// The r-th largest (1 <= r <= count) of the keys the block's threads visit, all within [lo, hi]:
// rounds of 4096 key bins over what is left of the range until a bin holds exactly the missing
// count (*all = true: every key of the bin is taken; the result is the bin's lower edge) or is one
// key wide (*all = false: the result is that key).  each(g) calls g(key, counted) for every member
// on the calling thread.  *above: the count of keys above the result's bin.  hist: kHistBins
// words; scratch: 35 words.
template <class Each>
__device__ __forceinline__ uint32_t block_rth_largest(Each each, uint32_t lo, uint32_t hi, uint32_t r, uint32_t* hist,
                                                      uint32_t* scratch, uint32_t* above, bool* all) {
  uint32_t gt = 0;
  uint32_t base = lo, range = hi - lo;
  for (;;) {
    const int sh = range >= (uint32_t)kHistBins ? 32 - __clz(range) - 12 : 0;
    for (int b = threadIdx.x; b < kHistBins; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    each([&](uint32_t v, bool counted) {
      if (counted && v >= base && v - base <= range) atomicAdd(&hist[(v - base) >> sh], 1u);
    });
    __syncthreads();
    const Bucket bk = block_bucket_bits(hist, kHistBins, 0, 0u, r, scratch);  // bin in prefix
    gt += r - bk.need;
    r = bk.need;
    const uint32_t edge = base + (bk.prefix << sh);
    if (bk.eq == r || sh == 0) {
      *above = gt;
      *all = bk.eq == r;
      return edge;
    }
    range = min(range - (bk.prefix << sh), (1u << sh) - 1u);
    base = edge;
  }
}

// Top `need` of the c list entries (c >= need, keys within [lo, hi]) in shared memory, handed to
// emit(slot, i, entry) (list entry i goes to output slot < need; every slot once, in no particular
// order).  Rounds of 4096 bins narrow a key interval [ilo, ihi]
// that holds the need-th entry: the first round bins the keys themselves when they share one sign
// (order keys are close to logarithmic in the score, so outliers do not crowd the bulk into a few
// bins) and bins linearly in the score otherwise; later rounds bin the interval's keys.  Once the
// interval holds at most 256 entries (or one key), one pass writes every entry above it and moves
// the interval's entries and their list indices into the histogram's words (hist: 16-byte
// aligned), where a rank count (score, then token) places them.  An exact tie of more than 1365
// entries at one key takes the lowest tokens by a search over the tokens.  The list is only read.  ctr: 2 words; mm: 2 words;
// scratch: 35 words.
template <int NT, class Emit>
__device__ void select_list_exact_emit(const uint2* list, int c, uint32_t need, uint32_t lo, uint32_t hi,
                                       uint32_t* hist, uint32_t* ctr, uint32_t* mm, uint32_t* scratch, Emit emit) {
  constexpr uint32_t kRank = 256;            // interval entries a rank count orders
  constexpr uint32_t kBuf = kHistBins / 3;   // (key, token) pairs and their list indices the histogram holds
  const int tid = threadIdx.x;
  uint32_t ilo = lo, ihi = hi, r = need, eq = (uint32_t)c;
  const bool one_sign = lo >= 0x80000000u || hi < 0x80000000u;
  for (int round = 0; round < 4 && eq > kRank && ihi > ilo; ++round) {
    const float vlo = key_to_float(ilo);
    const float scale = (float)kHistBins / (key_to_float(ihi) - vlo);
    const bool lin = round == 0 && !one_sign && scale > 0.f && scale < 3.0e38f;
    const uint32_t range = ihi - ilo;
    const int sh = range >= (uint32_t)kHistBins ? 32 - __clz(range) - 12 : 0;
    auto bin_of = [&](uint32_t k) { return lin ? linear_bin(k, vlo, scale) : (k - ilo) >> sh; };
    for (int b = tid; b < kHistBins; b += NT) hist[b] = 0;
    __syncthreads();
    for (int i = tid; i < c; i += NT) {
      const uint32_t k = list[i].x;
      if (k >= ilo && k <= ihi) atomicAdd(&hist[bin_of(k)], 1u);
    }
    __syncthreads();
    const Bucket bk = block_bucket_bits(hist, kHistBins, 0, 0u, r, scratch);  // bin in prefix
    r = bk.need;
    eq = bk.eq;
    if (lin) {  // the bin's key range (linear_bin is monotone)
      if (tid == 0) {
        mm[0] = 0xffffffffu;
        mm[1] = 0u;
      }
      __syncthreads();
      uint32_t blo = 0xffffffffu, bhi = 0u;
      for (int i = tid; i < c; i += NT) {
        const uint32_t k = list[i].x;
        if (k >= ilo && k <= ihi && bin_of(k) == bk.prefix) {
          blo = min(blo, k);
          bhi = max(bhi, k);
        }
      }
      block_min_max(blo, bhi, mm);
      __syncthreads();
      ilo = mm[0];
      ihi = mm[1];
      __syncthreads();
    } else {
      const uint32_t base = ilo + (bk.prefix << sh);
      ihi = min(ihi, base + ((1u << sh) - 1u));
      ilo = base;
    }
  }
  const uint32_t n_gt = need - r;  // entries above the interval, all taken
  if (eq <= kBuf) {
    uint2* bl = reinterpret_cast<uint2*>(hist);
    uint32_t* bi = hist + 2 * kBuf;
    if (tid == 0) {
      ctr[0] = 0;
      ctr[1] = 0;
    }
    __syncthreads();
    const int steps = (c + NT - 1) / NT;
    for (int j = 0; j < steps; ++j) {
      const int i = j * NT + tid;
      const uint2 e = i < c ? list[i] : make_uint2(0u, 0u);
      const bool gt = i < c && e.x > ihi, in = i < c && e.x >= ilo && e.x <= ihi;
      const uint32_t slot = warp_slot(gt, &ctr[0]);
      if (gt) emit(slot, (uint32_t)i, e);
      const uint32_t s2 = warp_slot(in, &ctr[1]);
      if (in) {
        bl[s2] = e;
        bi[s2] = (uint32_t)i;
      }
    }
    __syncthreads();
    for (uint32_t j = tid; j < eq; j += NT) {
      const uint2 m = bl[j];
      uint32_t rk = 0;
      for (uint32_t i = 0; i < eq; ++i) {
        const uint2 o = bl[i];
        rk += (o.x > m.x) || (o.x == m.x && o.y < m.y);
      }
      if (rk < r) emit(n_gt + rk, bi[j], m);
    }
    return;
  }
  // more than kBuf entries share the key ilo == ihi: the r lowest tokens among them, as the largest
  // values of 0xffffffff - token
  if (tid == 0) {
    mm[0] = 0xffffffffu;
    mm[1] = 0u;
  }
  __syncthreads();
  uint32_t tlo = 0xffffffffu, thi = 0u;
  for (int i = tid; i < c; i += NT)
    if (list[i].x == ilo) {
      tlo = min(tlo, 0xffffffffu - list[i].y);
      thi = max(thi, 0xffffffffu - list[i].y);
    }
  block_min_max(tlo, thi, mm);
  __syncthreads();
  tlo = mm[0];
  thi = mm[1];
  uint32_t a2;
  bool all2;
  const uint32_t tok = 0xffffffffu - block_rth_largest(
                                         [&](auto g) {
                                           for (int i = tid; i < c; i += NT) {
                                             const uint2 e = list[i];
                                             g(0xffffffffu - e.y, e.x == ilo);
                                           }
                                         },
                                         tlo, thi, r, hist, scratch, &a2, &all2);
  if (tid == 0) ctr[0] = 0;
  __syncthreads();
  const int steps = (c + NT - 1) / NT;
  for (int j = 0; j < steps; ++j) {
    const int i = j * NT + tid;
    const uint2 e = i < c ? list[i] : make_uint2(0u, 0u);
    const bool sel = i < c && (e.x > ihi || (e.x == ilo && e.y <= tok));
    const uint32_t slot = warp_slot(sel, &ctr[0]);
    if (sel) emit(slot, (uint32_t)i, e);
  }
}

// select_list_exact_emit writing token and value: oi[slot] (and ov[slot]).
template <int NT>
__device__ void select_list_exact(const uint2* list, int c, uint32_t need, uint32_t lo, uint32_t hi, uint32_t* hist,
                                  uint32_t* ctr, uint32_t* mm, uint32_t* scratch, int32_t* oi, float* ov) {
  select_list_exact_emit<NT>(list, c, need, lo, hi, hist, ctr, mm, scratch, [&](uint32_t slot, uint32_t, uint2 e) {
    oi[slot] = (int32_t)e.y;
    if (ov) ov[slot] = key_to_float(e.x);
  });
}

// Exact top-k of the score row [0, nt) by one CTA (tie: lower token): a full level-0 histogram of
// the keys, the keys above the boundary bucket written out, the bucket's keys ranked from the list
// (or from global memory when they overflow it).  Slots past the selection get -1 (and 0).
// list: LIST entries; hp: kHistPadded words; cnt: 2 words; scratch: 35 words.
template <int NT, int LIST>
__device__ void row_exact_topk(const float* row, int nt, bool vec, int topk, uint2* list, uint32_t* hp, uint32_t* cnt,
                               uint32_t* scratch, int32_t* oi, float* ov) {
  const int tid = threadIdx.x;
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

// Rows of scores [T, ld]; ids == nullptr: entry p < n_t is token p; otherwise entry p < P is token
// ids[t P + p] (empty when outside [0, n_t)), and P <= LIST.  lists (optional): the candidate lists
// a scoring kernel appended, [T][lcap] (key, token) with lcnt[t] entries (kNoList: the row has
// none) and every key at or above lcut[t] among them; a row whose list has at least
// min(topk, n_t) entries at or above lcut[t] and lost none past lcap is selected from those
// entries.  Any other row takes the exact path over its scores, or, with no score rows behind the
// lists (scores == nullptr), is left unselected with redo[t] = n_t (redo[t] = 0 for the rows
// answered).  only (optional): rows with only[t] <= 0 are skipped and keep their outputs.
template <int NT, int LIST, int MINB>
__global__ void __launch_bounds__(NT, MINB) row_topk_kernel(const float* __restrict__ scores, int64_t ld,
                                                            const int32_t* __restrict__ ids_all, int P,
                                                            const int32_t* __restrict__ n, int L, int topk,
                                                            int32_t* __restrict__ idx, float* __restrict__ score_opt,
                                                            const uint2* __restrict__ lists,
                                                            const uint32_t* __restrict__ lcnt,
                                                            const uint32_t* __restrict__ lcut, int lcap,
                                                            int64_t lstride, int32_t* __restrict__ redo,
                                                            const int32_t* __restrict__ only) {
  extern __shared__ uint2 list[];  // [LIST]
  __shared__ __align__(16) uint32_t hp[kHistPadded];
  __shared__ uint32_t scratch[35];
  __shared__ uint32_t cnt[2];
  __shared__ uint32_t mm[2];
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (only && only[t] <= 0) return;
  const int nt = clamp_len(n[t], L);
  const float* row = scores ? scores + (int64_t)t * ld : nullptr;
  const int32_t* ids = ids_all ? ids_all + (int64_t)t * P : nullptr;
  const int np = ids ? P : nt;  // entries of the row
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  const int tid = threadIdx.x;
  if (!ids && nt <= topk && row) {  // every prefix token is selected
    for (int a = tid; a < topk; a += NT) {
      oi[a] = a < nt ? a : -1;
      if (ov) ov[a] = a < nt ? row[a] : 0.f;
    }
    return;
  }
  const bool vec = row && (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  if (tid < 2) cnt[tid] = 0;
  if (tid == 0) {
    mm[0] = 0xffffffffu;
    mm[1] = 0u;
  }

  // ---- 1. candidates ----
  // the answer needs min(topk, n_t) entries (a prefix of at most topk keys is selected whole)
  const uint32_t need = (uint32_t)((!ids && nt < topk) ? nt : topk);
  bool exact = false, listed = false;
  uint32_t c_in = 0;
  if (lists) {
    c_in = __ldcg(lcnt + t);
    if (c_in != kNoList) {
      listed = c_in >= need && c_in <= (uint32_t)min(lcap, LIST);
      exact = !listed;  // too few entries, or entries dropped past the list's end
    }
  }
  if (listed) {  // copy the list in: every entry of a built list is at or above the row's cut
    const uint2* src = lists + (int64_t)t * lstride;
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (uint32_t i0 = 0; i0 < c_in; i0 += 4 * NT) {
      uint2 e[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t i = i0 + u * NT + tid;
        e[u] = i < c_in ? __ldcg(src + i) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t i = i0 + u * NT + tid;
        if (i < c_in) {
          list[i] = e[u];
          lo = min(lo, e[u].x);
          hi = max(hi, e[u].x);
        }
      }
    }
    if (tid == 0) cnt[0] = c_in;
    block_min_max(lo, hi, mm);
    __syncthreads();
  } else if (!exact) {
    float thr = -INFINITY;
    constexpr int ns = kRowSegments * kRowSegLen;
    const uint32_t rank = sample_rank(topk, np);
    if (np > LIST && rank > (uint32_t)ns) {
      exact = true;  // k close to n_t: the sample cannot place the cut
      __syncthreads();
    } else if (np > LIST) {
      const int seg = (np / kRowSegments) & ~(kRowSegLen - 1);  // >= 32 here
      constexpr int per = ns / NT;
      uint32_t sk[per];
#pragma unroll
      for (int u = 0; u < per; ++u) {
        const int i = u * NT + tid;
        sk[u] = order_key(__ldcg(row + (int64_t)(i / kRowSegLen) * seg + (i % kRowSegLen)));
      }
      __syncthreads();  // mm initialised
      thr = sample_cut<per>(sk, rank, hp, mm, scratch);
    } else {
      __syncthreads();
    }
    if (!exact && ids) {  // P <= LIST (checked on the host)
      // a candidate list: every entry with a valid token is kept; four entries a thread and step,
      // one block scan places a step's entries (no per-entry atomics or reloads)
      uint32_t lo = 0xffffffffu, hi = 0u, base = 0;
      const bool vec4 = vec && (reinterpret_cast<uintptr_t>(ids) & 15) == 0;
      for (int p0 = 0; p0 < np; p0 += 4 * NT) {
        const int p = p0 + 4 * tid;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        int32_t id[4] = {-1, -1, -1, -1};
        if (vec4 && p + 3 < np) {
          const float4 x = __ldcg(reinterpret_cast<const float4*>(row + p));
          const int4 y = __ldcg(reinterpret_cast<const int4*>(ids + p));
          v[0] = x.x, v[1] = x.y, v[2] = x.z, v[3] = x.w;
          id[0] = y.x, id[1] = y.y, id[2] = y.z, id[3] = y.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (p + e < np) {
              v[e] = __ldcg(row + p + e);
              id[e] = __ldcg(ids + p + e);
            }
        }
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) m |= (uint32_t)(id[e] >= 0 && id[e] < nt) << e;
        uint32_t total;
        uint32_t pos = base + block_exclusive_scan((uint32_t)__popc(m), scratch, &total);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((m >> e) & 1u) {
            const uint32_t k = order_key(v[e]);
            lo = min(lo, k);
            hi = max(hi, k);
            list[pos++] = make_uint2(k, (uint32_t)id[e]);
          }
        base += total;
      }
      if (tid == 0) cnt[0] = base;
      block_min_max(lo, hi, mm);
    } else if (!exact) {
      collect_above<NT>(row, np, vec, thr, list, LIST, &cnt[0], mm);
    }
  } else {
    __syncthreads();
  }
  if (redo && tid == 0) redo[t] = exact ? nt : 0;
  if (exact && !row) return;  // no score rows behind the list: the caller redoes this row

  // ---- 2. selection from the candidates ----
  if (!exact) {
    __syncthreads();
    const uint32_t c = cnt[0];
    if ((!listed || need < (uint32_t)topk) && np <= LIST && c <= (uint32_t)topk) {  // every entry is selected
      for (uint32_t i = tid; i < (uint32_t)topk; i += NT) {
        oi[i] = i < c ? (int32_t)list[i].y : -1;
        if (ov) ov[i] = i < c ? key_to_float(list[i].x) : 0.f;
      }
      return;
    }
    if (c >= (uint32_t)topk && c <= (uint32_t)LIST) {
      const uint32_t lo = mm[0], hi = mm[1];
      __syncthreads();  // mm is reused as scratch
      select_list_exact<NT>(list, (int)c, (uint32_t)topk, lo, hi, hp, cnt, mm, scratch, oi, ov);
      return;  // c >= topk entries: every slot is filled
    }
    __syncthreads();
  }

  // ---- exact path (score rows only) ----
  row_exact_topk<NT, LIST>(row, nt, vec, topk, list, hp, cnt, scratch, oi, ov);
}

template <int NT, int LIST, int MINB>
void launch_row_topk(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T, int L,
                     int topk, int32_t* idx, float* score_opt, const ListState* lst, const int32_t* only,
                     cudaStream_t s) {
  const size_t smem = sizeof(uint2) * (size_t)LIST;
  cudaFuncSetAttribute(row_topk_kernel<NT, LIST, MINB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(row_topk_kernel<NT, LIST, MINB>, T, NT, smem, s, scores, ld, ids, P, n, L, topk, idx, score_opt,
                                                      lst ? lst->list : nullptr, lst ? lst->cnt : nullptr,
                                                      lst ? lst->cutkey : nullptr, lst ? lst->cap : 0,
                                                      lst ? lst->stride : 0, lst ? lst->redo : nullptr, only);
}

// ---- candidate lists of long score rows --------------------------------------------------------

constexpr int kCutThreads = 1024;
constexpr int kSweepThreads = 256;
constexpr int kSweepPer = 32;                              // scores per thread (8 x float4)
constexpr int kSweepChunk = kSweepThreads * kSweepPer;     // 8192 scores per CTA

// One CTA per row: the row's cut from the same sample the row kernel takes (256 evenly spaced runs
// of 8 scores; rank: the expected sample count above the k-th score plus three standard
// deviations and a margin), as an order key in lcut[t], and lcnt[t] = 0.  Rows of at most cap
// entries, rows whose sample cannot place the cut and rows whose list is not expected to fit get
// no list (lcnt[t] = kNoList) and take the row kernel's own path.
__global__ void __launch_bounds__(kCutThreads) list_cut_kernel(const float* __restrict__ scores, int64_t ld,
                                                                const int32_t* __restrict__ n, int L, int topk,
                                                                int cap, uint32_t* __restrict__ lcnt,
                                                                uint32_t* __restrict__ lcut) {
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scratch[35];
  __shared__ uint32_t mm[2];
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  const int nt = clamp_len(n[t], L);
  constexpr int ns = kSampleRuns * kSampleRunLen;
  const uint32_t rank = sample_rank(topk, nt);
  // the list is expected to hold about rank / ns of the row; keep a tenth of the cap in reserve
  if (nt <= cap || rank > (uint32_t)ns || (double)rank * nt > 0.9 * (double)cap * ns) {
    if (threadIdx.x == 0) lcnt[t] = kNoList;
    return;
  }
  const float* row = scores + (int64_t)t * ld;
  const int seg = (nt / kSampleRuns) & ~(kSampleRunLen - 1);
  constexpr int per = ns / kCutThreads;
  uint32_t sk[per];
#pragma unroll
  for (int u = 0; u < per; ++u) {
    const int i = u * kCutThreads + (int)threadIdx.x;
    sk[u] = order_key(__ldcg(row + (int64_t)(i / kSampleRunLen) * seg + (i % kSampleRunLen)));
  }
  if (threadIdx.x == 0) {
    mm[0] = 0xffffffffu;
    mm[1] = 0u;
  }
  __syncthreads();
  const float thr = sample_cut<per>(sk, rank, hist, mm, scratch);
  if (threadIdx.x == 0) {
    lcnt[t] = 0u;
    lcut[t] = order_key(thr);
  }
}

// One CTA per (chunk of 8192 scores, row): every entry at or above the row's cut goes to the row's
// list; one block scan and one atomic per CTA place them (entries past cap are counted, not
// written).  Scores are compared as floats with the cut's value (the same order as their keys).
__global__ void __launch_bounds__(kSweepThreads, 4) list_sweep_kernel(const float* __restrict__ scores, int64_t ld,
                                                                      const int32_t* __restrict__ n, int L,
                                                                      uint2* __restrict__ lists, int64_t stride,
                                                                      uint32_t* __restrict__ lcnt,
                                                                      const uint32_t* __restrict__ lcut, int cap) {
  __shared__ uint32_t scratch[35];
  __shared__ uint32_t sbase;
  const int t = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int nt = clamp_len(n[t], L);
  const int s0 = blockIdx.x * kSweepChunk;
  if (s0 >= nt || __ldcg(lcnt + t) == kNoList) return;  // uniform across the block
  const int len = min(kSweepChunk, nt - s0);
  const float* row = scores + (int64_t)t * ld + s0;
  const float thr = key_to_float(__ldcg(lcut + t));
  const int tid = threadIdx.x;
  // element 4 (u * 256 + tid) + e of the chunk is v[4 u + e] and bit 4 u + e of the mask
  float v[kSweepPer];
  if (len == kSweepChunk && (reinterpret_cast<uintptr_t>(row) & 15) == 0) {
#pragma unroll
    for (int u = 0; u < kSweepPer / 4; ++u) {
      const float4 x = __ldcg(reinterpret_cast<const float4*>(row) + u * kSweepThreads + tid);
      v[4 * u] = x.x;
      v[4 * u + 1] = x.y;
      v[4 * u + 2] = x.z;
      v[4 * u + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kSweepPer; ++i) {
      const int p = 4 * ((i >> 2) * kSweepThreads + tid) + (i & 3);
      v[i] = p < len ? __ldcg(row + p) : -INFINITY;  // never at or above a cut of a finite score
    }
  }
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < kSweepPer; ++i) m |= (uint32_t)(v[i] >= thr) << i;
  uint32_t total;
  uint32_t slot = block_exclusive_scan((uint32_t)__popc(m), scratch, &total);
  if (tid == 0) sbase = total ? atomicAdd(lcnt + t, total) : 0u;
  __syncthreads();
  if (!m) return;
  slot += sbase;
  uint2* lt = lists + (int64_t)t * stride;
#pragma unroll
  for (int i = 0; i < kSweepPer; ++i)
    if ((m >> i) & 1u) {
      if (slot < (uint32_t)cap)
        lt[slot] = make_uint2(order_key(v[i]), (uint32_t)(s0 + 4 * ((i >> 2) * kSweepThreads + tid) + (i & 3)));
      ++slot;
    }
}

// One warp per row: the top-k of the row's candidate list (warp_list_select).  A row without a
// list, whose list lost entries past cap, or whose list holds fewer than min(k, n_t) entries at or
// above its cut gets redo[t] = n_t and no output; the others redo[t] = 0.
__global__ void __launch_bounds__(32 * kSelWarps, 3) list_select_warp_kernel(const int32_t* __restrict__ n, int L, int T,
                                                                          int topk, const uint2* __restrict__ lists,
                                                                          int64_t stride, int cap,
                                                                          const uint32_t* __restrict__ lcnt,
                                                                          const uint32_t* __restrict__ lcut,
                                                                          int32_t* __restrict__ redo,
                                                                          int32_t* __restrict__ idx,
                                                                          float* __restrict__ score_opt,
                                                                          const float* __restrict__ lhi) {
  __shared__ uint32_t hist[kSelWarps][kWarpBinWords];
  __shared__ uint2 bnd[kSelWarps][kWarpBound];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelWarps + warp;
  if (t >= T) return;  // uniform across the warp
  const int nt = clamp_len(n[t], L);
  const uint32_t c = __ldcg(lcnt + t);
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  if (nt == 0) {  // empty prefix: nothing to select
    for (int a = lane; a < topk; a += 32) {
      oi[a] = -1;
      if (ov) ov[a] = 0.f;
    }
    if (lane == 0) redo[t] = 0;
    return;
  }
  bool ok = c <= (uint32_t)cap;  // kNoList, or entries lost past cap: redone
  if (ok) {
    const uint2* lt = lists + (int64_t)t * stride;
    const uint32_t cut = __ldcg(lcut + t), need = (uint32_t)min(topk, nt);
    // two passes when the list's score range is known (a cut placed from a sample), else the
    // general rounds
    int r = 2;
    if (lhi && cut != 0u && cut != 0xffffffffu)
      r = warp_list_select_binned(lt, (int)c, cut, key_to_float(cut), __ldcg(lhi + t), need, topk, hist[warp],
                                  bnd[warp], oi, ov);
    ok = r == 1 || (r == 2 && warp_list_select(lt, (int)c, cut, need, topk, hist[warp], oi, ov));
  }
  if (lane == 0) redo[t] = ok ? 0 : nt;
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

// Candidate-list state of one selection (kernels.cuh): cnt [T] and cutkey [T] in one piece, then
// list [T][kListCap] (key, token); each piece 256-byte aligned.
namespace {
size_t al(size_t x) { return (x + 255) / 256 * 256; }
}  // namespace

size_t list_state_bytes(int T, int cap) {
  if (T <= 0) return 0;
  return al(sizeof(uint32_t) * 2 * (size_t)T) + al(sizeof(int32_t) * (size_t)T) + al(sizeof(uint2) * (size_t)T * cap);
}

ListState list_state(void* ws, int T, int topk, int cap) {
  char* p = static_cast<char*>(ws);
  ListState l;
  l.cnt = reinterpret_cast<uint32_t*>(p);
  l.cutkey = l.cnt + T;
  p += al(sizeof(uint32_t) * 2 * (size_t)T);
  l.redo = reinterpret_cast<int32_t*>(p);
  p += al(sizeof(int32_t) * (size_t)T);
  l.list = reinterpret_cast<uint2*>(p);
  // many rows take the 512-thread row kernel, whose list holds 8192 entries
  l.cap = T >= kRowKernelMinRows && cap > 8192 ? 8192 : cap;
  l.stride = cap;
  l.topk = topk;
  return l;
}

bool launch_list_build(const float* scores, int64_t ld, const int32_t* n, int T, int L, const ListState& l,
                       cudaStream_t s) {
  if (T <= 0) return false;
  // lists pay off for a few rows longer than the row kernel's own list: the pass over each row is
  // spread over every SM instead of one CTA per row; many rows fill the GPU with row CTAs already
  // (measured: lists built for prefill chunks of 4096 rows were slower than the row kernel alone)
  if (T >= kRowKernelMinRows || L <= l.cap) {
    mark_no_lists(l, T, s);
    return false;
  }
  launch_pdl(list_cut_kernel, T, kCutThreads, 0, s, scores, ld, n, L, l.topk, l.cap, l.cnt, l.cutkey);
  const int chunks = (L + kSweepChunk - 1) / kSweepChunk;
  launch_pdl(list_sweep_kernel, dim3(chunks, T), kSweepThreads, 0, s, scores, ld, n, L, l.list, l.stride, l.cnt,
             l.cutkey, l.cap);
  return true;
}

void launch_list_select_warp(const int32_t* n, int T, int L, int topk, const ListState& l, int32_t* idx,
                             float* score_opt, cudaStream_t s, const float* hi) {
  if (T <= 0) return;
  list_select_warp_kernel<<<(T + kSelWarps - 1) / kSelWarps, 32 * kSelWarps, 0, s>>>(
      n, L, T, topk, l.list, l.stride, l.cap, l.cnt, l.cutkey, l.redo, idx, score_opt, hi);
}

void mark_no_lists(const ListState& l, int T, cudaStream_t s) {
  if (T > 0) cudaMemsetAsync(l.cnt, 0xff, sizeof(uint32_t) * (size_t)T, s);
}

// ---- MISA-dagger selection over dense lists -----------------------------------------------------

// One CTA per row: the top-k' of the row's dense list by the routed score (ties to the lower token),
// then the top-k of those by their dense score.  Both selections stay in shared memory: the list's
// entries and dense scores are copied in, the first selection marks its entries, one compaction
// pass rewrites the marked ones as (dense score key, token) in place, and the second selection
// writes the output.  A row its list cannot answer (no list, fewer than k' entries, entries lost
// past the cap) takes the exact top-k' of its routed score row (into ctok, [T][kp] scratch) and
// scores those candidates with all H_I heads here (as the scorer does: one warp per 16 candidates
// on the tensor cores).
template <int NT, int LIST>
__global__ void __launch_bounds__(NT, 1)
    hier_select_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n, int L, int kp,
                       int topk, DenseList dl, const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                       const __nv_bfloat16* __restrict__ k, int64_t k_seq_stride, int H_I, int32_t* __restrict__ ctok,
                       int32_t* __restrict__ idx, float* __restrict__ score_opt) {
  extern __shared__ uint2 list[];                                    // [LIST]
  float* fl = reinterpret_cast<float*>(list + LIST);                 // [LIST] dense scores
  uint32_t* mark = reinterpret_cast<uint32_t*>(fl + LIST);           // [LIST / 32] selected entries
  __shared__ __align__(16) uint32_t hp[kHistPadded];
  __shared__ uint32_t scratch[35];
  __shared__ uint32_t cnt[2];
  __shared__ uint32_t mm[2];
  const int t = blockIdx.x, tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const int nt = clamp_len(n[t], L);
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  const int c1 = min(kp, nt);  // candidates
  const uint32_t c_in = __ldcg(dl.cnt + t);
  const bool listed = c_in != kNoList && c_in >= (uint32_t)kp && c_in <= (uint32_t)min(dl.cap, LIST);
  if (tid == 0) {
    mm[0] = 0xffffffffu;
    mm[1] = 0u;
  }

  // ---- 1. the k' candidates as (dense score key, token) in list[0, c1) ----
  if (listed) {
    const uint2* src = dl.list + (int64_t)t * dl.stride;
    const float* fsrc = dl.f + (int64_t)t * dl.stride;
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (uint32_t i = tid; i < c_in; i += NT) {
      const uint2 e = __ldcg(src + i);
      list[i] = e;
      fl[i] = __ldcg(fsrc + i);
      lo = min(lo, e.x);
      hi = max(hi, e.x);
    }
    for (uint32_t i = tid; i < (c_in + 31) / 32; i += NT) mark[i] = 0u;
    block_min_max(lo, hi, mm);
    __syncthreads();
    lo = mm[0];
    hi = mm[1];
    __syncthreads();  // mm is reused as scratch
    select_list_exact_emit<NT>(list, (int)c_in, (uint32_t)kp, lo, hi, hp, cnt, mm, scratch,
                               [&](uint32_t, uint32_t i, uint2) { atomicOr(&mark[i >> 5], 1u << (i & 31)); });
    __syncthreads();
    // compaction in place, NT entries a step: every entry moves down (or stays), so a step only
    // overwrites entries its threads have read (the barrier between reads and writes)
    uint32_t base = 0;
    for (uint32_t i0 = 0; i0 < c_in; i0 += NT) {
      const uint32_t i = i0 + tid;
      const bool sel = i < c_in && ((mark[i >> 5] >> (i & 31)) & 1u);
      const uint2 e = sel ? list[i] : make_uint2(0u, 0u);
      const float v = sel ? fl[i] : 0.f;
      uint32_t total;
      const uint32_t pos = base + block_exclusive_scan((uint32_t)sel, scratch, &total);
      __syncthreads();
      if (sel) list[pos] = make_uint2(order_key(v), e.y);
      base += total;
    }
  } else {
    int32_t* ct = ctok + (int64_t)t * kp;
    if (nt <= kp) {
      for (int p = tid; p < nt; p += NT) ct[p] = p;
    } else {
      const float* row = scores + (int64_t)t * ld;
      const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
      row_exact_topk<NT, LIST>(row, nt, vec, kp, list, hp, cnt, scratch, ct, nullptr);
    }
    const int ngf = (H_I + 7) / 8;
    uint2(*frag)[8][32] = reinterpret_cast<uint2(*)[8][32]>(fl);  // the dense-score array is free here
    float* wall = reinterpret_cast<float*>(fl) + ngf * 8 * 32 * 2;
    stage_all_head_frags<NT>(frag, q + (int64_t)t * H_I * kD, H_I, ngf);
    for (int e = tid; e < ngf * 8; e += NT) wall[e] = e < H_I ? w[(int64_t)t * H_I + e] : 0.f;
    __syncthreads();  // the candidates are written (global memory, this block) and the heads staged
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
    const __nv_bfloat16* kt = k + (int64_t)t * k_seq_stride;
    for (int s0 = warp * 16; s0 < c1; s0 += (NT / 32) * 16) {
      const int ra = s0 + g < c1 ? __ldcg(ct + s0 + g) : -1;
      const int rb = s0 + g + 8 < c1 ? __ldcg(ct + s0 + g + 8) : -1;
      uint4 A[4], B[4];
      load_rows(ra >= 0 && ra < nt ? kt + (int64_t)ra * kD : nullptr, rb >= 0 && rb < nt ? kt + (int64_t)rb * kD : nullptr,
                c, A, B);
      float flo, fhi;
      score_rows_rt(A, B, frag, wall, ngf, lane, flo, fhi);
      if (c == 0 && s0 + g < c1) list[s0 + g] = make_uint2(order_key(flo), (uint32_t)ra);
      if (c == 1 && s0 + g + 8 < c1) list[s0 + g + 8] = make_uint2(order_key(fhi), (uint32_t)rb);
    }
  }
  __syncthreads();

  // ---- 2. the top-k of the candidates by the dense score ----
  if (tid == 0) {
    mm[0] = 0xffffffffu;
    mm[1] = 0u;
  }
  uint32_t lo = 0xffffffffu, hi = 0u;
  for (int i = tid; i < c1; i += NT) {
    lo = min(lo, list[i].x);
    hi = max(hi, list[i].x);
  }
  block_min_max(lo, hi, mm);
  __syncthreads();
  if (c1 <= topk) {  // every candidate is selected
    for (int i = tid; i < topk; i += NT) {
      oi[i] = i < c1 ? (int32_t)list[i].y : -1;
      if (ov) ov[i] = i < c1 ? key_to_float(list[i].x) : 0.f;
    }
    return;
  }
  lo = mm[0];
  hi = mm[1];
  __syncthreads();  // mm is reused as scratch
  select_list_exact<NT>(list, c1, (uint32_t)topk, lo, hi, hp, cnt, mm, scratch, oi, ov);
}

void launch_list_cut(const float* scores, int64_t ld, const int32_t* n, int T, int L, int topk, int cap,
                     uint32_t* lcnt, uint32_t* lcut, cudaStream_t s) {
  if (T <= 0) return;
  launch_pdl(list_cut_kernel, T, kCutThreads, 0, s, scores, ld, n, L, topk, cap, lcnt, lcut);
}

void launch_hier_select(const float* scores, int64_t ld, const int32_t* n, int T, int L, int kp, int topk,
                        const DenseList& dl, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                        int H_I, int32_t* ctok, int32_t* idx, float* score_opt, cudaStream_t s) {
  if (T <= 0) return;
  constexpr int NT = 1024, LIST = kRowListLarge;
  const size_t smem = (sizeof(uint2) + sizeof(float)) * (size_t)LIST + sizeof(uint32_t) * (LIST / 32);
  cudaFuncSetAttribute(hier_select_kernel<NT, LIST>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(hier_select_kernel<NT, LIST>, T, NT, smem, s, scores, ld, n, L, kp, topk, dl,
             static_cast<const __nv_bfloat16*>(q), w, static_cast<const __nv_bfloat16*>(k), k_seq_stride, H_I, ctok,
             idx, score_opt);
}

void launch_topk_rows(const float* scores, int64_t ld, const int32_t* ids, int P, const int32_t* n, int T, int L,
                      int topk, const ListState* lst, int32_t* idx, float* score_opt, cudaStream_t s,
                      const int32_t* only) {
  if (T <= 0) return;
  if (!ids && (!lst || lst->cap <= 8192) && T >= kRowKernelMinRows)
    launch_row_topk<512, 8192, 2>(scores, ld, nullptr, 0, n, T, L, topk, idx, score_opt, lst, only, s);
  else
    launch_row_topk<1024, kRowListLarge, 1>(scores, ld, ids, P, n, T, L, topk, idx, score_opt, lst, only, s);
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
