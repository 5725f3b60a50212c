// Device helpers of the top-k selection.
//
// Selection rule ("MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// Technical Summary, "Sparse Token Scoring" and "Hierarchical Variant (MISA-dagger)": keep the k
// best tokens): score descending, exact ties to the lower token id.  Scores become
// order-preserving 32-bit keys (common.cuh).  Radix levels, most significant first:
//   level 0: bits 31..20 (4096 buckets)   level 1: bits 19..10   level 2: bits 9..0
// and, when equal keys straddle the boundary, the same three levels on (0xffffffff - id), which
// ranks smaller ids higher.
#pragma once

#include "common.cuh"

namespace misa {

constexpr int kHistBins = 4096;

// Sampled cut of a long row: kSampleRuns evenly spaced runs of kSampleRunLen consecutive entries.
constexpr int kSampleRuns = 256;
constexpr int kSampleRunLen = 8;  // one 32-byte sector of fp32 scores
// Candidate lists the decode scoring kernel appends (entries per query), and the count that marks
// a row without one.
constexpr int kListCap = 16384;
constexpr uint32_t kNoList = 0xffffffffu;

__device__ __forceinline__ int level_shift(int l) { return l == 0 ? 20 : (l == 1 ? 10 : 0); }
__device__ __forceinline__ int level_bins(int l) { return l == 0 ? 4096 : 1024; }

struct Bucket {
  uint32_t prefix, need, eq;
};

// Histogram increment in shared memory.  A plain atomic per item: on B200 aggregating the lanes
// of a warp that share a bin with __match_any_sync first was three times slower on real score
// rows (22.7 us against 7.4 us for 32 x 131072 scores; the rows spread over ~70 buckets).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  if (active) atomicAdd(&hist[bin], 1u);
}

// Find the bucket (of nb bins holding key bits shift..) that holds the need-th largest key among
// those counted in hist[nb].  All threads of the block get the same answer.  `scratch` holds 32
// words of shared memory for the scan and 3 words for the answer.
__device__ __forceinline__ Bucket block_bucket_bits(const uint32_t* hist, int nb, int sh, uint32_t prefix,
                                                    uint32_t need, uint32_t* scratch) {
  const int per = (nb + (int)blockDim.x - 1) / (int)blockDim.x;
  uint32_t local = 0;
  for (int d = 0; d < per; ++d) {
    const int b = nb - 1 - ((int)threadIdx.x * per + d);
    if (b >= 0) local += hist[b];
  }
  uint32_t total;
  uint32_t cum = block_exclusive_scan(local, scratch, &total);
  for (int d = 0; d < per; ++d) {
    const int b = nb - 1 - ((int)threadIdx.x * per + d);
    if (b < 0) break;
    const uint32_t hb = hist[b];
    if (cum < need && cum + hb >= need) {
      scratch[32] = prefix | ((uint32_t)b << sh);
      scratch[33] = need - cum;
      scratch[34] = hb;
    }
    cum += hb;
  }
  __syncthreads();
  const Bucket r{scratch[32], scratch[33], scratch[34]};
  __syncthreads();
  return r;
}

// Shared-memory index of bin b in a padded histogram: one extra word per 16 bins, so threads that
// each read 16 contiguous bins hit different banks.
__device__ __forceinline__ int hpad(int b) { return b + (b >> 4); }
constexpr int kHistPadded = kHistBins + kHistBins / 16;

// Bucket search over a padded shared histogram of kHistBins bins (key bits 31..20): each thread
// owns kHistBins / blockDim contiguous bins (at most 16), read without bank conflicts.
__device__ __forceinline__ Bucket bucket_search_padded(const uint32_t* hp, uint32_t need, uint32_t* scratch) {
  const int per = kHistBins / (int)blockDim.x;
  uint32_t local = 0;
  for (int d = 0; d < per; ++d) local += hp[hpad(kHistBins - 1 - ((int)threadIdx.x * per + d))];
  uint32_t total;
  uint32_t cum = block_exclusive_scan(local, scratch, &total);
  for (int d = 0; d < per; ++d) {
    const int b = kHistBins - 1 - ((int)threadIdx.x * per + d);
    const uint32_t hb = hp[hpad(b)];
    if (cum < need && cum + hb >= need) {
      scratch[32] = (uint32_t)b << 20;
      scratch[33] = need - cum;
      scratch[34] = hb;
    }
    cum += hb;
  }
  __syncthreads();
  const Bucket r{scratch[32], scratch[33], scratch[34]};
  __syncthreads();
  return r;
}

// Level-0 boundary of one row from its complete global histogram hist_t[kHistBins]: returns
// (prefix of the bucket holding the k-th largest key, keys still needed from it).  With fewer
// than k counted keys every key is taken; with none the prefix is 0xffffffff.  hp: padded
// shared scratch of kHistPadded words.  Every thread of the block must call it.
template <int NT>  // = blockDim.x; every thread issues its loads of the histogram together
__device__ __forceinline__ Bucket level0_boundary(const uint32_t* hist_t, uint32_t topk, uint32_t* hp,
                                                  uint32_t* scratch) {
  constexpr int kPer = kHistBins / NT;
  uint32_t v[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) v[i] = __ldcg(hist_t + threadIdx.x + i * NT);
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    hp[hpad((int)threadIdx.x + i * NT)] = v[i];
    local += v[i];
  }
  uint32_t total;
  block_exclusive_scan(local, scratch, &total);  // also orders the stores above
  const uint32_t need = min(topk, total);
  if (need == 0) return Bucket{0xffffffffu, 0u, 0u};
  return bucket_search_padded(hp, need, scratch);
}

// Sample rank whose score cuts a row of np entries for a top-k: the expected number of samples
// above the k-th entry plus three standard deviations and a margin.  Above
// kSampleRuns * kSampleRunLen the sample cannot place the cut.
__host__ __device__ __forceinline__ uint32_t sample_rank(int topk, int np) {
  const float ns = (float)(kSampleRuns * kSampleRunLen);
  const float mean = (float)topk * ns / (float)(np > 1 ? np : 1);
  return (uint32_t)(mean + 3.f * sqrtf(mean) + 8.f);
}

// Smallest lo and largest hi over the block into mm[0] and mm[1], which hold 0xffffffff and 0 on
// entry.  Every thread calls it; it synchronises before its shared atomics, the caller after.
__device__ __forceinline__ void block_min_max(uint32_t lo, uint32_t hi, uint32_t* mm) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) {
    atomicMin(&mm[0], lo);
    atomicMax(&mm[1], hi);
  }
}

// Linear bin of an order key's score: 4096 bins over [vlo, vlo + 4096 / scale].  Non-decreasing in
// the score (the subtraction and the multiplication by a positive scale keep order under
// round-to-nearest), so every entry of a higher bin is at least every entry of a lower one.
__device__ __forceinline__ uint32_t linear_bin(uint32_t key, float vlo, float scale) {
  const float x = (key_to_float(key) - vlo) * scale;
  return (uint32_t)min(__float2int_rz(x), kHistBins - 1);
}

// Smallest key among the calling threads' keys that `take` accepts, over the block (0xffffffff for
// none).  mm[0] is used; every thread calls it.
template <class Each, class Take>
__device__ __forceinline__ uint32_t block_min_of(Each each, Take take, uint32_t* mm) {
  if (threadIdx.x == 0) mm[0] = 0xffffffffu;
  __syncthreads();
  uint32_t mn = 0xffffffffu;
  each([&](uint32_t k) {
    if (take(k)) mn = min(mn, k);
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  if ((threadIdx.x & 31) == 0) atomicMin(&mm[0], mn);
  __syncthreads();
  const uint32_t v = mm[0];
  __syncthreads();
  return v;
}

// Cut for the r-th largest of a set of keys spread over the block: each(f) calls f(key) for every
// key of the calling thread; lo and hi are the block's smallest and largest key.  Returns the
// smallest key of a narrow bin holding the r-th largest key, so at least r keys are at or above it
// and only that bin's keys beyond.  Round 1 bins the key range itself in 4096 bins: order keys are
// close to logarithmic in the score within one sign, so a few outliers (far larger scores) do not
// crowd the bulk of the set into a few bins.  When the boundary bin still holds more than 64 keys
// (scores of both signs put 8 bins in a factor of two), round 2 bins that bin's own score range
// linearly.  A set of one value returns lo, which keeps every key.  hist: 4096 words of shared
// memory; mm: 2 words; scratch: 35 words.  Every thread calls it.
template <class Each>
__device__ __forceinline__ uint32_t linear_cut(Each each, uint32_t lo, uint32_t hi, uint32_t r, uint32_t* hist,
                                               uint32_t* mm, uint32_t* scratch) {
  if (hi <= lo) return lo;
  const uint32_t range = hi - lo;
  const int sh = range >= 4096u ? 32 - __clz(range) - 12 : 0;
  for (int b = threadIdx.x; b < kHistBins; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  each([&](uint32_t k) { hist_add(hist, (k - lo) >> sh, true); });
  __syncthreads();
  const Bucket bk = block_bucket_bits(hist, kHistBins, sh, 0u, r, scratch);
  const uint32_t b = bk.prefix >> sh;
  auto in_bin = [&](uint32_t k) { return ((k - lo) >> sh) == b; };
  if (bk.eq <= 64u) return block_min_of(each, in_bin, mm);
  // round 2: the boundary bin's keys, 4096 bins linear in their score
  if (threadIdx.x == 0) {
    mm[0] = 0xffffffffu;
    mm[1] = 0u;
  }
  uint32_t blo = 0xffffffffu, bhi = 0u;
  each([&](uint32_t k) {
    if (in_bin(k)) {
      blo = min(blo, k);
      bhi = max(bhi, k);
    }
  });
  block_min_max(blo, bhi, mm);
  __syncthreads();
  blo = mm[0];
  bhi = mm[1];
  __syncthreads();
  const float vlo = key_to_float(blo), vhi = key_to_float(bhi);
  const float scale = (float)kHistBins / (vhi - vlo);
  if (!(vhi > vlo) || !(scale > 0.f) || !(scale < 3.0e38f)) return blo;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  each([&](uint32_t k) { hist_add(hist, linear_bin(k, vlo, scale), in_bin(k)); });
  __syncthreads();
  const uint32_t b2 = block_bucket_bits(hist, kHistBins, 0, 0u, bk.need, scratch).prefix;
  return block_min_of(each, [&](uint32_t k) { return in_bin(k) && linear_bin(k, vlo, scale) == b2; }, mm);
}

// Cut from a sample of keys: the smallest score of the narrow bin holding the rank-th largest
// sample key (linear_cut), so at least `rank` sample keys are at or above the returned value.  PER
// keys per thread; hist: 4096 words of shared memory; mm: 2 words holding 0xffffffff and 0 on entry
// (and again on return); scratch: 35 words.  Every thread calls it.
template <int PER>
__device__ __forceinline__ float sample_cut(const uint32_t (&sk)[PER], uint32_t rank, uint32_t* hist, uint32_t* mm,
                                            uint32_t* scratch);

__device__ __forceinline__ Bucket block_bucket(const uint32_t* hist, int lvl, uint32_t prefix, uint32_t need,
                                               uint32_t* scratch) {
  return block_bucket_bits(hist, level_bins(lvl), level_shift(lvl), prefix, need, scratch);
}

template <int PER>
__device__ __forceinline__ float sample_cut(const uint32_t (&sk)[PER], uint32_t rank, uint32_t* hist, uint32_t* mm,
                                            uint32_t* scratch) {
  uint32_t slo = 0xffffffffu, shi = 0u;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    slo = min(slo, sk[u]);
    shi = max(shi, sk[u]);
  }
  block_min_max(slo, shi, mm);
  __syncthreads();
  slo = mm[0];
  shi = mm[1];
  __syncthreads();
  const uint32_t cut = linear_cut(
      [&](auto f) {
#pragma unroll
        for (int u = 0; u < PER; ++u) f(sk[u]);
      },
      slo, shi, rank, hist, mm, scratch);
  if (threadIdx.x == 0) {
    mm[0] = 0xffffffffu;
    mm[1] = 0u;
  }
  __syncthreads();
  return key_to_float(cut);  // the scores >= this value are the keys >= cut
}

// Radix select over m items given by acc.key(i) (0 = absent) and acc.id(i); acc.value(i) is the
// score written out for a selected item.  Starts at level
// `lvl0` with the boundary prefix/mask already fixed by earlier levels.  On return the selection
// is: items of class 1 (surely selected) and the first `need` items of class 2 in item order.
// hist: shared memory of kHistBins words; scratch: 35 words.
struct SelectResult {
  uint32_t prefix, mask, need;
  bool by_id;
  uint32_t prefix2, mask2, need2;
};

template <class Acc>
__device__ SelectResult radix_select_items(const Acc& acc, int m, uint32_t need, int lvl0, uint32_t prefix,
                                           uint32_t mask, uint32_t* hist, uint32_t* scratch) {
  SelectResult r{prefix, mask, need, false, 0u, 0u, 0u};
  uint32_t eq = 0;
  bool done = false;
  for (int lvl = lvl0; lvl < 3 && !done; ++lvl) {
    const int nb = level_bins(lvl), sh = level_shift(lvl);
    for (int b = threadIdx.x; b < nb; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const int iters = (m + (int)blockDim.x - 1) / (int)blockDim.x;
    for (int j = 0; j < iters; ++j) {
      const int i = j * (int)blockDim.x + (int)threadIdx.x;
      const uint32_t k = i < m ? acc.key(i) : 0u;
      hist_add(hist, (k >> sh) & (uint32_t)(nb - 1), k != 0u && (k & r.mask) == r.prefix);
    }
    __syncthreads();
    const Bucket bk = block_bucket(hist, lvl, r.prefix, r.need, scratch);
    r.prefix = bk.prefix;
    r.need = bk.need;
    eq = bk.eq;
    r.mask |= (uint32_t)(nb - 1) << sh;
    done = eq == r.need;
  }
  if (eq > r.need) {  // equal keys straddle the boundary: rank them by id
    r.by_id = true;
    r.need2 = r.need;
    for (int lvl = 0; lvl < 3; ++lvl) {
      const int nb = level_bins(lvl), sh = level_shift(lvl);
      for (int b = threadIdx.x; b < nb; b += blockDim.x) hist[b] = 0;
      __syncthreads();
      const int iters = (m + (int)blockDim.x - 1) / (int)blockDim.x;
      for (int j = 0; j < iters; ++j) {
        const int i = j * (int)blockDim.x + (int)threadIdx.x;
        const uint32_t k = i < m ? acc.key(i) : 0u;
        const bool in = k != 0u && (k & r.mask) == r.prefix;
        const uint32_t k2 = in ? 0xffffffffu - acc.id(i) : 0u;
        hist_add(hist, (k2 >> sh) & (uint32_t)(nb - 1), in && (k2 & r.mask2) == r.prefix2);
      }
      __syncthreads();
      const Bucket bk = block_bucket(hist, lvl, r.prefix2, r.need2, scratch);
      r.prefix2 = bk.prefix;
      r.need2 = bk.need;
      r.mask2 |= (uint32_t)(nb - 1) << sh;
      if (bk.eq == r.need2) break;
    }
  }
  return r;
}

// Class of item i under a select result: 1 surely selected, 2 selected by rank, 0 not.
template <class Acc>
__device__ __forceinline__ int select_class(const Acc& acc, int i, const SelectResult& r) {
  const uint32_t k = acc.key(i);
  if (k == 0u) return 0;
  const uint32_t u = k & r.mask;
  if (u > r.prefix) return 1;
  if (u < r.prefix) return 0;
  if (!r.by_id) return 2;
  const uint32_t u2 = (0xffffffffu - acc.id(i)) & r.mask2;
  return u2 > r.prefix2 ? 1 : (u2 == r.prefix2 ? 2 : 0);
}

// Write the selection in item order: out_id[pos], out_val[pos] for pos < kk (kk = selected count).
// Every thread takes a contiguous run of items; one block scan places the runs.
template <class Acc>
__device__ void write_selection(const Acc& acc, int m, const SelectResult& r, bool take_all, int32_t* out_id,
                                float* out_val, uint32_t kk, uint32_t* scratch) {
  const uint32_t needF = r.by_id ? r.need2 : r.need;
  const int run = (m + (int)blockDim.x - 1) / (int)blockDim.x;
  const int e0 = min((int)threadIdx.x * run, m), e1 = min(e0 + run, m);
  uint32_t c1 = 0, c2 = 0;
  for (int e = e0; e < e1; ++e) {
    const int c = take_all ? (acc.key(e) != 0u ? 1 : 0) : select_class(acc, e, r);
    c1 += c == 1;
    c2 += c == 2;
  }
  uint32_t tot;
  uint32_t r1 = block_exclusive_scan(c1, scratch, &tot);
  uint32_t r2 = block_exclusive_scan(c2, scratch, &tot);
  for (int e = e0; e < e1; ++e) {
    const int c = take_all ? (acc.key(e) != 0u ? 1 : 0) : select_class(acc, e, r);
    uint32_t pos = 0xffffffffu;
    if (c == 1) {
      pos = r1 + (take_all ? 0u : min(r2, needF));
      ++r1;
    } else if (c == 2) {
      if (r2 < needF) pos = r1 + r2;
      ++r2;
    }
    if (pos < kk) {
      out_id[pos] = (int32_t)acc.id(e);
      if (out_val) out_val[pos] = acc.value(e);
    }
  }
}

}  // namespace misa
