// Warp-level selection: one warp per row, no block barriers, for many rows at once (prefill
// chunks of thousands of queries).
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", "Methodology: MISA",
// "Sparse Token Scoring": the top-k tokens of a query by its routed score.  The primitive is the
// r-th largest of a set of order keys (select.cuh: order_key is monotone in the score), found by
// rounds of a 1024-bin histogram over what is left of the key range; list_select_warp ranks a
// query's candidate list with it, exact ties to the lower token.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace misa {

constexpr int kSelWarps = 8;                        // rows per CTA: one warp each
constexpr int kWarpBins = 1024;                     // histogram bins of a warp
constexpr int kWarpBinWords = kWarpBins + kWarpBins / 32;  // padded: a lane's 32 bins in distinct banks
constexpr int kWarpUnroll = 8;                      // loads in flight per lane

__device__ __forceinline__ int warp_bin_word(uint32_t b) { return (int)(b + (b >> 5)); }

// The bin holding the need-th largest counted key of a warp's padded 1024-bin histogram (bin 1023
// the largest): the bin, the count in higher bins and the bin's own count.  Lane l sums bins
// [1023 - 32 l - 31, 1023 - 32 l]; one warp scan finds the lane, which walks its bins.
struct WarpBin {
  uint32_t bin, above, in;
};
__device__ __forceinline__ WarpBin warp_bin(const uint32_t* h, uint32_t need) {
  const int lane = threadIdx.x & 31;
  const uint32_t b0 = (uint32_t)(kWarpBins - 32 * (lane + 1));  // lowest bin of the lane
  uint32_t c[32];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    c[j] = h[warp_bin_word(b0 + j)];
    local += c[j];
  }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - local;
  WarpBin r{0u, 0u, 0u};
  const bool mine = excl < need && incl >= need;
  if (mine) {
    uint32_t cum = excl;
#pragma unroll
    for (int j = 31; j >= 0; --j) {
      if (cum < need && cum + c[j] >= need) {
        r.bin = b0 + j;
        r.above = cum;
        r.in = c[j];
      }
      cum += c[j];
    }
  }
  const unsigned who = __ballot_sync(0xffffffffu, mine);
  const int src = who ? __ffs(who) - 1 : 0;
  r.bin = __shfl_sync(0xffffffffu, r.bin, src);
  r.above = __shfl_sync(0xffffffffu, r.above, src);
  r.in = __shfl_sync(0xffffffffu, r.in, src);
  return r;
}

// Calls f(i, load(i)) for every i < c (and f(i, {0, 0}) for the padding up to a multiple of
// 32 kWarpUnroll, so that every lane takes the same steps), lanes strided, kWarpUnroll loads in
// flight per lane.
template <class Load, class F>
__device__ __forceinline__ void warp_each(int c, Load load, F f) {
  const int lane = threadIdx.x & 31;
  for (int i0 = 0; i0 < c; i0 += 32 * kWarpUnroll) {
    uint2 e[kWarpUnroll];
#pragma unroll
    for (int u = 0; u < kWarpUnroll; ++u) {
      const int i = i0 + 32 * u + lane;
      e[u] = i < c ? load(i) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kWarpUnroll; ++u) f(i0 + 32 * u + lane, e[u]);
  }
}

// r-th largest value (1 <= r <= the number of values) of a warp's set, all within [lo, hi]: rounds
// of 1024 bins over what is left of the range (the first over [lo, hi]) until a bin holds exactly
// the missing count (*all = true: every value of the bin is taken, and the result is the bin's
// lower edge) or is one value wide (*all = false: the result is that value, and ties with it may
// straddle the r-th place).  each(g) calls g(value, counted) for every member of the set on every
// lane.  *above: the count of values strictly above the result's bin.  h: kWarpBinWords words of
// the warp's own shared memory.
template <class Each>
__device__ __forceinline__ uint32_t warp_rth_largest(Each each, uint32_t lo, uint32_t hi, uint32_t r, uint32_t* h,
                                                     uint32_t* above, bool* all) {
  const int lane = threadIdx.x & 31;
  uint32_t base = lo, range = hi - lo, gt = 0;
  for (;;) {
    const int sh = range >= (uint32_t)kWarpBins ? 32 - __clz(range) - 10 : 0;
#pragma unroll
    for (int j = 0; j < (kWarpBinWords + 31) / 32; ++j)
      if (32 * j + lane < kWarpBinWords) h[32 * j + lane] = 0u;
    __syncwarp();
    each([&](uint32_t v, bool counted) {
      if (counted && v >= base && v - base <= range) atomicAdd(&h[warp_bin_word((v - base) >> sh)], 1u);
    });
    __syncwarp();
    const WarpBin wb = warp_bin(h, r);
    __syncwarp();
    gt += wb.above;
    r -= wb.above;
    const uint32_t edge = base + (wb.bin << sh);
    if (wb.in == r || sh == 0) {
      *above = gt;
      *all = wb.in == r;
      return edge;
    }
    range = min(range - (wb.bin << sh), (1u << sh) - 1u);
    base = edge;
  }
}

// Smallest and largest of the lanes' lo / hi over the warp.
__device__ __forceinline__ void warp_min_max(uint32_t& lo, uint32_t& hi) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
}

// Cut of a query from a sample of its keys: the lower edge of the narrow bin holding the sample's
// rank-th largest key, so at least rank sample keys are at or above it.  key(i) is sample key i
// < ns (rank <= ns).
template <class Key>
__device__ __forceinline__ uint32_t warp_sample_cut(int ns, Key key, uint32_t rank, uint32_t* h,
                                                    uint32_t* smax = nullptr) {
  auto load = [&](int i) { return make_uint2(key(i), 0u); };
  uint32_t lo = 0xffffffffu, hi = 0u;
  warp_each(ns, load, [&](int i, uint2 e) {
    if (i < ns) {
      lo = min(lo, e.x);
      hi = max(hi, e.x);
    }
  });
  warp_min_max(lo, hi);
  if (smax) *smax = hi;
  uint32_t above;
  bool all;
  return warp_rth_largest([&](auto g) { warp_each(ns, load, [&](int i, uint2 e) { g(e.x, i < ns); }); }, lo, hi,
                          rank, h, &above, &all);
}

// Top-k of a candidate list whose entries (keys at or above cut; key 0 is an empty slot) lie
// mostly in [vlo, vhi] (the cut's score and the largest score of the sample that placed it;
// larger scores go to the top bin), in two passes: one bins the entries linearly in 1024 bins,
// the other writes the entries of the bins above the need-th entry's bin and keeps that bin's own
// entries in bnd (kWarpBound of them at most), where a rank count (score, then token) orders them.
// Returns 0 when fewer than need entries qualify, 2 when the bin holds more than kWarpBound
// entries or the range is empty (nothing written in either case), 1 when the selection is written
// to oi/ov [0, need) and padding to [need, topk).
constexpr int kWarpBound = 128;
__device__ __forceinline__ int warp_list_select_binned(const uint2* lt, int c, uint32_t cut, float vlo, float vhi,
                                                       uint32_t need, int topk, uint32_t* h, uint2* bnd,
                                                       int32_t* oi, float* ov) {
  const int lane = threadIdx.x & 31;
  const float scale = (float)kWarpBins / (vhi - vlo);
  if (!(vhi > vlo) || !(scale > 0.f) || !(scale < 3.0e38f)) return 2;
  auto load = [&](int i) { return __ldcg(lt + i); };
  auto valid = [&](int i, uint2 e) { return i < c && e.x != 0u && e.x >= cut; };
  auto bin = [&](uint32_t k) {
    return (uint32_t)max(0, min(__float2int_rz((key_to_float(k) - vlo) * scale), kWarpBins - 1));
  };
#pragma unroll
  for (int j = 0; j < (kWarpBinWords + 31) / 32; ++j)
    if (32 * j + lane < kWarpBinWords) h[32 * j + lane] = 0u;
  __syncwarp();
  uint32_t cnt = 0;
  warp_each(c, load, [&](int i, uint2 e) {
    if (valid(i, e)) {
      atomicAdd(&h[warp_bin_word(bin(e.x))], 1u);
      ++cnt;
    }
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (cnt < need) return 0;
  __syncwarp();
  const WarpBin wb = warp_bin(h, need);
  if (wb.in > (uint32_t)kWarpBound) return 2;
  const uint32_t need_in = need - wb.above;
  const uint32_t below = (1u << lane) - 1u;
  uint32_t pg = 0, pb = 0;
  warp_each(c, load, [&](int i, uint2 e) {
    const bool ok = valid(i, e);
    const uint32_t b = ok ? bin(e.x) : 0u;
    const bool gt = ok && b > wb.bin, eq = ok && b == wb.bin;
    const unsigned mg = __ballot_sync(0xffffffffu, gt), me = __ballot_sync(0xffffffffu, eq);
    if (gt) {
      const uint32_t s = pg + (uint32_t)__popc(mg & below);
      oi[s] = (int32_t)e.y;
      if (ov) ov[s] = key_to_float(e.x);
    }
    if (eq) bnd[pb + (uint32_t)__popc(me & below)] = e;
    pg += (uint32_t)__popc(mg);
    pb += (uint32_t)__popc(me);
  });
  __syncwarp();
  // the bin's entries: rank by score, then token; the first need_in are taken
  for (uint32_t j = lane; j < wb.in; j += 32) {
    const uint2 m = bnd[j];
    uint32_t r = 0;
    for (uint32_t i = 0; i < wb.in; ++i) {
      const uint2 o = bnd[i];
      r += (o.x > m.x) || (o.x == m.x && o.y < m.y);
    }
    if (r < need_in) {
      oi[wb.above + r] = (int32_t)m.y;
      if (ov) ov[wb.above + r] = key_to_float(m.x);
    }
  }
  for (int a = (int)need + lane; a < topk; a += 32) {
    oi[a] = -1;
    if (ov) ov[a] = 0.f;
  }
  return 1;
}

// Top-k of one query's candidate list lt[0, c) of (order key, token): the entries with a key at or
// above cut (key 0 never is a score's key), exact ties to the lower token.  Returns false, writing
// nothing, when fewer than need = min(topk, n_t) entries qualify; otherwise writes the selection to
// oi/ov [0, need) in no particular order and -1 / 0 to [need, topk).
__device__ __forceinline__ bool warp_list_select(const uint2* lt, int c, uint32_t cut, uint32_t need, int topk,
                                                 uint32_t* h, int32_t* oi, float* ov) {
  const int lane = threadIdx.x & 31;
  auto load = [&](int i) { return __ldcg(lt + i); };
  auto valid = [&](int i, uint2 e) { return i < c && e.x != 0u && e.x >= cut; };
  uint32_t cnt = 0, lo = 0xffffffffu, hi = 0u;
  warp_each(c, load, [&](int i, uint2 e) {
    if (valid(i, e)) {
      ++cnt;
      lo = min(lo, e.x);
      hi = max(hi, e.x);
    }
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  warp_min_max(lo, hi);
  if (cnt < need) return false;
  // selected: key > kstar, or key == kstar and (every such entry, or token <= tok)
  uint32_t kstar = lo, tok = 0xffffffffu;
  bool take_eq_all = true;
  if (cnt > need) {
    uint32_t above;
    bool all;
    kstar = warp_rth_largest([&](auto g) { warp_each(c, load, [&](int i, uint2 e) { g(e.x, valid(i, e)); }); }, lo,
                             hi, need, h, &above, &all);
    if (!all) {
      // exact ties at kstar straddle the need-th place: the lowest tokens among them, as the
      // largest values of 0xffffffff - token
      uint32_t tlo = 0xffffffffu, thi = 0u;
      warp_each(c, load, [&](int i, uint2 e) {
        if (valid(i, e) && e.x == kstar) {
          tlo = min(tlo, 0xffffffffu - e.y);
          thi = max(thi, 0xffffffffu - e.y);
        }
      });
      warp_min_max(tlo, thi);
      uint32_t a2;
      bool all2;
      tok = 0xffffffffu - warp_rth_largest(
                              [&](auto g) {
                                warp_each(c, load, [&](int i, uint2 e) { g(0xffffffffu - e.y, valid(i, e) && e.x == kstar); });
                              },
                              tlo, thi, need - above, h, &a2, &all2);
      take_eq_all = false;
    }
  }
  // one ballot per step places the lanes' selected entries
  const uint32_t below = (1u << lane) - 1u;
  uint32_t pos = 0;
  warp_each(c, load, [&](int i, uint2 e) {
    const bool sel = valid(i, e) && (e.x > kstar || (e.x == kstar && (take_eq_all || e.y <= tok)));
    const unsigned m = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const uint32_t slot = pos + (uint32_t)__popc(m & below);
      oi[slot] = (int32_t)e.y;
      if (ov) ov[slot] = key_to_float(e.x);
    }
    pos += (uint32_t)__popc(m);
  });
  for (int a = (int)need + lane; a < topk; a += 32) {
    oi[a] = -1;
    if (ov) ov[a] = 0.f;
  }
  return true;
}

}  // namespace misa
