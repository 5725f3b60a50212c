// Top-k selection by radix select.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", Technical Summary,
// "Methodology: MISA", "Sparse Token Scoring": the final top-k tokens are selected on the reduced
// scores; "Hierarchical Variant (MISA-dagger)": the k' candidates are narrowed to the top-k by
// their dense scores.  Selection rule: score descending, exact ties to the lower token index.
//
// Every score becomes an order-preserving 32-bit key.  Three histogram passes (11, 11 and 10
// bits, most significant first, each counting only keys whose higher bits match the prefix found
// so far) pin the key tau of the k-th largest element and how many elements equal to tau are
// still needed; a pass stops early once the bucket holding the k-th element is taken whole.  A
// last pass walks the row in index order with a block-wide scan and writes every key above
// tau and the first `need` keys equal to tau, so the output is in ascending index order and the
// tie rule holds exactly.  One CTA of 1024 threads per query.
//
// Candidate lists (re-rank) live in shared memory; if equal scores straddle the boundary, a
// second select over the token ids (smaller id wins) settles them, so the result does not depend
// on the order of the candidate list.
#include "kernels.cuh"

namespace misa {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kBins = 2048;

struct SelectState {
  uint32_t prefix, mask, need, eq;  // keys k with (k & mask) == prefix are "equal"; take `need` of them
};

// Radix select over `count` keys fetched by key_at(i) (key 0 = absent).  Leaves the boundary in
// *st: keys with (key & mask) > prefix are selected, and `need` of the `eq` keys with
// (key & mask) == prefix.  Requires need <= number of present keys.
template <class KeyAt>
__device__ void radix_select(KeyAt key_at, int count, uint32_t need, uint32_t* hist, uint32_t* wtot,
                             SelectState* st) {
  uint32_t prefix = 0, mask = 0;
  uint32_t eq = 0;
  const int shifts[3] = {21, 10, 0};
  const int nbits[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int nb = 1 << nbits[pass], sh = shifts[pass];
    for (int b = threadIdx.x; b < kBins; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < count; i += blockDim.x) {
      const uint32_t u = key_at(i);
      if (u != 0u && (u & mask) == prefix) atomicAdd(&hist[(u >> sh) & (nb - 1)], 1u);
    }
    __syncthreads();
    // Thread x owns `per` consecutive bins in descending bin order.
    const int per = (nb + blockDim.x - 1) / blockDim.x;
    uint32_t local = 0;
    for (int d = 0; d < per; ++d) {
      const int b = nb - 1 - (threadIdx.x * per + d);
      if (b >= 0) local += hist[b];
    }
    uint32_t total;
    uint32_t cum = block_exclusive_scan(local, wtot, &total);
    for (int d = 0; d < per; ++d) {
      const int b = nb - 1 - (threadIdx.x * per + d);
      if (b < 0) break;
      const uint32_t hb = hist[b];
      if (cum < need && cum + hb >= need) {
        st->prefix = prefix | ((uint32_t)b << sh);
        st->need = need - cum;
        st->eq = hb;
      }
      cum += hb;
    }
    __syncthreads();
    prefix = st->prefix;
    need = st->need;
    eq = st->eq;
    mask |= (uint32_t)(nb - 1) << sh;
    __syncthreads();
    if (eq == need) break;  // the boundary bucket is taken whole
  }
  if (threadIdx.x == 0) {
    st->prefix = prefix;
    st->mask = mask;
    st->need = need;
    st->eq = eq;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(const float* __restrict__ scores, int64_t ld,
                                                                 const int32_t* __restrict__ n, int L, int topk,
                                                                 int32_t* __restrict__ idx,
                                                                 float* __restrict__ score_opt) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t wtot[32];
  __shared__ SelectState st;
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const float* row = scores + (int64_t)t * ld;
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  if (nt <= topk) {
    for (int s = threadIdx.x; s < topk; s += blockDim.x) {
      oi[s] = s < nt ? s : -1;
      if (ov) ov[s] = s < nt ? row[s] : 0.f;
    }
    return;
  }
  auto key_at = [&](int i) { return order_key(row[i]); };
  radix_select(key_at, nt, (uint32_t)topk, hist, wtot, &st);
  const uint32_t prefix = st.prefix, mask = st.mask, need = st.need;
  const uint32_t n_gt = (uint32_t)topk - need;
  uint32_t base_gt = 0, base_eq = 0;
  for (int s0 = 0; s0 < nt; s0 += blockDim.x) {
    const int s = s0 + threadIdx.x;
    float v = 0.f;
    uint32_t gt = 0, eq = 0;
    if (s < nt) {
      v = row[s];
      const uint32_t key = order_key(v);
      const uint32_t u = key & mask;
      gt = key != 0u && u > prefix;  // key 0 (only an all-ones NaN) is never selected
      eq = key != 0u && u == prefix;
    }
    uint32_t tot;
    const uint32_t ex = block_exclusive_scan(gt | (eq << 16), wtot, &tot);
    const uint32_t gt_before = base_gt + (ex & 0xffffu), eq_before = base_eq + (ex >> 16);
    if (gt || (eq && eq_before < need)) {
      const uint32_t pos = gt_before + min(eq_before, need);
      if (pos < (uint32_t)topk) {
        oi[pos] = s;
        if (ov) ov[pos] = v;
      }
    }
    base_gt += tot & 0xffffu;
    base_eq += tot >> 16;
    if (base_gt == n_gt && base_eq >= need) break;  // uniform: every selected index is written
  }
}

// Candidate lists: F[t, P] with ids cand[t, P]; dynamic shared memory holds keys[P] and ids[P].
__global__ void __launch_bounds__(kTopkThreads) topk_cand_kernel(const float* __restrict__ F,
                                                                 const int32_t* __restrict__ cand,
                                                                 const int32_t* __restrict__ n, int L, int P,
                                                                 int topk, int32_t* __restrict__ idx,
                                                                 float* __restrict__ score_opt) {
  extern __shared__ uint32_t csm[];
  uint32_t* keys = csm;       // [P] order keys, 0 = empty slot
  uint32_t* ids = csm + P;    // [P] token ids
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t wtot[32];
  __shared__ SelectState st, st2;
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const float* ft = F + (int64_t)t * P;
  const int32_t* ct = cand + (int64_t)t * P;
  int32_t* oi = idx + (int64_t)t * topk;
  float* ov = score_opt ? score_opt + (int64_t)t * topk : nullptr;
  uint32_t cnt = 0;
  for (int i = threadIdx.x; i < P; i += blockDim.x) {
    const int32_t id = ct[i];
    const bool ok = id >= 0 && id < nt;
    keys[i] = ok ? order_key(ft[i]) : 0u;
    ids[i] = ok ? (uint32_t)id : 0u;
    cnt += ok;
  }
  uint32_t nvalid;
  block_exclusive_scan(cnt, wtot, &nvalid);
  const uint32_t kk = (uint32_t)topk < nvalid ? (uint32_t)topk : nvalid;
  uint32_t prefix = 0, mask = 0, need = 0;
  bool tie_by_id = false;
  uint32_t prefix2 = 0, mask2 = 0, need2 = 0;
  if (kk < nvalid) {
    radix_select([&](int i) { return keys[i]; }, P, kk, hist, wtot, &st);
    prefix = st.prefix;
    mask = st.mask;
    need = st.need;
    if (st.eq > need) {
      // equal scores straddle the boundary: among them keep the `need` smallest ids
      tie_by_id = true;
      radix_select(
          [&](int i) { return (keys[i] != 0u && (keys[i] & mask) == prefix) ? 0xffffffffu - ids[i] : 0u; }, P,
          need, hist, wtot, &st2);
      prefix2 = st2.prefix;
      mask2 = st2.mask;
      need2 = st2.need;
    }
  }
  uint32_t base = 0, base_eq2 = 0;
  for (int i0 = 0; i0 < P; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    uint32_t sel = 0, eq2 = 0;
    if (i < P && keys[i] != 0u) {
      if (kk == nvalid) {
        sel = 1;
      } else {
        const uint32_t u = keys[i] & mask;
        if (u > prefix) sel = 1;
        else if (u == prefix) {
          if (!tie_by_id) sel = 1;  // the whole equal group is needed (eq == need)
          else {
            const uint32_t u2 = (0xffffffffu - ids[i]) & mask2;
            if (u2 > prefix2) sel = 1;
            else if (u2 == prefix2) eq2 = 1;
          }
        }
      }
    }
    uint32_t tot;
    const uint32_t ex = block_exclusive_scan(sel | (eq2 << 16), wtot, &tot);
    const uint32_t eq2_before = base_eq2 + (ex >> 16);
    if (eq2 && eq2_before < need2) sel = 1;
    // positions: recount with the resolved flags
    uint32_t tot2;
    const uint32_t pos = base + block_exclusive_scan(sel, wtot, &tot2);
    if (sel && pos < (uint32_t)topk) {
      oi[pos] = (int32_t)ids[i];
      if (ov) ov[pos] = key_to_float(keys[i]);
    }
    base += tot2;
    base_eq2 += tot >> 16;
  }
  for (int a = (int)kk + threadIdx.x; a < topk; a += blockDim.x) {
    oi[a] = -1;
    if (ov) ov[a] = 0.f;
  }
}

}  // namespace

void launch_topk_rows(const float* scores, int64_t ld, const int32_t* n, int T, int L, int topk, int32_t* idx,
                      float* score_opt, cudaStream_t s) {
  if (T <= 0) return;
  topk_rows_kernel<<<T, kTopkThreads, 0, s>>>(scores, ld, n, L, topk, idx, score_opt);
}

size_t topk_cand_smem(int P) { return sizeof(uint32_t) * 2 * (size_t)P; }

void launch_topk_cand(const float* F, const int32_t* cand, const int32_t* n, int T, int L, int P, int topk,
                      int32_t* idx, float* score_opt, cudaStream_t s) {
  if (T <= 0) return;
  const size_t smem = topk_cand_smem(P);
  cudaFuncSetAttribute(topk_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  topk_cand_kernel<<<T, kTopkThreads, smem, s>>>(F, cand, n, L, P, topk, idx, score_opt);
}

}  // namespace misa
