// Token scoring with a list of indexer heads:  out[t, p] = sum_{j in list} w_{t,j} relu(q_{t,j} . k_s)
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", Technical Summary,
// "Methodology: MISA", "Sparse Token Scoring" (the list is the h routed heads), "Hierarchical
// Variant (MISA-dagger)" (the list is all H_I heads and the tokens are gathered candidates) and
// "Problem Statement" (the dense indexer: all heads, all prefix tokens).
//
// bf16 path.  Per key the work is h x 128 multiply-adds against 256 bytes read, so with h = 8 a
// CUDA-core dot product would spend more issue slots on FMAs and shuffles than HBM allows; the
// contraction runs on the tensor cores instead (mma_frag.cuh: key rows go from global memory
// straight into A fragments).  Heads are summed in ascending head index (the routed list is
// sorted, padded to a multiple of 8 with zero-weight slots), so the routed score with h = H_I is
// the dense score bit for bit.
//
// Three kernels here (shared bf16 caches go to score_tc.cu first):
//   score_persist_kernel  decode (one cache per query): persistent, 2 CTAs per SM; the actual
//       work (ceil(n_t/128) tiles of 128 rows per query) is flattened and split evenly over the
//       CTAs, each taking one contiguous range.  Each warp owns 16 rows of every tile and holds
//       the next tile in registers while the current one is multiplied.  (Measured on B200 with
//       32 x 131072 keys: 178 us against 185 us for the grid kernel; an added bulk L2 prefetch
//       of the rows four tiles ahead made it slower, 202 us, and was dropped.)
//       The same schedule serves gathered candidate lists (re-rank): positions instead of rows.
//   score_grid_kernel     one CTA per (query, chunk of positions): shared caches when the
//       tensor-core kernel (score_tc.cu, which takes shared bf16 caches) cannot run, and more
//       queries than the persistent schedule takes.
//   score_f32_kernel      fp32 inputs: one warp per key row on CUDA cores, exact fp32 products.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "mma_frag.cuh"
#include "select.cuh"

namespace misa {

namespace {

constexpr int kScoreThreads = 256;   // 8 warps
constexpr int kRowsPerChunk = 1024;  // positions per CTA of the grid kernel
constexpr int kGatherRowsPerChunk = 256;
constexpr int kTileRows = 128;       // persistent kernel: 8 warps x 16 rows
constexpr int kMaxPersistQueries = 8192;

// Shared staging of one query's head list: ascending head ids (padded), weights and the B
// fragments in fragment order.
template <int NG>
struct HeadStage {
  uint2 frag[NG][8][32];
  float wsel[NG * 8];
  int hl[NG * 8];
  int m;
};

// Thread 0 sorts the heads; pads reuse head hl[0] with weight 0.  Head ids outside [0, H_I) are
// clamped into range (the router never produces them).  Without a list (all heads, already in
// order) the threads fill it together.
__device__ __forceinline__ void stage_head_list(const int32_t* heads, int h, int H_I, int t, int slots,
                                                int* hl, int* m_out) {
  if (!heads) {
    for (int a = threadIdx.x; a < slots; a += blockDim.x) hl[a] = a < H_I ? a : 0;
    if (threadIdx.x == 0) *m_out = H_I;
    return;
  }
  // every id is loaded at once (one per thread), then one thread sorts them in shared memory
  for (int a = threadIdx.x; a < h; a += blockDim.x) {
    int v = heads[(int64_t)t * h + a];
    count_bad_id(kBadHead, v < 0 || v >= H_I);
    hl[a] = v < 0 ? 0 : (v >= H_I ? H_I - 1 : v);  // out-of-range ids are clamped, never dereferenced
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int a = 1; a < h; ++a) {
      const int v = hl[a];
      int b = a;
      while (b > 0 && hl[b - 1] > v) {
        hl[b] = hl[b - 1];
        --b;
      }
      hl[b] = v;
    }
    for (int a = h; a < slots; ++a) hl[a] = hl[0];
    *m_out = h;
  }
}

template <int NG>
__device__ __forceinline__ void stage_query(HeadStage<NG>& st, const __nv_bfloat16* q, const float* w,
                                            const int32_t* heads, int h, int H_I, int t) {
  stage_head_list(heads, h, H_I, t, NG * 8, st.hl, &st.m);
  __syncthreads();
  if (threadIdx.x < NG * 8)
    st.wsel[threadIdx.x] = (int)threadIdx.x < st.m ? w[(int64_t)t * H_I + st.hl[threadIdx.x]] : 0.f;
  stage_q_frags<NG, kScoreThreads>(st.frag, q + (int64_t)t * H_I * kD, st.hl);
  __syncthreads();
}

// Work of the persistent scorer.
enum : int {
  kModeRows = 0,    // every prefix position of each query: out[t, p] for p < n_t
  kModeGather = 1,  // gathered candidates: out[t, p] = score of token rows[t, p] for p < P
  kModeSample = 2,  // only the list cut's sample of each row longer than the list cap (kSampleRuns
                    // evenly spaced runs of kSampleRunLen tokens): out[t, s] at those tokens s
  kModeList = 3,    // as kModeRows, and every token whose score is at or above its row's cut is
                    // appended to the row's list with its dense score over all H_I heads
};

// Per-warp staging of kModeList: key rows at or above the cut wait here (a ring of 32 rows of
// 256 bytes, plus their (order key, token)) until 16 of them fill one tensor-core group.
constexpr int kRing = 32;

// kModeList: the first m <= 16 rows staged in a warp's ring (slots head .. head + m - 1, mod kRing)
// scored with all heads (frag / wall: ngf head groups) and appended to row t's list with one atomic
// (entries past the cap are counted, not written).  Called by the whole warp; rare (once per 16
// rows at or above the cut), so it is kept out of line, away from the scoring loop's registers.
__device__ __noinline__ void flush_ring(const uint8_t* ring, const uint2* meta, int head, int m,
                                        const uint2 (*frag)[8][32], const float* wall, int ngf, DenseList dl, int t) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  __syncwarp();
  const int sa = (head + g) & (kRing - 1), sb = (head + g + 8) & (kRing - 1);
  uint4 A[4], B[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    A[i] = g < m ? *reinterpret_cast<const uint4*>(ring + sa * kD * 2 + (4 * i + c) * 16) : make_uint4(0, 0, 0, 0);
    B[i] = g + 8 < m ? *reinterpret_cast<const uint4*>(ring + sb * kD * 2 + (4 * i + c) * 16) : make_uint4(0, 0, 0, 0);
  }
  float flo, fhi;
  score_rows_any(A, B, frag, wall, ngf, lane, flo, fhi);
  uint32_t base = 0;
  if (lane == 0) base = atomicAdd(dl.cnt + t, (uint32_t)m);
  base = __shfl_sync(0xffffffffu, base, 0);
  uint2* lt = dl.list + (int64_t)t * dl.stride;
  float* ft = dl.f + (int64_t)t * dl.stride;
  if (c == 0 && g < m && base + g < (uint32_t)dl.cap) {
    lt[base + g] = meta[sa];
    ft[base + g] = flo;
  }
  if (c == 1 && g + 8 < m && base + g + 8 < (uint32_t)dl.cap) {
    lt[base + g + 8] = meta[sb];
    ft[base + g + 8] = fhi;
  }
  __syncwarp();  // the slots are read before they are written again
}

template <int NG, int MODE>
__global__ void __launch_bounds__(kScoreThreads, 2)
    score_persist_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                         const __nv_bfloat16* __restrict__ k, int64_t k_seq_stride, const int32_t* __restrict__ n,
                         const int32_t* __restrict__ heads, int h, int H_I, int L, int T,
                         const int32_t* __restrict__ rows, int P, float* __restrict__ out, int64_t ld,
                         DenseList dl) {
  extern __shared__ __align__(16) uint8_t dsm[];
  int* tile_base = reinterpret_cast<int*>(dsm);  // [T + 1] flattened tile prefix
  __shared__ HeadStage<NG> st;
  __shared__ uint32_t wtot[35];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  // kModeList: all heads' fragments and weights, and this warp's ring (after the tile prefix)
  const int ngf = (H_I + 7) / 8;
  uint8_t* lsm = dsm + (((size_t)T + 1) * sizeof(int) + 15) / 16 * 16;
  uint2(*frag_all)[8][32] = reinterpret_cast<uint2(*)[8][32]>(lsm);
  float* wall = reinterpret_cast<float*>(lsm + (size_t)ngf * 8 * 32 * sizeof(uint2));
  uint8_t* ring = lsm + (size_t)ngf * 8 * 32 * sizeof(uint2) + kMaxHeads * sizeof(float) +
                  (size_t)warp * kRing * (kD * 2 + sizeof(uint2));
  uint2* meta = reinterpret_cast<uint2*>(ring + kRing * kD * 2);
  pdl_wait();
  pdl_trigger();

  // positions of query t: n_t (rows, list), P (gather), the sample of a row longer than the cap
  auto npos_of = [&](int nt) {
    if (MODE == kModeGather) return P;
    if (MODE == kModeSample) return nt > dl.cap ? kSampleRuns * kSampleRunLen : 0;
    return nt;
  };
  const int per = (T + kScoreThreads - 1) / kScoreThreads;
  const int q0 = min((int)threadIdx.x * per, T), q1 = min(q0 + per, T);
  uint32_t mine = 0;
  for (int t = q0; t < q1; ++t) mine += (npos_of(clamp_len(n[t], L)) + kTileRows - 1) / kTileRows;
  uint32_t total;
  uint32_t run = block_exclusive_scan(mine, wtot, &total);
  for (int t = q0; t < q1; ++t) {
    tile_base[t] = (int)run;
    run += (npos_of(clamp_len(n[t], L)) + kTileRows - 1) / kTileRows;
  }
  if (threadIdx.x == 0) tile_base[T] = (int)total;
  __syncthreads();
  const int64_t tb = (int64_t)blockIdx.x * total / gridDim.x;
  const int64_t te = (int64_t)(blockIdx.x + 1) * total / gridDim.x;

  int64_t pos = tb;
  while (pos < te) {
    int lo = 0, hi = T - 1;  // last query whose first tile is at or before pos
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tile_base[mid] <= pos) lo = mid;
      else hi = mid - 1;
    }
    const int t = lo;
    const int64_t seg_end = min(te, (int64_t)tile_base[t + 1]);
    const int first = (int)(pos - tile_base[t]);
    const int ntile = (int)(seg_end - pos);
    const int nt = clamp_len(n[t], L);
    const int npos = npos_of(nt);
    const int32_t* rt = MODE == kModeGather ? rows + (int64_t)t * P : nullptr;
    const int seg = (nt / kSampleRuns) & ~(kSampleRunLen - 1);  // kModeSample: run spacing
    // kModeList: the row's cut (no list: nothing is appended)
    bool listing = false;
    float cutv = 0.f;  // compared as a float: the same order as the keys (the cut is a finite score)
    if (MODE == kModeList) {
      listing = __ldcg(dl.cnt + t) != kNoList;
      cutv = key_to_float(__ldcg(dl.cut + t));
    }

    const __nv_bfloat16* kt = k + (int64_t)t * k_seq_stride;
    auto row_of = [&](int j) { return (first + j) * kTileRows + warp * 16; };
    // position p -> key row: p itself, the p-th sampled token, or rows[t, p] when gathering
    // (outside [0, n_t): empty).  Gathered row ids are fetched two tiles ahead, so a tile's row
    // loads never wait for its ids.
    auto raw_id = [&](int p) -> int {
      if (p >= npos) return -1;
      if (MODE == kModeSample) return (p / kSampleRunLen) * seg + (p % kSampleRunLen);
      if (MODE != kModeGather) return p;
      const int id = __ldg(rt + p);
      count_bad_id(kBadCandidate, c == 0 && id != -1 && (id < 0 || id >= nt));  // one lane of the quad
      return id;
    };
    auto valid_row = [&](int r) -> int { return (r >= 0 && r < nt) ? r : -1; };
    auto load_ids = [&](int ra, int rb, uint4 (&A)[4], uint4 (&B)[4]) {
      ra = valid_row(ra);
      rb = valid_row(rb);
      load_rows(ra >= 0 ? kt + (int64_t)ra * kD : nullptr, rb >= 0 ? kt + (int64_t)rb * kD : nullptr, c, A, B);
    };
    // the first tile's rows are read while the query's heads are staged
    int ida = raw_id(row_of(0) + g), idb = raw_id(row_of(0) + g + 8);
    int nia = MODE == kModeGather && ntile > 1 ? raw_id(row_of(1) + g) : -1;
    int nib = MODE == kModeGather && ntile > 1 ? raw_id(row_of(1) + g + 8) : -1;
    uint4 RA[4], RB[4];
    load_ids(ida, idb, RA, RB);

    __syncthreads();  // the previous segment's fragments are no longer read
    if (MODE == kModeList && listing) {
      stage_all_head_frags<kScoreThreads>(frag_all, q + (int64_t)t * H_I * kD, H_I, ngf);
      for (int e = threadIdx.x; e < ngf * 8; e += kScoreThreads) wall[e] = e < H_I ? w[(int64_t)t * H_I + e] : 0.f;
    }
    stage_query<NG>(st, q, w, heads, h, H_I, t);
    float wa[NG], wb[NG];
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      wa[ng] = st.wsel[ng * 8 + 2 * c];
      wb[ng] = st.wsel[ng * 8 + 2 * c + 1];
    }
    float* ot = out + (int64_t)t * ld;
    // kModeList: the staged rows [head, head + ns) of the ring; flush scores the first m <= 16 of
    // them with all heads and appends them to the row's list (one atomic per flush)
    int ns = 0, head = 0;
    auto flush = [&](int m) {
      flush_ring(ring, meta, head, m, frag_all, wall, ngf, dl, t);
      head = (head + m) & (kRing - 1);
      ns -= m;
    };
    for (int j = 0; j < ntile; ++j) {
      // the rows staged by the previous tile, before the next tile's loads are in flight
      if (MODE == kModeList && listing && ns >= 16) flush(16);
      uint4 NA[4], NB[4];
      int ra = -1, rb = -1;
      if (j + 1 < ntile) {
        if (MODE == kModeGather) {
          ra = nia;
          rb = nib;
          nia = j + 2 < ntile ? raw_id(row_of(j + 2) + g) : -1;
          nib = j + 2 < ntile ? raw_id(row_of(j + 2) + g + 8) : -1;
        } else {
          ra = raw_id(row_of(j + 1) + g);
          rb = raw_id(row_of(j + 1) + g + 8);
        }
        load_ids(ra, rb, NA, NB);
      }
      float slo, shi;
      score_rows<NG>(RA, RB, st.frag, wa, wb, lane, slo, shi);
      const int r = row_of(j) + g;
      if (MODE == kModeSample) {
        if (c == 0 && ida >= 0) ot[ida] = slo;
        if (c == 1 && idb >= 0) ot[idb] = shi;
      } else {
        if (c == 0 && r < npos) ot[r] = slo;
        if (c == 1 && r + 8 < npos) ot[r + 8] = shi;
      }
      if (MODE == kModeList && listing) {
        const bool pa = r < npos && slo >= cutv;
        const bool pb = r + 8 < npos && shi >= cutv;
        // bit 4 g' (lane (g', 0)): row g' passes; bit 4 g' + 1 (lane (g', 1)): row g' + 8
        const uint32_t bab = __ballot_sync(0xffffffffu, c == 0 ? pa : (c == 1 && pb));
        if (bab) {
          const uint32_t ba = bab & 0x11111111u, bb = (bab >> 1) & 0x11111111u;
          const uint32_t below = (1u << (4 * g)) - 1u;
          const int na = __popc(ba);
          if (pa) {
            const int sl = (head + ns + __popc(ba & below)) & (kRing - 1);
#pragma unroll
            for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(ring + sl * kD * 2 + (4 * i + c) * 16) = RA[i];
            if (c == 0) meta[sl] = make_uint2(order_key(slo), (uint32_t)r);
          }
          if (pb) {
            const int sl = (head + ns + na + __popc(bb & below)) & (kRing - 1);
#pragma unroll
            for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(ring + sl * kD * 2 + (4 * i + c) * 16) = RB[i];
            if (c == 0) meta[sl] = make_uint2(order_key(shi), (uint32_t)(r + 8));
          }
          ns += na + __popc(bb);  // at most 31: the ring holds them
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        RA[i] = NA[i];
        RB[i] = NB[i];
      }
      if (MODE == kModeSample) {
        ida = ra;
        idb = rb;
      }
    }
    if (MODE == kModeList && listing) {
      if (ns >= 16) flush(16);
      if (ns > 0) flush(ns);
    }
    pos = seg_end;
  }
}

template <int NG, bool GATHER>
__global__ void __launch_bounds__(kScoreThreads, 2)
    score_grid_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                      const __nv_bfloat16* __restrict__ k, int64_t k_seq_stride, const int32_t* __restrict__ n,
                      const int32_t* __restrict__ heads, int h, int H_I, int L,
                      const int32_t* __restrict__ rows, int P, float* __restrict__ out, int64_t ld) {
  constexpr int kChunk = GATHER ? kGatherRowsPerChunk : kRowsPerChunk;
  __shared__ HeadStage<NG> st;
  const int t = blockIdx.y;
  const int nt = clamp_len(n[t], L);
  const int npos = GATHER ? P : nt;
  const int p0 = blockIdx.x * kChunk;
  if (p0 >= npos) return;
  const int p1 = min(p0 + kChunk, npos);
  stage_query<NG>(st, q, w, heads, h, H_I, t);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  float wa[NG], wb[NG];
#pragma unroll
  for (int ng = 0; ng < NG; ++ng) {
    wa[ng] = st.wsel[ng * 8 + 2 * c];
    wb[ng] = st.wsel[ng * 8 + 2 * c + 1];
  }
  const __nv_bfloat16* kt = k + (int64_t)t * k_seq_stride;
  float* ot = out + (int64_t)t * ld;
  const int32_t* rt = GATHER ? rows + (int64_t)t * P : nullptr;

  auto load = [&](int r0, uint4 (&RA)[4], uint4 (&RB)[4], bool& va, bool& vb) {
    const int pa = r0 + g, pb = r0 + g + 8;
    int sa = pa, sb = pb;
    va = pa < p1;
    vb = pb < p1;
    if (GATHER) {
      sa = va ? __ldg(rt + pa) : -1;
      sb = vb ? __ldg(rt + pb) : -1;
      va = va && sa >= 0 && sa < nt;
      vb = vb && sb >= 0 && sb < nt;
    }
    load_rows(va ? kt + (int64_t)sa * kD : nullptr, vb ? kt + (int64_t)sb * kD : nullptr, c, RA, RB);
  };

  int r0 = p0 + warp * 16;
  uint4 RA[4], RB[4];
  bool va = false, vb = false;
  if (r0 < p1) load(r0, RA, RB, va, vb);
  for (; r0 < p1; r0 += 8 * 16) {
    uint4 NA[4], NB[4];
    bool na = false, nb = false;
    const int rn = r0 + 8 * 16;
    if (rn < p1) load(rn, NA, NB, na, nb);
    float slo, shi;
    score_rows<NG>(RA, RB, st.frag, wa, wb, lane, slo, shi);
    if (c == 0 && va) ot[r0 + g] = slo;
    if (c == 1 && vb) ot[r0 + g + 8] = shi;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      RA[i] = NA[i];
      RB[i] = NB[i];
    }
    va = na;
    vb = nb;
  }
}

// fp32: one warp per row; lane l holds dims 4l..4l+3.  Shared: head list + q rows [m][128].
template <bool GATHER>
__global__ void __launch_bounds__(kScoreThreads)
    score_f32_kernel(const float* __restrict__ q, const float* __restrict__ w, const float* __restrict__ k,
                     int64_t k_seq_stride, const int32_t* __restrict__ n, const int32_t* __restrict__ heads,
                     int h, int H_I, int L, const int32_t* __restrict__ rows, int P, float* __restrict__ out,
                     int64_t ld) {
  extern __shared__ __align__(16) float qs[];  // [H_I or h][kD]
  __shared__ int hl[kMaxHeads];
  __shared__ float wsel[kMaxHeads];
  __shared__ int m_sh;
  const int t = blockIdx.y;
  const int nt = clamp_len(n[t], L);
  const int npos = GATHER ? P : nt;
  const int p0 = blockIdx.x * kRowsPerChunk;
  if (p0 >= npos) return;
  const int p1 = min(p0 + kRowsPerChunk, npos);
  stage_head_list(heads, h, H_I, t, heads ? h : H_I, hl, &m_sh);
  __syncthreads();
  const int m = m_sh;
  if ((int)threadIdx.x < m) wsel[threadIdx.x] = w[(int64_t)t * H_I + hl[threadIdx.x]];
  for (int e = threadIdx.x; e < m * kD; e += kScoreThreads)
    qs[e] = q[((int64_t)t * H_I + hl[e / kD]) * kD + (e % kD)];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* kt = k + (int64_t)t * k_seq_stride;
  for (int p = p0 + warp; p < p1; p += kScoreThreads / 32) {
    int s = p;
    bool valid = true;
    if (GATHER) {
      s = rows[(int64_t)t * P + p];
      valid = s >= 0 && s < nt;
    }
    if (!valid) continue;  // warp-uniform
    const float4 kv = reinterpret_cast<const float4*>(kt + (int64_t)s * kD)[lane];
    float acc = 0.f;
    for (int a = 0; a < m; ++a) {
      const float4 qv = reinterpret_cast<const float4*>(qs + a * kD)[lane];
      float d = qv.x * kv.x;
      d = fmaf(qv.y, kv.y, d);
      d = fmaf(qv.z, kv.z, d);
      d = fmaf(qv.w, kv.w, d);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      acc = fmaf(wsel[a], relu(d), acc);
    }
    if (lane == 0) out[(int64_t)t * ld + p] = __fadd_rn(acc, 0.0f);
  }
}

int num_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    sms = v > 0 ? v : 148;
  }
  return sms;
}

template <int NG>
void launch_bf16(bool gather, bool persist, cudaStream_t s, const void* q, const float* w, const void* k,
                 int64_t k_seq_stride, const int32_t* n, const int32_t* heads, int h, int H_I, int T, int L,
                 const int32_t* rows, int P, float* out, int64_t ld) {
  auto qb = static_cast<const __nv_bfloat16*>(q);
  auto kb = static_cast<const __nv_bfloat16*>(k);
  if (persist) {
    const size_t smem = sizeof(int) * ((size_t)T + 1);
    const DenseList none{};
    if (gather) {
      cudaFuncSetAttribute(score_persist_kernel<NG, kModeGather>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      launch_pdl(score_persist_kernel<NG, kModeGather>, 2 * num_sms(), kScoreThreads, smem, s, qb, w, kb,
                 k_seq_stride, n, heads, h, H_I, L, T, rows, P, out, ld, none);
    } else {
      cudaFuncSetAttribute(score_persist_kernel<NG, kModeRows>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      launch_pdl(score_persist_kernel<NG, kModeRows>, 2 * num_sms(), kScoreThreads, smem, s, qb, w, kb,
                 k_seq_stride, n, heads, h, H_I, L, T, rows, P, out, ld, none);
    }
  } else if (gather) {
    const dim3 grid((P + kGatherRowsPerChunk - 1) / kGatherRowsPerChunk, T);
    score_grid_kernel<NG, true><<<grid, kScoreThreads, 0, s>>>(qb, w, kb, k_seq_stride, n, heads, h, H_I, L, rows, P,
                                                               out, ld);
  } else {
    const dim3 grid((L + kRowsPerChunk - 1) / kRowsPerChunk, T);
    score_grid_kernel<NG, false><<<grid, kScoreThreads, 0, s>>>(qb, w, kb, k_seq_stride, n, heads, h, H_I, L, rows,
                                                                P, out, ld);
  }
}

}  // namespace

void launch_scores(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                   const int32_t* n, const int32_t* heads, int T, int L, int H_I, int h, const int32_t* rows,
                   int P, float* out, int64_t ld, cudaStream_t s) {
  if (T <= 0) return;
  const int npos = rows ? P : L;
  if (npos <= 0) return;
  const bool gather = rows != nullptr;
  if (dt == DType::F32) {
    const dim3 grid((npos + kRowsPerChunk - 1) / kRowsPerChunk, T);
    const int m = heads ? h : H_I;
    const size_t smem = sizeof(float) * (size_t)m * kD;
    if (gather) {
      cudaFuncSetAttribute(score_f32_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      score_f32_kernel<true><<<grid, kScoreThreads, smem, s>>>(
          static_cast<const float*>(q), w, static_cast<const float*>(k), k_seq_stride, n, heads, h, H_I, L, rows,
          P, out, ld);
    } else {
      cudaFuncSetAttribute(score_f32_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      score_f32_kernel<false><<<grid, kScoreThreads, smem, s>>>(
          static_cast<const float*>(q), w, static_cast<const float*>(k), k_seq_stride, n, heads, h, H_I, L, rows,
          P, out, ld);
    }
    return;
  }
  // one shared cache: tensor-core contraction over blocks of queries
  if (!gather && k_seq_stride == 0 && launch_scores_tc(q, w, k, n, heads, T, L, H_I, h, out, ld, s)) return;
  // dense scores of gathered candidates (MISA-dagger re-rank): tensor-core contraction per 128 rows
  if (gather && !heads && launch_rerank_tc(q, w, k, k_seq_stride, n, T, L, H_I, rows, P, out, ld, s)) return;
  const int m = heads ? h : H_I;
  const int ng = (m + 7) / 8;
  // persistent schedule for per-query caches and for gathered candidate lists
  const bool persist = (gather || k_seq_stride != 0) && T <= kMaxPersistQueries;
  switch (ng) {
#define MISA_NG_CASE(NGV)                                                                               \
  case NGV:                                                                                             \
    launch_bf16<NGV>(gather, persist, s, q, w, k, k_seq_stride, n, heads, h, H_I, T, L, rows, P, out, ld); \
    break;
    MISA_NG_CASE(1)
    MISA_NG_CASE(2)
    MISA_NG_CASE(3)
    MISA_NG_CASE(4)
    MISA_NG_CASE(5)
    MISA_NG_CASE(6)
    MISA_NG_CASE(7)
    MISA_NG_CASE(8)
    MISA_NG_CASE(9)
    MISA_NG_CASE(10)
    MISA_NG_CASE(11)
    MISA_NG_CASE(12)
    MISA_NG_CASE(13)
    MISA_NG_CASE(14)
    MISA_NG_CASE(15)
    MISA_NG_CASE(16)
#undef MISA_NG_CASE
    default:
      break;
  }
}

size_t dense_list_smem(int T, int H_I) {
  const int ngf = (H_I + 7) / 8;
  return ((size_t)T + 1) * sizeof(int) + 15 + (size_t)ngf * 8 * 32 * sizeof(uint2) + kMaxHeads * sizeof(float) +
         (size_t)(kScoreThreads / 32) * kRing * (kD * 2 + sizeof(uint2));
}

bool launch_scores_sample(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n,
                          const int32_t* heads, int T, int L, int H_I, int h, int cap, float* out, int64_t ld,
                          cudaStream_t s) {
  if (h < 1 || h > 8 || T < 1 || T > kMaxPersistQueries || k_seq_stride == 0) return false;
  DenseList dl{};
  dl.cap = cap;
  const size_t smem = sizeof(int) * ((size_t)T + 1);
  cudaFuncSetAttribute(score_persist_kernel<1, kModeSample>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(score_persist_kernel<1, kModeSample>, 2 * num_sms(), kScoreThreads, smem, s,
             static_cast<const __nv_bfloat16*>(q), w, static_cast<const __nv_bfloat16*>(k), k_seq_stride, n, heads, h,
             H_I, L, T, static_cast<const int32_t*>(nullptr), 0, out, ld, dl);
  return true;
}

bool launch_scores_dense_list(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n,
                              const int32_t* heads, int T, int L, int H_I, int h, float* out, int64_t ld,
                              const DenseList& dl, cudaStream_t s) {
  if (h < 1 || h > 8 || T < 1 || T > kMaxPersistQueries || k_seq_stride == 0 || H_I > kMaxHeads) return false;
  const size_t smem = dense_list_smem(T, H_I);
  if (smem > kDenseListMaxSmem) return false;
  cudaFuncSetAttribute(score_persist_kernel<1, kModeList>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(score_persist_kernel<1, kModeList>, 2 * num_sms(), kScoreThreads, smem, s,
             static_cast<const __nv_bfloat16*>(q), w, static_cast<const __nv_bfloat16*>(k), k_seq_stride, n, heads, h,
             H_I, L, T, static_cast<const int32_t*>(nullptr), 0, out, ld, dl);
  return true;
}

MISA_BAD_ID_READER(read_and_clear_bad_ids_score)

}  // namespace misa
