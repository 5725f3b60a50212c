// Block mean-pool of the index-key cache and the block-pooled router.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", Technical
// Summary, "Methodology: MISA", "Lightweight Block-Pooled Router": the prefix is cut into
// M = ceil(L/B) blocks, each block is represented by the mean of its index keys, the per-head
// affinities against those pooled keys are aggregated into one score per head, and the top-h
// heads are routed.  Aggregation used here: r_{t,j} = w_{t,j} * sum_b max(0, q_{t,j} . kbar_b).
//
// Data layout: keys [L, 128] (bf16 or fp32) per cache, pooled keys kbar [M, 128] fp32 per cache.
// Every router path reads the pooled keys of all blocks of a prefix but the last from kbar and
// averages the last block (full or partial) from the keys, so the newest key is always seen and a
// decode loop pools a block only once the prefix has moved past it.
// bf16 queries: one kernel.  One CTA per (query, tile of 128 pooled blocks) multiplies the tile
// with the query's H_I head vectors on the tensor cores (see route_affinity_mma_kernel); the CTA
// whose tile holds the last block averages that block's keys itself; per-tile sums go to
// workspace and the query's last tile to finish adds them in tile order (deterministic), applies
// w and picks the top-h heads with warp shuffles.
// fp32 queries: CUDA cores, one CTA per (query, tile of 64 blocks) with a 4-head x 4-block
// register tile per thread, then a one-warp-per-query selection kernel.
#include <cuda_bf16.h>

#include <algorithm>

#include "kernels.cuh"

namespace misa {

namespace {

// One CTA of 1024 threads per block: 16 row groups x 64 column pairs, so a 128-key block is read
// with every load in flight at once.
template <DType DT>
__global__ void __launch_bounds__(1024) pool_kernel(const void* k, int64_t k_seq_stride, int L, int B,
                                                    float* kbar, int64_t kbar_seq_stride, int b0) {
  constexpr int RG = 16;
  __shared__ float part[RG][kD];
  const int b = b0 + blockIdx.x, seq = blockIdx.y;
  const size_t esz = DT == DType::BF16 ? 2 : 4;
  const void* kseq = static_cast<const char*>(k) + (int64_t)seq * k_seq_stride * esz;
  const int s0 = b * B, s1 = min(s0 + B, L);
  const int cp = threadIdx.x & 63, rg = threadIdx.x >> 6;
  float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
  for (int s = s0 + rg; s < s1; s += RG) {
    if (DT == DType::BF16) {
      const uint32_t x = reinterpret_cast<const uint32_t*>(kseq)[(int64_t)s * (kD / 2) + cp];
      a0 += bf16_lo(x);
      a1 += bf16_hi(x);
    } else {
      const float2 x = reinterpret_cast<const float2*>(kseq)[(int64_t)s * (kD / 2) + cp];
      a0 += x.x;
      a1 += x.y;
    }
  }
  part[rg][2 * cp] = a0;
  part[rg][2 * cp + 1] = a1;
  __syncthreads();
  if (threadIdx.x < kD) {
    float sum = 0.f;
#pragma unroll
    for (int r = 0; r < RG; ++r) sum += part[r][threadIdx.x];
    kbar[(int64_t)seq * kbar_seq_stride + (int64_t)b * kD + threadIdx.x] = sum / (float)(s1 - s0);
  }
}

// Mean of the last block [kbar_blocks(n_t, B) * B, n_t) of every query's prefix (full or partial).
template <DType DT>
__global__ void __launch_bounds__(256) partial_mean_kernel(const void* k, int64_t k_seq_stride,
                                                           const int32_t* n, int L, int B, float* pm) {
  __shared__ float part[16 * kD];
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  if (nt == 0) return;
  const size_t esz = DT == DType::BF16 ? 2 : 4;
  const void* kseq = static_cast<const char*>(k) + (int64_t)t * k_seq_stride * esz;
  const float m = block_mean_rows<DT>(kseq, kbar_blocks(nt, B) * B, nt, part);
  if (threadIdx.x < kD) pm[(int64_t)t * kD + threadIdx.x] = m;
}

// Per (query, 64-block tile): partial[t, c, j] = sum over the tile's blocks b < M_t of
// max(0, q_{t,j} . kbar_b).  blockDim = 4*H_I threads: (H_I/4 head groups) x 16 block lanes.
template <DType DT>
__global__ void __launch_bounds__(512) route_affinity_kernel(const void* q, const float* kbar,
                                                             int64_t kbar_seq_stride, const float* pm,
                                                             const int32_t* n, int L, int H_I, int B,
                                                             int nch, float* partial) {
  extern __shared__ __align__(16) float smem[];
  const int t = blockIdx.y, c = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const int nfull = kbar_blocks(nt, B), Mt = (nt + B - 1) / B;  // block nfull (< Mt) is the last
  const int bb = c * kRouteTile;
  if (bb >= Mt) return;
  const int QS = H_I + 4, KS = kRouteTile + 4;
  float* qT = smem;            // [kD][QS]  q of the H_I heads, transposed
  float* kT = smem + kD * QS;  // [kD][KS]  pooled keys of the tile, transposed
  const int nthr = blockDim.x, tid = threadIdx.x;
  for (int e = tid; e < H_I * kD; e += nthr) {
    const int j = e / kD, dd = e % kD;
    float v;
    if (DT == DType::BF16) {
      const uint16_t x = reinterpret_cast<const uint16_t*>(q)[((int64_t)t * H_I + j) * kD + dd];
      v = __uint_as_float((uint32_t)x << 16);
    } else {
      v = reinterpret_cast<const float*>(q)[((int64_t)t * H_I + j) * kD + dd];
    }
    qT[dd * QS + j] = v;
  }
  const float* kb = kbar + (int64_t)t * kbar_seq_stride;
  for (int e = tid; e < kRouteTile * kD; e += nthr) {
    const int bl = e / kD, dd = e % kD, b = bb + bl;
    float v = 0.f;
    if (b < nfull) v = kb[(int64_t)b * kD + dd];
    else if (b < Mt) v = pm[(int64_t)t * kD + dd];  // the last block, averaged from the keys
    kT[dd * KS + bl] = v;
  }
  __syncthreads();

  const int hg = tid >> 4, bl = tid & 15;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int dd = 0; dd < kD; ++dd) {
    const float4 a = *reinterpret_cast<const float4*>(&qT[dd * QS + 4 * hg]);
    const float4 b = *reinterpret_cast<const float4*>(&kT[dd * KS + 4 * bl]);
    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
  float hs[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (bb + 4 * bl + j < Mt) s += relu(acc[i][j]);
    hs[i] = s;
  }
#pragma unroll
  for (int o = 1; o < 16; o <<= 1)
#pragma unroll
    for (int i = 0; i < 4; ++i) hs[i] += __shfl_xor_sync(0xffffffffu, hs[i], o);
  if (bl == 0) {
    float* dst = partial + ((int64_t)t * nch + c) * H_I + 4 * hg;
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = hs[i];
  }
}

__device__ __forceinline__ bool head_better(float av, int aj, float bv, int bj) {
  return av > bv || (av == bv && aj < bj);
}

// One warp: the top-h heads by (r desc, j asc) with warp shuffles; lane l holds r of heads
// l + 32 i in v[i], live[i] false past H_I.
__device__ __forceinline__ void pick_heads_warp(float (&v)[kMaxHeads / 32], bool (&live)[kMaxHeads / 32], int h,
                                                int32_t* heads_t) {
  const int lane = threadIdx.x & 31;
  for (int rnd = 0; rnd < h; ++rnd) {
    float bv = 0.f;
    int bj = 0x7fffffff;
    bool have = false;
#pragma unroll
    for (int i = 0; i < kMaxHeads / 32; ++i) {
      const int j = lane + 32 * i;
      if (live[i] && (!have || head_better(v[i], j, bv, bj))) {
        bv = v[i];
        bj = j;
        have = true;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (oj != 0x7fffffff && (bj == 0x7fffffff || head_better(ov, oj, bv, bj))) {
        bv = ov;
        bj = oj;
      }
    }
    if (lane == 0) heads_t[rnd] = bj;
#pragma unroll
    for (int i = 0; i < kMaxHeads / 32; ++i)
      if (lane + 32 * i == bj) live[i] = false;
  }
}

// One warp: r_j = w_j * (sum of the nc per-tile partial sums in global memory, in tile order),
// then the top-h heads.  partial_t is [nch][H_I] for this query.
__device__ __forceinline__ void select_heads_warp(const float* partial_t, int nc, const float* w_t, int H_I, int h,
                                                  int32_t* heads_t, float* r_t) {
  const int lane = threadIdx.x & 31;
  float v[kMaxHeads / 32];
  bool live[kMaxHeads / 32];
#pragma unroll
  for (int i = 0; i < kMaxHeads / 32; ++i) {
    const int j = lane + 32 * i;
    live[i] = j < H_I;
    v[i] = 0.f;
    if (live[i]) {
      float s = 0.f;
#pragma unroll 8
      for (int c = 0; c < nc; ++c) s += __ldcg(partial_t + (int64_t)c * H_I + j);
      v[i] = w_t[j] * s;
      if (r_t) r_t[j] = v[i];
    }
  }
  pick_heads_warp(v, live, h, heads_t);
}

// One warp per query (fp32 path).
__global__ void __launch_bounds__(32) route_select_kernel(const float* partial, const float* w,
                                                          const int32_t* n, int L, int H_I, int B,
                                                          int nch, int tile, int h, int32_t* heads,
                                                          float* r_opt) {
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const int Mt = (nt + B - 1) / B;
  select_heads_warp(partial + (int64_t)t * nch * H_I, (Mt + tile - 1) / tile, w + (int64_t)t * H_I, H_I, h,
                    heads + (int64_t)t * h, r_opt ? r_opt + (int64_t)t * H_I : nullptr);
}

constexpr int kRouteMmaTile = 128;  // pooled blocks per CTA of the tensor-core router (8 warps x 16)

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// x = hi + mid + lo exactly up to the last ~24 bits: each part is the bf16 rounding of what the
// previous parts leave (the subtractions are exact in fp32).
__device__ __forceinline__ void split3(float x, float& hi, float& mid, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  const float r1 = x - hi;
  mid = __bfloat162float(__float2bfloat16_rn(r1));
  lo = r1 - mid;
}

// Tensor-core router for bf16 queries.  Per (query, tile of 128 pooled blocks): the GEMM
// kbar[128 blocks, 128] x q^T[128, H_I] on mma.m16n8k16.  bf16 q is exact; each fp32 pooled key is
// split into three bf16 parts and the three products are accumulated in fp32, which keeps the
// dot products at fp32 accuracy.  The pooled keys are loaded straight into A fragments (lane
// (g, c) of a warp holds dims 16kk + 4c .. +3 of blocks g and g+8 at k-step kk, and the q
// fragments staged in shared memory use the same dimension order).  Blocks below
// kbar_blocks(n_t, B) come from kbar; the last block of the prefix is averaged from the keys by
// the CTA whose tile holds it (pm_in: averaged beforehand).  Every thread issues its pooled-key
// loads first, then the q-fragment loads, then (one CTA per query) the last block's key loads,
// so the three overlap.  Epilogue: relu, sum over the tile's blocks per head (quad shuffles, then
// a fixed-order sum over the 8 warps).
template <int NG>
__global__ void __launch_bounds__(256) route_affinity_mma_kernel(const __nv_bfloat16* __restrict__ q,
                                                                 const float* __restrict__ w,
                                                                 const __nv_bfloat16* __restrict__ k,
                                                                 int64_t k_seq_stride,
                                                                 const float* __restrict__ kbar,
                                                                 int64_t kbar_seq_stride,
                                                                 const int32_t* __restrict__ n, int L, int B, int h,
                                                                 int nch, float* __restrict__ partial,
                                                                 uint32_t* __restrict__ done,
                                                                 int32_t* __restrict__ heads, float* __restrict__ r_opt,
                                                                 const float* __restrict__ pm_in) {
  constexpr int H = NG * 8;
  __shared__ uint2 frag[NG][8][32];
  __shared__ float wsum[8][H];
  __shared__ float part[16 * kD];
  __shared__ __align__(16) float pms[kD];  // mean of the last block
  __shared__ int last;
  const int t = blockIdx.y, c0 = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  const int nt = clamp_len(n[t], L);
  const int nk = kbar_blocks(nt, B), Mt = (nt + B - 1) / B;
  const int nc = (Mt + kRouteMmaTile - 1) / kRouteMmaTile;
  const int bb = c0 * kRouteMmaTile;
  if (bb >= Mt) {
    if (Mt == 0 && c0 == 0 && threadIdx.x < 32)  // empty prefix: every router score is 0
      select_heads_warp(partial, 0, w + (int64_t)t * H, H, h, heads + (int64_t)t * h,
                        r_opt ? r_opt + (int64_t)t * H : nullptr);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int ba = bb + warp * 16 + g, bq = ba + 8;
  const float* kb = kbar + (int64_t)t * kbar_seq_stride;
  float4 XA[8], XB[8];  // the warp's two pooled-key rows, all loads in flight at once
  {
    const float* rowa = ba < nk ? kb + (int64_t)ba * kD : nullptr;
    const float* rowb = bq < nk ? kb + (int64_t)bq * kD : nullptr;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      XA[kk] = rowa ? __ldg(reinterpret_cast<const float4*>(rowa + 16 * kk + 4 * c)) : make_float4(0, 0, 0, 0);
      XB[kk] = rowb ? __ldg(reinterpret_cast<const float4*>(rowb + 16 * kk + 4 * c)) : make_float4(0, 0, 0, 0);
    }
  }
  {  // q fragments: every thread issues its loads together (256 threads)
    constexpr int kPer = (NG * 8 * 32 + 255) / 256;
    uint2 v[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = (int)threadIdx.x + 256 * i;
      if (e < NG * 8 * 32) {
        const int ng = e >> 8, kk = (e >> 5) & 7, ln = e & 31;
        const int gg = ln >> 2, cc = ln & 3;
        v[i] = __ldg(reinterpret_cast<const uint2*>(q + ((int64_t)t * H + ng * 8 + gg) * kD + 16 * kk + 4 * cc));
      }
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = (int)threadIdx.x + 256 * i;
      if (e < NG * 8 * 32) frag[e >> 8][(e >> 5) & 7][e & 31] = v[i];
    }
  }
  if (nk >= bb && nk < bb + kRouteMmaTile) {  // this tile holds the last block
    if (pm_in) {  // averaged beforehand (paged caches)
      if (threadIdx.x < kD) pms[threadIdx.x] = pm_in[(int64_t)t * kD + threadIdx.x];
    } else {
      const float m = block_mean_rows<DType::BF16>(k + (int64_t)t * k_seq_stride, nk * B, nt, part);
      if (threadIdx.x < kD) pms[threadIdx.x] = m;
    }
  }
  __syncthreads();
  if (ba == nk) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) XA[kk] = *reinterpret_cast<const float4*>(pms + 16 * kk + 4 * c);
  }
  if (bq == nk) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) XB[kk] = *reinterpret_cast<const float4*>(pms + 16 * kk + 4 * c);
  }
  float acc[NG][4];
#pragma unroll
  for (int ng = 0; ng < NG; ++ng) acc[ng][0] = acc[ng][1] = acc[ng][2] = acc[ng][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const float4 xa = XA[kk], xb = XB[kk];
    float ah[4], am[4], al[4], bh[4], bm[4], bl[4];
    split3(xa.x, ah[0], am[0], al[0]);
    split3(xa.y, ah[1], am[1], al[1]);
    split3(xa.z, ah[2], am[2], al[2]);
    split3(xa.w, ah[3], am[3], al[3]);
    split3(xb.x, bh[0], bm[0], bl[0]);
    split3(xb.y, bh[1], bm[1], bl[1]);
    split3(xb.z, bh[2], bm[2], bl[2]);
    split3(xb.w, bh[3], bm[3], bl[3]);
    const uint32_t A[3][4] = {
        {pack_bf16x2(ah[0], ah[1]), pack_bf16x2(bh[0], bh[1]), pack_bf16x2(ah[2], ah[3]), pack_bf16x2(bh[2], bh[3])},
        {pack_bf16x2(am[0], am[1]), pack_bf16x2(bm[0], bm[1]), pack_bf16x2(am[2], am[3]), pack_bf16x2(bm[2], bm[3])},
        {pack_bf16x2(al[0], al[1]), pack_bf16x2(bl[0], bl[1]), pack_bf16x2(al[2], al[3]), pack_bf16x2(bl[2], bl[3])}};
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      const uint2 bf = frag[ng][kk][lane];
#pragma unroll
      for (int p = 0; p < 3; ++p) mma_16816(acc[ng], A[p][0], A[p][1], A[p][2], A[p][3], bf.x, bf.y);
    }
  }
  const bool va = ba < Mt, vb = bq < Mt;
#pragma unroll
  for (int ng = 0; ng < NG; ++ng) {
    float h0 = (va ? relu(acc[ng][0]) : 0.f) + (vb ? relu(acc[ng][2]) : 0.f);
    float h1 = (va ? relu(acc[ng][1]) : 0.f) + (vb ? relu(acc[ng][3]) : 0.f);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      h0 += __shfl_xor_sync(0xffffffffu, h0, o);
      h1 += __shfl_xor_sync(0xffffffffu, h1, o);
    }
    if (g == 0) {
      wsum[warp][ng * 8 + 2 * c] = h0;
      wsum[warp][ng * 8 + 2 * c + 1] = h1;
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < H; j += blockDim.x) {
    float s = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < 8; ++w8) s += wsum[w8][j];
    partial[((int64_t)t * nch + c0) * H + j] = s;
  }
  // the query's last tile to finish sums the tiles in order and picks the heads
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(done + t, 1u) == (uint32_t)(nc - 1);
  __syncthreads();
  if (last && threadIdx.x < 32) {
    __threadfence();
    select_heads_warp(partial + (int64_t)t * nch * H, nc, w + (int64_t)t * H, H, h, heads + (int64_t)t * h,
                      r_opt ? r_opt + (int64_t)t * H : nullptr);
  }
}

// kbar [M, 128] fp32 -> parts [3][M][128] bf16 with kbar = hi + mid + lo to fp32 accuracy (the
// operands of the tensor-core router for one shared cache).
__global__ void __launch_bounds__(256) kbar_split_kernel(const float* __restrict__ kbar, int64_t count,
                                                         __nv_bfloat16* __restrict__ parts) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    float hi, mid, lo;
    split3(kbar[i], hi, mid, lo);
    parts[i] = __float2bfloat16_rn(hi);
    parts[count + i] = __float2bfloat16_rn(mid);
    parts[2 * count + i] = __float2bfloat16_rn(lo);
  }
}

// One CTA per query, after the tensor-core router's per-tile sums Sp[t][tile][j] over the pooled
// blocks below kbar_blocks(n_t, B): adds max(0, q_{t,j} . mean of the last block) (keys
// [kbar_blocks(n_t, B) B, n_t), averaged here), then r_j = w_j * total and the top-h heads.  The q
// rows and the per-tile sums are requested before the mean is formed, so their loads overlap it.
__global__ void __launch_bounds__(256) route_finish_kernel(const __nv_bfloat16* __restrict__ q,
                                                           const float* __restrict__ w,
                                                           const __nv_bfloat16* __restrict__ k,
                                                           const int32_t* __restrict__ n, int L, int H_I, int B,
                                                           int h, const float* __restrict__ Sp, int nch,
                                                           int tile, int32_t* __restrict__ heads,
                                                           float* __restrict__ r_opt) {
  constexpr int kHeadsPerWarp = kMaxHeads / 8;
  __shared__ float part[16 * kD];
  __shared__ __align__(16) float pm[kD];
  __shared__ float pmd[kMaxHeads];
  __shared__ float tot[kMaxHeads];
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const int nf = kbar_blocks(nt, B), c = nt - nf * B;  // c keys in the last block (0: empty prefix)
  const int ntiles = (nf + tile - 1) / tile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint2 qv[kHeadsPerWarp];  // lane's 4 dims of this warp's heads warp, warp + 8, ...
#pragma unroll
  for (int i = 0; i < kHeadsPerWarp; ++i) {
    const int j = warp + 8 * i;
    qv[i] = (c > 0 && j < H_I) ? *reinterpret_cast<const uint2*>(q + ((int64_t)t * H_I + j) * kD + 4 * lane)
                               : make_uint2(0u, 0u);
  }
  float spsum = 0.f;
  if ((int)threadIdx.x < H_I) {
#pragma unroll 4
    for (int i = 0; i < ntiles; ++i) spsum += __ldcg(Sp + ((int64_t)t * nch + i) * H_I + threadIdx.x);
  }
  if (c > 0) {
    const float m = block_mean_rows<DType::BF16>(k, nt - c, nt, part);
    if (threadIdx.x < kD) pm[threadIdx.x] = m;
  }
  __syncthreads();
  if (c > 0) {
    const float4 p4 = *reinterpret_cast<const float4*>(pm + 4 * lane);
#pragma unroll
    for (int i = 0; i < kHeadsPerWarp; ++i) {
      const int j = warp + 8 * i;
      if (j < H_I) {  // uniform across the warp
        const uint2 x = qv[i];
        float d = bf16_lo(x.x) * p4.x + bf16_hi(x.x) * p4.y + bf16_lo(x.y) * p4.z + bf16_hi(x.y) * p4.w;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) pmd[j] = relu(d);
      }
    }
  }
  __syncthreads();
  if ((int)threadIdx.x < H_I) tot[threadIdx.x] = spsum + (c > 0 ? pmd[threadIdx.x] : 0.f);
  __syncthreads();
  if (warp == 0) {
    float v[kMaxHeads / 32];
    bool live[kMaxHeads / 32];
#pragma unroll
    for (int i = 0; i < kMaxHeads / 32; ++i) {
      const int j = lane + 32 * i;
      live[i] = j < H_I;
      v[i] = live[i] ? w[(int64_t)t * H_I + j] * tot[j] : 0.f;
      if (live[i] && r_opt) r_opt[(int64_t)t * H_I + j] = v[i];
    }
    pick_heads_warp(v, live, h, heads + (int64_t)t * h);
  }
}

}  // namespace

void launch_kbar_split(const float* kbar, int M, __nv_bfloat16* parts, cudaStream_t s) {
  const int64_t count = (int64_t)M * kD;
  const int grid = (int)std::min<int64_t>((count + 255) / 256, 4096);
  if (count > 0) kbar_split_kernel<<<grid, 256, 0, s>>>(kbar, count, parts);
}

void launch_route_finish(const __nv_bfloat16* q, const float* w, const __nv_bfloat16* k, const int32_t* n, int T,
                         int L, int H_I, int B, int h, const float* Sp, int nch, int tile, int32_t* heads,
                         float* r_opt, cudaStream_t s) {
  if (T > 0) route_finish_kernel<<<T, 256, 0, s>>>(q, w, k, n, L, H_I, B, h, Sp, nch, tile, heads, r_opt);
}

void launch_pool(DType dt, const void* k, int64_t k_seq_stride, int n_seq, int L, int B, float* kbar,
                 int64_t kbar_seq_stride, int b0, int b1, cudaStream_t s) {
  if (b1 <= b0 || n_seq <= 0) return;
  dim3 grid(b1 - b0, n_seq);
  if (dt == DType::BF16)
    pool_kernel<DType::BF16><<<grid, 1024, 0, s>>>(k, k_seq_stride, L, B, kbar, kbar_seq_stride, b0);
  else
    pool_kernel<DType::F32><<<grid, 1024, 0, s>>>(k, k_seq_stride, L, B, kbar, kbar_seq_stride, b0);
}

int route_chunks(int L, int B) {
  const int M = (L + B - 1) / B;
  return (M + kRouteTile - 1) / kRouteTile;
}

void launch_route(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                  const float* kbar, int64_t kbar_seq_stride, const int32_t* n, int T, int L, int H_I,
                  int B, int h, int32_t* heads, float* r_opt, float* pm, float* partial, uint32_t* done,
                  __nv_bfloat16* kbar_parts, const float* pm_in, cudaStream_t s) {
  if (T <= 0) return;
  const int M = (L + B - 1) / B;
  // many queries on one shared cache: tensor-core contraction over blocks of queries
  if (dt == DType::BF16 && !pm_in && k_seq_stride == 0 && kbar_seq_stride == 0 && T >= kRouteTcMinQueries &&
      launch_route_tc(q, w, k, kbar, n, T, L, H_I, B, h, heads, r_opt, kbar_parts, partial, route_chunks(L, B), s))
    return;
  if (dt == DType::BF16) {
    const int nch = (M + kRouteMmaTile - 1) / kRouteMmaTile;
    const dim3 grid(nch, T);
    cudaMemsetAsync(done, 0, sizeof(uint32_t) * (size_t)T, s);
    auto qb = static_cast<const __nv_bfloat16*>(q);
    auto kb = static_cast<const __nv_bfloat16*>(k);
    switch (H_I / 8) {
#define MISA_ROUTE_CASE(NGV)                                                                                  \
  case NGV:                                                                                                   \
    launch_pdl(route_affinity_mma_kernel<NGV>, grid, 256, 0, s, qb, w, kb, k_seq_stride, kbar, kbar_seq_stride, n, L, \
               B, h, nch, partial, done, heads, r_opt, pm_in);                                                \
    break;
      MISA_ROUTE_CASE(1)
      MISA_ROUTE_CASE(2)
      MISA_ROUTE_CASE(3)
      MISA_ROUTE_CASE(4)
      MISA_ROUTE_CASE(5)
      MISA_ROUTE_CASE(6)
      MISA_ROUTE_CASE(7)
      MISA_ROUTE_CASE(8)
      MISA_ROUTE_CASE(9)
      MISA_ROUTE_CASE(10)
      MISA_ROUTE_CASE(11)
      MISA_ROUTE_CASE(12)
      MISA_ROUTE_CASE(13)
      MISA_ROUTE_CASE(14)
      MISA_ROUTE_CASE(15)
      MISA_ROUTE_CASE(16)
#undef MISA_ROUTE_CASE
      default:
        break;
    }
  } else {
    const int nch = route_chunks(L, B);
    const size_t smem = sizeof(float) * (size_t)kD * ((H_I + 4) + (kRouteTile + 4));
    if (pm_in)
      pm = const_cast<float*>(pm_in);
    else
      partial_mean_kernel<DType::F32><<<T, 256, 0, s>>>(k, k_seq_stride, n, L, B, pm);
    cudaFuncSetAttribute(route_affinity_kernel<DType::F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    route_affinity_kernel<DType::F32><<<dim3(nch, T), 4 * H_I, smem, s>>>(q, kbar, kbar_seq_stride, pm, n, L,
                                                                           H_I, B, nch, partial);
    route_select_kernel<<<T, 32, 0, s>>>(partial, w, n, L, H_I, B, nch, kRouteTile, h, heads, r_opt);
  }
}

}  // namespace misa
