// Block mean-pool of the index-key cache and the block-pooled router.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", Technical
// Summary, "Methodology: MISA", "Lightweight Block-Pooled Router": the prefix is cut into
// M = ceil(L/B) blocks, each block is represented by the mean of its index keys, the per-head
// affinities against those pooled keys are aggregated into one score per head, and the top-h
// heads are routed.  Aggregation used here: r_{t,j} = w_{t,j} * sum_b max(0, q_{t,j} . kbar_b).
//
// Data layout: keys [L, 128] (bf16 or fp32) per cache, pooled keys kbar [M, 128] fp32 per cache.
// Work split for the router: one CTA per (query, tile of 64 blocks); the CTA holds the query's
// H_I head vectors and the 64 pooled keys transposed in shared memory and every thread owns a
// 4-head x 4-block register tile, so each pair of float4 shared loads feeds 16 FMAs.  Partial
// sums per tile go to workspace and a one-warp-per-query kernel adds them in a fixed order
// (deterministic), applies w and picks the top-h heads with warp shuffles.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace misa {

namespace {

// Sum of key rows [s0, s1) of one cache, 256 threads: 4 row groups x 64 column pairs.
// Returns, in threads 0..127, the mean of column threadIdx.x (IEEE division by the count).
template <DType DT>
__device__ __forceinline__ float block_mean_256(const void* kseq, int s0, int s1, float (*part)[kD]) {
  const int cp = threadIdx.x & 63, rg = threadIdx.x >> 6;
  float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
  for (int s = s0 + rg; s < s1; s += 4) {
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
  float mean = 0.f;
  if (threadIdx.x < kD) {
    const int i = threadIdx.x;
    const float sum = ((part[0][i] + part[1][i]) + part[2][i]) + part[3][i];
    mean = sum / (float)(s1 - s0);
  }
  return mean;
}

template <DType DT>
__global__ void __launch_bounds__(256) pool_kernel(const void* k, int64_t k_seq_stride, int L, int B,
                                                   float* kbar, int64_t kbar_seq_stride, int b0) {
  __shared__ float part[4][kD];
  const int b = b0 + blockIdx.x, seq = blockIdx.y;
  const size_t esz = DT == DType::BF16 ? 2 : 4;
  const void* kseq = static_cast<const char*>(k) + (int64_t)seq * k_seq_stride * esz;
  const int s0 = b * B, s1 = min(s0 + B, L);
  const float m = block_mean_256<DT>(kseq, s0, s1, part);
  if (threadIdx.x < kD) kbar[(int64_t)seq * kbar_seq_stride + (int64_t)b * kD + threadIdx.x] = m;
}

// Mean of the partial last block [floor(n_t/B)*B, n_t) of every query whose prefix is not a
// multiple of B.
template <DType DT>
__global__ void __launch_bounds__(256) partial_mean_kernel(const void* k, int64_t k_seq_stride,
                                                           const int32_t* n, int L, int B, float* pm) {
  __shared__ float part[4][kD];
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const int c = nt % B;
  if (c == 0) return;
  const size_t esz = DT == DType::BF16 ? 2 : 4;
  const void* kseq = static_cast<const char*>(k) + (int64_t)t * k_seq_stride * esz;
  const float m = block_mean_256<DT>(kseq, nt - c, nt, part);
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
  const int nfull = nt / B, Mt = (nt + B - 1) / B;
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
    else if (b < Mt) v = pm[(int64_t)t * kD + dd];  // the partial last block
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

// One warp per query: r_j = w_j * sum over tiles; top-h heads by (r desc, j asc).
__global__ void __launch_bounds__(32) route_select_kernel(const float* partial, const float* w,
                                                          const int32_t* n, int L, int H_I, int B,
                                                          int nch, int h, int32_t* heads, float* r_opt) {
  const int t = blockIdx.x, lane = threadIdx.x;
  const int nt = clamp_len(n[t], L);
  const int Mt = (nt + B - 1) / B;
  const int nc = (Mt + kRouteTile - 1) / kRouteTile;
  float v[kMaxHeads / 32];
  bool live[kMaxHeads / 32];
#pragma unroll
  for (int i = 0; i < kMaxHeads / 32; ++i) {
    const int j = lane + 32 * i;
    live[i] = j < H_I;
    v[i] = 0.f;
    if (live[i]) {
      float s = 0.f;
      for (int c = 0; c < nc; ++c) s += partial[((int64_t)t * nch + c) * H_I + j];
      v[i] = w[(int64_t)t * H_I + j] * s;
      if (r_opt) r_opt[(int64_t)t * H_I + j] = v[i];
    }
  }
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
    if (lane == 0) heads[(int64_t)t * h + rnd] = bj;
#pragma unroll
    for (int i = 0; i < kMaxHeads / 32; ++i)
      if (lane + 32 * i == bj) live[i] = false;
  }
}

}  // namespace

void launch_pool(DType dt, const void* k, int64_t k_seq_stride, int n_seq, int L, int B, float* kbar,
                 int64_t kbar_seq_stride, int b0, int b1, cudaStream_t s) {
  if (b1 <= b0 || n_seq <= 0) return;
  dim3 grid(b1 - b0, n_seq);
  if (dt == DType::BF16)
    pool_kernel<DType::BF16><<<grid, 256, 0, s>>>(k, k_seq_stride, L, B, kbar, kbar_seq_stride, b0);
  else
    pool_kernel<DType::F32><<<grid, 256, 0, s>>>(k, k_seq_stride, L, B, kbar, kbar_seq_stride, b0);
}

int route_chunks(int L, int B) {
  const int M = (L + B - 1) / B;
  return (M + kRouteTile - 1) / kRouteTile;
}

void launch_route(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                  const float* kbar, int64_t kbar_seq_stride, const int32_t* n, int T, int L, int H_I,
                  int B, int h, int32_t* heads, float* r_opt, float* pm, float* partial, cudaStream_t s) {
  if (T <= 0) return;
  const int nch = route_chunks(L, B);
  const size_t smem = sizeof(float) * (size_t)kD * ((H_I + 4) + (kRouteTile + 4));
  if (dt == DType::BF16) {
    partial_mean_kernel<DType::BF16><<<T, 256, 0, s>>>(k, k_seq_stride, n, L, B, pm);
    cudaFuncSetAttribute(route_affinity_kernel<DType::BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    route_affinity_kernel<DType::BF16><<<dim3(nch, T), 4 * H_I, smem, s>>>(q, kbar, kbar_seq_stride, pm, n, L,
                                                                            H_I, B, nch, partial);
  } else {
    partial_mean_kernel<DType::F32><<<T, 256, 0, s>>>(k, k_seq_stride, n, L, B, pm);
    cudaFuncSetAttribute(route_affinity_kernel<DType::F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    route_affinity_kernel<DType::F32><<<dim3(nch, T), 4 * H_I, smem, s>>>(q, kbar, kbar_seq_stride, pm, n, L,
                                                                           H_I, B, nch, partial);
  }
  route_select_kernel<<<T, 32, 0, s>>>(partial, w, n, L, H_I, B, nch, h, heads, r_opt);
}

}  // namespace misa
