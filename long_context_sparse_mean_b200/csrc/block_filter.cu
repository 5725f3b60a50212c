// Token-axis block filter composed with MISA.
//
// "HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse Attention" (arXiv 2603.28458),
// abstract: a block-level coarse stage scores pooled block representatives and discards regions,
// then the indexer runs only on the tokens of the kept candidate blocks.  "MISA: Mixture of Indexer
// Sparse Attention for Long-Context LLM Inference", "Problem Statement" and "Significance and
// Claims": that token-axis saving and MISA's head-axis routing are complementary.
//
// Composition computed here, for query t with routed heads R_t:
//   S_{t,b} = sum_{j in R_t} w_{t,j} * max(0, q_{t,j} . kbar_b)      (b < M_t = ceil(n_t/B))
// with kbar_b the router's block means (the last block, full or partial, averaged from the keys).  The
// m best blocks are kept by the per-row top-k, expand_blocks_kernel turns them into token ids, and
// the gather scorer and the per-row top-k score and select those tokens with the routed heads.
//
// Cost per query: M_t pooled keys (fp32, 512 B each) for the block scores, then m*B keys instead of
// n_t for the token scores.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace misa {

namespace {

constexpr int kBlockScoreThreads = 256;  // 8 warps
constexpr int kBlocksPerCta = 64;        // pooled blocks per CTA (8 per warp)

// Block scores of one query over pooled blocks [blockIdx.x * 64, +64) ∩ [0, M_t).  The routed
// heads' q rows are staged in shared memory as fp32 (dynamic, h * 128 floats).  A warp takes one
// pooled block at a time: lane l holds columns 4l..4l+3 of kbar_b, each head's dot product is a
// warp reduction.  The CTA whose range holds the last block first averages that block's keys.
template <DType DT>
__global__ void __launch_bounds__(kBlockScoreThreads) block_score_kernel(
    const void* __restrict__ q, const float* __restrict__ w, const void* __restrict__ k, int64_t k_seq_stride,
    const float* __restrict__ kbar, int64_t kbar_seq_stride, const int32_t* __restrict__ n,
    const int32_t* __restrict__ heads, int L, int H_I, int B, int h, float* __restrict__ S, int64_t ldS,
    int32_t* __restrict__ Mt_out) {
  extern __shared__ __align__(16) float qs[];  // [h][kD]
  __shared__ float ws_[kMaxHeads];
  __shared__ __align__(16) float pmean[kD];
  __shared__ float part[16 * kD];
  const int t = blockIdx.y;
  const int nt = clamp_len(n[t], L);
  const int Mt = (nt + B - 1) / B;
  const int nfull = kbar_blocks(nt, B);  // blocks read from kbar; block nfull (< Mt) is the last
  if (blockIdx.x == 0 && threadIdx.x == 0) Mt_out[t] = Mt;
  const int b0 = blockIdx.x * kBlocksPerCta;
  if (b0 >= Mt) return;
  const int b1 = min(b0 + kBlocksPerCta, Mt);
  const int tid = threadIdx.x;

  // routed heads: weight (0 for an index outside [0, H_I)) and q row in fp32
  for (int a = tid; a < h; a += kBlockScoreThreads) {
    const int j = heads[(int64_t)t * h + a];
    count_bad_id(kBadHead, blockIdx.x == 0 && (j < 0 || j >= H_I));  // once per query
    ws_[a] = (j >= 0 && j < H_I) ? w[(int64_t)t * H_I + j] : 0.f;
  }
  for (int e = tid; e < h * kD; e += kBlockScoreThreads) {
    const int a = e / kD, i = e % kD;
    const int j = heads[(int64_t)t * h + a];
    float v = 0.f;
    if (j >= 0 && j < H_I) {
      const int64_t off = ((int64_t)t * H_I + j) * kD + i;
      v = DT == DType::BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off])
                            : static_cast<const float*>(q)[off];
    }
    qs[e] = v;
  }
  // mean of the last block [nfull * B, nt)
  if (nfull < Mt && nfull >= b0 && nfull < b1) {
    const size_t esz = DT == DType::BF16 ? 2 : 4;
    const void* kseq = static_cast<const char*>(k) + (int64_t)t * k_seq_stride * esz;
    const float m = block_mean_rows<DT>(kseq, nfull * B, nt, part);
    if (tid < kD) pmean[tid] = m;
  }
  __syncthreads();

  const int lane = tid & 31, warp = tid >> 5;
  const float* kb_t = kbar + (int64_t)t * kbar_seq_stride;
  for (int b = b0 + warp; b < b1; b += kBlockScoreThreads / 32) {
    const float4 kv = b < nfull ? __ldg(reinterpret_cast<const float4*>(kb_t + (int64_t)b * kD) + lane)
                                : reinterpret_cast<const float4*>(pmean)[lane];
    float acc = 0.f;
    for (int a = 0; a < h; ++a) {
      const float4 qv = reinterpret_cast<const float4*>(qs + a * kD)[lane];
      float dot = qv.x * kv.x;
      dot = fmaf(qv.y, kv.y, dot);
      dot = fmaf(qv.z, kv.z, dot);
      dot = fmaf(qv.w, kv.w, dot);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      acc = fmaf(ws_[a], relu(dot), acc);
    }
    if (lane == 0) S[(int64_t)t * ldS + b] = acc;
  }
}

// Token ids of the kept blocks: position a*B + i of query t is token blocks[t, a]*B + i, or -1 when
// the slot is empty or the token lies past the prefix.
__global__ void expand_blocks_kernel(const int32_t* __restrict__ blocks, int m, const int32_t* __restrict__ n,
                                     int L, int B, int32_t* __restrict__ rows) {
  const int t = blockIdx.y;
  const int P = m * B;
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= P) return;
  const int nt = clamp_len(n[t], L);
  const int b = blocks[(int64_t)t * m + p / B];
  const int64_t s = (int64_t)b * B + p % B;
  rows[(int64_t)t * P + p] = (b >= 0 && s < nt) ? (int32_t)s : -1;
}

}  // namespace

void launch_block_scores(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                         const float* kbar, int64_t kbar_seq_stride, const int32_t* n, const int32_t* heads, int T,
                         int L, int H_I, int B, int h, float* S, int64_t ldS, int32_t* Mt, cudaStream_t s) {
  if (T <= 0) return;
  const int M = (L + B - 1) / B;
  const dim3 grid((M + kBlocksPerCta - 1) / kBlocksPerCta, T);
  const size_t smem = sizeof(float) * (size_t)h * kD;
  if (dt == DType::BF16) {
    cudaFuncSetAttribute(block_score_kernel<DType::BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    block_score_kernel<DType::BF16><<<grid, kBlockScoreThreads, smem, s>>>(
        q, w, k, k_seq_stride, kbar, kbar_seq_stride, n, heads, L, H_I, B, h, S, ldS, Mt);
  } else {
    cudaFuncSetAttribute(block_score_kernel<DType::F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    block_score_kernel<DType::F32><<<grid, kBlockScoreThreads, smem, s>>>(
        q, w, k, k_seq_stride, kbar, kbar_seq_stride, n, heads, L, H_I, B, h, S, ldS, Mt);
  }
}

void launch_expand_blocks(const int32_t* blocks, int m, const int32_t* n, int T, int L, int B, int32_t* rows,
                          cudaStream_t s) {
  if (T <= 0 || m <= 0) return;
  const int P = m * B;
  const dim3 grid((P + 255) / 256, T);
  expand_blocks_kernel<<<grid, 256, 0, s>>>(blocks, m, n, L, B, rows);
}

MISA_BAD_ID_READER(read_and_clear_bad_ids_block_filter)

}  // namespace misa
