// Token scoring with a list of indexer heads:  out[t, p] = sum_{j in list} w_{t,j} relu(q_{t,j} . k_s)
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", Technical Summary,
// "Methodology: MISA", "Sparse Token Scoring" (the list is the h routed heads), "Hierarchical
// Variant (MISA-dagger)" (the list is all H_I heads and the tokens are gathered candidates) and
// "Problem Statement" (the dense indexer: all heads, all prefix tokens).
//
// bf16 path.  Per key the work is h x 128 multiply-adds against 256 bytes read, so with h = 8 a
// CUDA-core dot product would spend more issue slots on FMAs and shuffles than HBM allows; the
// contraction K[rows,128] x Q[128, heads] instead runs on the tensor cores with
// mma.m16n8k16 (bf16 in, fp32 accumulate).  Key rows are loaded straight from global memory
// into the A-fragment registers: the dot product is invariant under any permutation of the 128
// dimensions applied to both operands, so lane (g, c) of a warp loads the 16-byte chunks
// c, c+4, c+8, c+12 of rows g and g+8 (every load instruction of the warp reads 8 rows x 64
// contiguous bytes, all of each 32-byte sector used) and the query fragments staged in shared
// memory use the same dimension order.  No shared-memory round trip for K, no ldmatrix.  The
// epilogue applies relu, weights and sums the heads of a row inside the thread and over the 4
// lanes of a quad, and writes one fp32 score per key.
//
// Heads are summed in ascending head index (the routed list is sorted first, padded to a
// multiple of 8 with zero-weight slots), so the routed score with h = H_I is the dense score bit
// for bit.  -0 is normalised to +0.
//
// fp32 path (q and k in fp32): one warp per key row on CUDA cores, exact fp32 products.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace misa {

namespace {

constexpr int kScoreThreads = 256;   // 8 warps
constexpr int kRowsPerChunk = 1024;  // positions per CTA

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_row_chunk(const __nv_bfloat16* row, int chunk) {
  return __ldg(reinterpret_cast<const uint4*>(row) + chunk);
}

// Shared staging of one query's head list: ascending head ids (padded), weights and, for the
// bf16 path, the B fragments in fragment order.
template <int NG>
struct HeadStage {
  uint2 frag[NG][8][32];
  float wsel[NG * 8];
  int hl[NG * 8];
  int m;
};

// Thread 0 sorts the heads; pads reuse head hl[0] with weight 0.  Head ids outside [0, H_I) are
// clamped into range (the router never produces them).
__device__ __forceinline__ void stage_head_list(const int32_t* heads, int h, int H_I, int t, int slots,
                                                int* hl, int* m_out) {
  if (threadIdx.x == 0) {
    const int m = heads ? h : H_I;
    for (int a = 0; a < m; ++a) {
      int v = heads ? heads[(int64_t)t * h + a] : a;
      v = v < 0 ? 0 : (v >= H_I ? H_I - 1 : v);  // out-of-range ids are clamped, never dereferenced
      int b = a;
      while (b > 0 && hl[b - 1] > v) {
        hl[b] = hl[b - 1];
        --b;
      }
      hl[b] = v;
    }
    for (int a = m; a < slots; ++a) hl[a] = hl[0];
    *m_out = m;
  }
}

template <int NG, bool GATHER>
__global__ void __launch_bounds__(kScoreThreads, 2)
    score_bf16_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                      const __nv_bfloat16* __restrict__ k, int64_t k_seq_stride, const int32_t* __restrict__ n,
                      const int32_t* __restrict__ heads, int h, int H_I, int L,
                      const int32_t* __restrict__ rows, int P, float* __restrict__ out, int64_t ld) {
  __shared__ HeadStage<NG> st;
  const int t = blockIdx.y;
  const int nt = clamp_len(n[t], L);
  const int npos = GATHER ? P : nt;
  const int p0 = blockIdx.x * kRowsPerChunk;
  if (p0 >= npos) return;
  const int p1 = min(p0 + kRowsPerChunk, npos);

  stage_head_list(heads, h, H_I, t, NG * 8, st.hl, &st.m);
  __syncthreads();
  if (threadIdx.x < NG * 8)
    st.wsel[threadIdx.x] = threadIdx.x < st.m ? w[(int64_t)t * H_I + st.hl[threadIdx.x]] : 0.f;
  for (int e = threadIdx.x; e < NG * 8 * 32; e += kScoreThreads) {
    const int ng = e >> 8, kk = (e >> 5) & 7, ln = e & 31;
    const int g = ln >> 2, c = ln & 3;
    const int base = 32 * (kk >> 1) + 8 * c + 4 * (kk & 1);
    const __nv_bfloat16* src = q + ((int64_t)t * H_I + st.hl[ng * 8 + g]) * kD + base;
    st.frag[ng][kk][ln] = *reinterpret_cast<const uint2*>(src);
  }
  __syncthreads();

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
    const __nv_bfloat16* ra = kt + (int64_t)(va ? sa : 0) * kD;
    const __nv_bfloat16* rb = kt + (int64_t)(vb ? sb : 0) * kD;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      RA[i] = va ? ldg_row_chunk(ra, 4 * i + c) : make_uint4(0, 0, 0, 0);
      RB[i] = vb ? ldg_row_chunk(rb, 4 * i + c) : make_uint4(0, 0, 0, 0);
    }
  };

  int r0 = p0 + warp * 16;
  uint4 RA[4], RB[4];
  bool va, vb;
  if (r0 < p1) load(r0, RA, RB, va, vb);
  for (; r0 < p1; r0 += 8 * 16) {
    uint4 NA[4], NB[4];
    bool na = false, nb = false;
    const int rn = r0 + 8 * 16;
    if (rn < p1) load(rn, NA, NB, na, nb);

    float slo = 0.f, shi = 0.f;
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint4 xa = RA[kk >> 1], xb = RB[kk >> 1];
        const uint2 bf = st.frag[ng][kk][lane];
        if (kk & 1)
          mma_bf16_16816(acc, xa.z, xb.z, xa.w, xb.w, bf.x, bf.y);
        else
          mma_bf16_16816(acc, xa.x, xb.x, xa.y, xb.y, bf.x, bf.y);
      }
      slo = fmaf(wa[ng], relu(acc[0]), slo);
      slo = fmaf(wb[ng], relu(acc[1]), slo);
      shi = fmaf(wa[ng], relu(acc[2]), shi);
      shi = fmaf(wb[ng], relu(acc[3]), shi);
    }
    slo += __shfl_xor_sync(0xffffffffu, slo, 1);
    shi += __shfl_xor_sync(0xffffffffu, shi, 1);
    slo += __shfl_xor_sync(0xffffffffu, slo, 2);
    shi += __shfl_xor_sync(0xffffffffu, shi, 2);
    slo = __fadd_rn(slo, 0.0f);
    shi = __fadd_rn(shi, 0.0f);
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
  if (threadIdx.x < m) wsel[threadIdx.x] = w[(int64_t)t * H_I + hl[threadIdx.x]];
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

template <int NG>
void launch_bf16(bool gather, dim3 grid, cudaStream_t s, const void* q, const float* w, const void* k,
                 int64_t k_seq_stride, const int32_t* n, const int32_t* heads, int h, int H_I, int L,
                 const int32_t* rows, int P, float* out, int64_t ld) {
  auto qb = static_cast<const __nv_bfloat16*>(q);
  auto kb = static_cast<const __nv_bfloat16*>(k);
  if (gather)
    score_bf16_kernel<NG, true><<<grid, kScoreThreads, 0, s>>>(qb, w, kb, k_seq_stride, n, heads, h, H_I, L, rows,
                                                               P, out, ld);
  else
    score_bf16_kernel<NG, false><<<grid, kScoreThreads, 0, s>>>(qb, w, kb, k_seq_stride, n, heads, h, H_I, L,
                                                                rows, P, out, ld);
}

}  // namespace

void launch_scores(DType dt, const void* q, const float* w, const void* k, int64_t k_seq_stride,
                   const int32_t* n, const int32_t* heads, int T, int L, int H_I, int h, const int32_t* rows,
                   int P, float* out, int64_t ld, cudaStream_t s) {
  if (T <= 0) return;
  const int npos = rows ? P : L;
  if (npos <= 0) return;
  dim3 grid((npos + kRowsPerChunk - 1) / kRowsPerChunk, T);
  const bool gather = rows != nullptr;
  if (dt == DType::F32) {
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
  const int m = heads ? h : H_I;
  const int ng = (m + 7) / 8;
  switch (ng) {
#define MISA_NG_CASE(NGV) \
  case NGV:               \
    launch_bf16<NGV>(gather, grid, s, q, w, k, k_seq_stride, n, heads, h, H_I, L, rows, P, out, ld); \
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

}  // namespace misa
