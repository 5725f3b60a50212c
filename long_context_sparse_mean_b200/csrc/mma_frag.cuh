// Warp-level bf16 tensor-core fragments for scoring key rows against a list of head vectors.
//
// Contraction per 16 key rows: K[16, 128] x Q[128, 8 heads] on mma.m16n8k16 (bf16 in, fp32
// accumulate).  The dot product does not depend on the order of the 128 dimensions as long as
// both operands use the same order, so lane (g, c) of a warp loads the 16-byte chunks c, c+4,
// c+8, c+12 of rows g and g+8 straight from global memory (each load instruction of the warp
// covers 8 rows x 64 contiguous bytes) and uses them as A fragments; the query fragments are
// staged in shared memory in the matching order:  at k-step kk, fragment slot e of lane (g, c)
// holds dimension 32*(kk/2) + 8c + 4*(kk%2) + e of head g.
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "common.cuh"

namespace misa {

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// First element of the 4 query dimensions held by lane (g, c) at k-step kk.
__device__ __forceinline__ int frag_dim(int kk, int c) { return 32 * (kk >> 1) + 8 * c + 4 * (kk & 1); }

// Stage the B fragments of NG groups of 8 heads: frag[ng][kk][lane] = 4 bf16 of head hl[8 ng + g].
// NT = threads of the block; every thread issues all its loads before its first store.
template <int NG, int NT>
__device__ __forceinline__ void stage_q_frags(uint2 (*frag)[8][32], const __nv_bfloat16* qt, const int* hl) {
  constexpr int kElems = NG * 8 * 32;
  constexpr int kPer = (kElems + NT - 1) / NT;
  uint2 v[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = (int)threadIdx.x + i * NT;
    if (e < kElems) {
      const int ng = e >> 8, kk = (e >> 5) & 7, ln = e & 31;
      const int g = ln >> 2, c = ln & 3;
      v[i] = *reinterpret_cast<const uint2*>(qt + (int64_t)hl[ng * 8 + g] * kD + frag_dim(kk, c));
    }
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = (int)threadIdx.x + i * NT;
    if (e < kElems) frag[e >> 8][(e >> 5) & 7][e & 31] = v[i];
  }
}

// The B fragments of all H_I heads in head order, ngf = ceil(H_I / 8) groups (slots past H_I repeat
// head 0; their weight is 0), by the NT threads of the block.  Same layout as stage_q_frags.
template <int NT>
__device__ __forceinline__ void stage_all_head_frags(uint2 (*frag)[8][32], const __nv_bfloat16* qt, int H_I,
                                                     int ngf) {
  for (int e = (int)threadIdx.x; e < ngf * 256; e += NT) {
    const int ng = e >> 8, kk = (e >> 5) & 7, ln = e & 31;
    const int hd = ng * 8 + (ln >> 2);
    frag[ng][kk][ln] = *reinterpret_cast<const uint2*>(qt + (int64_t)(hd < H_I ? hd : 0) * kD + frag_dim(kk, ln & 3));
  }
}

// Load the A data of one 16-row group: rows ra (lane row g) and rb (row g+8); null = zeros.
__device__ __forceinline__ void load_rows(const __nv_bfloat16* ra, const __nv_bfloat16* rb, int c, uint4 (&A)[4],
                                          uint4 (&Bq)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    A[i] = ra ? __ldg(reinterpret_cast<const uint4*>(ra) + 4 * i + c) : make_uint4(0, 0, 0, 0);
    Bq[i] = rb ? __ldg(reinterpret_cast<const uint4*>(rb) + 4 * i + c) : make_uint4(0, 0, 0, 0);
  }
}

// Scores of the 16 rows for NG head groups: s_lo (row g) and s_hi (row g+8) in every lane of
// the quad, sum_j w_j relu(q_j . k) with heads in list order; -0 is returned as +0.
template <int NG>
__device__ __forceinline__ void score_rows(const uint4 (&A)[4], const uint4 (&Bq)[4], const uint2 (*frag)[8][32],
                                           const float* wa, const float* wb, int lane, float& s_lo, float& s_hi) {
  float slo = 0.f, shi = 0.f;
#pragma unroll
  for (int ng = 0; ng < NG; ++ng) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint4 xa = A[kk >> 1], xb = Bq[kk >> 1];
      const uint2 bf = frag[ng][kk][lane];
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
  s_lo = __fadd_rn(slo, 0.0f);
  s_hi = __fadd_rn(shi, 0.0f);
}

// score_rows for a run-time number of head groups ng_count, weights from shared memory (wsel[8 ng +
// e] for slot e of group ng): the same operations in the same order, so the result is score_rows<NG>
// bit for bit.
__device__ __forceinline__ void score_rows_rt(const uint4 (&A)[4], const uint4 (&Bq)[4], const uint2 (*frag)[8][32],
                                              const float* wsel, int ng_count, int lane, float& s_lo, float& s_hi) {
  const int c = lane & 3;
  float slo = 0.f, shi = 0.f;
  for (int ng = 0; ng < ng_count; ++ng) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint4 xa = A[kk >> 1], xb = Bq[kk >> 1];
      const uint2 bf = frag[ng][kk][lane];
      if (kk & 1)
        mma_bf16_16816(acc, xa.z, xb.z, xa.w, xb.w, bf.x, bf.y);
      else
        mma_bf16_16816(acc, xa.x, xb.x, xa.y, xb.y, bf.x, bf.y);
    }
    const float wa = wsel[ng * 8 + 2 * c], wb = wsel[ng * 8 + 2 * c + 1];
    slo = fmaf(wa, relu(acc[0]), slo);
    slo = fmaf(wb, relu(acc[1]), slo);
    shi = fmaf(wa, relu(acc[2]), shi);
    shi = fmaf(wb, relu(acc[3]), shi);
  }
  slo += __shfl_xor_sync(0xffffffffu, slo, 1);
  shi += __shfl_xor_sync(0xffffffffu, shi, 1);
  slo += __shfl_xor_sync(0xffffffffu, slo, 2);
  shi += __shfl_xor_sync(0xffffffffu, shi, 2);
  s_lo = __fadd_rn(slo, 0.0f);
  s_hi = __fadd_rn(shi, 0.0f);
}

// score_rows_rt with the group count known at compile time for the common head pools (H_I = 32, 64,
// 128): the groups' accumulator chains are unrolled and independent, so their MMAs overlap.
__device__ __forceinline__ void score_rows_any(const uint4 (&A)[4], const uint4 (&Bq)[4], const uint2 (*frag)[8][32],
                                               const float* wsel, int ng_count, int lane, float& s_lo, float& s_hi) {
  const int c = lane & 3;
  auto fixed = [&](auto ngc) {
    constexpr int NGC = decltype(ngc)::value;
    float wa[NGC], wb[NGC];
#pragma unroll
    for (int ng = 0; ng < NGC; ++ng) {
      wa[ng] = wsel[ng * 8 + 2 * c];
      wb[ng] = wsel[ng * 8 + 2 * c + 1];
    }
    score_rows<NGC>(A, Bq, frag, wa, wb, lane, s_lo, s_hi);
  };
  if (ng_count == 8)
    fixed(std::integral_constant<int, 8>{});
  else if (ng_count == 4)
    fixed(std::integral_constant<int, 4>{});
  else if (ng_count == 16)
    fixed(std::integral_constant<int, 16>{});
  else
    score_rows_rt(A, Bq, frag, wsel, ng_count, lane, s_lo, s_hi);
}

}  // namespace misa
