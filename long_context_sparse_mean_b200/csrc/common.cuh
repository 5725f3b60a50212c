// Device helpers shared by the MISA indexer kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace misa {

constexpr int kD = 128;          // index-key width handled by every kernel
constexpr int kMaxHeads = 128;   // largest indexer-head pool H_I
constexpr int kRouteTile = 64;   // router blocks per CTA tile

// Element type of q and k.
enum class DType : int { BF16 = 0, F32 = 1 };

// Order-preserving map of a finite fp32 value onto uint32: a > b  <=>  key(a) > key(b), and
// -0 and +0 map to the same key (they are the same score).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// Two bf16 values packed in one 32-bit word (element 0 in the low half) widened to fp32.
__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

__device__ __forceinline__ float relu(float x) { return fmaxf(x, 0.0f); }

// Clamp a device-side prefix length to [0, L].
__device__ __forceinline__ int clamp_len(int n, int L) { return n < 0 ? 0 : (n > L ? L : n); }

// Exclusive scan over the threads of a block (blockDim.x a multiple of 32, at most 1024).
// `warp_tot` is shared scratch of 32 words.  Returns the exclusive prefix; *total gets the sum.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < nwarps ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const uint32_t before = warp == 0 ? 0u : warp_tot[warp - 1];
  *total = warp_tot[nwarps - 1];
  __syncthreads();  // warp_tot may be reused right after
  return before + x - v;
}

}  // namespace misa
