// Device helpers shared by the MISA indexer kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace misa {

// Programmatic dependent launch: a kernel launched with launch_pdl may start while the previous
// kernel on its stream is finishing; pdl_wait() (at the top of such a kernel, before it reads
// anything the previous kernel writes) waits for that kernel to complete and its memory to be
// visible, and pdl_trigger() lets the next kernel launch its CTAs early.  Both are no-ops in a
// kernel launched the ordinary way.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <class... KArgs, class... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

constexpr int kD = 128;          // index-key width handled by every kernel
constexpr int kMaxHeads = 128;   // largest indexer-head pool H_I
constexpr int kRouteTile = 64;   // router blocks per CTA tile

// Element type of q and k.
enum class DType : int { BF16 = 0, F32 = 1 };

// Bounds-checked build (compiled with MISA_CHECKED): every id a kernel skips because it lies
// outside its range is counted by kind in its translation unit's counters, which the C ABI reads
// (misa_device_check, misa_bad_index_counts).  Such ids are never dereferenced in either build.
enum BadIdKind : int {
  kBadHead = 0,       // a routed head id outside [0, H_I)
  kBadCandidate = 1,  // a candidate token id outside [0, n_t) other than the empty marker -1
  kBadPage = 2,       // a page-table entry inside a prefix outside [0, num_pages)
  kBadIdKinds = 3
};
#ifdef MISA_CHECKED
static __device__ unsigned int g_bad_ids[kBadIdKinds];
__device__ __forceinline__ void count_bad_id(int kind, bool bad) {
  if (bad) atomicAdd(&g_bad_ids[kind], 1u);
}
// Host side: adds this translation unit's counters to out[kBadIdKinds] and clears them; false if
// the copy failed.
#define MISA_BAD_ID_READER(name)                                                          \
  bool name(unsigned int* out) {                                                          \
    unsigned int v[kBadIdKinds] = {0, 0, 0};                                              \
    if (cudaMemcpyFromSymbol(v, g_bad_ids, sizeof(v)) != cudaSuccess) return false;       \
    const unsigned int z[kBadIdKinds] = {0, 0, 0};                                        \
    if (cudaMemcpyToSymbol(g_bad_ids, z, sizeof(z)) != cudaSuccess) return false;         \
    for (int i = 0; i < kBadIdKinds; ++i) out[i] += v[i];                                 \
    return true;                                                                          \
  }
#else
__device__ __forceinline__ void count_bad_id(int, bool) {}
#define MISA_BAD_ID_READER(name) \
  bool name(unsigned int*) { return true; }
#endif

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

// Pooled blocks of a prefix of nt keys that are read from the pooled-key cache: every block but
// the last.  The last block, keys [kbar_blocks(nt, B) * B, nt) (full or partial), is averaged from
// the keys by the kernel that needs it, so a decode loop pools a block once its prefix has moved
// past it, and the newest key is always seen.
__device__ __forceinline__ int kbar_blocks(int nt, int B) { return nt > 0 ? (nt - 1) / B : 0; }

// Mean of key rows [s0, s1) of one cache ([*, 128], bf16 or fp32), all 256 threads of the block:
// every thread owns one 16-byte column chunk of a row group and issues the loads of up to 128 rows
// at once.  part: shared scratch of 16 x 128 floats.  Returns the mean of column threadIdx.x in
// threads 0..127 (IEEE division by the count); every thread must call it (it synchronises).
template <DType DT>
__device__ __forceinline__ float block_mean_rows(const void* kseq, int s0, int s1, float* part) {
  constexpr int EPC = DT == DType::BF16 ? 8 : 4;  // elements per 16-byte chunk
  constexpr int CPR = kD / EPC;                   // chunks per row
  constexpr int RG = 256 / CPR;                   // row groups
  constexpr int IT = 128 / RG;                    // rows a thread loads per batch
  const int cc = threadIdx.x % CPR, rg = threadIdx.x / CPR;
  const uint4* base = reinterpret_cast<const uint4*>(kseq);
  float acc[EPC];
#pragma unroll
  for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
  for (int s = s0 + rg; s < s1; s += RG * IT) {
    uint4 x[IT];
#pragma unroll
    for (int i = 0; i < IT; ++i) {
      const int r = s + i * RG;
      x[i] = r < s1 ? __ldg(base + (int64_t)r * CPR + cc) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < IT; ++i) {
      const uint32_t u[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
      if (DT == DType::BF16) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += __uint_as_float(u[e] << 16);
          acc[2 * e + 1] += __uint_as_float(u[e] & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] += __uint_as_float(u[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPC; ++e) part[rg * kD + cc * EPC + e] = acc[e];
  __syncthreads();
  float mean = 0.f;
  if (threadIdx.x < kD) {
    float sum = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) sum += part[g * kD + threadIdx.x];
    mean = sum / (float)(s1 - s0);
  }
  __syncthreads();  // part may be reused right after
  return mean;
}

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
