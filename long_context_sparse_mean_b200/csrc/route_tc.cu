// Router affinities on the 5th-generation tensor cores for queries that share one key cache and
// its pooled keys (chunked prefill).
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", "Methodology:
// MISA", "Lightweight Block-Pooled Router": every head j of query t gets one affinity aggregated
// over the mean-pooled keys of its prefix, r_{t,j} = w_{t,j} sum_{b < M_t} max(0, q_{t,j} . kbar_b).
//
// This kernel computes, per tile of 256 pooled blocks, Sp[t][tile][j] = the sum over the tile's
// blocks b < kbar_blocks(n_t, B) (every block of the prefix but the last) of
// max(0, q_{t,j} . kbar_b); route_finish (pool_route.cu) adds the last block, averaged from the
// keys, applies w and picks the top-h.  As a contraction: A = the H_I query-head rows
// of 128 / H_I consecutive queries [128 rows x 128 dims], contiguous in q and loaded by TMA;
// B = 256 pooled keys in three bf16 parts (kbar = hi + mid + lo to fp32 accuracy, so the dot
// products keep the accuracy of fp32 pooled keys) [256 x 128] each; D = A (hi + mid + lo)^T
// accumulates in tensor memory with TMEM lane = query-head row and column = pooled block, so the
// epilogue thread that owns a row sums max(0, D) over its query's full blocks in registers.
//
// Per CTA (one per SM, persistent): a contiguous range of the flattened (query block, block tile)
// work.  Warps 0-3: epilogue (one TMEM lane quarter each); warp 4: TMA producer (A once per
// query block, double-buffered; B through a 4-stage ring of 256 blocks x 64 dims of one part);
// warp 5: MMA issuer and TMEM owner (two accumulators of 256 columns).  Waits are bounded in time
// as in the scoring kernel (score_tc.cu).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace misa {

// Nonzero after the router kernel gave up on a wait (read and cleared by misa_device_check).
__device__ int g_route_tc_status = 0;

namespace {

constexpr int kRows = 128;                          // UMMA M: query-head rows
constexpr int kBlocks = 256;                        // UMMA N: pooled blocks per tile
constexpr int kStages = 4;                          // B ring
constexpr int kStageBytes = kBlocks * 64 * 2;       // 32 KB: 64 dims of one part
constexpr int kAHalf = kRows * 64 * 2;              // 16 KB
constexpr int kABytes = 2 * kAHalf;                 // 32 KB
constexpr int kMaxBlocks = 4096;                    // query blocks per launch
constexpr int kEpiWarps = 4;
constexpr int kTmaWarp = 4, kMmaWarp = 5;
constexpr int kThreads = 6 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 1000000000ull;

constexpr int kOffA = 0;                                             // [2][32 KB]
constexpr int kOffB = kOffA + 2 * kABytes;                           // [kStages][32 KB]
constexpr int kOffPre = kOffB + kStages * kStageBytes;               // u32 [kMaxBlocks + 1]
constexpr int kOffBar = kOffPre + ((kMaxBlocks + 1) * 4 + 15) / 16 * 16;
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 4 * 36 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory of the tensor-core router exceeds 227 KB");

__device__ __forceinline__ void give_up(volatile int* abort) {
  *abort = 1;
  atomicExch(&g_route_tc_status, 1);
}

// max(0, x) summed over the 32 columns of one chunk whose block index is below lim.
template <int CC>
__device__ __forceinline__ float relu_sum_chunk(const uint32_t (&v)[32], int lim) {
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int u = 0; u < 32; u += 2) {
    const int c = CC * 32 + u;
    a += c < lim ? fmaxf(__uint_as_float(v[u]), 0.f) : 0.f;
    b += c + 1 < lim ? fmaxf(__uint_as_float(v[u + 1]), 0.f) : 0.f;
  }
  return a + b;
}

__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kbmap,
                    const int32_t* __restrict__ n, int L, int B, int H_I, int M, int T, float* __restrict__ Sp,
                    int nch) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* pre = reinterpret_cast<uint32_t*>(sm + kOffPre);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + kOffMisc);
  volatile uint32_t* tmem_slot = misc;
  volatile int* abort = reinterpret_cast<volatile int*>(misc + 1);
  uint32_t* warp_tot = misc + 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int QR = kRows / H_I;  // queries per block
  const int NB = (T + QR - 1) / QR;

  tc::block_tile_prefix(NB, QR, T, kBlocks, [&](int t) { return kbar_blocks(clamp_len(__ldg(n + t), L), B); }, pre,
                        warp_tot);
  const uint64_t W = pre[NB];
  const uint32_t a = (uint32_t)(W * blockIdx.x / gridDim.x);
  const uint32_t e = (uint32_t)(W * (blockIdx.x + 1) / gridDim.x);
  if (a >= e) return;

  const uint32_t bar0 = tc::smem_u32(sm + kOffBar);
  const uint32_t bfull = bar0, bempty = bfull + 8 * kStages, afull = bempty + 8 * kStages, aempty = afull + 16,
                 accfull = aempty + 16, accempty = accfull + 16, drain = accempty + 16;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(bfull + 8 * i, 1);
      tc::mbar_init(bempty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(afull + 8 * i, 1);
      tc::mbar_init(aempty + 8 * i, 1);
      tc::mbar_init(accfull + 8 * i, 1);
      tc::mbar_init(accempty + 8 * i, kEpiWarps);
    }
    tc::mbar_init(drain, 1);
    *abort = 0;
    tc::mbar_init_fence();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(tc::smem_u32((const void*)tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t abase = tc::smem_u32(sm + kOffA);
  const uint32_t bbase = tc::smem_u32(sm + kOffB);

  if (warp < kEpiWarps) {
    // ---------------- epilogue: one query-head row per thread ----------------
    const int r = warp * 32 + lane;
    const int qi = r / H_I, j = r % H_I;
    uint32_t i = 0, lo, hi;
    int blk;
    tc::TileSegments it(pre, NB, a, e);
    bool ok = true;
    while (ok && it.next(blk, lo, hi)) {
      const int t = blk * QR + qi;
      const bool real = qi < QR && t < T;
      const int nf = real ? kbar_blocks(clamp_len(__ldg(n + t), L), B) : 0;
      for (uint32_t tile = lo; tile < hi; ++tile, ++i) {
        const int ab = i & 1;
        if (!tc::mbar_wait(accfull + 8 * ab, (i >> 1) & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(ab * kBlocks);
        const int lim = nf - (int)tile * kBlocks;
        uint32_t va[32], vb[32];
        float sum = 0.f;
        tc::tmem_ld32(ta, va);
        tc::tmem_ld_wait(va);
        tc::tmem_ld32(ta + 32, vb);
        sum += relu_sum_chunk<0>(va, lim);
        tc::tmem_ld_wait(vb);
        tc::tmem_ld32(ta + 64, va);
        sum += relu_sum_chunk<1>(vb, lim);
        tc::tmem_ld_wait(va);
        tc::tmem_ld32(ta + 96, vb);
        sum += relu_sum_chunk<2>(va, lim);
        tc::tmem_ld_wait(vb);
        tc::tmem_ld32(ta + 128, va);
        sum += relu_sum_chunk<3>(vb, lim);
        tc::tmem_ld_wait(va);
        tc::tmem_ld32(ta + 160, vb);
        sum += relu_sum_chunk<4>(va, lim);
        tc::tmem_ld_wait(vb);
        tc::tmem_ld32(ta + 192, va);
        sum += relu_sum_chunk<5>(vb, lim);
        tc::tmem_ld_wait(va);
        tc::tmem_ld32(ta + 224, vb);
        sum += relu_sum_chunk<6>(va, lim);
        tc::tmem_ld_wait(vb);
        sum += relu_sum_chunk<7>(vb, lim);
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_relaxed(accempty + 8 * ab);
        if (real && lim > 0) Sp[((int64_t)t * nch + tile) * H_I + j] = sum;
      }
    }
    if (!ok) give_up(abort);
  } else if (warp == kTmaWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t f = 0, p = 0, lo, hi;
      int blk;
      tc::TileSegments it(pre, NB, a, e);
      bool ok = true;
      while (ok && it.next(blk, lo, hi)) {
        const int pb = p & 1;
        if (p >= 2 && !tc::mbar_wait(aempty + 8 * pb, ((p >> 1) - 1) & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc::mbar_arrive_expect_tx(afull + 8 * pb, kABytes);
        tc::tma_load_2d(abase + pb * kABytes, &qmap, 0, blk * kRows, afull + 8 * pb);
        tc::tma_load_2d(abase + pb * kABytes + kAHalf, &qmap, 64, blk * kRows, afull + 8 * pb);
        ++p;
        for (uint32_t tile = lo; ok && tile < hi; ++tile) {
          for (int sub = 0; sub < 6; ++sub, ++f) {  // (part, 64-dim half)
            const int st = f % kStages;
            if (f >= kStages && !tc::mbar_wait(bempty + 8 * st, ((f / kStages) - 1) & 1, abort, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc::mbar_arrive_expect_tx(bfull + 8 * st, kStageBytes);
            tc::tma_load_2d(bbase + st * kStageBytes, &kbmap, (sub & 1) * 64, (sub >> 1) * M + (int)tile * kBlocks,
                            bfull + 8 * st);
          }
        }
      }
      if (!ok) give_up(abort);
      for (uint32_t g = f > kStages ? f - kStages : 0; g < f; ++g)
        tc::mbar_wait(bfull + 8 * (g % kStages), (g / kStages) & 1, nullptr, kWaitLimitNs);
      for (uint32_t g = p > 2 ? p - 2 : 0; g < p; ++g) tc::mbar_wait(afull + 8 * (g & 1), (g >> 1) & 1, nullptr, kWaitLimitNs);
    }
  } else {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kRows, kBlocks);
      uint32_t f = 0, i = 0, p = 0, lo, hi;
      int blk;
      tc::TileSegments it(pre, NB, a, e);
      bool ok = true;
      while (ok && it.next(blk, lo, hi)) {
        const int pb = p & 1;
        if (!tc::mbar_wait(afull + 8 * pb, (p >> 1) & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t ab_ = abase + pb * kABytes;
        for (uint32_t tile = lo; ok && tile < hi; ++tile, ++i) {
          const int ab = i & 1;
          if (i >= 2 && !tc::mbar_wait(accempty + 8 * ab, ((i >> 1) - 1) & 1, abort, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(ab * kBlocks);
          for (int sub = 0; sub < 6; ++sub, ++f) {
            const int st = f % kStages;
            if (!tc::mbar_wait(bfull + 8 * st, (f / kStages) & 1, abort, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc::tc_fence_after();
            const uint64_t ad = tc::sw128_kmajor_desc(ab_ + (sub & 1) * kAHalf);
            const uint64_t bd = tc::sw128_kmajor_desc(bbase + st * kStageBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (sub | kk) != 0);
            tc::mma_commit(bempty + 8 * st);
          }
          if (ok) tc::mma_commit(accfull + 8 * ab);
        }
        if (ok) tc::mma_commit(aempty + 8 * pb);
        ++p;
      }
      if (!ok) give_up(abort);
      tc::mma_commit(drain);
      tc::mbar_wait(drain, 0, nullptr, kWaitLimitNs);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int read_and_clear_route_tc_status() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_route_tc_status, sizeof(int)) != cudaSuccess) return -1;
  if (v) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_route_tc_status, &zero, sizeof(int));
  }
  return v;
}

bool launch_route_tc(const void* q, const float* w, const void* k, const float* kbar, const int32_t* n, int T,
                     int L, int H_I, int B, int h, int32_t* heads, float* r_opt, __nv_bfloat16* kbar_parts,
                     float* Sp, int nch, cudaStream_t s) {
  if (T <= 0) return true;
  if (kRows % H_I != 0 || !kbar_parts) return false;
  const int M = (L + B - 1) / B;
  CUtensorMap kbmap;
  if (!tmap_rows128_bf16(&kbmap, kbar_parts, 3 * (uint64_t)M, kBlocks)) return false;
  const int QR = kRows / H_I;
  const int per_launch = kMaxBlocks * QR;
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  // every query map first, so that nothing is launched unless all of them encode
  const int nl = (T + per_launch - 1) / per_launch;
  if (nl > 16) return false;
  CUtensorMap qmaps[16];
  for (int l = 0; l < nl; ++l) {
    const int t0 = l * per_launch, Tc = T - t0 < per_launch ? T - t0 : per_launch;
    if (!tmap_rows128_bf16(&qmaps[l], qb + (int64_t)t0 * H_I * kD, (uint64_t)Tc * H_I, kRows)) return false;
  }
  launch_kbar_split(kbar, M, kbar_parts, s);
  cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  const int grid = sm_count();
  for (int l = 0; l < nl; ++l) {
    const int t0 = l * per_launch, Tc = T - t0 < per_launch ? T - t0 : per_launch;
    route_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(qmaps[l], kbmap, n + t0, L, B, H_I, M, Tc,
                                                       Sp + (int64_t)t0 * nch * H_I, nch);
  }
  launch_route_finish(qb, w, static_cast<const __nv_bfloat16*>(k), n, T, L, H_I, B, h, Sp, nch, kBlocks, heads,
                      r_opt, s);
  return true;
}

}  // namespace misa
