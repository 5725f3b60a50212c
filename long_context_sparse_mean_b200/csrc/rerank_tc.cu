// MISA-dagger re-rank scores on the 5th-generation tensor cores: the dense score of gathered
// candidate tokens.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", "Hierarchical
// Variant (MISA-dagger)": the k' candidates of the routed pass are re-scored with all H_I heads,
// F_{t,s} = sum_{j < H_I} w_{t,j} max(0, q_{t,j} . k_s), and the top-k of F is kept.
//
// As one contraction per tile of 128 candidates of query t: A = the 128 gathered key rows [128 x
// 128 dims] (bf16), B = the query's H_I head rows [H_I x 128], D = A B^T [128 candidates x H_I
// heads] in tensor memory (fp32).  TMEM lane = candidate, so the epilogue thread that owns a
// candidate sums w_j max(0, D_j) over its H_I columns in registers.  At 64 heads a candidate costs
// 2 x 64 x 128 FLOPs for 256 bytes of key: the legacy warp-level MMA was the limit of the gather
// kernel, here the tensor cores take the contraction in 8 instructions a tile and the gather of
// the rows from HBM sets the pace.
//
// Per CTA (one per SM, persistent): a contiguous range of the flattened (query, tile) work.  Warp
// roles:
//   warps 0-3 epilogue (one TMEM lane quarter each): tcgen05.ld of the accumulator, w * ReLU sums,
//             one coalesced 128-byte store of 32 scores per warp
//   warps 4-7 gather: each thread copies 16-byte chunks of the candidate rows (16 threads a row,
//             so a warp instruction reads two whole 256-byte rows) with cp.async into a 4-stage
//             ring in the 128-byte swizzled K-major layout; empty slots (ids outside [0, n_t))
//             are zero-filled; also the query's head rows and weights, double-buffered
//   warp 8    MMA issuer (one thread) and TMEM owner: two accumulators
// Every wait is bounded in time; a wait that runs out sets a device status word and all roles
// leave their loops, wait for their own copies and MMAs, and free tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace misa {

// Nonzero after the re-rank kernel gave up on a wait (read and cleared by misa_device_check).
__device__ int g_rerank_tc_status = 0;

namespace {

constexpr int kRows = 128;                       // candidates per tile (UMMA M, TMEM lanes)
constexpr int kStages = 4;                       // A ring
constexpr int kAHalf = kRows * 128;              // 16 KB: 128 rows x 64 dims
constexpr int kATile = 2 * kAHalf;               // 32 KB
constexpr int kMaxH = 128;
constexpr int kBMax = 2 * kMaxH * 128;           // 32 KB: 128 head rows x 128 dims
constexpr int kEpiWarps = 4, kProdWarps = 4;
constexpr int kProdWarp0 = kEpiWarps, kMmaWarp = kEpiWarps + kProdWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kProdThreads = kProdWarps * 32;
constexpr uint32_t kTmemCols = 256;              // two accumulators at columns 0 and 128
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kStages * kATile;
constexpr int kOffW = kOffB + 2 * kBMax;                 // [2][kMaxH] f32
constexpr int kOffBar = kOffW + 2 * kMaxH * 4;
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;          // tmem base, abort
constexpr int kSmemBytes = kOffMisc + 16 + 1024;          // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory of the re-rank kernel exceeds 227 KB");

struct Bars {
  uint32_t afull, aempty, bfull, bempty, accfull, accempty, drain;
  __device__ uint32_t af(int i) const { return afull + 8 * i; }
  __device__ uint32_t ae(int i) const { return aempty + 8 * i; }
  __device__ uint32_t bf(int i) const { return bfull + 8 * i; }
  __device__ uint32_t be(int i) const { return bempty + 8 * i; }
  __device__ uint32_t cf(int i) const { return accfull + 8 * i; }
  __device__ uint32_t ce(int i) const { return accempty + 8 * i; }
};

__device__ __forceinline__ void give_up(volatile int* abort) {
  *abort = 1;
  atomicExch(&g_rerank_tc_status, 1);
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Waits until at most N of this thread's committed cp.async groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Shared address of 16-byte chunk c (0..15) of row `row` in a K-major operand of `rows` rows stored
// as two 64-column halves in the 128-byte swizzled layout.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t base, int rows, int row, int c) {
  return base + (uint32_t)((c >> 3) * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128) +
         ((((uint32_t)c & 7u) ^ ((uint32_t)row & 7u)) << 4);
}

// out[t, p] = F_{t, cand[t, p]} for p < P (0 for an empty slot).
__global__ void __launch_bounds__(kThreads, 1)
    rerank_tc_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                     const __nv_bfloat16* __restrict__ k, int64_t k_seq_stride, const int32_t* __restrict__ n,
                     int L, int T, int H, const int32_t* __restrict__ cand, int P, float* __restrict__ out,
                     int64_t ld) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* wsm = reinterpret_cast<float*>(sm + kOffW);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + kOffMisc);
  volatile uint32_t* tmem_slot = misc;
  volatile int* abort = reinterpret_cast<volatile int*>(misc + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();

  const int ntile = (P + kRows - 1) / kRows;
  const int64_t W = (int64_t)T * ntile;
  const int64_t a = W * blockIdx.x / gridDim.x, e = W * (blockIdx.x + 1) / gridDim.x;
  if (a >= e) return;  // uniform: nothing allocated yet
  // the work item after `x` belongs to another query (or there is none): the query's last tile here
  auto last_of_query = [&](int64_t x) { return x + 1 >= e || (x + 1) / ntile != x / ntile; };

  const uint32_t bar0 = tc::smem_u32(sm + kOffBar);
  Bars bars;
  bars.afull = bar0;
  bars.aempty = bars.afull + 8 * kStages;
  bars.bfull = bars.aempty + 8 * kStages;
  bars.bempty = bars.bfull + 16;
  bars.accfull = bars.bempty + 16;
  bars.accempty = bars.accfull + 16;
  bars.drain = bars.accempty + 16;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(bars.af(i), kProdThreads);
      tc::mbar_init(bars.ae(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(bars.bf(i), kProdThreads);
      tc::mbar_init(bars.be(i), 1 + kEpiWarps);
      tc::mbar_init(bars.cf(i), 1);
      tc::mbar_init(bars.ce(i), kEpiWarps);
    }
    tc::mbar_init(bars.drain, 1);
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
    // ---------------- epilogue: candidate row = TMEM lane ----------------
    const int row = warp * 32 + lane;
    uint32_t i = 0, p = 0;
    bool ok = true;
    for (int64_t x = a; ok && x < e; ++x) {
      const int t = (int)(x / ntile), tile = (int)(x % ntile);
      const int pb = p & 1;
      if (x == a || x % ntile == 0) {  // a new query: its weights
        if (!tc::mbar_wait(bars.bf(pb), (p >> 1) & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
      }
      const int ab = i & 1;
      if (!tc::mbar_wait(bars.cf(ab), (i >> 1) & 1, abort, kWaitLimitNs)) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const float* wr = wsm + pb * kMaxH;
      const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(ab * 128);
      float f = 0.f;
      for (int c0 = 0; c0 < H; c0 += 32) {
        uint32_t v[32];
        tc::tmem_ld32(ta + (uint32_t)c0, v);
        tc::tmem_ld_wait(v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < H) f = fmaf(wr[c0 + j], relu(__uint_as_float(v[j])), f);
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_relaxed(bars.ce(ab));
      const int pos = tile * kRows + row;
      if (pos < P) out[(int64_t)t * ld + pos] = __fadd_rn(f, 0.0f);
      if (last_of_query(x)) {
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bars.be(pb));
        ++p;
      }
      ++i;
    }
    if (!ok) give_up(abort);
  } else if (warp < kMmaWarp) {
    // ---------------- gather: key rows of the candidates, head rows of the queries ----------------
    const int pt = threadIdx.x - kProdWarp0 * 32;  // 0..127
    const int c = pt & 15, r0 = pt >> 4;           // 16 threads per row, 8 rows per instruction
    uint32_t f = 0, arrived = 0, p = 0;  // stages issued, stages handed to the MMA, queries staged
    // every stage issued lands and goes to the MMA (before any wait that the MMA may have to
    // release, so that it never waits for a stage held back here)
    auto flush = [&]() {
      tc::cp_async_wait_all();
      tc::fence_proxy_async_smem();
      for (; arrived < f; ++arrived) tc::mbar_arrive(bars.af(arrived % kStages));
    };
    // the candidate ids of a tile: 16 rows a thread, loaded one tile ahead of their copies
    auto load_ids = [&](int64_t x, int (&id)[kRows / 8]) {
      const int t = (int)(x / ntile), tile = (int)(x % ntile);
      const int32_t* ct = cand + (int64_t)t * P;
#pragma unroll
      for (int i2 = 0; i2 < kRows / 8; ++i2) {
        const int pos = tile * kRows + i2 * 8 + r0;
        id[i2] = pos < P ? __ldg(ct + pos) : -1;
      }
    };
    int idn[kRows / 8];
    load_ids(a, idn);
    bool ok = true;
    for (int64_t x = a; ok && x < e; ++x) {
      const int t = (int)(x / ntile);
      if (x == a || x % ntile == 0) {  // a new query: stage its head rows and weights
        const int pb = p & 1;
        if (p >= 2) {
          // the buffer is free once the MMA is done with query p - 2: every stage issued goes to the
          // MMA first, so that it never waits for a stage held back here
          flush();
          if (!tc::mbar_wait(bars.be(pb), ((p >> 1) - 1) & 1, abort, kWaitLimitNs)) {
            ok = false;
            break;
          }
        }
        // plain loads (the stages in flight keep flying), then the async proxy sees the stores
        const uint32_t bb = bbase + pb * kBMax;
#pragma unroll 4
        for (int hr = r0; hr < H; hr += 8) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(q + ((int64_t)t * H + hr) * kD + c * 8));
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sw128_chunk(bb, H, hr, c)), "r"(v.x), "r"(v.y),
                       "r"(v.z), "r"(v.w)
                       : "memory");
        }
        for (int j = pt; j < H; j += kProdThreads) wsm[pb * kMaxH + j] = __ldg(w + (int64_t)t * H + j);
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(bars.bf(pb));
        ++p;
      }
      const int st = f % kStages;
      // the MMA has released stage f - kStages (handed over when stage f - 1 was issued)
      if (f >= kStages && !tc::mbar_wait(bars.ae(st), ((f / kStages) - 1) & 1, abort, kWaitLimitNs)) {
        ok = false;
        break;
      }
      const int nt = clamp_len(__ldg(n + t), L);
      const __nv_bfloat16* kt = k + (int64_t)t * k_seq_stride;
      int id[kRows / 8];
#pragma unroll
      for (int i2 = 0; i2 < kRows / 8; ++i2) {
        id[i2] = idn[i2];
        // bounds-checked build: an id other than -1 outside [0, n_t), once per row (chunk 0)
        count_bad_id(kBadCandidate, c == 0 && id[i2] != -1 && (id[i2] < 0 || id[i2] >= nt));
      }
      if (x + 1 < e) load_ids(x + 1, idn);
      const uint32_t sa = abase + st * kATile;
#pragma unroll
      for (int i2 = 0; i2 < kRows / 8; ++i2) {
        const int rr = i2 * 8 + r0;
        const bool valid = id[i2] >= 0 && id[i2] < nt;
        const __nv_bfloat16* src = valid ? kt + (int64_t)id[i2] * kD + c * 8 : kt;
        tc::cp_async_16(sw128_chunk(sa, kRows, rr, c), src, valid ? 16u : 0u);
      }
      cp_async_commit();
      ++f;
      // at most kStages - 1 stages stay in flight: hand the older ones to the MMA
      if (f - arrived > kStages - 1) {
        cp_async_wait_group<kStages - 1>();
        tc::fence_proxy_async_smem();
        for (; f - arrived > kStages - 1; ++arrived) tc::mbar_arrive(bars.af(arrived % kStages));
      }
    }
    flush();  // the stages still in flight land before the CTA exits
    if (!ok) give_up(abort);
  } else {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kRows, H);
      uint32_t f = 0, i = 0, p = 0;
      bool ok = true;
      for (int64_t x = a; ok && x < e; ++x) {
        const int pb = p & 1;
        if (x == a || x % ntile == 0) {
          if (!tc::mbar_wait(bars.bf(pb), (p >> 1) & 1, abort, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
        }
        const int ab = i & 1;
        if (i >= 2 && !tc::mbar_wait(bars.ce(ab), ((i >> 1) - 1) & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        const int st = f % kStages;
        if (!tc::mbar_wait(bars.af(st), (f / kStages) & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * 128);
        const uint32_t sa = abase + st * kATile, sb = bbase + pb * kBMax;
        for (int half = 0; half < 2; ++half) {
          const uint64_t ad = tc::sw128_kmajor_desc(sa + half * kAHalf);
          const uint64_t bd = tc::sw128_kmajor_desc(sb + half * H * 128);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (half | kk) != 0);
        }
        tc::mma_commit(bars.ae(st));
        tc::mma_commit(bars.cf(ab));
        if (last_of_query(x)) {
          tc::mma_commit(bars.be(pb));
          ++p;
        }
        ++f;
        ++i;
      }
      if (!ok) give_up(abort);
      // every issued MMA completes before tensor memory is freed
      tc::mma_commit(bars.drain);
      tc::mbar_wait(bars.drain, 0, nullptr, kWaitLimitNs);
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

bool launch_rerank_tc(const void* q, const float* w, const void* k, int64_t k_seq_stride, const int32_t* n, int T,
                      int L, int H_I, const int32_t* cand, int P, float* out, int64_t ld, cudaStream_t s) {
  if (T <= 0 || P <= 0) return true;
  if (H_I < 16 || H_I > kMaxH || H_I % 16 != 0) return false;
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(k) & 15) || (k_seq_stride % 8) != 0)
    return false;
  const int64_t work = (int64_t)T * ((P + kRows - 1) / kRows);
  const int grid = (int)(work < sm_count() ? work : sm_count());
  cudaFuncSetAttribute(rerank_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  launch_pdl(rerank_tc_kernel, grid, kThreads, kSmemBytes, s, static_cast<const __nv_bfloat16*>(q), w,
                                                      static_cast<const __nv_bfloat16*>(k), k_seq_stride, n, L, T,
                                                      H_I, cand, P, out, ld);
  return true;
}

int read_and_clear_rerank_tc_status() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_rerank_tc_status, sizeof(int)) != cudaSuccess) return -1;
  if (v) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_rerank_tc_status, &zero, sizeof(int));
  }
  return v;
}

MISA_BAD_ID_READER(read_and_clear_bad_ids_rerank_tc)

}  // namespace misa
