// Routed-head token scoring on the 5th-generation tensor cores for queries that share one key
// cache (chunked causal prefill, and several queries decoding against the same cache).
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", "Methodology:
// MISA", "Sparse Token Scoring": with its routed head set R_t, query t scores every prefix token
// s < n_t as I_{t,s} = sum_{j in R_t} w_{t,j} max(0, q_{t,j} . k_s) (all H_I heads for the dense
// indexer of "Problem Statement").
//
// As one contraction: gather the routed query-head rows of a block of queries into a B operand
// [256 rows x 128 dims] (query-major, heads ascending, padded with zero-weight copies up to a
// power of two MP >= 8 per query), stream the shared keys as the A operand [128 keys x 128 dims],
// and accumulate D = K Q^T [128 keys x 256 query-heads] in tensor memory.  TMEM lane = key, so
// the epilogue thread that owns a key sums its query's MP head columns in registers
// (w * ReLU), with no cross-thread reduction, and stores one coalesced 128-byte row segment per
// query and warp.
//
// Per CTA (one per SM, persistent): a contiguous range of the flattened (query block, key tile)
// work, balanced to within one tile.  Warp roles:
//   warps 0-15 epilogue (TMEM lane quarter x column quarter): tcgen05.ld of the accumulator,
//              w * ReLU sums; a warp's (queries x 32 keys) block goes out as one TMA store from
//              shared memory when every key is inside every prefix, else as masked stores
//              (entries at s >= n_t are never written)
//   warp 16    query-head gather: sorts each query's head list, cp.async of the rows into the
//              swizzled operand layout (double-buffered across query blocks)
//   warp 17    TMA producer: 128-key x 64-dim tiles of K into a 4-stage ring
//   warp 18    MMA issuer (one thread) and TMEM owner: 2 accumulators of 256 fp32 columns
// Every wait is bounded in time; a wait that runs out sets a device status word and all roles
// leave their loops, wait for their own copies and MMAs, and free tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace misa {

// Nonzero after a tensor-core kernel gave up on a wait (read and cleared by misa_device_check).
__device__ int g_tc_status = 0;

namespace {

constexpr int kTileKeys = 128;                       // UMMA M: keys per accumulator (TMEM lanes)
constexpr int kTileCols = 256;                       // UMMA N: query-head rows per block
constexpr int kStages = 4;                           // K ring: 128 keys x 64 dims per stage
constexpr int kStageBytes = kTileKeys * 64 * 2;      // 16 KB
constexpr int kQHalfBytes = kTileCols * 64 * 2;      // 32 KB: 64 dims of all 256 rows
constexpr int kQBytes = 2 * kQHalfBytes;             // 64 KB per query block
constexpr int kMaxBlocks = 2048;                     // query blocks per launch
constexpr int kEpiWarps = 16;
constexpr int kLoaderWarp = 16, kTmaWarp = 17, kMmaWarp = 18;
constexpr int kThreads = 19 * 32;
constexpr uint32_t kTmemCols = 512;                  // two accumulators of 256 columns
constexpr uint64_t kWaitLimitNs = 1000000000ull;     // 1 s

// Shared-memory layout (offsets from a 1024-byte aligned base).
constexpr int kOffQ = 0;                                          // [2][64 KB]
constexpr int kOffK = kOffQ + 2 * kQBytes;                         // [kStages][16 KB]
constexpr int kStageOutFloats = 8 * 32;                           // per epilogue warp: 8 rows x 32 keys
constexpr int kOffOut = kOffK + kStages * kStageBytes;             // [kEpiWarps][8][32] f32 staged stores
constexpr int kOffPre = kOffOut + kEpiWarps * kStageOutFloats * 4; // [kMaxBlocks + 1] u32
constexpr int kOffW = kOffPre + ((kMaxBlocks + 1) * 4 + 15) / 16 * 16;  // [2][256] f32
constexpr int kOffHead = kOffW + 2 * kTileCols * 4;                // [2][256] i32
constexpr int kOffN = kOffHead + 2 * kTileCols * 4;                // [2][32] i32 prefix lengths
constexpr int kOffTau = kOffN + 2 * 32 * 4;                        // [2][32] f32 cuts (compact mode)
constexpr int kOffBar = kOffTau + 2 * 32 * 4;                      // mbarriers
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;                   // tmem base, abort, scan scratch
constexpr int kSmemBytes = kOffMisc + 4 * 36 + 1024;               // + alignment slack

struct Bars {
  uint32_t kfull, kempty, accfull, accempty, qfull, qempty, drain;  // shared addresses of arrays
  __device__ uint32_t kf(int i) const { return kfull + 8 * i; }
  __device__ uint32_t ke(int i) const { return kempty + 8 * i; }
  __device__ uint32_t af(int i) const { return accfull + 8 * i; }
  __device__ uint32_t ae(int i) const { return accempty + 8 * i; }
  __device__ uint32_t qf(int i) const { return qfull + 8 * i; }
  __device__ uint32_t qe(int i) const { return qempty + 8 * i; }
};

// w * ReLU of the 32 accumulator columns [32 CC, 32 CC + 32) of one epilogue thread, two columns
// per packed fp32x2 FMA: column c (counted from the warp's first column) belongs to query c / MP
// of the warp; its slot pair (c % MP) / 2 feeds float2 partial sum ((c % MP) / 2) % NF of that
// query.  wr holds the weights from the warp's first column on.
template <int MP, int NF, int CC>
__device__ __forceinline__ void accumulate_chunk(const uint32_t (&v)[32], const float* wr, float2* acc) {
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 wv = *reinterpret_cast<const float4*>(wr + CC * 32 + j);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const int c = CC * 32 + j + u;
      const int x = (c / MP) * NF + ((c % MP) / 2) % NF;
      const float2 r = make_float2(fmaxf(__uint_as_float(v[j + u]), 0.f), fmaxf(__uint_as_float(v[j + u + 1]), 0.f));
      const float2 ww = u == 0 ? make_float2(wv.x, wv.y) : make_float2(wv.z, wv.w);
      acc[x] = __ffma2_rn(ww, r, acc[x]);
    }
  }
}

__device__ __forceinline__ void give_up(volatile int* abort) {
  *abort = 1;
  atomicExch(&g_tc_status, 1);
}

// Output modes of the scorer:
//   kRows     score rows: out[t, s] for s < n_t (entries past the prefix are not written)
//   kSample   every tile_stride-th key tile only (tiles 0, S, 2S, ...), packed: sampled tile i of a
//             row goes to columns [128 i, 128 i + 128) of out
//   kCompact  no score row: each score at or above tau[t] is appended as (order key, token) to the
//             query's candidate list (lists [T][cap]); lcnt[t] counts every such score, also past
//             cap (then the list is incomplete and the caller redoes the query)
enum { kRows = 0, kSample = 1, kCompact = 2 };

template <int MP, int FM>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap omap,
                    int tma_store, const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                    const int32_t* __restrict__ n, const int32_t* __restrict__ heads, int h, int H_I, int L, int T,
                    float* __restrict__ out, int64_t ld, int tile_stride, const float* __restrict__ tau,
                    uint2* __restrict__ lists, uint32_t* __restrict__ lcnt, int cap) {
  constexpr int QT = kTileCols / MP;  // queries per block
  // key tile of work tile `tile` (the sample takes every tile_stride-th)
  auto key_tile = [&](uint32_t tile) -> int { return FM == kSample ? (int)tile * tile_stride : (int)tile; };
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* pre = reinterpret_cast<uint32_t*>(sm + kOffPre);
  float* wsm = reinterpret_cast<float*>(sm + kOffW);
  int* shead = reinterpret_cast<int*>(sm + kOffHead);  // sorted head of every B row
  int* hraw = shead + kTileCols;                         // the same, as given
  int* nsm = reinterpret_cast<int*>(sm + kOffN);         // n_t of the block's queries
  float* tsm = reinterpret_cast<float*>(sm + kOffTau);   // tau_t of the block's queries (compact mode)
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + kOffMisc);
  volatile uint32_t* tmem_slot = misc;
  volatile int* abort = reinterpret_cast<volatile int*>(misc + 1);
  uint32_t* warp_tot = misc + 4;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NB = (T + QT - 1) / QT;

  // ---- key tiles per query block and their prefix ----
  tc::block_tile_prefix(NB, QT, T, kTileKeys, [&](int t) {
    const int nt = clamp_len(__ldg(n + t), L);
    if (FM != kSample) return nt;
    const int kt = (nt + kTileKeys - 1) / kTileKeys;                   // key tiles of the prefix
    return (kt + tile_stride - 1) / tile_stride * kTileKeys;           // sampled tiles, as a length
  }, pre, warp_tot);
  const uint64_t W = pre[NB];
  const uint32_t a = (uint32_t)(W * blockIdx.x / gridDim.x);
  const uint32_t e = (uint32_t)(W * (blockIdx.x + 1) / gridDim.x);
  if (a >= e) return;  // uniform: nothing allocated yet

  const uint32_t bar0 = tc::smem_u32(sm + kOffBar);
  Bars bars;
  bars.kfull = bar0;
  bars.kempty = bars.kfull + 8 * kStages;
  bars.accfull = bars.kempty + 8 * kStages;
  bars.accempty = bars.accfull + 16;
  bars.qfull = bars.accempty + 16;
  bars.qempty = bars.qfull + 16;
  bars.drain = bars.qempty + 16;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(bars.kf(i), 1);
      tc::mbar_init(bars.ke(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(bars.af(i), 1);
      tc::mbar_init(bars.ae(i), kEpiWarps);
      tc::mbar_init(bars.qf(i), 1);
      tc::mbar_init(bars.qe(i), 1 + kEpiWarps);
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
  const uint32_t qbase = tc::smem_u32(sm + kOffQ);
  const uint32_t kbase = tc::smem_u32(sm + kOffK);

  if (warp < kEpiWarps) {
    // ---------------- epilogue ----------------
    // warp = (column quarter cq, TMEM lane quarter lq); with 128 rows per query the even quarters
    // take a whole query (128 columns) and the odd ones only hand the accumulator back
    constexpr int CW = MP > 64 ? 128 : 64;  // columns of an active warp
    constexpr int QW = CW / MP;              // its queries
    constexpr int NF = MP / 8;               // float2 partial sums per query: chains of 4 a tile
    const int lq = warp & 3, cq = warp >> 2;
    const int col0 = cq * 64;
    float* stage_out = reinterpret_cast<float*>(sm + kOffOut) + warp * kStageOutFloats;
    const bool active = (col0 % CW) == 0;
    uint32_t i = 0, p = 0, lo, hi;
    int blk;
    tc::TileSegments it(pre, NB, a, e);
    while (it.next(blk, lo, hi)) {
      const int pb = p & 1;
      if (!tc::mbar_wait(bars.qf(pb), (p >> 1) & 1, abort, kWaitLimitNs)) {
        give_up(abort);
        break;
      }
      const int tq = blk * QT + col0 / MP;
      const int* nr = nsm + pb * 32 + col0 / MP;
      const float* wr = wsm + pb * kTileCols + col0;
      int nmin = tma_store ? 0x7fffffff : 0;  // keys below it are inside every prefix of the warp
#pragma unroll
      for (int l = 0; l < QW; ++l) nmin = min(nmin, nr[l]);
      bool ok = true;
      for (uint32_t tile = lo; tile < hi; ++tile, ++i) {
        const int ab = i & 1;
        if (!tc::mbar_wait(bars.af(ab), (i >> 1) & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        float2 acc[QW * NF];
#pragma unroll
        for (int x = 0; x < QW * NF; ++x) acc[x] = make_float2(0.f, 0.f);
        if (active) {
          const uint32_t ta = tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(ab * kTileCols + col0);
          // 32-column loads, each overlapping the previous chunk's arithmetic
          uint32_t va[32], vb[32];
          tc::tmem_ld32(ta, va);
          tc::tmem_ld_wait(va);
          tc::tmem_ld32(ta + 32, vb);
          accumulate_chunk<MP, NF, 0>(va, wr, acc);
          tc::tmem_ld_wait(vb);
          if constexpr (CW == 128) {
            tc::tmem_ld32(ta + 64, va);
            accumulate_chunk<MP, NF, 1>(vb, wr, acc);
            tc::tmem_ld_wait(va);
            tc::tmem_ld32(ta + 96, vb);
            accumulate_chunk<MP, NF, 2>(va, wr, acc);
            tc::tmem_ld_wait(vb);
            accumulate_chunk<MP, NF, 3>(vb, wr, acc);
          } else {
            accumulate_chunk<MP, NF, 1>(vb, wr, acc);
          }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_relaxed(bars.ae(ab));
        if (active) {
          const int s0w = key_tile(tile) * kTileKeys + lq * 32;  // first key of the warp's 32
          const int s = s0w + lane;
          const int c0w = FM == kSample ? (int)tile * kTileKeys + lq * 32 : s0w;  // its output column
          float sum[QW];
#pragma unroll
          for (int l = 0; l < QW; ++l) {
#pragma unroll
            for (int st = NF / 2; st >= 1; st >>= 1)
#pragma unroll
              for (int x = 0; x < st; ++x) acc[l * NF + x] = __fadd2_rn(acc[l * NF + x], acc[l * NF + x + st]);
            sum[l] = acc[l * NF].x + acc[l * NF].y;
          }
          if (FM == kCompact) {
            // one ballot per query, then lane l reserves query l's slots: the warp's atomics to its
            // QW lists go out as one instruction, one round trip per tile
            const float* tr = tsm + pb * 32 + col0 / MP;
            unsigned mk[QW];
            uint32_t want = 0;
#pragma unroll
            for (int l = 0; l < QW; ++l) {
              mk[l] = __ballot_sync(0xffffffffu, s < nr[l] && sum[l] >= tr[l]);
              if (lane == l) want = (uint32_t)__popc(mk[l]);
            }
            uint32_t got = 0;
            if (lane < QW && want) got = atomicAdd(lcnt + tq + lane, want);
            const uint32_t below = (1u << lane) - 1u;
#pragma unroll
            for (int l = 0; l < QW; ++l) {
              const uint32_t base = __shfl_sync(0xffffffffu, got, l);
              if ((mk[l] >> lane) & 1u) {
                const uint32_t pos = base + (uint32_t)__popc(mk[l] & below);
                if (pos < (uint32_t)cap) lists[(int64_t)(tq + l) * cap + pos] = make_uint2(order_key(sum[l]), (uint32_t)s);
              }
            }
          } else if (s0w + 32 <= nmin) {  // the whole block: one TMA store
            if (lane == 0) tc::bulk_wait_read_all();  // the previous store has read the buffer
            __syncwarp();
#pragma unroll
            for (int l = 0; l < QW; ++l) stage_out[l * 32 + lane] = sum[l];
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tc::tma_store_2d(&omap, c0w, tq, tc::smem_u32(stage_out));
              tc::bulk_commit();
            }
          } else {
#pragma unroll
            for (int l = 0; l < QW; ++l)
              if (s < nr[l]) out[(int64_t)(tq + l) * ld + c0w + lane] = sum[l];
          }
        }
      }
      if (!ok) {
        give_up(abort);
        break;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bars.qe(pb));
      ++p;
    }
    if (lane == 0) tc::bulk_wait_all();  // staged stores complete before the CTA exits
    __syncwarp();
  } else if (warp == kLoaderWarp) {
    // ---------------- query-head gather ----------------
    const int m = heads ? h : H_I;
    uint32_t p = 0, lo, hi;
    int blk;
    tc::TileSegments it(pre, NB, a, e);
    while (it.next(blk, lo, hi)) {
      const int pb = p & 1;
      if (p >= 2 && !tc::mbar_wait(bars.qe(pb), ((p >> 1) - 1) & 1, abort, kWaitLimitNs)) {
        give_up(abort);
        break;
      }
      const int t0 = blk * QT;
      float* ws = wsm + pb * kTileCols;
      // raw head ids of every (query, slot); padding slots (j >= m) sort last
      for (int idx = lane; idx < kTileCols; idx += 32) {
        const int qi = idx / MP, j = idx % MP, t = t0 + qi;
        int v = 0x7fffffff;
        if (t < T && j < m) {
          v = heads ? __ldg(heads + (int64_t)t * h + j) : j;
          v = v < 0 ? 0 : (v >= H_I ? H_I - 1 : v);
        }
        hraw[idx] = v;
      }
      __syncwarp();
      // each query's heads ascending: the slot of an entry is its rank (ties by position)
      for (int idx = lane; idx < kTileCols; idx += 32) {
        if (!heads) {
          shead[idx] = hraw[idx];
          continue;
        }
        const int qi = idx / MP, j = idx % MP;
        const int* r = hraw + qi * MP;
        const int v = r[j];
        int rank = 0;
        for (int x = 0; x < MP; ++x) {
          const int u = r[x];
          rank += (u < v) || (u == v && x < j);
        }
        shead[qi * MP + rank] = v;
      }
      __syncwarp();
      for (int qi = lane; qi < QT; qi += 32) {
        const int t = t0 + qi;
        nsm[pb * 32 + qi] = t < T ? clamp_len(__ldg(n + t), L) : 0;
        if (FM == kCompact) tsm[pb * 32 + qi] = t < T ? __ldg(tau + t) : INFINITY;
      }
      // weights; padding slots repeat the query's first head with weight 0
      for (int idx = lane; idx < kTileCols; idx += 32) {
        const int qi = idx / MP, j = idx % MP, t = t0 + qi;
        float wv = 0.f;
        if (t < T && j < m)
          wv = __ldg(w + (int64_t)t * H_I + shead[idx]);
        else
          shead[idx] = t < T ? shead[qi * MP] : 0;
        ws[idx] = wv;
      }
      __syncwarp();
      const uint32_t qb = qbase + pb * kQBytes;
      for (int idx = lane; idx < kTileCols * 16; idx += 32) {
        const int row = idx >> 4, c = idx & 15;
        const int t = t0 + row / MP;
        const int tsrc = t < T ? t : T - 1;
        const __nv_bfloat16* src = q + ((int64_t)tsrc * H_I + shead[row]) * kD + c * 8;
        const uint32_t dst = qb + (c >> 3) * kQHalfBytes + (row >> 3) * 1024 + (row & 7) * 128 +
                             ((((uint32_t)c & 7u) ^ ((uint32_t)row & 7u)) << 4);
        tc::cp_async_16(dst, src, t < T ? 16u : 0u);
      }
      tc::cp_async_wait_all();
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bars.qf(pb));
      ++p;
    }
  } else if (warp == kTmaWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t f = 0, lo, hi;
      int blk;
      tc::TileSegments it(pre, NB, a, e);
      bool ok = true;
      while (ok && it.next(blk, lo, hi)) {
        for (uint32_t tile = lo; ok && tile < hi; ++tile) {
          for (int half = 0; half < 2; ++half, ++f) {
            const int st = f % kStages;
            if (f >= kStages && !tc::mbar_wait(bars.ke(st), ((f / kStages) - 1) & 1, abort, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc::mbar_arrive_expect_tx(bars.kf(st), kStageBytes);
            tc::tma_load_2d(kbase + st * kStageBytes, &kmap, half * 64, key_tile(tile) * kTileKeys, bars.kf(st));
          }
        }
      }
      if (!ok) give_up(abort);
      // every issued copy lands before the CTA exits
      for (uint32_t g = f > kStages ? f - kStages : 0; g < f; ++g)
        tc::mbar_wait(bars.kf(g % kStages), (g / kStages) & 1, nullptr, kWaitLimitNs);
    }
  } else {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kTileKeys, kTileCols);
      uint32_t f = 0, i = 0, p = 0, lo, hi;
      int blk;
      tc::TileSegments it(pre, NB, a, e);
      bool ok = true;
      while (ok && it.next(blk, lo, hi)) {
        const int pb = p & 1;
        if (!tc::mbar_wait(bars.qf(pb), (p >> 1) & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t qb = qbase + pb * kQBytes;
        for (uint32_t tile = lo; ok && tile < hi; ++tile, ++i) {
          const int ab = i & 1;
          if (i >= 2 && !tc::mbar_wait(bars.ae(ab), ((i >> 1) - 1) & 1, abort, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(ab * kTileCols);
          for (int half = 0; half < 2; ++half, ++f) {
            const int st = f % kStages;
            if (!tc::mbar_wait(bars.kf(st), (f / kStages) & 1, abort, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc::tc_fence_after();
            const uint64_t ad = tc::sw128_kmajor_desc(kbase + st * kStageBytes);
            const uint64_t bd = tc::sw128_kmajor_desc(qb + half * kQHalfBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc::mma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (half | kk) != 0);
            tc::mma_commit(bars.ke(st));
          }
          if (ok) tc::mma_commit(bars.af(ab));
        }
        if (ok) tc::mma_commit(bars.qe(pb));
        ++p;
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

// Output buffers of one scorer call: out [T, ld] with out_cols columns written at most (score
// rows, or the packed sample), or the candidate lists of compact mode.
struct TcOut {
  float* out;
  int64_t ld;
  int64_t out_cols;
  int tile_stride;
  const float* tau;
  uint2* lists;
  uint32_t* lcnt;
  int cap;
};

template <int MP, int FM>
void launch_mp(const CUtensorMap& map, const __nv_bfloat16* q, const float* w, const int32_t* n,
               const int32_t* heads, int h, int H_I, int L, int T, const TcOut& o, cudaStream_t s) {
  constexpr int QT = kTileCols / MP;
  constexpr int QW = (MP > 64 ? 128 : 64) / MP;  // rows of an epilogue warp's store box
  cudaFuncSetAttribute(score_tc_kernel<MP, FM>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  const int grid = sm_count();
  const int per_launch = kMaxBlocks * QT;
  for (int t0 = 0; t0 < T; t0 += per_launch) {
    const int Tc = T - t0 < per_launch ? T - t0 : per_launch;
    float* ot = FM == kCompact ? nullptr : o.out + (int64_t)t0 * o.ld;
    CUtensorMap omap;
    const bool tma = FM != kCompact &&
                     tmap_f32_rows(&omap, ot, (uint64_t)o.out_cols, (uint64_t)Tc, (uint64_t)o.ld, 32, QW);
    if (!tma) memset(&omap, 0, sizeof(omap));
    score_tc_kernel<MP, FM><<<grid, kThreads, kSmemBytes, s>>>(
        map, omap, tma ? 1 : 0, q + (int64_t)t0 * H_I * kD, w + (int64_t)t0 * H_I, n + t0,
        heads ? heads + (int64_t)t0 * h : nullptr, h, H_I, L, Tc, ot, o.ld, o.tile_stride,
        FM == kCompact ? o.tau + t0 : nullptr, FM == kCompact ? o.lists + (int64_t)t0 * o.cap : nullptr,
        FM == kCompact ? o.lcnt + t0 : nullptr, o.cap);
  }
}

template <int FM>
bool launch_tc_mode(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads, int T,
                    int L, int H_I, int h, const TcOut& o, cudaStream_t s) {
  if (T <= 0 || L <= 0) return true;
  if (reinterpret_cast<uintptr_t>(q) & 15) return false;
  CUtensorMap map;
  if (!tmap_rows128_bf16(&map, k, (uint64_t)L, kTileKeys)) return false;
  const int m = heads ? h : H_I;
  int mp = 8;
  while (mp < m) mp <<= 1;
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  switch (mp) {
    case 8:
      launch_mp<8, FM>(map, qb, w, n, heads, h, H_I, L, T, o, s);
      break;
    case 16:
      launch_mp<16, FM>(map, qb, w, n, heads, h, H_I, L, T, o, s);
      break;
    case 32:
      launch_mp<32, FM>(map, qb, w, n, heads, h, H_I, L, T, o, s);
      break;
    case 64:
      launch_mp<64, FM>(map, qb, w, n, heads, h, H_I, L, T, o, s);
      break;
    case 128:
      launch_mp<128, FM>(map, qb, w, n, heads, h, H_I, L, T, o, s);
      break;
    default:
      return false;
  }
  return true;
}

}  // namespace

static_assert(kSmemBytes <= 232448, "shared memory of the tensor-core scorer exceeds 227 KB");

int sm_count() {
  int dev = 0, v = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
  return v > 0 ? v : 1;
}

bool launch_scores_tc(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads, int T,
                      int L, int H_I, int h, float* out, int64_t ld, cudaStream_t s) {
  const TcOut o{out, ld, L, 1, nullptr, nullptr, nullptr, 0};
  return launch_tc_mode<kRows>(q, w, k, n, heads, T, L, H_I, h, o, s);
}

bool launch_scores_tc_sample(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads,
                             int T, int L, int H_I, int h, int tile_stride, float* sample, int64_t ld,
                             cudaStream_t s) {
  const int64_t cols = (int64_t)((L + kTileKeys - 1) / kTileKeys + tile_stride - 1) / tile_stride * kTileKeys;
  const TcOut o{sample, ld, cols, tile_stride, nullptr, nullptr, nullptr, 0};
  return launch_tc_mode<kSample>(q, w, k, n, heads, T, L, H_I, h, o, s);
}

bool launch_scores_tc_compact(const void* q, const float* w, const void* k, const int32_t* n, const int32_t* heads,
                              int T, int L, int H_I, int h, const float* tau, uint2* lists, uint32_t* lcnt, int cap,
                              cudaStream_t s) {
  const TcOut o{nullptr, 0, 0, 1, tau, lists, lcnt, cap};
  return launch_tc_mode<kCompact>(q, w, k, n, heads, T, L, H_I, h, o, s);
}

int read_and_clear_tc_status() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_status, sizeof(int)) != cudaSuccess) return -1;
  if (v) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(int));
  }
  return v;
}

}  // namespace misa
