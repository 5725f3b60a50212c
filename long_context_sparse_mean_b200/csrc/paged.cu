// Paged key caches: the keys of sequence t live in fixed-size pages of one shared pool
// [num_pages, page_size, 128], and its logical key s is row s % page_size of physical page
// page_table[t][s / page_size].  The indexer's definitions apply to the logical cache unchanged
// (the pages call MISA a drop-in replacement for the DSA indexer, "Key Contributions"; paging is the
// serving layout such a replacement has to read).
//
// The scoring and re-rank stages read a paged cache through the gather path of the scorer: the
// pool is one shared cache of num_pages * page_size rows, and paged_rows_kernel turns each query's
// logical positions (its prefix, or its candidate tokens) into physical rows, -1 where a position
// lies past the prefix or its page id is out of range.  Key rows stay 256 contiguous bytes, so the
// scorer's bound is the same as for contiguous caches plus 4 bytes of row id per key.
// Pooling and the router's partial-block mean read the pool through the same lookup.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace misa {

namespace {

// Physical row of logical key s of sequence t, or -1 (page past the table or out of the pool; a
// bounds-checked build counts an out-of-pool page when `count` is set).
__device__ __forceinline__ int64_t paged_row(const int32_t* table, int64_t max_pages, int64_t num_pages,
                                             int page_size, int t, int64_t s, bool count) {
  const int64_t lp = s / page_size;
  if (lp >= max_pages) return -1;
  const int32_t pg = __ldg(table + (int64_t)t * max_pages + lp);
  if (pg < 0 || pg >= num_pages) {
    count_bad_id(kBadPage, count);
    return -1;
  }
  return (int64_t)pg * page_size + s % page_size;
}

// rows[t, p] = physical row of logical token s = p (ids == nullptr) or ids[t, p], for 0 <= s < n_t;
// -1 otherwise.  n_phys[t] = pool_rows (every physical row is a valid gather target).
__global__ void paged_rows_kernel(const int32_t* __restrict__ table, int64_t max_pages, int64_t num_pages,
                                  int page_size, const int32_t* __restrict__ n, int L, const int32_t* __restrict__ ids,
                                  int P, int32_t* __restrict__ rows, int32_t* __restrict__ n_phys, int pool_rows) {
  const int t = blockIdx.y;
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p == 0) n_phys[t] = pool_rows;
  if (p >= P) return;
  const int nt = clamp_len(n[t], L);
  const int64_t s = ids ? (int64_t)ids[(int64_t)t * P + p] : (int64_t)p;
  count_bad_id(kBadCandidate, ids && s != -1 && (s < 0 || s >= nt));
  const int64_t r = (s >= 0 && s < nt) ? paged_row(table, max_pages, num_pages, page_size, t, s, true) : -1;
  rows[(int64_t)t * P + p] = (int32_t)r;
}

// Sum over logical keys [s0, s1) of sequence t, RG row groups x 64 column pairs (blockDim = 64 RG);
// rows whose page is out of range count as zero.  part[RG][kD] is shared scratch; the column sums
// end up in part[0][*] (after the barrier inside).
template <DType DT, int RG>
__device__ __forceinline__ void paged_sum(const void* pool, const int32_t* table, int64_t max_pages,
                                          int64_t num_pages, int page_size, int t, int s0, int s1,
                                          float (*part)[kD]) {
  const int cp = threadIdx.x & 63, rg = threadIdx.x >> 6;
  float a0 = 0.f, a1 = 0.f;
  for (int s = s0 + rg; s < s1; s += RG) {
    const int64_t r = paged_row(table, max_pages, num_pages, page_size, t, s, cp == 0);  // one count per row
    if (r < 0) continue;
    if (DT == DType::BF16) {
      const uint32_t x = __ldg(reinterpret_cast<const uint32_t*>(pool) + r * (kD / 2) + cp);
      a0 += bf16_lo(x);
      a1 += bf16_hi(x);
    } else {
      const float2 x = __ldg(reinterpret_cast<const float2*>(pool) + r * (kD / 2) + cp);
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
    for (int g = 0; g < RG; ++g) sum += part[g][threadIdx.x];
    part[0][threadIdx.x] = sum;  // only part[g][threadIdx.x] of this thread's column is touched
  }
  __syncthreads();
}

// kbar[seq, b] = mean of logical keys [bB, min((b+1)B, L)) of each sequence (1024 threads).
template <DType DT>
__global__ void __launch_bounds__(1024) pool_paged_kernel(const void* __restrict__ pool, int64_t num_pages,
                                                          int page_size, const int32_t* __restrict__ table,
                                                          int64_t max_pages, int L, int B, float* __restrict__ kbar,
                                                          int64_t kbar_seq_stride, int b0) {
  __shared__ float part[16][kD];
  const int b = b0 + blockIdx.x, seq = blockIdx.y;
  const int s0 = b * B, s1 = min(s0 + B, L);
  paged_sum<DT, 16>(pool, table, max_pages, num_pages, page_size, seq, s0, s1, part);
  if (threadIdx.x < kD)
    kbar[(int64_t)seq * kbar_seq_stride + (int64_t)b * kD + threadIdx.x] = part[0][threadIdx.x] / (float)(s1 - s0);
}

// pm[t] = mean of the last block of query t's prefix, logical keys [kbar_blocks(n_t, B) B, n_t)
// (full or partial; untouched for an empty prefix), 256 threads.
template <DType DT>
__global__ void __launch_bounds__(256) partial_mean_paged_kernel(const void* __restrict__ pool, int64_t num_pages,
                                                                 int page_size, const int32_t* __restrict__ table,
                                                                 int64_t max_pages, const int32_t* __restrict__ n,
                                                                 int L, int B, float* __restrict__ pm) {
  __shared__ float part[4][kD];
  const int t = blockIdx.x;
  const int nt = clamp_len(n[t], L);
  const int c = nt - kbar_blocks(nt, B) * B;
  if (c == 0) return;
  paged_sum<DT, 4>(pool, table, max_pages, num_pages, page_size, t, nt - c, nt, part);
  if (threadIdx.x < kD) pm[(int64_t)t * kD + threadIdx.x] = part[0][threadIdx.x] / (float)c;
}

}  // namespace

void launch_paged_rows(const int32_t* table, int64_t max_pages, int64_t num_pages, int page_size, const int32_t* n,
                       int T, int L, const int32_t* ids, int P, int32_t* rows, int32_t* n_phys, cudaStream_t s) {
  if (T <= 0 || P <= 0) return;
  const dim3 grid((P + 255) / 256, T);
  paged_rows_kernel<<<grid, 256, 0, s>>>(table, max_pages, num_pages, page_size, n, L, ids, P, rows, n_phys,
                                         (int)(num_pages * page_size));
}

void launch_pool_paged(DType dt, const void* pool, int64_t num_pages, int page_size, const int32_t* table,
                       int64_t max_pages, int n_seq, int L, int B, float* kbar, int64_t kbar_seq_stride, int b0,
                       int b1, cudaStream_t s) {
  if (n_seq <= 0 || b1 <= b0) return;
  const dim3 grid(b1 - b0, n_seq);
  if (dt == DType::BF16)
    pool_paged_kernel<DType::BF16><<<grid, 1024, 0, s>>>(pool, num_pages, page_size, table, max_pages, L, B, kbar,
                                                         kbar_seq_stride, b0);
  else
    pool_paged_kernel<DType::F32><<<grid, 1024, 0, s>>>(pool, num_pages, page_size, table, max_pages, L, B, kbar,
                                                        kbar_seq_stride, b0);
}

void launch_partial_mean_paged(DType dt, const void* pool, int64_t num_pages, int page_size, const int32_t* table,
                               int64_t max_pages, const int32_t* n, int T, int L, int B, float* pm, cudaStream_t s) {
  if (T <= 0) return;
  if (dt == DType::BF16)
    partial_mean_paged_kernel<DType::BF16><<<T, 256, 0, s>>>(pool, num_pages, page_size, table, max_pages, n, L, B,
                                                             pm);
  else
    partial_mean_paged_kernel<DType::F32><<<T, 256, 0, s>>>(pool, num_pages, page_size, table, max_pages, n, L, B,
                                                            pm);
}

MISA_BAD_ID_READER(read_and_clear_bad_ids_paged)

}  // namespace misa
