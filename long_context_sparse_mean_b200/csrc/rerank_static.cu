// misa_hier_rerank_static: the MISA-dagger re-rank for callers that cannot allocate device memory.
//
// misa_hier_rerank needs T * k' floats of scratch for the dense scores of the candidates and
// takes them from a caller-provided workspace.  Some callers have no way to provide one: a
// plugin that a host framework hands only its input and output buffers (the framework owns the
// device memory pool and exposes no allocator), or a latency-critical decode loop that must not
// risk an allocation failure or the device synchronisation that cudaMalloc / cudaFree can cause
// in the middle of a step.  This variant keeps that scratch in a fixed array compiled into the
// library instead, so the call allocates nothing: no cudaMalloc, no cudaFree, no allocating
// library routine.
//
// Limits and sharing:
//   - the array holds MISA_STATIC_RERANK_SCRATCH_FLOATS floats (4 MiB); every GPU that loads the
//     library keeps it until the process exits.  Calls with T * kp above that return
//     MISA_ERR_WORKSPACE and launch nothing.
//   - every call on a device uses the same array and leaves its contents behind.  Nothing in it
//     has to start at zero: each entry the selection reads was written earlier in the same call.
//     Two calls whose kernels overlap on the GPU (different streams, no ordering between them)
//     race on the array and both results are undefined; order such calls on one stream or with
//     events.
//   - the array's device address is looked up once per device (cudaGetSymbolAddress, with that
//     device current) by the first call on that device; make that first call before any stream
//     capture.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/misa.h"
#include "kernels.cuh"

namespace {

// Dense re-rank scores F[T, kp] of the current call.
static __device__ __align__(256) float g_rerank_scratch[MISA_STATIC_RERANK_SCRATCH_FLOATS];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_rerank_scratch on the current device (the host-side name of the array is
// only a stand-in and must never reach a kernel).
misa_status scratch_on_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MISA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_rerank_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MISA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MISA_OK;
}

}  // namespace

extern "C" misa_status misa_hier_rerank_static(const void* q, const float* w, const void* k,
                                               int64_t k_seq_stride, const int32_t* n, const int32_t* cand,
                                               int T, int L, int H_I, int d, int kp, int topk, int dtype,
                                               int32_t* idx, float* score_opt, void* stream) {
  if (T < 0 || L < 1 || k_seq_stride < 0 || topk < 1 || kp < topk) return MISA_ERR_INVALID_ARG;
  if (dtype != MISA_BF16 && dtype != MISA_F32) return MISA_ERR_UNSUPPORTED;
  if (d != misa::kD || H_I < 8 || H_I > misa::kMaxHeads || H_I % 8 != 0) return MISA_ERR_UNSUPPORTED;
  if (kp > MISA_MAX_KP) return MISA_ERR_UNSUPPORTED;
  if (k_seq_stride != 0 && k_seq_stride < (int64_t)L * d) return MISA_ERR_INVALID_ARG;
  if (T == 0) return MISA_OK;
  if (!q || !w || !k || !n || !cand || !idx) return MISA_ERR_INVALID_ARG;
  if ((int64_t)T * kp > (int64_t)MISA_STATIC_RERANK_SCRATCH_FLOATS) return MISA_ERR_WORKSPACE;
  float* F = nullptr;
  const misa_status st = scratch_on_current_device(&F);
  if (st != MISA_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const misa::DType dt = dtype == MISA_F32 ? misa::DType::F32 : misa::DType::BF16;
  misa::launch_scores(dt, q, w, k, k_seq_stride, n, nullptr, T, L, H_I, H_I, cand, kp, F, kp, s);
  misa::launch_topk_cand(F, cand, n, T, L, kp, topk, idx, score_opt, s);
  return cudaGetLastError() == cudaSuccess ? MISA_OK : MISA_ERR_CUDA;
}
