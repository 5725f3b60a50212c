// Host side of the TMA loads: 2-D tensor maps over row-major bf16 matrices with 128 columns,
// encoded through the driver entry point obtained from the runtime (no link against libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace misa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tmap_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      (void)cudaGetLastError();
  });
  return fn;
}

// Map over a [rows, 128] bf16 matrix (row stride 256 bytes) loading boxes of 64 columns x
// box_rows rows into the 128-byte swizzled layout; rows past the end read as zero.  False if the
// base is not 16-byte aligned or the encoder is unavailable.
inline bool tmap_rows128_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  if (reinterpret_cast<uintptr_t>(base) & 15) return false;
  const EncodeTiledFn encode = tmap_encoder();
  if (!encode || rows == 0) return false;
  const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over a row-major fp32 matrix [rows, cols] with a row stride of ld elements, for stores of
// box_cols x box_rows boxes (no swizzle); writes outside the matrix are dropped.  False unless
// the base is 16-byte aligned and ld is a multiple of 4.
inline bool tmap_f32_rows(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t ld,
                          uint32_t box_cols, uint32_t box_rows) {
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld % 4) != 0 || cols == 0 || rows == 0) return false;
  const EncodeTiledFn encode = tmap_encoder();
  if (!encode) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count();  // multiprocessors of the current device (score_tc.cu)

}  // namespace misa
