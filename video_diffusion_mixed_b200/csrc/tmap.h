// tmap.h -- host-side construction of TMA tensor maps (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so the library needs no link-time dependency on libcuda).
#pragma once

#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace sb {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// A [rows][K] bf16 row-major tensor (K a multiple of 64) seen as 128-byte chunks:
// dims {64, K/64, rows}; one box = 16 chunks of one row = a 1024-element row segment (2 KB),
// 128B swizzle. Chunks past K and rows past the end read as zero.
inline bool make_row_segment_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K) {
  auto fn = tmap_encoder();
  if (!fn || K % 64 != 0 || (reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)(K / 64), (cuuint64_t)rows};
  cuuint64_t strides[2] = {128, (cuuint64_t)K * 2};
  cuuint32_t box[3] = {64, 16, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A [rows][K] bf16 row-major tensor (K a multiple of 64) seen as one column of 128-byte half
// blocks: dims {64, rows * K / 64}; one box = 64 consecutive half blocks = 32 Hadamard blocks of
// 128 channels (8 KB), 128B swizzle. Half blocks past the end read as zero. The half-block count
// must fit a signed 32-bit coordinate.
inline bool make_halfblock_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K) {
  auto fn = tmap_encoder();
  if (!fn || K % 64 != 0 || (reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  const int64_t n = rows * (K / 64);
  if (n <= 0 || n >= (int64_t(1) << 31)) return false;
  cuuint64_t dims[2] = {64, (cuuint64_t)n};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sb
