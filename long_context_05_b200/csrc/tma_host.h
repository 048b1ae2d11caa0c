// Host helper: encode 2-D TMA tensor maps through the driver entry point
// (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

namespace dsa {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major matrix of `rows` rows, each `row_elems` elements of `elem_bytes`
// (row pitch `pitch_bytes`, a multiple of 16), read in boxes of box_rows x
// box_elems.  The inner box extent in bytes must be a multiple of 16 and, with
// swizzling, no larger than the swizzle span.
inline bool make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* base,
                         uint64_t rows, uint64_t row_elems, uint64_t pitch_bytes, uint32_t box_rows,
                         uint32_t box_elems, CUtensorMapSwizzle swizzle) {
  auto enc = tmap_encoder();
  if (enc == nullptr) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0 || pitch_bytes % 16 != 0) return false;
  if ((box_elems * elem_bytes) % 16 != 0) return false;
  cuuint64_t dims[2] = {row_elems, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_elems, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace dsa
