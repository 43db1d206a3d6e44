// tmap.h -- host-side creation of TMA tensor maps (driver entry point fetched
// through the runtime, so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace msa {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D view [rows][cols] of 16-bit elements (row pitch `pitch_elems`), box
// [box_rows][box_cols].  Returns false if the driver rejects the map
// (alignment, box or stride rules).
inline bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base,
                         uint64_t rows, uint64_t cols, uint64_t pitch_elems, uint32_t box_rows,
                         uint32_t box_cols, CUtensorMapSwizzle swizzle) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                              uint64_t pitch_elems, uint32_t box_rows, uint32_t box_cols,
                              CUtensorMapSwizzle swizzle) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rows, cols, pitch_elems,
                      box_rows, box_cols, swizzle);
}

// 3-D view [d2][d1][d0] of 16-bit elements (element strides: 1, pitch1,
// pitch2; the strides need not grow with the dimension), box [b2][b1][b0].
inline bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType type, const void* base,
                         uint64_t d0, uint64_t d1, uint64_t d2, uint64_t pitch1_elems,
                         uint64_t pitch2_elems, uint32_t b0, uint32_t b1, uint32_t b2,
                         CUtensorMapSwizzle swizzle) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {pitch1_elems * 2, pitch2_elems * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 version; used e.g. for one group's rows of a [tokens][groups][dim] tensor.
inline bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                              uint64_t d2, uint64_t pitch1_elems, uint64_t pitch2_elems,
                              uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle swizzle) {
  return make_tmap_3d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, d0, d1, d2, pitch1_elems,
                      pitch2_elems, b0, b1, b2, swizzle);
}

}  // namespace msa
