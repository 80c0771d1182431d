// tmap.cu -- host-side TMA tensor-map construction through the driver entry
// point (no link-time dependency on libcuda).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "sm100_primitives.cuh"

namespace dsa {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_once;

void resolve() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

}  // namespace

namespace {

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType type, uint32_t elem_bytes, const void* base,
                  uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                  CUtensorMapSwizzle swizzle) {
  std::call_once(g_once, resolve);
  if (!g_encode) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                       uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, cols, rows, box_cols,
                      box_rows, swizzle);
}

bool make_tmap_u8_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                     uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, cols, rows, box_cols, box_rows,
                      swizzle);
}

}  // namespace dsa
