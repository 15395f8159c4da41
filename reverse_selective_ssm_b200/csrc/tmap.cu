// TMA tensor-map encoding through the runtime's driver entry point, so the
// library needs no link-time dependency on libcuda.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tmap.h"

namespace r2l {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // Resolved once per process; the pointer never changes afterwards.
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

}  // namespace

bool make_tmap_2d(CUtensorMap* m, const void* base, int elem_bytes, long long inner, long long rows,
                  long long ld_bytes, int box_inner, int box_rows, int swizzle_bytes) {
  auto enc = encode_fn();
  if (!enc || inner <= 0 || rows <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
             : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                   : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_rows_by_parity(CUtensorMap* m, const void* base, int elem_bytes, long long inner, long long rows,
                              long long ld_bytes, int box_inner, int box_rows, int swizzle_bytes) {
  auto enc = encode_fn();
  if (!enc || inner <= 0 || rows <= 0 || (rows & 1)) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, 2u, (cuuint64_t)(rows / 2)};
  cuuint64_t strides[2] = {(cuuint64_t)ld_bytes, (cuuint64_t)(2 * ld_bytes)};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1u, 1u, 1u};
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
             : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                   : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace r2l
