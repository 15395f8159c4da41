// Host launcher of the tcgen05 GEMM (gemm_tc.cuh): TMA descriptor encoding,
// tile-width choice and the persistent launch (one CTA per SM).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gemm_tc.cuh"
#include "tc_gemm.h"

namespace r2l {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // Resolved once per process through the runtime, so the library needs no
  // link-time dependency on libcuda.  The pointer never changes afterwards.
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

// Row-major bf16 matrix [rows, inner] with row stride `ld` elements, read in
// boxes of 64 (inner) × box_rows with 128-byte swizzle; out-of-range elements
// read as zero.
bool make_tmap(CUtensorMap* m, const void* base, int inner, long long rows, int ld, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int BN, typename TOut>
cudaError_t launch(const TcGemm& g, cudaStream_t st) {
  using Cfg = TcGemmCfg<BN>;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, g.A, g.K, g.M, g.lda, Cfg::BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, g.B, g.K, g.N, g.ldb, BN)) return cudaErrorInvalidValue;
  auto kern = gemm_tc_kernel<BN, TOut>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)((g.M + Cfg::BM - 1) / Cfg::BM) * ((g.N + BN - 1) / BN);
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, 192, Cfg::SMEM_BYTES, st>>>(ta, tb, static_cast<TOut*>(g.C), g.ldc, g.C2, g.ldc2, g.c2_cols,
                                            g.M, g.N, g.K, g.len, g.L, g.err);
  return cudaPeekAtLastError();
}

template <typename TOut>
cudaError_t dispatch(const TcGemm& g, cudaStream_t st) {
  // widest tile that divides N; else the narrowest that covers it; else 256 with a ragged edge
  if (g.N % 256 == 0) return launch<256, TOut>(g, st);
  if (g.N <= 64) return launch<64, TOut>(g, st);
  if (g.N <= 128) return launch<128, TOut>(g, st);
  if (g.N <= 160) return launch<160, TOut>(g, st);
  if (g.N % 128 == 0) return launch<128, TOut>(g, st);
  return launch<256, TOut>(g, st);
}

}  // namespace

cudaError_t tc_gemm(const TcGemm& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return cudaSuccess;
  if ((g.lda % 8) || (g.ldb % 8) || (g.K % 8)) return cudaErrorInvalidValue;  // TMA: 16-byte strides
  return g.c_fp32 ? dispatch<float>(g, st) : dispatch<bf16>(g, st);
}

}  // namespace r2l
