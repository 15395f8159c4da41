// Host launcher of the tcgen05 GEMM (gemm_tc.cuh): TMA descriptor encoding,
// tile-width choice and the persistent launch (one CTA per SM).
#include <cuda.h>

#include <type_traits>

#include "gemm_convx.cuh"
#include "gemm_tc.cuh"
#include "tc_gemm.h"
#include "tmap.h"

namespace r2l {
namespace {

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// 256 × 256 tiles (two M = 128 MMA blocks per CTA) for 256-multiple N (0: 128 × BN only).
#ifndef R2L_GEMM_MB2
#define R2L_GEMM_MB2 1
#endif
// shortest K for which the 256 × 256 tile pays (its epilogue does not overlap the next tile)
#ifndef R2L_GEMM_MB2_MIN_K
#define R2L_GEMM_MB2_MIN_K 0
#endif

template <int BN, typename TOut, int MB = 1>
cudaError_t launch(const TcGemm& g, cudaStream_t st) {
  using Cfg = TcGemmCfg<BN, TOut, MB>;
  CUtensorMap ta, tb, tc;
  if (!make_tmap_2d(&ta, g.A, 2, g.K, g.M, (long long)g.lda * 2, Cfg::BK, Cfg::BM, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, g.B, 2, g.K, g.N, (long long)g.ldb * 2, Cfg::BK, BN, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tc, g.C, (int)sizeof(TOut), g.N, g.M, (long long)g.ldc * sizeof(TOut), 32, 32, Cfg::STG_SWIZZLE))
    return cudaErrorInvalidValue;
  auto kern = gemm_tc_kernel<BN, TOut, MB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)((g.M + Cfg::BM - 1) / Cfg::BM) * ((g.N + BN - 1) / BN);
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, st>>>(ta, tb, tc, g.C2, g.ldc2, g.c2_cols,
                                            g.M, g.N, g.K, g.len, g.L, g.err);
  return cudaPeekAtLastError();
}

template <typename TOut>
cudaError_t dispatch(const TcGemm& g, cudaStream_t st) {
  // widest tile that divides N; else the narrowest that covers it; else 256 with a ragged edge
  if (g.N % 256 == 0) {
    // 256 × 256 tiles only when there are enough of them to give every SM one
    if constexpr (std::is_same<TOut, bf16>::value)
      if (R2L_GEMM_MB2 && g.K >= R2L_GEMM_MB2_MIN_K &&
          (long long)((g.M + 255) / 256) * (g.N / 256) >= sm_count())
        return launch<256, TOut, 2>(g, st);
    return launch<256, TOut>(g, st);
  }
  if (g.N <= 64) return launch<64, TOut>(g, st);
  if (g.N <= 128) return launch<128, TOut>(g, st);
  if (g.N <= 160) return launch<160, TOut>(g, st);
  if (g.N % 128 == 0) return launch<128, TOut>(g, st);
  return launch<256, TOut>(g, st);
}

template <bool FWD>
cudaError_t launch_convx(const ConvX& g, cudaStream_t st) {
  namespace cx = convx;
  CUtensorMap tx, tb, tc, tw4, tcb;
  if (!make_tmap_2d(&tx, g.x, 2, g.E, g.M, g.ldx * 2, cx::BK, cx::XR, 0) ||
      !make_tmap_2d(&tb, g.W, 2, g.E, cx::BN, (long long)g.E * 2, cx::BK, cx::BN, 128) ||
      !make_tmap_2d(&tc, g.C, 4, cx::BN, g.M, (long long)g.ldc * 4, 32, 32, 128) ||
      !make_tmap_2d(&tw4, g.conv_w, 4, 4, g.E, 16, 4, cx::BK, 0) ||
      !make_tmap_2d(&tcb, g.conv_b, 4, g.E, 1, (long long)g.E * 4, cx::BK, 1, 0))
    return cudaErrorInvalidValue;
  auto kern = cx::gemm_convx_kernel<FWD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cx::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long tiles = (g.M + cx::BM - 1) / cx::BM;
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  if (grid <= 0) return cudaSuccess;
  cx::Args a;
  a.x = g.x; a.ldx = g.ldx; a.conv_w = g.conv_w; a.conv_b = g.conv_b; a.u = g.u; a.ldu = g.ldu;
  a.M = g.M; a.K = g.E; a.C2 = g.C2; a.ldc2 = g.ldc2; a.c2_cols = g.c2_cols; a.len = g.len; a.L = g.L;
  a.err = g.err;
  kern<<<grid, cx::THREADS, cx::SMEM_BYTES, st>>>(tx, tb, tc, tw4, tcb, a);
  return cudaPeekAtLastError();
}

}  // namespace

bool convx_supported(int N, int E) { return N == convx::BN && E > 0 && E % convx::BK == 0; }

bool convx_worthwhile(long long M) { return (M + convx::BM - 1) / convx::BM >= sm_count(); }

cudaError_t convx_gemm(const ConvX& g, cudaStream_t st) {
  if (g.M <= 0) return cudaSuccess;
  if (!convx_supported(160, g.E) || (g.ldx % 8) || (g.ldu % 2) || (g.ldc * 4) % 16) return cudaErrorInvalidValue;
  return g.fwd ? launch_convx<true>(g, st) : launch_convx<false>(g, st);
}

cudaError_t tc_gemm(const TcGemm& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return cudaSuccess;
  if ((g.lda % 8) || (g.ldb % 8) || (g.K % 8)) return cudaErrorInvalidValue;  // TMA: 16-byte strides
  if ((g.ldc * (g.c_fp32 ? 4 : 2)) % 16) return cudaErrorInvalidValue;
  return g.c_fp32 ? dispatch<float>(g, st) : dispatch<bf16>(g, st);
}

}  // namespace r2l
