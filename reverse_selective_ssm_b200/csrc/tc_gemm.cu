// Host launcher of the tcgen05 GEMM (gemm_tc.cuh): TMA descriptor encoding,
// tile-width choice and the persistent launch (one CTA per SM).
#include <cuda.h>

#include <type_traits>

#include "gemm_convx.cuh"
#include "gemm_tc.cuh"
#include "launch_pdl.h"
#include "tc_gemm.h"
#include "tmap.h"

namespace r2l {

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

namespace {

// 256 × 256 tiles (two M = 128 MMA blocks per CTA) for 256-multiple N (0: 128 × BN only).
#ifndef R2L_GEMM_MB2
#define R2L_GEMM_MB2 1
#endif
// split-K for fp32-output GEMMs with fewer tiles than SMs (0: off)
#ifndef R2L_GEMM_SPLITK
#define R2L_GEMM_SPLITK 1
#endif
// shortest K for which the 256 × 256 tile pays (its epilogue does not overlap the next tile)
#ifndef R2L_GEMM_MB2_MIN_K
#define R2L_GEMM_MB2_MIN_K 0
#endif

// Split-K: C[m, c] = Σ_s P[s·Mp + m, c], slices added in order s = 0, 1, …
// (deterministic); C2[m, c] = bf16 of it for c < c2_cols on valid rows.
__global__ void splitk_sum_kernel(const float* __restrict__ P, int splits, long long Mp, int N,
                                  float* __restrict__ C, int ldc, bf16* __restrict__ C2, int ldc2, int c2_cols,
                                  int M, const int* __restrict__ len, int L) {
  grid_dep_wait();
  grid_dep_launch();
  const int m = blockIdx.x;
  if (m >= M) return;
  const bool valid = !len || row_valid(len, L, m);
  for (int c = threadIdx.x; c < N; c += blockDim.x) {
    float acc = 0.0f;
    for (int sp = 0; sp < splits; ++sp) acc += P[((long long)sp * Mp + m) * N + c];
    C[(long long)m * ldc + c] = acc;
    if (C2 && valid && c < c2_cols) C2[(long long)m * ldc2 + c] = __float2bfloat16_rn(acc);
  }
}

// The same sum, four columns per thread (N and ldc multiples of 4, P and C
// 16-byte aligned): up to eight slices' loads are in flight before their adds,
// which keep the order above, so both kernels give the same bits.
__global__ void splitk_sum4_kernel(const float* __restrict__ P, int splits, long long Mp, int N,
                                   float* __restrict__ C, int ldc, bf16* __restrict__ C2, int ldc2, int c2_cols,
                                   int M, const int* __restrict__ len, int L) {
  grid_dep_wait();
  grid_dep_launch();
  const int n4 = N >> 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)M * n4) return;
  const int m = (int)(idx / n4);
  const int c = (int)(idx - (long long)m * n4) * 4;
  const float* p = P + (long long)m * N + c;
  const long long slice = Mp * N;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int s0 = 0; s0 < splits; s0 += 8) {
    float4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (s0 + i < splits) v[i] = *reinterpret_cast<const float4*>(p + (s0 + i) * slice);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (s0 + i < splits) {
        acc.x += v[i].x;
        acc.y += v[i].y;
        acc.z += v[i].z;
        acc.w += v[i].w;
      }
  }
  *reinterpret_cast<float4*>(C + (long long)m * ldc + c) = acc;
  if (C2 && c < c2_cols && (!len || row_valid(len, L, m))) {
    const float a[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (c + i < c2_cols) C2[(long long)m * ldc2 + c + i] = __float2bfloat16_rn(a[i]);
  }
}

}  // namespace

cudaError_t tc_gemm_add_partials(const float* P, int splits, long long Mp, int N, float* C, int ldc, bf16* C2,
                                 int ldc2, int c2_cols, int M, const int* len, int L, cudaStream_t st) {
  if ((N | ldc) & 3 || ((reinterpret_cast<uintptr_t>(P) | reinterpret_cast<uintptr_t>(C)) & 15)) return cudaErrorInvalidValue;
  const long long n = (long long)M * (N / 4);
  if (n <= 0) return cudaSuccess;
  return launch_pdl(splitk_sum4_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, P, splits, Mp, N, C, ldc,
                    C2, ldc2, c2_cols, M, len, L);
}

int tc_gemm_kept_splits(long long M, int N, int K) {
  if (N % 256 != 0 || M <= 0) return 0;
  const long long tiles = (M + 127) / 128 * (N / 256);
  const int sms = sm_count();
  if (tiles >= sms) return 0;
  const int num_k = (K + 63) / 64;
  int sp = (int)(sms / tiles);             // one wave of (tile, split) units
  if (sp > 8) sp = 8;
  while (sp > 1 && num_k / sp < 8) --sp;
  return sp < 1 ? 1 : sp;
}

namespace {

int tile_width(int N) {   // the BN dispatch() picks for an fp32-output GEMM of this width
  if (N % 256 == 0) return 256;
  if (N <= 64) return 64;
  if (N <= 128) return 128;
  if (N <= 160) return 160;
  if (N % 128 == 0) return 128;
  return 256;
}

// K splits for an fp32-output GEMM with fewer tiles than SMs (0 ⇒ none):
// enough (tile, split) units to cover the SMs, at least 4 K blocks each,
// every split non-empty.
int choose_splits(long long tiles, int num_k) {
  const int sms = sm_count();
  if (tiles * 2 > sms || num_k < 8) return 1;
  int want = (int)(sms / tiles);
  if (want > num_k / 4) want = num_k / 4;
  if (want < 2) return 1;
  const int kps = (num_k + want - 1) / want;
  return (num_k + kps - 1) / kps;
}

template <int BN, typename TOut, int MB = 1, int AMN = 0, int BMN = 0>
cudaError_t launch(const TcGemm& g, cudaStream_t st) {
  using Cfg = TcGemmCfg<BN, TOut, MB>;
  CUtensorMap ta, tb, tc;
  // K-major: boxes of 64 K × BM (BN) rows; MN-major: boxes of 64 M (N) × 64 K rows
  if (AMN ? !make_tmap_2d(&ta, g.A, 2, g.M, g.K, (long long)g.lda * 2, 64, Cfg::BK, 128)
          : !make_tmap_2d(&ta, g.A, 2, g.K, g.M, (long long)g.lda * 2, Cfg::BK, Cfg::BM, 128))
    return cudaErrorInvalidValue;
  if (BMN ? !make_tmap_2d(&tb, g.B, 2, g.N, g.K, (long long)g.ldb * 2, 64, Cfg::BK, 128)
          : !make_tmap_2d(&tb, g.B, 2, g.K, g.N, (long long)g.ldb * 2, Cfg::BK, BN, 128))
    return cudaErrorInvalidValue;
  if (!g.keep_partials &&
      !make_tmap_2d(&tc, g.C, (int)sizeof(TOut), g.N, g.M, (long long)g.ldc * sizeof(TOut), 32, 32, Cfg::STG_SWIZZLE))
    return cudaErrorInvalidValue;
  auto kern = gemm_tc_kernel<BN, TOut, MB, AMN, BMN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long num_m = (g.M + Cfg::BM - 1) / Cfg::BM;
  const long long tiles = num_m * ((g.N + BN - 1) / BN);
  int splits = 1;
  if constexpr (std::is_same<TOut, float>::value) {
    if (g.keep_partials) {
      const int sp = g.kept_splits;
      const size_t need = (size_t)sp * num_m * Cfg::BM * g.N * sizeof(float);
      if (BN != 256 || MB != 1 || sp < 1 || !g.partial || g.partial_bytes < need) return cudaErrorInvalidValue;
      splits = sp;
      if (!make_tmap_2d(&tc, g.partial, 4, g.N, (long long)sp * num_m * Cfg::BM, (long long)g.N * 4, 32, 32,
                        Cfg::STG_SWIZZLE))
        return cudaErrorInvalidValue;
    }
  }
  if constexpr (std::is_same<TOut, float>::value) {
    const int sp = g.keep_partials ? 1 : choose_splits(tiles, (g.K + Cfg::BK - 1) / Cfg::BK);
    const size_t need = (size_t)sp * num_m * Cfg::BM * g.N * sizeof(float);
    if (R2L_GEMM_SPLITK && sp > 1 && g.partial && g.partial_bytes >= need) {
      splits = sp;
      if (!make_tmap_2d(&tc, g.partial, 4, g.N, (long long)sp * num_m * Cfg::BM, (long long)g.N * 4, 32, 32,
                        Cfg::STG_SWIZZLE))
        return cudaErrorInvalidValue;
    }
  }
  const long long units = tiles * splits;
  const int grid = (int)(units < sm_count() ? units : sm_count());
  if (grid <= 0) return cudaSuccess;
  const cudaError_t el = launch_pdl(kern, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM_BYTES, st, ta, tb, tc, g.C2,
                                    g.ldc2, g.c2_cols, g.M, g.N, g.K, g.len, g.L, g.err, splits);
  if (el != cudaSuccess) return el;
  cudaError_t e2 = cudaPeekAtLastError();
  if (e2 != cudaSuccess || splits == 1 || g.keep_partials) return e2;
  if (((g.N | g.ldc) & 3) == 0 && ((reinterpret_cast<uintptr_t>(g.partial) | reinterpret_cast<uintptr_t>(g.C)) & 15) == 0) {
    const long long n = (long long)g.M * (g.N / 4);
    const cudaError_t es = launch_pdl(splitk_sum4_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st,
                                      (const float*)g.partial, splits, (long long)(num_m * Cfg::BM), g.N,
                                      reinterpret_cast<float*>(g.C), g.ldc, g.C2, g.ldc2, g.c2_cols, g.M, g.len, g.L);
    if (es != cudaSuccess) return es;
  } else {
    const cudaError_t es = launch_pdl(splitk_sum_kernel, dim3((unsigned)g.M), dim3(128), 0, st,
                                      (const float*)g.partial, splits, (long long)(num_m * Cfg::BM), g.N,
                                      reinterpret_cast<float*>(g.C), g.ldc, g.C2, g.ldc2, g.c2_cols, g.M, g.len, g.L);
    if (es != cudaSuccess) return es;
  }
  return cudaPeekAtLastError();
}

template <typename TOut>
cudaError_t dispatch(const TcGemm& g, cudaStream_t st) {
  // widest tile that divides N; else the narrowest that covers it; else 256 with a ragged edge
  if (g.N % 256 == 0) {
    // 256 × 256 tiles when there are enough of them for three SMs in four: one
    // wave of them beats 1.7 waves of 128 × 256 tiles (M = 1024, N = 8192).  Not
    // for ragged rows: a 256-row tile ending a sequence computes up to 255
    // padding rows (B = 256 × 512, lengths U[64, 512]: 40 % of the rows computed
    // against 20 % with 128-row tiles, 6.31 → 6.01 ms per forward)
    if constexpr (std::is_same<TOut, bf16>::value)
      if (R2L_GEMM_MB2 && !g.ragged && g.K >= R2L_GEMM_MB2_MIN_K &&
          (long long)((g.M + 255) / 256) * (g.N / 256) * 4 >= (long long)sm_count() * 3)
        return launch<256, TOut, 2>(g, st);
    // fewer 128 × 256 tiles than SMs: 128-wide tiles give twice as many
    if ((long long)((g.M + 127) / 128) * (g.N / 256) < sm_count()) return launch<128, TOut>(g, st);
    return launch<256, TOut>(g, st);
  }
  if (g.N <= 64) return launch<64, TOut>(g, st);
  if (g.N <= 128) return launch<128, TOut>(g, st);
  if (g.N <= 160) return launch<160, TOut>(g, st);
  if (g.N % 128 == 0) return launch<128, TOut>(g, st);
  return launch<256, TOut>(g, st);
}

// fp32-output GEMMs with MN-major operands (the weight gradients): the tile
// width as dispatch() picks it, in whole 64-column boxes when B is MN-major.
template <int AMN, int BMN>
cudaError_t dispatch_mn(const TcGemm& g, cudaStream_t st) {
  if (g.N % 256 == 0) {
    if ((long long)((g.M + 127) / 128) * (g.N / 256) < sm_count()) return launch<128, float, 1, AMN, BMN>(g, st);
    return launch<256, float, 1, AMN, BMN>(g, st);
  }
  if (g.N <= 64) return launch<64, float, 1, AMN, BMN>(g, st);
  if (g.N <= 128) return launch<128, float, 1, AMN, BMN>(g, st);
  if constexpr (!BMN)
    if (g.N <= 160) return launch<160, float, 1, AMN, BMN>(g, st);
  if (g.N % 128 == 0) return launch<128, float, 1, AMN, BMN>(g, st);
  return launch<256, float, 1, AMN, BMN>(g, st);
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
  const cudaError_t el = launch_pdl(kern, dim3(grid), dim3(cx::THREADS), cx::SMEM_BYTES, st, tx, tb, tc, tw4, tcb, a);
  if (el != cudaSuccess) return el;
  return cudaPeekAtLastError();
}

}  // namespace

size_t tc_gemm_partial_bytes(long long M, int N, int K) {
  const int BN = tile_width(N);
  const long long num_m = (M + 127) / 128;
  const int sp = choose_splits(num_m * ((N + BN - 1) / BN), (K + 63) / 64);
  return sp > 1 ? (size_t)sp * num_m * 128 * N * sizeof(float) : 0;
}

bool convx_supported(int N, int E) { return N == convx::BN && E > 0 && E % convx::BK == 0; }

bool convx_worthwhile(long long M) { return (M + convx::BM - 1) / convx::BM >= sm_count(); }

cudaError_t convx_gemm(const ConvX& g, cudaStream_t st) {
  if (g.M <= 0) return cudaSuccess;
  if (!convx_supported(160, g.E) || (g.ldx % 8) || (g.ldu % 2) || (g.ldc * 4) % 16) return cudaErrorInvalidValue;
  return g.fwd ? launch_convx<true>(g, st) : launch_convx<false>(g, st);
}

cudaError_t tc_gemm(const TcGemm& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return cudaSuccess;
  // TMA: 16-byte row strides; a K-major operand's K is its inner extent
  if ((g.lda % 8) || (g.ldb % 8) || (!g.a_mn && (g.K % 8))) return cudaErrorInvalidValue;
  if (g.keep_partials) {
    if (!g.c_fp32 || g.a_mn || g.b_mn || g.C2) return cudaErrorInvalidValue;
    return launch<256, float>(g, st);
  }
  if ((g.ldc * (g.c_fp32 ? 4 : 2)) % 16) return cudaErrorInvalidValue;
  if (g.a_mn || g.b_mn) {
    if (!g.c_fp32 || !g.a_mn || g.C2) return cudaErrorInvalidValue;
    return g.b_mn ? dispatch_mn<1, 1>(g, st) : dispatch_mn<1, 0>(g, st);
  }
  return g.c_fp32 ? dispatch<float>(g, st) : dispatch<bf16>(g, st);
}

}  // namespace r2l
