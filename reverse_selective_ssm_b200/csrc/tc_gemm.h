// Host interface of the tcgen05 bf16 GEMM: C[m, n] = Σ_k A[m, k] · B[n, k].
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace r2l {

struct TcGemm {
  const __nv_bfloat16* A;  // [M, K] row stride lda (elements), 16-byte aligned
  int lda;
  const __nv_bfloat16* B;  // [N, K] row stride ldb
  int ldb;
  void* C;                 // [M, N] row stride ldc; bf16, or fp32 when c_fp32
  int ldc;
  bool c_fp32;
  __nv_bfloat16* C2;       // optional bf16 copy of columns < c2_cols (row stride ldc2)
  int ldc2;
  int c2_cols;
  int M, N, K;
  const int* len;          // device lengths [B] (rows i >= len[b] of each sequence are skipped)
  int L;
  unsigned* err;           // device status word (timeout flag)
};

// Enqueues the GEMM on `st`.  Requires lda, ldb, K to be multiples of 8.
cudaError_t tc_gemm(const TcGemm& g, cudaStream_t st);

}  // namespace r2l
