// Host interface of the tcgen05 bf16 GEMM: C[m, n] = Σ_k A[m, k] · B[n, k].
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace r2l {

struct TcGemm {
  const __nv_bfloat16* A;  // [M, K] row stride lda (elements), 16-byte aligned; [K, M] when a_mn
  int lda;
  const __nv_bfloat16* B;  // [N, K] row stride ldb; [K, N] when b_mn
  int ldb;
  // MN-major operands (fp32 C only): A stored [K, M], B stored [K, N], rows of
  // stride lda / ldb.  Supported: a_mn alone, or a_mn with b_mn.
  bool a_mn, b_mn;
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
  float* partial;          // optional scratch for split-K partial sums (fp32 C only), or null
  size_t partial_bytes;
  // keep_partials (fp32 C only): run on 128 × 256 tiles with kept_splits (≥ 1,
  // normally tc_gemm_kept_splits of the shape, decided by the caller so that it
  // and the code adding the slices agree) K splits and leave the partial sums
  // in `partial` as [kept_splits][Mp][N], Mp = M rounded up to 128, for the
  // caller to add in split order; C is not written.
  bool keep_partials;
  int kept_splits;
  // the rows come from sequences of different lengths (right-padded): 128-row
  // tiles, which waste fewer padding rows at each sequence's end than 256-row ones
  bool ragged;
};

// Streaming multiprocessors of the current device (148 on B200).
int sm_count();

// C2[m, c] = bf16(Σ_s P[s·Mp + m, c]) for c < c2_cols on valid rows (and C = the
// fp32 sum, which may be P itself), slices added in split order: the sum a
// keep_partials GEMM leaves to its caller.
cudaError_t tc_gemm_add_partials(const float* P, int splits, long long Mp, int N, float* C, int ldc,
                                 __nv_bfloat16* C2, int ldc2, int c2_cols, int M, const int* len, int L,
                                 cudaStream_t st);

// Splits a keep_partials GEMM of this shape uses: 0 when N is not a multiple
// of 256 or its 128 × 256 tiles alone fill the SMs; else the fewest splits (at
// most 8, each of at least 8 K blocks of 64) that give every SM a unit.
int tc_gemm_kept_splits(long long M, int N, int K);

// Scratch an fp32-output GEMM of this shape uses for split-K partial sums
// (0 when it runs unsplit).  With less, it runs unsplit.
size_t tc_gemm_partial_bytes(long long M, int N, int K);

// Enqueues the GEMM on `st`.  Requires lda, ldb, K to be multiples of 8.
cudaError_t tc_gemm(const TcGemm& g, cudaStream_t st);

// conv + SiLU fused into x_proj (gemm_convx.cuh): u = SiLU(conv(x)) written to
// `u` for the valid rows, and [Δr | B | C] = u·W_xᵀ into C (fp32), Δr also into
// C2 (bf16).  For N = 160 (dt_rank 128, d_state 16) and E a multiple of 64.
struct ConvX {
  const __nv_bfloat16* x;  // [M, E] row stride ldx (the x half of xz)
  long long ldx;
  const float* conv_w;     // [E, 4]
  const float* conv_b;     // [E]
  __nv_bfloat16* u;        // [M, E] row stride ldu
  long long ldu;
  const __nv_bfloat16* W;  // x_proj weight [160, E]
  float* C;                // [M, 160]
  int ldc;
  __nv_bfloat16* C2;       // [M, ldc2], columns < c2_cols
  int ldc2;
  int c2_cols;
  int M, E;
  const int* len;
  int L;
  unsigned* err;
  bool fwd;                // causal conv of the left-to-right block
};

bool convx_supported(int N, int E);
// The fused kernel runs one 128-row tile per CTA at a time; below one tile per
// SM the standalone conv kernel, which spreads over all SMs, is faster.
bool convx_worthwhile(long long M);
cudaError_t convx_gemm(const ConvX& g, cudaStream_t st);

}  // namespace r2l
