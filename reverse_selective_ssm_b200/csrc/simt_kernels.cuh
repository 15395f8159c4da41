// SIMT kernels of the R2L sidecar: the fp32 GEMM path (true fp32, no TF32),
// length preparation, the anti-causal conv + SiLU, and the LayerNorm + tanh(s)
// gated residual epilogue.
//
// Layer: "Bifocal Diffusion Language Models" (arXiv 2606.27732v1), §3.4 steps
// ❶–❹; Mamba-1 block internals per step ❷ (d_conv = 4, §4.1).
#pragma once

#include "common.cuh"

namespace r2l {

// ---------------------------------------------------------------------------
// lengths: clamp to [0, L] into the workspace copy every later kernel reads;
// flag any value that had to be clamped.  lengths == nullptr means all L.
// ---------------------------------------------------------------------------
__global__ void prep_lengths_kernel(const int32_t* __restrict__ lengths, int* __restrict__ len_ws,
                                    int B, int L, unsigned* __restrict__ status) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int v = lengths ? lengths[b] : L;
  if (v < 0 || v > L) {
    atomicOr(status, 1u);
    v = v < 0 ? 0 : L;
  }
  len_ws[b] = v;
}

// ---------------------------------------------------------------------------
// C[m, n] = Σ_k A[m, k] · W[n, k]   (nn.Linear: y = x Wᵀ), fp32 accumulation.
// 64×64 output tile per 256-thread block, 4×4 per thread, BK = 16.  Tiles with
// no valid row (all padding) are skipped; padding rows are never stored.
// ---------------------------------------------------------------------------
template <typename TA, typename TW, typename TC>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(const TA* __restrict__ A, int lda, const TW* __restrict__ W, int ldw,
                 TC* __restrict__ C, int ldc, int M, int N, int K,
                 const int* __restrict__ len, int L) {
  __shared__ float As[16][64 + 4];
  __shared__ float Ws[16][64 + 4];
  const int tid = threadIdx.x;
  const long long m0 = (long long)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  int any = 0;
  if (tid < 64 && m0 + tid < M) any = row_valid(len, L, m0 + tid);
  if (!__syncthreads_or(any)) return;

  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
    for (int e = tid; e < 64 * 16; e += 256) {
      const int rr = e >> 4, kk = e & 15;
      const long long gm = m0 + rr;
      const int gk = k0 + kk;
      As[kk][rr] = (gm < M && gk < K) ? to_f32(A[gm * lda + gk]) : 0.0f;
      const int gn = n0 + rr;
      Ws[kk][rr] = (gn < N && gk < K) ? to_f32(W[(long long)gn * ldw + gk]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long gm = m0 + ty * 4 + i;
    if (gm >= M || !row_valid(len, L, gm)) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn < N) C[gm * ldc + gn] = from_f32<TC>(acc[i][j]);
    }
  }
}

// ---------------------------------------------------------------------------
// Anti-causal depthwise conv (width 4) + SiLU:
//   u[i, c] = SiLU(conv_b[c] + Σ_{k=0..3} conv_w[c, 3-k] · x[i+k, c]),  x[j] = 0 for j ≥ len.
// x is read from the in_proj output (row stride ldx).  One thread per (b, i, c).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void conv_silu_kernel(const T* __restrict__ x, int ldx, T* __restrict__ u, int E,
                                 const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                                 const int* __restrict__ len, int L) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int i = blockIdx.y;
  const int b = blockIdx.z;
  const int n = len[b];
  if (c >= E || i >= n) return;
  const long long row = (long long)b * L + i;
  float acc = conv_b[c];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (i + k < n) acc = fmaf(conv_w[c * 4 + 3 - k], to_f32(x[(row + k) * ldx + c]), acc);
  u[row * E + c] = from_f32<T>(silu_f(acc));
}

// ---------------------------------------------------------------------------
// Block-wide sum over 256 threads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < 8 ? red[lane] : 0.0f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);  // every lane gets the total
  return t;
}

// ---------------------------------------------------------------------------
// Stream-local LayerNorm (§3.4 ❸) and gated residual (§3.4 ❹), one block of 256
// threads per valid row:  h ← RN(h + g · (γ ⊙ (o − μ) / sqrt(σ² + 1e-5) + β)).
// Two-pass mean / variance in fp32.  HAS_LN = false: ĥ = o.
// ---------------------------------------------------------------------------
template <typename T, bool HAS_LN>
__global__ void __launch_bounds__(256)
ln_gate_residual_kernel(T* __restrict__ h, const T* __restrict__ o, const float* __restrict__ ln_w,
                        const float* __restrict__ ln_b, float g, int d,
                        const int* __restrict__ len, int L, float* __restrict__ hhat_out) {
  __shared__ float red[8];
  const long long row = blockIdx.x;
  const long long b = row / L;
  const int i = (int)(row - b * L);
  if (i >= len[b]) return;
  const T* orow = o + row * d;
  T* hrow = h + row * d;
  float mean = 0.0f, rstd = 1.0f;
  if (HAS_LN) {
    float s = 0.0f;
    for (int j = threadIdx.x; j < d; j += 256) s += to_f32(orow[j]);
    mean = block_sum_256(s, red) / (float)d;
    float q = 0.0f;
    for (int j = threadIdx.x; j < d; j += 256) {
      const float t = to_f32(orow[j]) - mean;
      q = fmaf(t, t, q);
    }
    const float var = block_sum_256(q, red) / (float)d;
    rstd = rsqrtf(var + 1e-5f);
  }
  for (int j = threadIdx.x; j < d; j += 256) {
    float v = to_f32(orow[j]);
    if (HAS_LN) v = fmaf((v - mean) * rstd, ln_w[j], ln_b[j]);
    if (hhat_out) hhat_out[row * d + j] = v;
    hrow[j] = from_f32<T>(fmaf(g, v, to_f32(hrow[j])));
  }
}

}  // namespace r2l
