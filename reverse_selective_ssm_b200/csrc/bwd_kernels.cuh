// Device kernels of the sidecar hook's gradient (r2l_sidecar_backward), other
// than the GEMMs (tcgen05, gemm_tc.cuh) and the scan's own gradient
// (scan_bwd.cu).  The chain rule of one hook of "Bifocal Diffusion Language
// Models" (arXiv 2606.27732v1, §3.4 steps ❶–❹), taken in reverse order:
//
//   ❹ gate:      ĝ = tanh(s)·dh⁺,  ds = (1 − tanh²(s))·Σ dh⁺ ⊙ ĥ
//   ❸ LayerNorm: n̂ = (o − μ)·rstd,  dγ = Σ ĝ ⊙ n̂,  dβ = Σ ĝ,
//                do = rstd·(γĝ − mean(γĝ) − n̂·mean(γĝ ⊙ n̂))   (per row)
//   conv+SiLU:   dpre = du ⊙ SiLU'(pre),  dx_j = Σ_k w[W−1−k]·dpre_{j−k},
//                dw[W−1−k] = Σ_i dpre_i·x_{i+k},  db = Σ_i dpre_i
//
// Every sum over positions runs in a fixed order (per-chunk partial sums, then
// the chunks in order), so the gradients are bitwise reproducible.  Rows of
// padding (position ≥ the sequence's length) contribute nothing.
#pragma once

#include "common.cuh"

namespace r2l {
namespace bwd {

constexpr int ROW_CHUNK = 64;      // positions per partial sum of a column reduction

__device__ __forceinline__ bool valid_row(const int* len, int L, long long m) {
  return len == nullptr || row_valid(len, L, m);
}

// out[c, m] = bf16(in[m, c]) for the valid rows m < M, 0 for padding rows and
// for m in [M, Mp) (Mp = the leading dimension of out, a multiple of 8).  A
// 32 × 32 tile per block through shared memory: reads and writes coalesced.
template <typename TIn>
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const TIn* __restrict__ in, long long ld_in, int M, int C,
                                                             bf16* __restrict__ out, long long ld_out,
                                                             const int* __restrict__ len, int L) {
  __shared__ float tile[32][33];
  const int c0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 × 8
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const long long m = m0 + r;
    const int c = c0 + tx;
    float v = 0.0f;
    if (m < M && c < C && valid_row(len, L, m)) v = to_f32(in[m * ld_in + c]);
    tile[r][tx] = v;
  }
  __syncthreads();
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int c = c0 + r;
    const long long m = m0 + tx;
    if (c < C && m < ld_out) out[(long long)c * ld_out + m] = __float2bfloat16_rn(tile[tx][r]);
  }
}

// out[m, c] = bf16(in[m, c]) on valid rows, 0 on padding rows (m < M, c < C).
template <typename TIn>
__global__ void to_bf16_rows_kernel(const TIn* __restrict__ in, long long ld_in, int M, int C, bf16* __restrict__ out,
                                    long long ld_out, const int* __restrict__ len, int L) {
  const long long total = (long long)M * C;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long m = t / C;
    const int c = (int)(t - m * C);
    const float v = valid_row(len, L, m) ? to_f32(in[m * ld_in + c]) : 0.0f;
    out[m * ld_out + c] = __float2bfloat16_rn(v);
  }
}

// ❹ + ❸ per row (one warp per row): the row's LayerNorm statistics (kept for
// the column sums), its share of Σ dh⁺ ⊙ ĥ, and do (bf16, 0 on padding rows).
// Without LayerNorm, ĥ = o and do = ĝ.
template <bool HAS_LN>
__global__ void __launch_bounds__(256) ln_gate_bwd_rows_kernel(const bf16* __restrict__ o, const float* __restrict__ dh_out,
                                                               const float* __restrict__ gamma,
                                                               const float* __restrict__ beta, float g, int d,
                                                               const int* __restrict__ len, int L, long long M,
                                                               float2* __restrict__ stats, float* __restrict__ ds_row,
                                                               bf16* __restrict__ dout) {
  const long long m = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const bf16* orow = o + m * d;
  const float* grow = dh_out + m * d;
  bf16* drow = dout + m * d;
  if (!valid_row(len, L, m)) {
    for (int j = lane; j < d; j += 32) drow[j] = __float2bfloat16_rn(0.0f);
    if (lane == 0) {
      ds_row[m] = 0.0f;
      stats[m] = make_float2(0.0f, 0.0f);
    }
    return;
  }
  float mu = 0.0f, rstd = 1.0f;
  if (HAS_LN) {
    float s = 0.0f;
    for (int j = lane; j < d; j += 32) s += __bfloat162float(orow[j]);
#pragma unroll
    for (int k = 16; k; k >>= 1) s += __shfl_xor_sync(0xffffffffu, s, k);
    mu = s / (float)d;
    float q = 0.0f;
    for (int j = lane; j < d; j += 32) {
      const float t = __bfloat162float(orow[j]) - mu;
      q += t * t;
    }
#pragma unroll
    for (int k = 16; k; k >>= 1) q += __shfl_xor_sync(0xffffffffu, q, k);
    rstd = rsqrtf(q / (float)d + 1e-5f);
  }
  // Σ dh⁺ ⊙ ĥ, Σ γĝ and Σ γĝ ⊙ n̂ over the row
  float sh = 0.0f, s1 = 0.0f, s2 = 0.0f;
  for (int j = lane; j < d; j += 32) {
    const float ov = __bfloat162float(orow[j]);
    const float gv = grow[j];
    if (HAS_LN) {
      const float nh = (ov - mu) * rstd;
      sh += gv * (gamma[j] * nh + beta[j]);
      const float gg = g * gv * gamma[j];
      s1 += gg;
      s2 += gg * nh;
    } else {
      sh += gv * ov;
    }
  }
#pragma unroll
  for (int k = 16; k; k >>= 1) {
    sh += __shfl_xor_sync(0xffffffffu, sh, k);
    s1 += __shfl_xor_sync(0xffffffffu, s1, k);
    s2 += __shfl_xor_sync(0xffffffffu, s2, k);
  }
  const float m1 = s1 / (float)d, m2 = s2 / (float)d;
  for (int j = lane; j < d; j += 32) {
    const float gv = g * grow[j];
    float dv;
    if (HAS_LN) {
      const float nh = (__bfloat162float(orow[j]) - mu) * rstd;
      dv = rstd * (gamma[j] * gv - m1 - nh * m2);
    } else {
      dv = gv;
    }
    drow[j] = __float2bfloat16_rn(dv);
  }
  if (lane == 0) {
    ds_row[m] = sh;
    stats[m] = make_float2(mu, rstd);
  }
}

// ❸ column sums, chunk y of ROW_CHUNK rows: dγ and dβ partials
// part[y][0][j] = Σ ĝ ⊙ n̂, part[y][1][j] = Σ ĝ over the chunk's valid rows.
__global__ void ln_bwd_cols_kernel(const bf16* __restrict__ o, const float* __restrict__ dh_out, float g, int d,
                                   const int* __restrict__ len, int L, long long M, const float2* __restrict__ stats,
                                   float* __restrict__ part) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  const long long r0 = (long long)blockIdx.y * ROW_CHUNK;
  const long long r1 = r0 + ROW_CHUNK < M ? r0 + ROW_CHUNK : M;
  float a = 0.0f, bsum = 0.0f;
  for (long long m = r0; m < r1; ++m) {
    if (!valid_row(len, L, m)) continue;
    const float2 st = stats[m];
    const float gv = g * dh_out[m * d + j];
    a += gv * (__bfloat162float(o[m * d + j]) - st.x) * st.y;
    bsum += gv;
  }
  part[((long long)blockIdx.y * 2 + 0) * d + j] = a;
  part[((long long)blockIdx.y * 2 + 1) * d + j] = bsum;
}

// out[c] = scale · Σ_p part[p·stride + c], p = 0, 1, … in order.
__global__ void colsum_kernel(const float* __restrict__ part, int nparts, long long stride, int C, float scale,
                              float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  float s = 0.0f;
  for (int p = 0; p < nparts; ++p) s += part[p * stride + c];
  out[c] = scale * s;
}

// *out = scale · Σ_m v[m] over m = 0 … n − 1: one block, fixed order (each
// thread a strided partial, then a fixed tree).
__global__ void __launch_bounds__(1024) sum_kernel(const float* __restrict__ v, long long n, float scale,
                                                   float* __restrict__ out) {
  __shared__ float sh[1024];
  float s = 0.0f;
  for (long long i = threadIdx.x; i < n; i += 1024) s += v[i];
  sh[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w; w >>= 1) {
    if ((int)threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = scale * sh[0];
}

// conv + SiLU, step 1: dpre[m, c] = (du_s + du_x)[m, c] · SiLU'(pre[m, c]) on
// valid rows (0 on padding), with pre = conv_b + Σ_k w[W−1−k]·x_{i+k} (x_j = 0
// for j ≥ len_b) recomputed from x.
__global__ void conv_silu_bwd_pre_kernel(const bf16* __restrict__ x, long long ldx, const float* __restrict__ conv_w,
                                         const float* __restrict__ conv_b, const float* __restrict__ du_s,
                                         const float* __restrict__ du_x, int E, const int* __restrict__ len, int L,
                                         long long M, float* __restrict__ dpre) {
  const long long total = M * E;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long m = t / E;
    const int c = (int)(t - m * E);
    const long long b = m / L;
    const int i = (int)(m - b * L);
    const int n = len ? len[b] : L;
    float dv = 0.0f;
    if (i < n) {
      float pre = conv_b[c];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (i + k < n) pre += conv_w[c * 4 + 3 - k] * __bfloat162float(x[(m + k) * ldx + c]);
      const float sg = 1.0f / (1.0f + expf(-pre));
      dv = (du_s[t] + du_x[t]) * sg * (1.0f + pre * (1.0f - sg));
    }
    dpre[t] = dv;
  }
}

// conv + SiLU, step 2: dx_j = Σ_k w[W−1−k]·dpre_{j−k} (k ≤ j), as bf16 into
// dxz (columns 0 … E−1; 0 on padding rows).
__global__ void conv_bwd_dx_kernel(const float* __restrict__ dpre, const float* __restrict__ conv_w, int E,
                                   const int* __restrict__ len, int L, long long M, bf16* __restrict__ dxz,
                                   long long lddxz) {
  const long long total = M * E;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long m = t / E;
    const int c = (int)(t - m * E);
    const long long b = m / L;
    const int j = (int)(m - b * L);
    const int n = len ? len[b] : L;
    float v = 0.0f;
    if (j < n) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (j - k >= 0) v += conv_w[c * 4 + 3 - k] * dpre[(m - k) * E + c];
    }
    dxz[m * lddxz + c] = __float2bfloat16_rn(v);
  }
}

// conv + SiLU, step 3, chunk y of ROW_CHUNK rows: parameter partials
// part[y][k][c] = Σ_i dpre_i·x_{i+k} (k = 0..3, the tap w[W−1−k]; x_j = 0 for
// j ≥ len_b) and part[y][4][c] = Σ_i dpre_i.
__global__ void conv_bwd_params_kernel(const float* __restrict__ dpre, const bf16* __restrict__ x, long long ldx,
                                       int E, const int* __restrict__ len, int L, long long M,
                                       float* __restrict__ part) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= E) return;
  const long long r0 = (long long)blockIdx.y * ROW_CHUNK;
  const long long r1 = r0 + ROW_CHUNK < M ? r0 + ROW_CHUNK : M;
  float s[5] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  for (long long m = r0; m < r1; ++m) {
    const long long b = m / L;
    const int i = (int)(m - b * L);
    const int n = len ? len[b] : L;
    if (i >= n) continue;
    const float dv = dpre[m * E + c];
    s[4] += dv;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (i + k < n) s[k] += dv * __bfloat162float(x[(m + k) * ldx + c]);
  }
#pragma unroll
  for (int k = 0; k < 5; ++k) part[((long long)blockIdx.y * 5 + k) * E + c] = s[k];
}

// dconv_w[c][W−1−k] and dconv_b[c] from the chunk partials, chunks in order.
__global__ void conv_bwd_reduce_kernel(const float* __restrict__ part, int nchunks, int E, float* __restrict__ dconv_w,
                                       float* __restrict__ dconv_b) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= E) return;
  float s[5] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  for (int y = 0; y < nchunks; ++y)
#pragma unroll
    for (int k = 0; k < 5; ++k) s[k] += part[((long long)y * 5 + k) * E + c];
#pragma unroll
  for (int k = 0; k < 4; ++k) dconv_w[c * 4 + 3 - k] = s[k];
  dconv_b[c] = s[4];
}

// dh = dh⁺ + tmp on valid rows, dh⁺ on padding rows (the hook neither reads
// nor writes them).
__global__ void add_rows_kernel(const float* __restrict__ dh_out, const float* __restrict__ tmp, int d,
                                const int* __restrict__ len, int L, long long M, float* __restrict__ dh) {
  const long long total = M * d;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long m = t / d;
    dh[t] = valid_row(len, L, m) ? dh_out[t] + tmp[t] : dh_out[t];
  }
}

}  // namespace bwd
}  // namespace r2l
