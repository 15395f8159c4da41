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
// The scan's power path: when A is the S4D-real initialisation A[c][m] =
// −(m+1), the 16 decays of a (token, channel) are the powers r, r², …, r¹⁶ of
// r = e^{−Δ}, and no per-state exponential is needed.  The path is decided once
// per call, exactly: it is taken when every A_log[c][m] equals, bit for bit,
// ln_bits[m] (the float nearest ln(m+1), computed on the host), and then the
// scan uses A_m = −(m+1) exactly.  One block reads all E·16 entries and
// writes 0 (power path) or 1 (general path) to *general for every later
// kernel of the call to read.
// ---------------------------------------------------------------------------
struct LnTable {
  uint32_t bits[16];
};

// The A_log arrays of up to kMaxCheckedHooks hooks, checked by one launch
// (block k checks hook k and writes general[k]).
constexpr int kMaxCheckedHooks = 64;
struct ALogSet {
  const float* a[kMaxCheckedHooks];
};

__global__ void __launch_bounds__(1024)
a_log_check_kernel(const __grid_constant__ ALogSet set, int E, const __grid_constant__ LnTable tab,
                   unsigned* __restrict__ general) {
  // A_log is [E, 16] and 16-byte aligned: thread t reads uint4 number t +
  // 1024·k, whose four entries are states 4·(t mod 4) … 4·(t mod 4) + 3;
  // eight independent loads per thread are in flight at a time
  const uint4* a4 = reinterpret_cast<const uint4*>(set.a[blockIdx.x]);
  const int m0 = (threadIdx.x & 3) * 4;
  const uint32_t t0 = tab.bits[m0], t1 = tab.bits[m0 + 1], t2 = tab.bits[m0 + 2], t3 = tab.bits[m0 + 3];
  const int n4 = E * 4;
  constexpr int U = 8;                 // loads in flight per thread
  int bad = 0;
  for (int base = threadIdx.x; base < n4; base += U * blockDim.x) {
    uint4 v[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int i = base + k * blockDim.x;
      v[k] = i < n4 ? a4[i] : make_uint4(t0, t1, t2, t3);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) bad |= (v[k].x != t0) | (v[k].y != t1) | (v[k].z != t2) | (v[k].w != t3);
  }
  bad = __syncthreads_or(bad);
  if (threadIdx.x == 0) general[blockIdx.x] = bad ? 1u : 0u;
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
// fwd = true: the causal conv of the left-to-right block instead,
//   u[i, c] = SiLU(conv_b[c] + Σ_{k=0..3} conv_w[c, 3-k] · x[i-k, c]),  x[j] = 0 for j < 0.
template <typename T>
__global__ void conv_silu_kernel(const T* __restrict__ x, int ldx, T* __restrict__ u, int E,
                                 const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                                 const int* __restrict__ len, int L, bool fwd) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int i = blockIdx.y;
  const int b = blockIdx.z;
  const int n = len[b];
  if (c >= E || i >= n) return;
  const long long row = (long long)b * L + i;
  float acc = conv_b[c];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = fwd ? i - k : i + k;
    if (j >= 0 && j < n) acc = fmaf(conv_w[c * 4 + 3 - k], to_f32(x[((long long)b * L + j) * ldx + c]), acc);
  }
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

// ---------------------------------------------------------------------------
// bf16 path of the LayerNorm + gated residual: one warp per valid row, 16-byte
// accesses, the row of o held in registers (NV chunks of 8 per lane, so
// d ≤ 256·NV) for a two-pass mean / variance without re-reading memory.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// SPLIT: o arrives as `splits` fp32 partial sums P[s][row][col] (slices of
// `slice` floats, the K-split out_proj of a small batch); the row's o is their
// sum in split order rounded to bf16, the value the unsplit GEMM would have
// stored up to the order of its fp32 additions, and it is written to o_out
// when that is set.
template <int NV, bool HAS_LN, bool SPLIT = false>
__global__ void __launch_bounds__(128)
ln_residual_bf16_kernel(bf16* __restrict__ h, const bf16* __restrict__ o, const float* __restrict__ ln_w,
                        const float* __restrict__ ln_b, float g, int d, const int* __restrict__ len, int L,
                        long long M, float* __restrict__ hhat_out, const float* __restrict__ P = nullptr,
                        int splits = 0, long long slice = 0, bf16* __restrict__ o_out = nullptr) {
  grid_dep_wait();
  grid_dep_launch();
  const long long row = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const long long b = row / L;
  if ((int)(row - b * L) >= len[b]) return;
  const bf16* orow = o + row * d;
  bf16* hrow = h + row * d;
  // both rows are requested before any arithmetic, so a warp keeps 8 KB in flight
  uint4 oraw[NV], hraw_all[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int col = (k * 32 + lane) * 8;
    if (col < d) {
      if (!SPLIT) oraw[k] = *reinterpret_cast<const uint4*>(orow + col);
      hraw_all[k] = *reinterpret_cast<const uint4*>(hrow + col);
    }
  }
  float v[NV][8];
  if (SPLIT) {
    // slice by slice, all of a slice's loads of the row in flight at once
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
      for (int q = 0; q < 8; ++q) v[k][q] = 0.0f;
    for (int sp = 0; sp < splits; ++sp) {
      const float* prow = P + sp * slice + row * d;
      float4 pr[NV][2];
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int col = (k * 32 + lane) * 8;
        if (col < d) {
          pr[k][0] = *reinterpret_cast<const float4*>(prow + col);
          pr[k][1] = *reinterpret_cast<const float4*>(prow + col + 4);
        }
      }
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int col = (k * 32 + lane) * 8;
        if (col < d) {
          v[k][0] += pr[k][0].x; v[k][1] += pr[k][0].y; v[k][2] += pr[k][0].z; v[k][3] += pr[k][0].w;
          v[k][4] += pr[k][1].x; v[k][5] += pr[k][1].y; v[k][6] += pr[k][1].z; v[k][7] += pr[k][1].w;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int col = (k * 32 + lane) * 8;
      if (col < d) {
        __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&oraw[k]);
#pragma unroll
        for (int q = 0; q < 4; ++q) o2[q] = __floats2bfloat162_rn(v[k][2 * q], v[k][2 * q + 1]);
        if (o_out) *reinterpret_cast<uint4*>(o_out + row * d + col) = oraw[k];
      }
    }
  }
  float s = 0.0f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int col = (k * 32 + lane) * 8;
    if (col < d) {
      const uint4 raw = oraw[k];
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(p2[q]);
        v[k][2 * q] = f.x;
        v[k][2 * q + 1] = f.y;
        s += f.x + f.y;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[k][q] = 0.0f;
    }
  }
  float mean = 0.0f, rstd = 1.0f;
  if (HAS_LN) {
    mean = warp_sum(s) / (float)d;
    float q2 = 0.0f;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int col = (k * 32 + lane) * 8;
      if (col < d) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float t = v[k][q] - mean;
          q2 = fmaf(t, t, q2);
        }
      }
    }
    rstd = rsqrtf(warp_sum(q2) / (float)d + 1e-5f);
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int col = (k * 32 + lane) * 8;
    if (col >= d) continue;
    float hv[8];
    if (HAS_LN) {
      const float4 w0 = *reinterpret_cast<const float4*>(ln_w + col);
      const float4 w1 = *reinterpret_cast<const float4*>(ln_w + col + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(ln_b + col);
      const float4 b1 = *reinterpret_cast<const float4*>(ln_b + col + 4);
      const float gw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      const float gb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) hv[q] = fmaf((v[k][q] - mean) * rstd, gw[q], gb[q]);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) hv[q] = v[k][q];
    }
    if (hhat_out) {
      float4* dst = reinterpret_cast<float4*>(hhat_out + row * d + col);
      dst[0] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      dst[1] = make_float4(hv[4], hv[5], hv[6], hv[7]);
    }
    uint4 hraw = hraw_all[k];
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&hraw);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(h2[q]);
      h2[q] = __floats2bfloat162_rn(fmaf(g, hv[2 * q], f.x), fmaf(g, hv[2 * q + 1], f.y));
    }
    *reinterpret_cast<uint4*>(hrow + col) = hraw;
  }
}

}  // namespace r2l
