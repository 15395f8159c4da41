// Anti-causal depthwise conv (width 4) + SiLU for the bf16 path:
//   u[i, c] = SiLU(conv_b[c] + Σ_{k=0..3} conv_w[c, 3-k] · x[i+k, c]),   x[j] = 0 for j ≥ len
// ("Bifocal Diffusion Language Models", arXiv 2606.27732v1, §3.4 steps ❶–❷:
// the Mamba-1 causal conv seen through the flip).  One thread covers 8
// channels (16-byte loads and stores) × CT consecutive tokens and keeps the
// CT + 3 input rows it needs in registers (as packed bf16, unpacked per use),
// all requested before the first output is computed.
#pragma once

#include "common.cuh"

namespace r2l {
namespace conv {

constexpr int CT = 16;       // tokens per thread
constexpr int THREADS = 128;

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 t = __bfloat1622float2(p[q]);
    f[2 * q] = t.x;
    f[2 * q + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 v;
  uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * q], f[2 * q + 1]);
    w[q] = *reinterpret_cast<uint32_t*>(&t);
  }
  return v;
}

// SiLU(v) = v / (1 + e^{-v}) with the hardware exponential and division
// (relative error ~1e-6, far below the bf16 rounding of u).
__device__ __forceinline__ float silu_hw(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// x: row stride ldx (elements, multiple of 8); u: [B·L, E].  E % 8 == 0.
// FWD: the causal conv of the left-to-right block (taps on x[i-k], x[j<0] = 0).
template <bool FWD>
__global__ void __launch_bounds__(THREADS)
conv_silu_bf16_kernel(const bf16* __restrict__ x, int ldx, bf16* __restrict__ u, int E,
                      const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                      const int* __restrict__ len, int L) {
  const int cg = blockIdx.x * THREADS + threadIdx.x;
  const int c0 = cg * 8;
  const int t0 = blockIdx.y * CT;
  const int b = blockIdx.z;
  const int n = len[b];
  if (c0 >= E || t0 >= n) return;
  float w[8][4], bias[8];
  {
    const float4* wp = reinterpret_cast<const float4*>(conv_w + (long long)c0 * 4);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const float4 t = wp[ch];
      w[ch][0] = t.x; w[ch][1] = t.y; w[ch][2] = t.z; w[ch][3] = t.w;
    }
    const float4* bp = reinterpret_cast<const float4*>(conv_b + c0);
    const float4 b0 = bp[0], b1 = bp[1];
    bias[0] = b0.x; bias[1] = b0.y; bias[2] = b0.z; bias[3] = b0.w;
    bias[4] = b1.x; bias[5] = b1.y; bias[6] = b1.z; bias[7] = b1.w;
  }
  const long long row0 = (long long)b * L + t0;
  // window rows: token t0 + r (reverse block) or t0 - 3 + r (forward block)
  const int first = FWD ? t0 - 3 : t0;
  uint4 xr[CT + 3];
#pragma unroll
  for (int r = 0; r < CT + 3; ++r) {
    const int tok = first + r;
    xr[r] = (tok >= 0 && tok < n) ? *reinterpret_cast<const uint4*>(x + ((long long)b * L + tok) * ldx + c0)
                                  : make_uint4(0u, 0u, 0u, 0u);
  }
  // rolling window of 4 unpacked rows: win[k] holds window row t + k
  float win[4][8];
#pragma unroll
  for (int k = 0; k < 3; ++k) unpack8(xr[k], win[k]);
#pragma unroll
  for (int t = 0; t < CT; ++t) {
    unpack8(xr[t + 3], win[(t + 3) & 3]);
    if (t0 + t >= n) break;
    float o[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      float acc = bias[ch];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc = fmaf(w[ch][3 - k], win[((FWD ? 3 - k : k) + t) & 3][ch], acc);
      o[ch] = silu_hw(acc);
    }
    *reinterpret_cast<uint4*>(u + (row0 + t) * E + c0) = pack8(o);
  }
}

}  // namespace conv
}  // namespace r2l
