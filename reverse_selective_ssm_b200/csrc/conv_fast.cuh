// Anti-causal depthwise conv (width 4) + SiLU for the bf16 path:
//   u[i, c] = SiLU(conv_b[c] + Σ_{k=0..3} conv_w[c, 3-k] · x[i+k, c]),   x[j] = 0 for j ≥ len
// ("Bifocal Diffusion Language Models", arXiv 2606.27732v1, §3.4 steps ❶–❷:
// the Mamba-1 causal conv seen through the flip).  One thread covers 8
// channels (16-byte loads and stores) × NT consecutive tokens and keeps the
// NT + 3 input rows it needs in registers (as packed bf16, unpacked per use),
// all requested before the first output is computed.  NT = 16, or 8 when 16
// would give fewer than two blocks per SM (a denoising block of 1024 tokens:
// 512 blocks instead of 256 spread the work over the SMs more evenly).
#pragma once

#include "common.cuh"

namespace r2l {
namespace conv {

constexpr int THREADS = 128;

// Tokens per thread for a grid over B sequences of L tokens and E channels.
inline int tokens_per_thread(int B, int L, int E, int sms) {
  const long long blocks16 = (long long)((E / 8 + THREADS - 1) / THREADS) * ((L + 15) / 16) * B;
  return blocks16 < 2LL * sms ? 8 : 16;
}

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

__device__ __forceinline__ float ex2_hw(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_hw(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The same on a pair of channels: packed f32x2 multiply-adds around two
// hardware exponentials (e^{-v} = 2^{-v·log2 e}) and reciprocals.
__device__ __forceinline__ float2 silu_hw2(float2 v) {
  const float2 t = __fmul2_rn(v, make_float2(-1.4426950408889634f, -1.4426950408889634f));
  const float2 den = __fadd2_rn(make_float2(ex2_hw(t.x), ex2_hw(t.y)), make_float2(1.0f, 1.0f));
  return __fmul2_rn(v, make_float2(rcp_hw(den.x), rcp_hw(den.y)));
}

// bf16x2 word → (low, high) as floats: the bf16 bits are the top half of the fp32.
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// x: row stride ldx (elements, multiple of 8); u: [B·L, E].  E % 8 == 0.
// FWD: the causal conv of the left-to-right block (taps on x[i-k], x[j<0] = 0).
template <bool FWD, int NT>
__global__ void __launch_bounds__(THREADS)
conv_silu_bf16_kernel(const bf16* __restrict__ x, int ldx, bf16* __restrict__ u, int E,
                      const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                      const int* __restrict__ len, int L) {
  grid_dep_wait();
  grid_dep_launch();
  const int cg = blockIdx.x * THREADS + threadIdx.x;
  const int c0 = cg * 8;
  const int t0 = blockIdx.y * NT;
  const int b = blockIdx.z;
  const int n = len[b];
  if (c0 >= E || t0 >= n) return;
  // taps and bias of the thread's 8 channels as 4 channel pairs: w2[p][k] = (w[2p][k], w[2p+1][k])
  float2 w2[4][4], bias2[4];
  {
    const float4* wp = reinterpret_cast<const float4*>(conv_w + (long long)c0 * 4);
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) {
      const float4 a = wp[2 * pp], b = wp[2 * pp + 1];
      w2[pp][0] = make_float2(a.x, b.x); w2[pp][1] = make_float2(a.y, b.y);
      w2[pp][2] = make_float2(a.z, b.z); w2[pp][3] = make_float2(a.w, b.w);
    }
    const float4* bp = reinterpret_cast<const float4*>(conv_b + c0);
    const float4 b0 = bp[0], b1 = bp[1];
    bias2[0] = make_float2(b0.x, b0.y); bias2[1] = make_float2(b0.z, b0.w);
    bias2[2] = make_float2(b1.x, b1.y); bias2[3] = make_float2(b1.z, b1.w);
  }
  const long long row0 = (long long)b * L + t0;
  // window rows: token t0 + r (reverse block) or t0 - 3 + r (forward block)
  const int first = FWD ? t0 - 3 : t0;
  uint4 xr[NT + 3];
#pragma unroll
  for (int r = 0; r < NT + 3; ++r) {
    const int tok = first + r;
    xr[r] = (tok >= 0 && tok < n) ? *reinterpret_cast<const uint4*>(x + ((long long)b * L + tok) * ldx + c0)
                                  : make_uint4(0u, 0u, 0u, 0u);
  }
  // rolling window of 4 unpacked rows as channel pairs: win[k & 3] holds window row k
  float2 win[4][4];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    win[k][0] = bf2_to_f2(xr[k].x); win[k][1] = bf2_to_f2(xr[k].y);
    win[k][2] = bf2_to_f2(xr[k].z); win[k][3] = bf2_to_f2(xr[k].w);
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    {
      const int r = (t + 3) & 3;
      win[r][0] = bf2_to_f2(xr[t + 3].x); win[r][1] = bf2_to_f2(xr[t + 3].y);
      win[r][2] = bf2_to_f2(xr[t + 3].z); win[r][3] = bf2_to_f2(xr[t + 3].w);
    }
    if (t0 + t >= n) break;
    uint4 packed;
    uint32_t* pw = reinterpret_cast<uint32_t*>(&packed);
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) {
      float2 acc = bias2[pp];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc = __ffma2_rn(w2[pp][3 - k], win[((FWD ? 3 - k : k) + t) & 3][pp], acc);
      const float2 o = silu_hw2(acc);
      __nv_bfloat162 ob = __floats2bfloat162_rn(o.x, o.y);
      pw[pp] = *reinterpret_cast<uint32_t*>(&ob);
    }
    *reinterpret_cast<uint4*>(u + (row0 + t) * E + c0) = packed;
  }
}

}  // namespace conv
}  // namespace r2l
