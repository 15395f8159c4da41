// Sequential reverse selective scan: one thread per (sequence b, channel c),
// walking i = len_b-1 … 0 (or 0 … len_b-1 for the left-to-right block, fwd)
// with the d_state = 16 state in registers.  Used for
// the fp32 path (config-0 sizes) where parallelism is not the point.
//
// "Bifocal Diffusion Language Models" (arXiv 2606.27732v1), §3.4 step ❷ (the
// Mamba-1 selective scan on the flipped sequence), written in original
// coordinates:
//   Δ_i = softplus(dt_raw_i + dt_b)
//   H_i = exp(Δ_i A) ⊙ H_{i+1} + Δ_i u_i B_i,   H_len = 0
//   y_i = (⟨C_i, H_i⟩ + D u_i) · SiLU(z_i)
#pragma once

#include "common.cuh"

namespace r2l {

template <typename T>
__global__ void scan_simple_kernel(const T* __restrict__ u, const T* __restrict__ z, int ldz,
                                   const T* __restrict__ dt_raw, const float* __restrict__ dbc,
                                   int ldd, int R, const float* __restrict__ A_log,
                                   const float* __restrict__ Dv, const float* __restrict__ dt_b,
                                   T* __restrict__ y, int E, const int* __restrict__ len, int L,
                                   bool fwd) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (c >= E) return;
  const int n = len[b];
  float A[16], H[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    A[m] = -expf(A_log[c * 16 + m]);
    H[m] = 0.0f;
  }
  const float Dc = Dv[c], bc = dt_b[c];
  for (int step = 0; step < n; ++step) {
    const int i = fwd ? step : n - 1 - step;     // fwd: the left-to-right block
    const long long row = (long long)b * L + i;
    const float uu = to_f32(u[row * E + c]);
    const float delta = softplus_f(to_f32(dt_raw[row * E + c]) + bc);
    const float* Bp = dbc + row * ldd + R;
    const float* Cp = Bp + 16;
    const float du = delta * uu;
    float acc = 0.0f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      H[m] = fmaf(expf(delta * A[m]), H[m], du * Bp[m]);
      acc = fmaf(H[m], Cp[m], acc);
    }
    const float zz = to_f32(z[row * ldz + c]);
    y[row * E + c] = from_f32<T>(fmaf(Dc, uu, acc) * silu_f(zz));
  }
}

}  // namespace r2l
