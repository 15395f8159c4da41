// Shared device helpers for libr2l (type conversion, activations, row validity).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace r2l {

typedef __nv_bfloat16 bf16;

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// SiLU(v) = v / (1 + exp(-v)), the Mamba-1 block activation.
__device__ __forceinline__ float silu_f(float v) { return v / (1.0f + expf(-v)); }

// softplus(v) = log(1 + exp(v)), and v itself above 20 (Δ parameterisation).
__device__ __forceinline__ float softplus_f(float v) { return v > 20.0f ? v : log1pf(expf(v)); }

// Programmatic dependent launch.  grid_dep_wait: block until the grids this
// one was launched behind have completed and their writes are visible (it
// returns at once in a grid launched without the programmatic attribute).
// grid_dep_launch: let the next grid of the stream, when launched with the
// attribute, start once every CTA of this grid has issued it or exited.
// A kernel launched with the attribute (launch_pdl.h) calls grid_dep_wait
// before it touches global memory that earlier kernels of the stream write or
// read, and before it allocates tensor memory; it calls grid_dep_launch only
// after its own grid_dep_wait.  So at most two grids of a stream are resident
// at once, the later one waiting, and a tensor-memory allocation never waits
// for a grid that is still running.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Row m = b*L + i of a right-padded [B, L, ·] batch is valid when i < len[b].
__device__ __forceinline__ bool row_valid(const int* len, int L, long long m) {
  const long long b = m / L;
  const int i = (int)(m - b * L);
  return i < len[b];
}

}  // namespace r2l
