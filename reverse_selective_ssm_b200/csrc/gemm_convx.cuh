// conv + SiLU fused into x_proj ("Bifocal Diffusion Language Models",
// arXiv 2606.27732v1, §3.4 step ❷, the Mamba-1 block's depthwise conv and its
// input projection):
//
//     u[i, c]   = SiLU(conv_b[c] + Σ_{k=0..3} conv_w[c, 3−k] · x[i+k, c])   (x[j] = 0 for j ≥ len)
//     dbc[i, n] = Σ_c u[i, c] · W_x[n, c]                                   (n < 160: Δr | B | C)
//
// (with FWD the causal conv of the left-to-right block: taps on x[i−k],
// x[j] = 0 for j < 0).  The tcgen05 GEMM of gemm_tc.cuh with BN = 160 gets its
// A operand from eight converter warps instead of TMA: per 64-channel K slice
// they read a [128 + 3 rows × 64] tile of x (TMA, no swizzle), compute u with
// packed f32x2 arithmetic, write it into the A stage in the 128-byte-swizzled
// K-major layout the MMA reads, and store it to HBM once for the scan.  This
// replaces the conv kernel's pass over x and u and x_proj's second read of u.
//
// Roles (448 threads, one CTA per SM, persistent over 128-row tiles):
//   warp 0      TMA: x tile and W_x tile of each K slice into the stage ring
//   warp 1      TMEM allocation; one lane issues tcgen05.mma (M=128, N=160, K=16)
//   warps 2-5   epilogue, as in gemm_tc.cuh (fp32 dbc by TMA store, bf16 Δr copy)
//   warps 6-13  converters: warp v owns rows 16v … 16v+15 of the tile, lane l
//               the channel pair 2l, 2l+1 of the slice (a warp's lanes share
//               rows, so sequence-boundary masking is uniform across the warp)
// Every mbarrier wait is bounded (timeout flag, drain, return).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "sm100_primitives.cuh"

namespace r2l {
namespace convx {

constexpr int BM = 128, BN = 160, BK = 64;
constexpr int HALO = 3;                                   // d_conv − 1
constexpr int XR = BM + HALO;                             // x rows per tile
constexpr int CONV_WARPS = 16;
static_assert(BM % CONV_WARPS == 0 && (BM / CONV_WARPS) % 8 == 0, "rows per converter warp");
constexpr int ROWS_PER_WARP = BM / CONV_WARPS;            // 8 (a multiple of 8: the A swizzle phase)
constexpr int THREADS = (6 + CONV_WARPS) * 32;
constexpr uint32_t A_BYTES = BM * BK * 2;                 // 16 KB, 128-byte swizzle
constexpr uint32_t B_BYTES = BN * BK * 2;                 // 20 KB, 128-byte swizzle
constexpr uint32_t X_BYTES = XR * BK * 2;                 // 16,768 B, row-major, no swizzle
constexpr uint32_t W4_BYTES = BK * 4 * 4;                // conv_w slice [64 × 4] fp32
constexpr uint32_t CB_BYTES = BK * 4;                     // conv_b slice [64] fp32
constexpr uint32_t X_ALLOC = (X_BYTES + W4_BYTES + CB_BYTES + 1023) / 1024 * 1024;   // x tile, then weights
constexpr int STAGES = 3;
constexpr uint32_t STG_BYTES = 32 * 32 * 4;               // epilogue staging (fp32)
constexpr uint32_t TMEM_COLS = 512;                       // two 160-column accumulators
constexpr size_t SMEM_BYTES = 1024 + STAGES * (size_t)(A_BYTES + B_BYTES + X_ALLOC) + 8 * STG_BYTES + 512;
static_assert(B_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle-atom alignment");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

struct Args {
  const bf16* x; long long ldx;        // [M, E] (the x half of xz)
  const float* conv_w;                 // [E, 4]
  const float* conv_b;                 // [E]
  bf16* u; long long ldu;              // [M, E] out
  int M, K;                            // K = E
  bf16* C2; int ldc2; int c2_cols;     // bf16 copy of columns < c2_cols (Δr)
  const int* len; int L;
  unsigned* err;
};

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
__device__ __forceinline__ float2 silu2(float2 v) {
  const float2 t = __fmul2_rn(v, make_float2(-1.4426950408889634f, -1.4426950408889634f));
  const float2 den = __fadd2_rn(make_float2(ex2_hw(t.x), ex2_hw(t.y)), make_float2(1.0f, 1.0f));
  return __fmul2_rn(v, make_float2(rcp_hw(den.x), rcp_hw(den.y)));
}
__device__ __forceinline__ float2 bf2f(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2bf(float2 v) {
  __nv_bfloat162 b = __floats2bfloat162_rn(v.x, v.y);
  return *reinterpret_cast<uint32_t*>(&b);
}

// One converter thread, one K slice: tile rows rbase … rbase+15 (rbase = 16v),
// channels c = kb·64 + 2l, +1.  sx: the stage's x tile (row 0 is tile row 0, or
// tile row −3 with FWD), followed by the slice's conv_w [64 × 4] and conv_b
// [64]; sa: the stage's A tile.  (r0, b0, i0, n0): global row, sequence,
// position and length of the thread's first row; `interior`: all 16 rows are
// valid rows of one sequence with every tap inside it (warp-uniform).
template <bool FWD>
__device__ __forceinline__ void convert_slice(const uint8_t* sx, uint8_t* sa, const Args& a, int r0, int b0,
                                              int i0, int n0, bool interior, int v, int l, int kb) {
  const int c = kb * BK + 2 * l;
  const float4 w0 = *reinterpret_cast<const float4*>(sx + X_BYTES + (2 * l) * 16);
  const float4 w1 = *reinterpret_cast<const float4*>(sx + X_BYTES + (2 * l + 1) * 16);
  const float2 wk[4] = {make_float2(w0.x, w1.x), make_float2(w0.y, w1.y), make_float2(w0.z, w1.z),
                        make_float2(w0.w, w1.w)};
  const float2 bias = *reinterpret_cast<const float2*>(sx + X_BYTES + W4_BYTES + l * 8);
  const int rbase = v * ROWS_PER_WARP;
  const uint8_t* xs = sx + rbase * (BK * 2) + l * 4;
  uint8_t* as = sa + rbase * 128 + ((l & 3) << 2);
  const int lc = l >> 2;
  bf16* ug = a.u + (long long)r0 * a.ldu + c;
  // rolling window of 4 unpacked x rows: win[q & 3] is window row q (x tile row rbase + q)
  float2 win[4];
#pragma unroll
  for (int q = 0; q < HALO; ++q) win[q] = bf2f(*reinterpret_cast<const uint32_t*>(xs + q * (BK * 2)));
  if (interior) {
#pragma unroll
    for (int t = 0; t < ROWS_PER_WARP; ++t) {
      win[(t + HALO) & 3] = bf2f(*reinterpret_cast<const uint32_t*>(xs + (t + HALO) * (BK * 2)));
      float2 acc = bias;
#pragma unroll
      for (int k = 0; k < 4; ++k) acc = __ffma2_rn(wk[3 - k], win[(FWD ? t + 3 - k : t + k) & 3], acc);
      const uint32_t uv = f2bf(silu2(acc));
      // A stage, K-major 128-byte swizzle: 16-byte chunk lc of row (rbase + t) sits at chunk lc ^ (t % 8)
      *reinterpret_cast<uint32_t*>(as + t * 128 + ((lc ^ (t & 7)) << 4)) = uv;
      *reinterpret_cast<uint32_t*>(ug + (long long)t * a.ldu) = uv;
    }
    return;
  }
  int r = r0, b = b0, i = i0, n = n0;
#pragma unroll
  for (int t = 0; t < ROWS_PER_WARP; ++t) {
    win[(t + HALO) & 3] = bf2f(*reinterpret_cast<const uint32_t*>(xs + (t + HALO) * (BK * 2)));
    if (i >= a.L) {                                // next sequence
      ++b;
      i = 0;
      n = (b * a.L < a.M) ? (a.len ? a.len[b] : a.L) : 0;
    }
    // taps: reverse block x[i+k] = window row t+k; forward block x[i−k] = window row t+3−k
    float2 acc = bias;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool in = FWD ? i - k >= 0 : i + k < n;
      if (in) acc = __ffma2_rn(wk[3 - k], win[(FWD ? t + 3 - k : t + k) & 3], acc);
    }
    const uint32_t uv = f2bf(silu2(acc));
    *reinterpret_cast<uint32_t*>(as + t * 128 + ((lc ^ (t & 7)) << 4)) = uv;
    if (i < n && r < a.M) *reinterpret_cast<uint32_t*>(ug + (long long)t * a.ldu) = uv;
    ++r;
    ++i;
  }
}

template <bool FWD>
__global__ void __launch_bounds__(THREADS, 1)
gemm_convx_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmW4,
                  const __grid_constant__ CUtensorMap tmCB, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sX = sB + STAGES * B_BYTES;
  uint8_t* sStg = sX + STAGES * X_ALLOC;
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + 8 * STG_BYTES);   // x and W_x landed
  uint64_t* afull = full + STAGES;                                      // A written by the converters
  uint64_t* empty = afull + STAGES;                                     // MMAs done with the stage
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = a.M, K = a.K;
  const int num_m = (M + BM - 1) / BM;
  const int num_k = K / BK;
  const long long total = num_m;          // N = 160 is one tile wide

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&afull[s], CONV_WARPS);
      sm100::mbar_init(&empty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      sm100::mbar_init(&tfull[q], 1);
      sm100::mbar_init(&tempty[q], 128);
    }
    sm100::mbar_init(drain, 1);
    sm100::fence_barrier_init();
    sm100::prefetch_tmap(&tmX);
    sm100::prefetch_tmap(&tmB);
    sm100::prefetch_tmap(&tmC);
    sm100::prefetch_tmap(&tmW4);
    sm100::prefetch_tmap(&tmCB);
  }
  grid_dep_wait();
  if (warp == 1) sm100::tmem_alloc(tmem_slot, TMEM_COLS);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_launch();

  auto tile_live = [&](long long t) -> bool {
    if (!a.len) return true;
    const long long r0 = t * BM;
    const long long r1 = r0 + BM < M ? r0 + BM : M;
    return rows_have_valid(a.len, a.L, r0, r1);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      bool ok = true;
      for (long long t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!tile_live(t)) continue;
        // the reverse block reads rows r0 … r0+130, the forward block r0−3 … r0+127
        // (rows outside [0, M) read as zero)
        const int xrow = (int)(t * BM) - (FWD ? HALO : 0);
        for (int kb = 0; kb < num_k; ++kb) {
          if (!sm100::mbar_wait(&empty[stage], phase ^ 1u, a.err)) { ok = false; break; }
          sm100::mbar_arrive_expect_tx(&full[stage], X_BYTES + W4_BYTES + CB_BYTES + B_BYTES);
          sm100::tma_load_2d(sX + stage * X_ALLOC, &tmX, kb * BK, xrow, &full[stage]);
          sm100::tma_load_2d(sX + stage * X_ALLOC + X_BYTES, &tmW4, 0, kb * BK, &full[stage]);
          sm100::tma_load_2d(sX + stage * X_ALLOC + X_BYTES + W4_BYTES, &tmCB, kb * BK, 0, &full[stage]);
          sm100::tma_load_2d(sB + stage * B_BYTES, &tmB, kb * BK, 0, &full[stage]);
          ++issued[stage];
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) sm100::mbar_wait(&full[s], (uint32_t)(issued[s] - 1) & 1u, nullptr, 1000000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (long long t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!tile_live(t)) continue;
        if (!sm100::mbar_wait(&tempty[acc], aphase ^ 1u, a.err)) { ok = false; break; }
        sm100::tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < num_k; ++kb) {
          // the converters waited for the x and W_x tiles before writing A
          if (!sm100::mbar_wait(&afull[stage], phase, a.err)) { ok = false; break; }
          sm100::tc_fence_after();
          const uint32_t a0 = sm100::smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = sm100::smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            sm100::mma_bf16(d_tmem, sm100::smem_desc_k128(a0 + k * 32), sm100::smem_desc_k128(b0 + k * 32),
                            idesc, (kb | k) != 0);
          sm100::mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        sm100::mma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) aphase ^= 1u;
      }
      sm100::mma_commit(drain);
      sm100::mbar_wait(drain, 0, a.err, 1000000000ull);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    uint8_t* stg = sStg + (warp - 2) * 2 * STG_BYTES;
    int acc = 0;
    uint32_t aphase = 0;
    int chunk = 0;
    for (long long t = blockIdx.x; t < total; t += gridDim.x) {
      if (!tile_live(t)) continue;
      if (!sm100::mbar_wait(&tfull[acc], aphase, a.err)) break;
      sm100::tc_fence_after();
      const long long row = t * BM + q * 32 + lane;
      const bool row_ok = row < M && (!a.len || row_valid(a.len, a.L, row));
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32, ++chunk) {
        float v[32];
        sm100::tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256 + c0), v);
        uint8_t* buf = stg + (chunk & 1) * STG_BYTES;
        if (lane == 0) sm100::bulk_wait_read_le1();
        __syncwarp();
        stage_row32<float>(buf, lane, v);
        sm100::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          sm100::tma_store_2d(&tmC, buf, c0, (int)(t * BM) + q * 32);
          sm100::bulk_commit();
        }
        if (a.C2 && row_ok && c0 < a.c2_cols) {
          bf16* d2 = a.C2 + row * (long long)a.ldc2 + c0;
          if (c0 + 32 <= a.c2_cols) {
            store_row32<bf16>(d2, v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < a.c2_cols - c0) d2[j] = __float2bfloat16_rn(v[j]);
          }
        }
      }
      sm100::tc_fence_before();
      sm100::mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) aphase ^= 1u;
    }
    if (lane == 0) sm100::bulk_wait_all();
  } else {
    // ------------------------------------------------------------ converters
    const int v = warp - 6;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (long long t = blockIdx.x; t < total && ok; t += gridDim.x) {
      if (!tile_live(t)) continue;
      const int r0 = (int)(t * BM) + v * ROWS_PER_WARP;
      const int b0 = r0 / a.L, i0 = r0 - b0 * a.L;
      const int n0 = r0 < M ? (a.len ? a.len[b0] : a.L) : 0;
      // all 16 rows valid in one sequence, every tap inside it
      const bool interior = r0 + ROWS_PER_WARP <= M &&
                            (FWD ? (i0 >= HALO && i0 + ROWS_PER_WARP <= n0)
                                 : (i0 + ROWS_PER_WARP - 1 + HALO < n0));
      for (int kb = 0; kb < num_k; ++kb) {
        // the MMAs that read this A slot retired before its x tile was reloaded
        if (!sm100::mbar_wait(&full[stage], phase, a.err)) { ok = false; break; }
        convert_slice<FWD>(sX + stage * X_ALLOC, sA + stage * A_BYTES, a, r0, b0, i0, n0, interior, v, lane, kb);
        sm100::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&afull[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 1) sm100::tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace convx
}  // namespace r2l
