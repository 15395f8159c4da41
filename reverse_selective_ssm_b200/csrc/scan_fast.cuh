// Reverse selective scan for the bf16 path ("Bifocal Diffusion Language
// Models", arXiv 2606.27732v1, §3.4 step ❷: the Mamba-1 selective scan on the
// flipped sequence, run here from each sequence's last valid token to its
// first):
//
//   Δ_i = softplus(dt_raw_i + dt_b),   dt_raw_i = W_dt · Δr_i
//   H_i = exp(Δ_i A) ⊙ H_{i+1} + Δ_i u_i B_i          (H entering the last token = 0)
//   y_i = (⟨C_i, H_i⟩ + D u_i) · SiLU(z_i)
//
// Work split: a CTA owns 128 channels of one sequence over one chunk of
// tokens; each of its 4 compute warps holds 32 channels, one channel per
// thread, with the 16-entry state in registers updated by packed f32x2
// arithmetic.  A producer warp streams [16 tokens × 128 channels] tiles of u
// and z, the [16 tokens × 32] tile of B|C, and either
// the dt_raw tile or, with DTMMA, the [16 tokens × R] tile of Δr, into a
// 4-deep shared-memory ring with TMA, from the chunk's right end to its left
// end; it writes each finished y tile back with a TMA store (tiles that cross
// the chunk's left edge are stored row by row by the compute threads, so no
// row outside the chunk is ever written).
//
// DTMMA (dt_proj fused, R = 128): a sixth warp keeps the CTA's W_dt slice
// [128 channels × R] in shared memory and, per tile, issues tcgen05.mma
// (M = 128 channels, N = 16 tokens, K = R) into a TMEM column block; the
// accumulator's lane is the channel, so each compute thread reads its 16
// dt_raw values with one tcgen05.ld.  dt_raw never touches HBM.  The layer
// itself runs the DTMMA scan as the two-threads-per-channel kernel of
// scan_pair.cuh; this one-thread DTMMA form is kept as its compile-time
// alternative (R2L_SCAN_IMPL=0), and the form without DTMMA serves dt_rank ≠ 128.
//
// When a sequence is split into several chunks (to give the GPU enough
// independent work), three launches cooperate through a small carry buffer:
//   1. chunk_scan_kernel<false>: each chunk scans from a zero state and stores
//      its final state S_k (the state at its first token) and Σ Δ over it;
//   2. chunk_carry_kernel: per (sequence, channel), from the last chunk to the
//      first, the state entering chunk k from the right is
//      H_in(k) = S_{k+1} + exp(A Σ_{k+1} Δ) ⊙ H_in(k+1), written over S_k;
//   3. chunk_scan_kernel<true>: each chunk rescans from H_in(k) and writes y.
// With one chunk per sequence only step 3 runs, from a zero state.
//
// FWD runs the same block left to right (the "L2R Mamba" control of Table 4):
// tiles stream from the chunk's left end, tokens are visited in increasing
// order, and chunk carries flow from each chunk to the one on its right.
//
// Decays: exp(Δ A_m) is exp2(Δ · A_m log2 e) on the MUFU unit.  When A is the
// S4D-real initialisation A_m = −(m+1) (decided once per call, exactly, by
// a_log_check_kernel), the 16 decays are the powers r, r², …, r¹⁶ of
// r = exp(−Δ) = 1 / (1 + e^v) for v = dt_raw + dt_b (since Δ = softplus(v)):
// one reciprocal and a depth-4 product tree per (token, channel).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace r2l {
namespace rscan {

constexpr int TS = 16;        // tokens per pipeline stage
constexpr int SUB = 8;        // tokens per phase-A / phase-B sub-tile
constexpr int STAGES = 4;
constexpr int CWARPS = 4;     // compute warps
constexpr int CTHREADS = CWARPS * 32;
constexpr int CH = CTHREADS;  // channels per CTA
constexpr int DT_R = 128;     // dt_rank of the fused dt_proj (kScanFusedDtRank)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

constexpr uint32_t ACT_TILE = TS * CH * 2;        // one bf16 [TS × CH] tile
constexpr uint32_t BC_TILE = TS * 32 * 4;         // one fp32 [TS × 32] tile
constexpr uint32_t DR_TILE = TS * DT_R * 2;       // one bf16 [TS × R] Δr tile (2 swizzle atoms)
constexpr uint32_t W_SLICE = CH * DT_R * 2;       // bf16 W_dt [CH × R] (2 atoms of 16 KB)
constexpr uint32_t TMEM_COLS = 64;                // STAGES × TS fp32 columns

// Shared-memory layout (offsets from a 1024-byte aligned base).  Without
// DTMMA: u, dt, z, y tiles, B|C tiles, barriers.  With DTMMA: W slice, Δr
// tiles, u, z, y tiles, B|C tiles, barriers.
template <bool DTMMA>
struct Smem {
  static constexpr uint32_t W = 0;
  static constexpr uint32_t DR = DTMMA ? W_SLICE : 0;
  static constexpr uint32_t U = DR + (DTMMA ? STAGES * DR_TILE : 0);
  static constexpr uint32_t DT = U + STAGES * ACT_TILE;           // unused with DTMMA
  static constexpr uint32_t Z = DT + (DTMMA ? 0 : STAGES * ACT_TILE);
  static constexpr uint32_t Y = Z + STAGES * ACT_TILE;
  static constexpr uint32_t BC = Y + STAGES * ACT_TILE;
  static constexpr uint32_t BAR = BC + STAGES * BC_TILE;          // full, empty, dtready [STAGES], wfull, drain
  static constexpr uint32_t SLOT = BAR + (3 * STAGES + 2) * 8;    // TMEM base address
  static constexpr size_t BYTES = 1024 + SLOT + 16;
  static constexpr int THREADS = CTHREADS + 32 + (DTMMA ? 32 : 0);
};

struct Params {
  const float* A_log;   // [E, 16]
  const float* D;       // [E]
  const float* dt_b;    // [E]
  bf16* y;              // [B·L, E] (row stride ldy)
  long long ldy;
  int E, L;
  int T;                // chunk length in tokens (multiple of TS)
  int nc;               // chunks per sequence
  const int* len;       // [B] valid lengths (already clamped to [0, L])
  float* carry;         // [B][nc][E][16]: S_k, then H_in(k)  (unused when nc == 1)
  float* carry_sum;     // [B][nc][E]: Σ Δ over chunk k
  unsigned* err;
  int force_general;
  const unsigned* a_general;  // 0: A is exactly −(1..16) (the power path), decided once per call
  int fwd;              // left-to-right block (chunk carry direction)
  float* hck;           // training mode: H at every position 16(k+1) < len, [B][nc16][E][16] (else null)
  int nc16;             // ⌈L/16⌉
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Δ = softplus(v) = log(1 + x), x = e^v (v itself above 20), and r = e^{-Δ} =
// 1 / (1 + x).  Δ = log2(w)·ln 2 with w = fl(1 + x): the rounding of 1 + x
// (2⁻²⁴/x relative) and the absolute error of the hardware log2 (≈1e-7 in Δ)
// leave a relative error near 1e-4 at the smallest steps of the Mamba
// parameterisation (Δ ≈ 1e-3), far below the bf16 rounding of the scan's
// output.  The decay r is exact to rounding.
__device__ __forceinline__ void softplus_and_decay(float v, float& delta, float& r) {
  const float x = ex2_approx(v * LOG2E);
  const float w = 1.0f + x;
  r = rcp_approx(w);
  delta = v > 20.0f ? v : lg2_approx(w) * LN2;
}

// SiLU(z) = z / (1 + e^{-z})
__device__ __forceinline__ float silu_fast(float z) {
  return __fdividef(z, 1.0f + ex2_approx(-z * LOG2E));
}

// Per-thread constants of one channel.
struct Ctx {
  float dtb, Dc;
  float A2[16];          // A_m · log2 e
};

// One sub-tile of SUB tokens [j0, j0 + SUB) of one channel, last token first.
// Phase A computes what does not depend on the state (softplus, the decay
// base, Δu, D·u, the gate) for all of its tokens; phase B runs the
// recurrence (tokens in decreasing order, increasing with FWD).  FULL: every
// token of the sub-tile is inside the chunk; otherwise only tokens
// j in [jlo, jhi) are.  dtv: the tile's 16 dt_raw values (DTMMA)
// or unused (read sdt).  Output: y rows to shared memory (ys, stride CH) for
// tiles stored by TMA, else to global (yg).
template <bool FINAL, bool POW, bool FULL, bool DTMMA, bool FWD>
__device__ __forceinline__ void scan_sub(const Ctx& cx, float2 (&H)[8], float& sumd, const bf16* su,
                                         const bf16* sdt, const float (&dtv)[16], const bf16* sz,
                                         const float* sbc, bf16* ys, bf16* yg, long long ldy, bool store_ok,
                                         int j0, int jlo, int jhi) {
  float dec[SUB], du[SUB], gz[SUB], Du[SUB];
#pragma unroll
  for (int t = 0; t < SUB; ++t) {
    const int j = j0 + t;
    if (!FULL && (j < jlo || j >= jhi)) continue;
    float delta, r;
    const float raw = DTMMA ? dtv[j] : __bfloat162float(sdt[j * CH]);
    softplus_and_decay(raw + cx.dtb, delta, r);
    const float uu = __bfloat162float(su[j * CH]);
    dec[t] = POW ? r : delta;
    du[t] = delta * uu;
    if (FINAL) {
      Du[t] = cx.Dc * uu;
      gz[t] = silu_fast(__bfloat162float(sz[j * CH]));
    } else {
      sumd += delta;
    }
  }
#pragma unroll
  for (int tt = 0; tt < SUB; ++tt) {
    const int t = FWD ? tt : SUB - 1 - tt;
    const int j = j0 + t;
    if (!FULL && (j < jlo || j >= jhi)) continue;
    const float4* bc4 = reinterpret_cast<const float4*>(sbc + j * 32);
    const float2 du2 = make_float2(du[t], du[t]);
    float2 a[8];
    if (POW) {
      // r^1 … r^16 by a depth-4 product tree
      const float r = dec[t];
      const float r2 = r * r;
      a[0] = make_float2(r, r2);
      a[1] = __fmul2_rn(a[0], make_float2(r2, r2));          // r3 r4
      const float r4 = a[1].y;
      a[2] = __fmul2_rn(a[0], make_float2(r4, r4));          // r5 r6
      a[3] = __fmul2_rn(a[1], make_float2(r4, r4));          // r7 r8
      const float r8 = a[3].y;
#pragma unroll
      for (int q = 0; q < 4; ++q) a[4 + q] = __fmul2_rn(a[q], make_float2(r8, r8));   // r9 … r16
    } else {
      const float delta = dec[t];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        a[q] = make_float2(ex2_approx(delta * cx.A2[2 * q]), ex2_approx(delta * cx.A2[2 * q + 1]));
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 Bq = bc4[q];
      H[2 * q] = __ffma2_rn(a[2 * q], H[2 * q], __fmul2_rn(du2, make_float2(Bq.x, Bq.y)));
      H[2 * q + 1] = __ffma2_rn(a[2 * q + 1], H[2 * q + 1], __fmul2_rn(du2, make_float2(Bq.z, Bq.w)));
    }
    if (FINAL) {
      float2 acc0 = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 Cq = bc4[4 + q];
        acc0 = __ffma2_rn(make_float2(Cq.x, Cq.y), H[2 * q], acc0);
        acc1 = __ffma2_rn(make_float2(Cq.z, Cq.w), H[2 * q + 1], acc1);
      }
      const float s = (acc0.x + acc0.y) + (acc1.x + acc1.y);
      const bf16 yv = __float2bfloat16_rn((s + Du[t]) * gz[t]);
      if (store_ok) {
        if (ys) ys[j * CH] = yv;
        else yg[(long long)j * ldy] = yv;
      }
    }
  }
}

// The TMA producer (one thread): streams the chunk's tiles right to left into
// the STAGES-deep ring and, for the final scan, writes each finished y tile
// that lies wholly inside the chunk back with a bulk tensor store.  With
// DTMMA it first loads the CTA's W_dt slice, and streams Δr tiles instead of
// dt_raw tiles.
template <class S, bool FINAL, bool DTMMA, bool FWD, int CHN = CH>
__device__ __forceinline__ void run_producer(const CUtensorMap* tm_u, const CUtensorMap* tm_z,
                                             const CUtensorMap* tm_dt, const CUtensorMap* tm_bc,
                                             const CUtensorMap* tm_y, const CUtensorMap* tm_w, uint8_t* smem,
                                             uint64_t* full, uint64_t* empty, uint64_t* wfull, int b, int cb,
                                             int s0, int e0, int ntiles, const Params& p) {
  bf16* s_u = reinterpret_cast<bf16*>(smem + S::U);
  bf16* s_dt = reinterpret_cast<bf16*>(smem + S::DT);
  bf16* s_z = reinterpret_cast<bf16*>(smem + S::Z);
  bf16* s_y = reinterpret_cast<bf16*>(smem + S::Y);
  float* s_bc = reinterpret_cast<float*>(smem + S::BC);
  sm100::prefetch_tmap(tm_u);
  sm100::prefetch_tmap(tm_dt);
  sm100::prefetch_tmap(tm_bc);
  if (FINAL) {
    sm100::prefetch_tmap(tm_z);
    sm100::prefetch_tmap(tm_y);
  }
  if (DTMMA) {
    sm100::prefetch_tmap(tm_w);
    sm100::mbar_arrive_expect_tx(wfull, (uint32_t)(CHN * DT_R * 2));
    for (int a = 0; a < DT_R / 64; ++a)
      sm100::tma_load_2d(smem + S::W + a * (CHN * 128), tm_w, a * 64, cb * CHN, wfull);
  }
  constexpr uint32_t act = TS * CHN * 2;
  constexpr uint32_t bytes = (FINAL ? 2 : 1) * act + BC_TILE + (DTMMA ? DR_TILE : act);
  int issued = 0;
  bool ok = true;
  const int iters = ntiles + (FINAL ? STAGES : 0);
  for (int it = 0; it < iters; ++it) {
    const int st = it % STAGES;
    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
    if (!sm100::mbar_wait(&empty[st], ph ^ 1u, p.err)) { ok = false; break; }
    if (FINAL && it >= STAGES) {
      const int pt = it - STAGES;                     // the tile just finished in this slot
      const int tb = FWD ? s0 + pt * TS : e0 - (pt + 1) * TS;
      if (FWD ? tb + TS <= e0 : tb >= s0) {           // whole tile inside the chunk: y sits in s_y
        sm100::tma_store_2d(tm_y, s_y + st * TS * CHN, cb * CHN, b * p.L + tb);
        sm100::bulk_commit();
        sm100::bulk_wait_read_all();                  // s_y[st] is rewritten STAGES tiles later
      }
    }
    if (it < ntiles) {
      // may start before row 0 (reverse, b = 0) or run past the last row (FWD): reads zeros
      const int row0 = b * p.L + (FWD ? s0 + it * TS : e0 - (it + 1) * TS);
      sm100::mbar_arrive_expect_tx(&full[st], bytes);
      sm100::tma_load_2d(s_u + st * TS * CHN, tm_u, cb * CHN, row0, &full[st]);
      if (DTMMA) {
        uint8_t* dr = smem + S::DR + st * DR_TILE;
        for (int a = 0; a < DT_R / 64; ++a) sm100::tma_load_2d(dr + a * (TS * 128), tm_dt, a * 64, row0, &full[st]);
      } else {
        sm100::tma_load_2d(s_dt + st * TS * CHN, tm_dt, cb * CHN, row0, &full[st]);
      }
      if (FINAL) sm100::tma_load_2d(s_z + st * TS * CHN, tm_z, cb * CHN, row0, &full[st]);
      sm100::tma_load_2d(s_bc + st * TS * 32, tm_bc, 0, row0, &full[st]);
      ++issued;
    }
  }
  if (FINAL) sm100::bulk_wait_all();
  if (!ok) {  // drain loads still in flight before the CTA can exit
    for (int it = issued - 1; it >= 0 && it >= issued - STAGES; --it)
      sm100::mbar_wait(&full[it % STAGES], (uint32_t)(it / STAGES) & 1u, nullptr, 1000000000ull);
    if (DTMMA) sm100::mbar_wait(wfull, 0, nullptr, 1000000000ull);
  }
}

// The dt_proj MMA issuer (one thread, DTMMA): per tile, dt_rawᵀ[128 ch × 16
// tokens] = W_dt slice · Δr tileᵀ into TMEM columns [16·st, 16·st + 16).
__device__ __forceinline__ void run_dt_mma(uint8_t* smem, uint32_t tmem_base, uint64_t* full, uint64_t* dtready,
                                           uint64_t* wfull, uint64_t* drain, int ntiles, unsigned* err) {
  using S = Smem<true>;
  constexpr uint32_t idesc = sm100::idesc_bf16_f32(128, TS);
  bool ok = sm100::mbar_wait(wfull, 0, err);
  const uint32_t w0 = sm100::smem_u32(smem + S::W);
  for (int it = 0; it < ntiles && ok; ++it) {
    const int st = it % STAGES;
    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
    if (!sm100::mbar_wait(&full[st], ph, err)) break;
    sm100::tc_fence_after();
    const uint32_t d0 = sm100::smem_u32(smem + S::DR + st * DR_TILE);
#pragma unroll
    for (int k = 0; k < DT_R / 16; ++k) {
      const uint32_t a_addr = w0 + (k / 4) * (CH * 128) + (k % 4) * 32;
      const uint32_t b_addr = d0 + (k / 4) * (TS * 128) + (k % 4) * 32;
      sm100::mma_bf16(tmem_base + (uint32_t)(st * TS), sm100::smem_desc_k128(a_addr), sm100::smem_desc_k128(b_addr),
                      idesc, k != 0);
    }
    sm100::mma_commit(&dtready[st]);
  }
  sm100::mma_commit(drain);
  sm100::mbar_wait(drain, 0, err, 1000000000ull);
}

template <bool FINAL, bool DTMMA, bool FWD>
__global__ void __launch_bounds__(Smem<DTMMA>::THREADS, 2)
chunk_scan_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_z,
                  const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ CUtensorMap tm_bc,
                  const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_w,
                  const Params p) {
  using S = Smem<DTMMA>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const bf16* s_u = reinterpret_cast<const bf16*>(smem + S::U);
  const bf16* s_dt = reinterpret_cast<const bf16*>(smem + S::DT);
  const bf16* s_z = reinterpret_cast<const bf16*>(smem + S::Z);
  bf16* s_y = reinterpret_cast<bf16*>(smem + S::Y);
  const float* s_bc = reinterpret_cast<const float*>(smem + S::BC);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* dtready = empty + STAGES;
  uint64_t* wfull = dtready + STAGES;
  uint64_t* drain = wfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::SLOT);

  const int cb = blockIdx.x, k = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool compute = tid < CTHREADS;
  const int ch = compute ? tid : 0;             // channel within the block
  const int c = cb * CH + ch;
  const bool cvalid = compute && c < p.E;
  const int n = p.len[b];
  const int s0 = k * p.T;
  const int e0 = min(s0 + p.T, n);

  if (s0 >= n) {  // chunk entirely in the padding: nothing to read or write
    if (!FINAL && cvalid) {
      float4* dst = reinterpret_cast<float4*>(p.carry + (((long long)b * p.nc + k) * p.E + c) * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      p.carry_sum[((long long)b * p.nc + k) * p.E + c] = 0.0f;
    }
    return;
  }
  const int ntiles = (e0 - s0 + TS - 1) / TS;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], CWARPS);
      sm100::mbar_init(&dtready[s], 1);
    }
    sm100::mbar_init(wfull, 1);
    sm100::mbar_init(drain, 1);
    sm100::fence_barrier_init();
  }
  if (DTMMA && warp == CWARPS + 1) sm100::tmem_alloc(tmem_slot, TMEM_COLS);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = DTMMA ? *tmem_slot : 0u;

  if (warp == CWARPS) {
    if (lane == 0)
      run_producer<S, FINAL, DTMMA, FWD>(&tm_u, &tm_z, &tm_dt, &tm_bc, &tm_y, &tm_w, smem, full, empty, wfull, b, cb, s0,
                                 e0, ntiles, p);
    return;   // the producer warp takes no part in the teardown below
  }
  if (DTMMA && warp == CWARPS + 1) {
    if (lane == 0) run_dt_mma(smem, tmem_base, full, dtready, wfull, drain, ntiles, p.err);
    __syncwarp();
    sm100::named_bar_sync(1, CTHREADS + 32);   // every compute warp has finished reading TMEM
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, TMEM_COLS);
    return;
  }

  // -------------------------------------------------------------- compute warps
  Ctx cx;
  cx.dtb = cvalid ? p.dt_b[c] : 0.0f;
  cx.Dc = cvalid ? p.D[c] : 0.0f;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const float a = cvalid ? -expf(p.A_log[c * 16 + m]) : -(float)(m + 1);
    cx.A2[m] = a * LOG2E;
  }
  const bool use_pow = !p.force_general && *p.a_general == 0u;

  float2 H[8];
  if (FINAL && p.nc > 1 && cvalid) {
    const float4* src = reinterpret_cast<const float4*>(p.carry + (((long long)b * p.nc + k) * p.E + c) * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = src[q];
      H[2 * q] = make_float2(v.x, v.y);
      H[2 * q + 1] = make_float2(v.z, v.w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) H[q] = make_float2(0.0f, 0.0f);
  }
  float sumd = 0.0f;
  float dtv[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) dtv[j] = 0.0f;

  for (int it = 0; it < ntiles; ++it) {
    const int st = it % STAGES;
    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
    if (!sm100::mbar_wait(&full[st], ph, p.err)) break;
    if (DTMMA) {
      if (!sm100::mbar_wait(&dtready[st], ph, p.err)) break;
      sm100::tc_fence_after();
      sm100::tmem_ld16(tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(st * TS), dtv);
    }
    const int tbase = FWD ? s0 + it * TS : e0 - (it + 1) * TS;   // sequence position of tile row 0
    const int jlo = (!FWD && s0 > tbase) ? s0 - tbase : 0;       // tokens [jlo, jhi) are in the chunk
    const int jhi = (FWD && e0 - tbase < TS) ? e0 - tbase : TS;
    const bool full = jlo == 0 && jhi == TS;
    const bf16* su = s_u + st * TS * CH + ch;
    const bf16* sdt = s_dt + st * TS * CH + ch;
    const bf16* sz = s_z + st * TS * CH + ch;
    const float* sbc = s_bc + st * TS * 32;
    // full tiles go out through shared memory and a TMA store; a tile that
    // crosses the chunk's edge is written row by row
    bf16* ys = full ? s_y + st * TS * CH + ch : nullptr;
    bf16* yg = p.y + ((long long)b * p.L + tbase) * p.ldy + c;
#pragma unroll
    for (int sb = 0; sb < TS / SUB; ++sb) {
      const int j0 = FWD ? sb * SUB : TS - SUB - sb * SUB;
      if (full) {
        if (use_pow)
          scan_sub<FINAL, true, true, DTMMA, FWD>(cx, H, sumd, su, sdt, dtv, sz, sbc, ys, yg, p.ldy, cvalid, j0, 0, TS);
        else
          scan_sub<FINAL, false, true, DTMMA, FWD>(cx, H, sumd, su, sdt, dtv, sz, sbc, ys, yg, p.ldy, cvalid, j0, 0, TS);
      } else if (j0 + SUB > jlo && j0 < jhi) {
        if (use_pow)
          scan_sub<FINAL, true, false, DTMMA, FWD>(cx, H, sumd, su, sdt, dtv, sz, sbc, ys, yg, p.ldy, cvalid, j0, jlo, jhi);
        else
          scan_sub<FINAL, false, false, DTMMA, FWD>(cx, H, sumd, su, sdt, dtv, sz, sbc, ys, yg, p.ldy, cvalid, j0, jlo, jhi);
      }
    }
    if (FINAL && ys) sm100::fence_proxy_async_smem();   // make the y tile visible to the TMA store
    if (DTMMA) sm100::tc_fence_before();
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty[st]);
  }

  if (!FINAL && cvalid) {
    float4* dst = reinterpret_cast<float4*>(p.carry + (((long long)b * p.nc + k) * p.E + c) * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_float4(H[2 * q].x, H[2 * q].y, H[2 * q + 1].x, H[2 * q + 1].y);
    p.carry_sum[((long long)b * p.nc + k) * p.E + c] = sumd;
  }
  if (DTMMA) {
    sm100::tc_fence_before();
    sm100::named_bar_sync(1, CTHREADS + 32);   // release TMEM to the dealloc
  }
}

// Operands of the tensor-core broadcast of B|C (scan_pair.cuh): no-swizzle
// K-major tf32 tiles with 32-byte rows.
constexpr uint32_t OPB_BYTES = 64 * 32;                 // 64 rows × (8 tf32)
constexpr uint32_t ONES_BYTES = 128 * 32;               // 128 rows × (8 tf32)

// Byte offset of row n of a no-swizzle K-major operand with 32-byte rows:
// 8-row core matrices of 16-byte rows, the two 16-byte halves of a row 128
// bytes apart (lbo), 8-row groups 256 bytes apart (sbo).
__device__ __forceinline__ uint32_t opnd_row(int n) { return (uint32_t)((n >> 3) * 256 + (n & 7) * 16); }

// Per (sequence, channel): turn chunk end states S_k into the states entering
// each chunk from the right (from the left with fwd), in place (see the
// header comment, step 2).
__global__ void chunk_carry_kernel(const Params p) {
  grid_dep_wait();
  grid_dep_launch();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (c >= p.E) return;
  const int n = p.len[b];
  if (n <= 0) return;
  const int nk = (n + p.T - 1) / p.T;
  float A[16], carry[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    A[m] = -expf(p.A_log[c * 16 + m]);
    carry[m] = 0.0f;
  }
  for (int kk = 0; kk < nk; ++kk) {
    const int k = p.fwd ? kk : nk - 1 - kk;   // from the chunk the state enters first
    float4* S = reinterpret_cast<float4*>(p.carry + (((long long)b * p.nc + k) * p.E + c) * 16);
    const float sd = p.carry_sum[((long long)b * p.nc + k) * p.E + c];
    float s[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = S[q];
      s[4 * q] = v.x; s[4 * q + 1] = v.y; s[4 * q + 2] = v.z; s[4 * q + 3] = v.w;
      S[q] = make_float4(carry[4 * q], carry[4 * q + 1], carry[4 * q + 2], carry[4 * q + 3]);
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) carry[m] = fmaf(expf(A[m] * sd), carry[m], s[m]);
  }
}

}  // namespace rscan
}  // namespace r2l
