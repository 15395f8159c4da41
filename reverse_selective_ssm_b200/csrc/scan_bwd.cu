// Gradient of the reverse selective scan (fp32), the step that training the
// sidecar alone back-propagates through ("Bifocal Diffusion Language Models",
// arXiv 2606.27732v1, §3.4 step ❷: the Mamba-1 scan run from each sequence's
// last valid position to its first, with softplus(Δ) in front and the SiLU(z)
// gate behind).  Forward, per sequence of n positions:
//
//   Δ_i = softplus(v_i), v_i = dt_raw_i + dt_b;   a_i = exp(Δ_i A), A = -exp(A_log)
//   H_n = 0,  H_i = a_i ⊙ H_{i+1} + Δ_i u_i B_i;   p_i = ⟨C_i, H_i⟩ + D u_i;   y_i = p_i SiLU(z_i)
//
// Backward for dy = ∂L/∂y (chain rule):
//
//   dp_i = dy_i SiLU(z_i),  dz_i = dy_i p_i SiLU'(z_i)
//   G_i  = ∂L/∂H_i = a_{i-1} ⊙ G_{i-1} + dp_i C_i,  G_{-1} = 0   (left to right)
//   dΔ_i = Σ_m G_im H_{i+1,m} a_im A_m + u_i Σ_m G_im B_im,   ddt_raw_i = dΔ_i softplus'(v_i)
//   du_i = D dp_i + Δ_i Σ_m G_im B_im
//   dB_i = Σ_c G_i Δ_i u_i,   dC_i = Σ_c dp_i H_i                 (sums over channels)
//   dA_log = A ⊙ Σ_i Δ_i G_i ⊙ H_{i+1} ⊙ a_i,  dD = Σ_i dp_i u_i,  ddt_b = Σ_i ddt_raw_i
//
// The adjoint G runs left to right while H runs right to left, so both are
// split into chunks of T positions, in 6 launches:
//   1. state: each chunk scans H right to left from zero (its end state and
//      Σ Δ over the chunk) and G left to right from zero (its end value and
//      Σ Δ over positions s-1 … e-2, the decays it crossed);
//   2. carry: per (sequence, channel, state), the state entering each chunk
//      from the right, H_in(k) = S_{k+1} + exp(A Σ_{k+1}Δ) H_in(k+1), and G
//      entering each chunk from the left, the same recurrence the other way;
//   3. final: each chunk recomputes its H from H_in(k), keeping every second
//      position, then walks G from the carried value two positions at a
//      time and writes every gradient;
//   4.-6. fixed-order reductions: the per-chunk parameter partials (two
//      levels) and the per-block partial sums of dB | dC (deterministic, no
//      atomics).
//
// Threads: four per channel, thread q holding states 4q … 4q+3 (float4 loads
// of B, C and the state rows), 64 channels per 256-thread block.  Sums over
// the four threads use two xor shuffles; the sum of dB | dC over a warp's 8
// channels is a 7-shuffle reduce-scatter that leaves each lane one of the 32
// columns.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "scan_bwd.h"

namespace r2l {
namespace sbwd {

constexpr int CPB = 64;                   // channels per block
constexpr int THREADS = CPB * 4;
constexpr int WARPS = THREADS / 32;

struct Args {
  const float* u;
  const float* z;
  const bf16* u16;         // bf16 u and z instead (when not null)
  const bf16* z16;
  int ldz;
  const float* dt;
  const float* bc;
  int ldbc;
  const float* A_log;
  const float* D;
  const float* dt_b;
  const float* dy;
  float* du;
  float* dz;
  int ld_dz;
  float* ddt;
  float* dbc;
  int ld_dbc;
  float* dA_log;
  float* dD;
  float* ddt_b;
  int B, L, E, T, nc;
  const int* lengths;      // caller's lengths, or null
  unsigned* status;
  float* hcar;             // [B][nc][E][16]: chunk end states, then H_in(k)
  float* hsd;              // [B][nc][E]
  float* gcar;             // [B][nc][E][16]: chunk end adjoints, then G entering from the left
  float* gsd;              // [B][nc][E]
  float* pA;               // [B][nc][E][16] Σ Δ G H_{i+1} a over the chunk
  float* pD;               // [B][nc][E]
  float* pb;               // [B][nc][E]
  float* pbc;              // [E/CPB][B·L][32] per-block partial dB | dC
  int nbc;                 // channel blocks in pbc
  int ckpt_ragged_only;    // the checkpoint pass skips sequences whose length is a multiple of 16
  bf16* ddt16;             // bf16 ddt_raw and dz instead of fp32 (the walk only), or null
  long long ld_ddt16;
  bf16* dz16;
  long long ld_dz16;
  uint32_t lnbits[16];     // float log(1) … log(16): the power-path A_log
};

__device__ __forceinline__ int seq_len(const Args& a, int b) {
  int n = a.lengths ? a.lengths[b] : a.L;
  if (n < 0 || n > a.L) {
    if (a.status && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(a.status, 0x1u);   // R2L_DEVFLAG_LENGTH_CLAMPED
    n = n < 0 ? 0 : a.L;
  }
  return n;
}

// softplus and its derivative σ, with the hardware exponential (relative
// error about 1e-6 over the range used, far under the fp32 path's tolerance)
// and the accurate log1p (Δ is small, log(1 + x) for small x).
__device__ __forceinline__ float softplus_fwd(float v) { return v > 20.0f ? v : log1pf(__expf(v)); }
__device__ __forceinline__ float sigmoid_fast(float v) { return __fdividef(1.0f, 1.0f + __expf(-v)); }
__device__ __forceinline__ float softplus_grad(float v) { return v > 20.0f ? 1.0f : sigmoid_fast(v); }

// 2^x on the MUFU unit (ex2.approx, relative error about 2^-22): the decays
// a = exp(Δ A) = 2^(Δ · A log2 e).
__device__ __forceinline__ float exp2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
// four consecutive bf16 (8-byte aligned) widened to fp32
__device__ __forceinline__ float4 ld4h(const bf16* p) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float get(const float4& v, int j) { return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w; }

__device__ __forceinline__ float sum4(float v) {         // over the channel's four threads
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

struct Lane {
  int c, q, b, k, s, e, n;
  float A[4];    // A_m of the thread's states
  float A2[4];   // A_m · log2 e
  float2 Ap[2];  // A as (states 0,1), (2,3) pairs for the packed f32x2 arithmetic
  float2 A2p[2];
};

__device__ __forceinline__ Lane lane_setup(const Args& a) {
  Lane l;
  l.c = blockIdx.x * CPB + (threadIdx.x >> 2);
  l.q = threadIdx.x & 3;
  l.k = blockIdx.y;
  l.b = blockIdx.z;
  l.n = seq_len(a, l.b);
  l.s = l.k * a.T;
  l.e = min(l.s + a.T, l.n);
  const float4 al = ld4(a.A_log + (size_t)l.c * 16 + 4 * l.q);
  l.A[0] = -expf(al.x); l.A[1] = -expf(al.y); l.A[2] = -expf(al.z); l.A[3] = -expf(al.w);
#pragma unroll
  for (int j = 0; j < 4; ++j) l.A2[j] = l.A[j] * kLog2e;
  l.Ap[0] = make_float2(l.A[0], l.A[1]);
  l.Ap[1] = make_float2(l.A[2], l.A[3]);
  l.A2p[0] = make_float2(l.A2[0], l.A2[1]);
  l.A2p[1] = make_float2(l.A2[2], l.A2[3]);
  return l;
}

__device__ __forceinline__ float2 lo2(const float4& v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4& v) { return make_float2(v.z, v.w); }
__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }

// The decays of the thread's 4 states for step Δ: exp(Δ A) = 2^(Δ A log2 e).
__device__ __forceinline__ void decays(const Lane& l, float delta, float2 (&a)[2]) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float2 t = __fmul2_rn(dup2(delta), l.A2p[k]);
    a[k] = make_float2(exp2_mufu(t.x), exp2_mufu(t.y));
  }
}

__device__ __forceinline__ size_t carry_idx(const Args& a, const Lane& l) {
  return (((size_t)l.b * a.nc + l.k) * a.E + l.c);
}

// Per-(position, channel) scalars of a chunk for the block's 64 channels,
// rows [s, e): computed once per element by the whole block from coalesced
// float4 reads (instead of once per state-holding thread), so the
// per-position loops below read shared memory only.  Arrays are [T][64]
// (row r = position s + r); bc is the raw [T][32] B | C rows.
//   U = u, DL = Δ, DU = Δ u, DP = dp = dy SiLU(z), FZ = dy SiLU'(z) (dz = p FZ),
//   SG = softplus'(v)
enum : unsigned { S_U = 1, S_DL = 2, S_DU = 4, S_DP = 8, S_FZ = 16, S_SG = 32 };
constexpr int NSTAGE = 6;

struct Stage {
  float* arr[NSTAGE];
  float* bc;
};

// Arrays sit 8 words apart in bank order (stride T·64 + 8 floats), so the
// three gradient rows that a channel's threads q = 0, 1, 2 leave in arrays
// 2, 5 and 4 fall in different banks.
constexpr int STAGE_PAD = 8;

__device__ __forceinline__ Stage stage_layout(float* base, int T) {
  Stage st;
#pragma unroll
  for (int k = 0; k < NSTAGE; ++k) st.arr[k] = base + (size_t)k * (T * CPB + STAGE_PAD);
  st.bc = base + (size_t)NSTAGE * (T * CPB + STAGE_PAD);
  return st;
}

constexpr size_t stage_floats(int T) { return (size_t)NSTAGE * (T * CPB + STAGE_PAD) + (size_t)T * 32; }

template <unsigned WANT>
__device__ __forceinline__ void stage_chunk(const Args& a, const Lane& l, const Stage& st) {
  const int nrows = l.e - l.s;
  if (nrows <= 0) return;
  const long long row0 = (long long)l.b * a.L + l.s;
  const int col0 = blockIdx.x * CPB;
  constexpr bool NEED_U = WANT & (S_U | S_DU);
  constexpr bool NEED_Z = WANT & (S_DP | S_FZ);
  for (int t = threadIdx.x; t < nrows * (CPB / 4); t += THREADS) {
    const int r = t / (CPB / 4), q4 = t % (CPB / 4);
    const long long row = row0 + r;
    const int col = col0 + 4 * q4;
    const float4 dtb = ld4(a.dt_b + col);
    const float4 v4 = ld4(a.dt + row * a.E + col);
    float4 u4 = make_float4(0.f, 0.f, 0.f, 0.f), z4 = u4, dy4 = u4;
    if (NEED_U) u4 = a.u16 ? ld4h(a.u16 + row * a.E + col) : ld4(a.u + row * a.E + col);
    if (NEED_Z) {
      z4 = a.z16 ? ld4h(a.z16 + row * a.ldz + col) : ld4(a.z + row * a.ldz + col);
      dy4 = ld4(a.dy + row * a.E + col);
    }
    float o[NSTAGE][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float v = get(v4, j) + get(dtb, j);
      const float delta = softplus_fwd(v);
      const float uu = get(u4, j), zz = get(z4, j), dyy = get(dy4, j);
      const float sg = sigmoid_fast(zz);
      o[0][j] = uu;
      o[1][j] = delta;
      o[2][j] = delta * uu;
      o[3][j] = dyy * zz * sg;
      o[4][j] = dyy * sg * (1.0f + zz * (1.0f - sg));
      o[5][j] = (WANT & S_SG) ? softplus_grad(v) : 0.0f;
    }
    const int off = r * CPB + 4 * q4;
#pragma unroll
    for (int k = 0; k < NSTAGE; ++k)
      if (WANT & (1u << k)) st4(st.arr[k] + off, make_float4(o[k][0], o[k][1], o[k][2], o[k][3]));
  }
  for (int t = threadIdx.x; t < nrows * 8; t += THREADS) {
    const int r = t >> 3, q4 = t & 7;
    st4(st.bc + r * 32 + 4 * q4, ld4(a.bc + (row0 + r) * a.ldbc + 4 * q4));
  }
}

// 1. + 3. Per chunk, from zero: H right to left (its end state and Σ Δ over
// the chunk) and G left to right (its end value and Σ Δ over positions
// s-1 … e-2, the decays it crosses), from one staging of the chunk.
__global__ void __launch_bounds__(THREADS) state_kernel(const Args a) {
  extern __shared__ float4 sm4[];
  const Lane l = lane_setup(a);
  const Stage sg = stage_layout(reinterpret_cast<float*>(sm4), a.T);
  stage_chunk<S_DL | S_DU | S_DP>(a, l, sg);
  const size_t ci = carry_idx(a, l);
  const int ch = threadIdx.x >> 2;
  const bool full = a.T == 16 && l.e - l.s == 16;
  float prev = 0.0f;                                   // Δ_{s-1}
  if (l.s > 0 && l.s < l.e) prev = softplus_fwd(a.dt[((size_t)l.b * a.L + l.s - 1) * a.E + l.c] + a.dt_b[l.c]);
  __syncthreads();
  {
    float2 H[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float sd = 0.0f;
    auto step = [&](int r) {
      const float delta = sg.arr[1][r * CPB + ch];
      const float2 du = dup2(sg.arr[2][r * CPB + ch]);
      const float4 Bq = ld4(sg.bc + r * 32 + 4 * l.q);
      sd += delta;
      float2 ad[2];
      decays(l, delta, ad);
      H[0] = __ffma2_rn(ad[0], H[0], __fmul2_rn(du, lo2(Bq)));
      H[1] = __ffma2_rn(ad[1], H[1], __fmul2_rn(du, hi2(Bq)));
    };
    if (full) {
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) step(15 - rr);
    } else {
      for (int r = l.e - l.s - 1; r >= 0; --r) step(r);
    }
    st4(a.hcar + ci * 16 + 4 * l.q, make_float4(H[0].x, H[0].y, H[1].x, H[1].y));
    if (l.q == 0) a.hsd[ci] = sd;
  }
  {
    float2 G[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float sd = 0.0f;
    auto step = [&](int r) {
      const float delta = sg.arr[1][r * CPB + ch];
      const float dp = sg.arr[3][r * CPB + ch];
      const float4 Cq = ld4(sg.bc + r * 32 + 16 + 4 * l.q);
      if (r > 0) {
        float2 ad[2];
        decays(l, prev, ad);
        G[0] = __fmul2_rn(G[0], ad[0]);
        G[1] = __fmul2_rn(G[1], ad[1]);
      }
      if (r > 0 || l.s > 0) sd += prev;
      G[0] = __ffma2_rn(dup2(dp), lo2(Cq), G[0]);
      G[1] = __ffma2_rn(dup2(dp), hi2(Cq), G[1]);
      prev = delta;
    };
    if (full) {
#pragma unroll
      for (int r = 0; r < 16; ++r) step(r);
    } else {
      for (int r = 0; r < l.e - l.s; ++r) step(r);
    }
    st4(a.gcar + ci * 16 + 4 * l.q, make_float4(G[0].x, G[0].y, G[1].x, G[1].y));
    if (l.q == 0) a.gsd[ci] = sd;
  }
}

// 2. + 4. Carries over the chunks of one (sequence, channel, state), for H
// (blockIdx.z = 0: right to left) and G (blockIdx.z = 1: left to right):
// buf[k] ← the value entering chunk k, running = buf_old[k] + exp(A·sd[k])·running.
__global__ void carry_kernel(const Args a) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // c·16 + m
  const int b = blockIdx.y;
  const bool rev = blockIdx.z == 0;
  float* buf = rev ? a.hcar : a.gcar;
  const float* sd = rev ? a.hsd : a.gsd;
  if (t >= (long long)a.E * 16) return;
  const int c = (int)(t >> 4), m = (int)(t & 15);
  const float A = -expf(a.A_log[(size_t)c * 16 + m]);
  float run = 0.0f;
  constexpr int PF = 8;                    // chunks whose loads are issued together
  for (int s0 = 0; s0 < a.nc; s0 += PF) {
    float old[PF], dec[PF];
#pragma unroll
    for (int j = 0; j < PF; ++j) {
      const int step = s0 + j;
      const int k = rev ? a.nc - 1 - step : step;
      const size_t ci = ((size_t)b * a.nc + (step < a.nc ? k : 0)) * a.E + c;
      old[j] = step < a.nc ? buf[ci * 16 + m] : 0.0f;
      dec[j] = step < a.nc ? sd[ci] : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < PF; ++j) {
      const int step = s0 + j;
      if (step < a.nc) {
        const int k = rev ? a.nc - 1 - step : step;
        buf[(((size_t)b * a.nc + k) * a.E + c) * 16 + m] = run;
        run = fmaf(expf(A * dec[j]), run, old[j]);
      }
    }
  }
}

// 5. Per chunk: H from H_in(k), right to left, keeping it at every second
// position (shared memory); then G from the carried value, left to right,
// two positions at a time: their H is recomputed in registers from the
// checkpoint on their right (with the decays the G steps reuse), and every
// gradient is formed.  TF = 16: a chunk of 16 valid positions, unrolled with
// static shared-memory offsets; TF = 0: any chunk (ragged ends, other chunk
// lengths).
template <int TF>
__device__ __forceinline__ void final_body(const Args& a, const Lane& l, const Stage& sg, float4* Hck, float* red,
                                           float4 Hr, float4 Gin, float (&aprev)[4], float (&dA)[4],
                                           float& dDacc, float& dbacc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ch = threadIdx.x >> 2;
  const int T = TF ? TF : a.T;
  const int nvalid = TF ? TF : l.e - l.s;                   // positions s … e-1
  const int nrows = TF ? TF : min(l.s + a.T, a.L) - l.s;    // rows of this chunk in the padded batch
  const float Dc = a.D[l.c];

  auto hcalc = [&](int r, const float4& Hright, float4& Hout, float2 (&ad)[2]) {
    const float delta = sg.arr[1][r * CPB + ch];
    const float2 du = dup2(sg.arr[2][r * CPB + ch]);
    const float4 Bq = ld4(sg.bc + r * 32 + 4 * l.q);
    decays(l, delta, ad);
    const float2 h0 = __ffma2_rn(ad[0], lo2(Hright), __fmul2_rn(du, lo2(Bq)));
    const float2 h1 = __ffma2_rn(ad[1], hi2(Hright), __fmul2_rn(du, hi2(Bq)));
    Hout = make_float4(h0.x, h0.y, h1.x, h1.y);
  };

  // H over the chunk, right to left, kept at the even positions 2, 4, …
  {
    float4 H = Hr;
    auto hstep = [&](int r) {
      float2 ad[2];
      hcalc(r, H, H, ad);
      if ((r & 1) == 0) Hck[(r >> 1) * THREADS + threadIdx.x] = H;
    };
    if constexpr (TF > 0) {
#pragma unroll
      for (int rr = 0; rr < TF - 2; ++rr) hstep(TF - 1 - rr);
    } else {
      for (int r = nvalid - 1; r >= 2; --r) hstep(r);
    }
  }

  float2 G[2] = {lo2(Gin), hi2(Gin)};
  float2 ap[2] = {make_float2(aprev[0], aprev[1]), make_float2(aprev[2], aprev[3])};
  float2 dAp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  // this lane's column of dB | dC after the reduce-scatter: value index
  // vi = 4·bit4 + 2·bit3 + bit2 of the lane → (vi < 4 ? 0 : 16) + 4q + (vi & 3)
  const int vi = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
  const int col = (vi < 4 ? 0 : 16) + 4 * l.q + (vi & 3);
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float* redw = red + (size_t)warp * T * 32 + col;
  // thread q of a channel leaves one per-position gradient in shared memory,
  // over the staged input it no longer needs: du over Δu (q = 0), ddt_raw
  // over softplus' (q = 1), dz over the dz factor (q = 2)
  float* outq = l.q == 0 ? sg.arr[2] : l.q == 1 ? sg.arr[5] : sg.arr[4];
  auto gstep = [&](int r, const float4& Hi, const float4& Hn, const float2 (&ai)[2]) {
    const float uu = sg.arr[0][r * CPB + ch];
    const float delta = sg.arr[1][r * CPB + ch];
    const float du_ = sg.arr[2][r * CPB + ch];
    const float dp = sg.arr[3][r * CPB + ch];
    const float fz = sg.arr[4][r * CPB + ch];
    const float spg = sg.arr[5][r * CPB + ch];
    const float4 Bq = ld4(sg.bc + r * 32 + 4 * l.q);
    const float4 Cq = ld4(sg.bc + r * 32 + 16 + 4 * l.q);
    const float2 dp2 = dup2(dp);
    G[0] = __ffma2_rn(ap[0], G[0], __fmul2_rn(dp2, lo2(Cq)));
    G[1] = __ffma2_rn(ap[1], G[1], __fmul2_rn(dp2, hi2(Cq)));
    const float2 pc2 = __ffma2_rn(hi2(Hi), hi2(Cq), __fmul2_rn(lo2(Hi), lo2(Cq)));
    const float2 gh0 = __fmul2_rn(__fmul2_rn(G[0], lo2(Hn)), ai[0]);
    const float2 gh1 = __fmul2_rn(__fmul2_rn(G[1], hi2(Hn)), ai[1]);
    const float2 sa2 = __ffma2_rn(gh1, l.Ap[1], __fmul2_rn(gh0, l.Ap[0]));
    const float2 sb2 = __ffma2_rn(G[1], hi2(Bq), __fmul2_rn(G[0], lo2(Bq)));
    const float2 d2 = dup2(delta);
    dAp[0] = __ffma2_rn(d2, gh0, dAp[0]);
    dAp[1] = __ffma2_rn(d2, gh1, dAp[1]);
    const float pc = sum4(pc2.x + pc2.y);
    const float sa = sum4(sa2.x + sa2.y);
    const float sb = sum4(sb2.x + sb2.y);
    const float p = fmaf(Dc, uu, pc);
    const float ddt = fmaf(sb, uu, sa) * spg;
    dDacc = fmaf(dp, uu, dDacc);
    dbacc += ddt;
    // dB (values 0-3) and dC (values 4-7) of states 4q … 4q+3, summed over
    // the warp's 8 channels by a reduce-scatter on lane bits 4, 3, 2
    const float2 gb0 = __fmul2_rn(G[0], dup2(du_)), gb1 = __fmul2_rn(G[1], dup2(du_));
    const float2 hc0 = __fmul2_rn(dp2, lo2(Hi)), hc1 = __fmul2_rn(dp2, hi2(Hi));
    const float vv[8] = {gb0.x, gb0.y, gb1.x, gb1.y, hc0.x, hc0.y, hc1.x, hc1.y};
    float w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float send = b4 ? vv[t] : vv[t + 4];
      const float keep = b4 ? vv[t + 4] : vv[t];
      w[t] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float x[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const float send = b3 ? w[t] : w[t + 2];
      const float keep = b3 ? w[t + 2] : w[t];
      x[t] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const float send = b2 ? x[0] : x[1];
    const float keep = b2 ? x[1] : x[0];
    redw[r * 32] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    const float outv = l.q == 0 ? fmaf(Dc, dp, delta * sb) : l.q == 1 ? ddt : p * fz;
    if (l.q < 3) outq[r * CPB + ch] = outv;
    ap[0] = ai[0];
    ap[1] = ai[1];
  };
  // positions r0 and r0 + 1 (the latter if valid): H_{r0+2} from the
  // checkpoint (H entering the chunk from the right past its end)
  auto pair = [&](int r0) {
    const bool two = r0 + 1 < nvalid;
    const float4 Hright = (r0 + 2 < nvalid) ? Hck[((r0 + 2) >> 1) * THREADS + threadIdx.x] : Hr;
    float4 H1 = Hright, H0;
    float2 a1[2], a0[2];
    if (two) hcalc(r0 + 1, Hright, H1, a1);
    hcalc(r0, H1, H0, a0);
    gstep(r0, H0, H1, a0);
    if (two) gstep(r0 + 1, H1, Hright, a1);
  };
  if constexpr (TF > 0) {
#pragma unroll
    for (int r0 = 0; r0 < TF; r0 += 2) pair(r0);
  } else {
    for (int r0 = 0; r0 < nvalid; r0 += 2) pair(r0);
    for (int r = nvalid > 0 ? nvalid : 0; r < nrows; ++r) {   // padding rows of the chunk
      if (l.q < 3) outq[r * CPB + ch] = 0.0f;
      redw[r * 32] = 0.0f;
    }
  }
  dA[0] = dAp[0].x; dA[1] = dAp[0].y; dA[2] = dAp[1].x; dA[3] = dAp[1].y;
}

__global__ void __launch_bounds__(THREADS, 3) final_kernel(const Args a) {
  extern __shared__ float4 sm4[];
  float4* Hs = sm4;                            // [(T+1)/2][THREADS]: H at positions 2, 4, … (index r/2)
  float* red = reinterpret_cast<float*>(sm4 + (size_t)((a.T + 1) / 2) * THREADS);   // [WARPS][T][32]
  const Lane l = lane_setup(a);
  const Stage sg = stage_layout(red + (size_t)WARPS * a.T * 32, a.T);
  stage_chunk<S_U | S_DL | S_DU | S_DP | S_FZ | S_SG>(a, l, sg);
  const size_t ci = carry_idx(a, l);
  const float4 Hr = ld4(a.hcar + ci * 16 + 4 * l.q);             // H_e, entering from the right
  const float4 Gin = ld4(a.gcar + ci * 16 + 4 * l.q);            // G_{s-1}, entering from the left
  float aprev[4] = {0.f, 0.f, 0.f, 0.f};                         // G_{-1} = 0 at s = 0
  if (l.s > 0 && l.s < l.e) {
    const float dprev = softplus_fwd(a.dt[((size_t)l.b * a.L + l.s - 1) * a.E + l.c] + a.dt_b[l.c]);
#pragma unroll
    for (int j = 0; j < 4; ++j) aprev[j] = exp2_mufu(dprev * l.A2[j]);
  }
  __syncthreads();
  float dA[4] = {0.f, 0.f, 0.f, 0.f};
  float dDacc = 0.0f, dbacc = 0.0f;
  if (a.T == 16 && l.e - l.s == 16)
    final_body<16>(a, l, sg, Hs, red, Hr, Gin, aprev, dA, dDacc, dbacc);
  else
    final_body<0>(a, l, sg, Hs, red, Hr, Gin, aprev, dA, dDacc, dbacc);
  __syncthreads();
  // the per-position gradients, [rows × 64 channels] each, as float4 rows
  const int T = a.T;
  const int nrows = min(l.s + T, a.L) - l.s;
  {
    const size_t row0 = (size_t)l.b * a.L + l.s;
    const int col0 = blockIdx.x * CPB;
    for (int t = threadIdx.x; t < nrows * (CPB / 4); t += THREADS) {
      const int r = t / (CPB / 4), q4 = t % (CPB / 4);
      const int off = r * CPB + 4 * q4;
      const size_t row = row0 + r;
      st4(a.du + row * a.E + col0 + 4 * q4, ld4(sg.arr[2] + off));
      st4(a.ddt + row * a.E + col0 + 4 * q4, ld4(sg.arr[5] + off));
      st4(a.dz + row * a.ld_dz + col0 + 4 * q4, ld4(sg.arr[4] + off));
    }
  }
  // fixed-order sum over the block's warps → per-block partial of dB | dC
  for (int t = threadIdx.x; t < nrows * 32; t += THREADS) {
    const int rr = t >> 5, cc = t & 31;
    float acc = 0.0f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) acc += red[((size_t)w * T + rr) * 32 + cc];
    a.pbc[((size_t)blockIdx.x * a.B * a.L + (size_t)l.b * a.L + l.s + rr) * 32 + cc] = acc;
  }
  st4(a.pA + ci * 16 + 4 * l.q, make_float4(dA[0], dA[1], dA[2], dA[3]));
  if (l.q == 0) {
    a.pD[ci] = dDacc;
    a.pb[ci] = dbacc;
  }
}

// 6a. dA_log, dD, ddt_b: sums over the B·nc (sequence, chunk) partials in a
// fixed order, in two levels: segment g of RSEG consecutive partials is
// summed by block row g into seg[g], then the segments in order.
constexpr int RSEG = 32;

__global__ void reduce_params_seg_kernel(const Args a, float* seg) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // c·16 + m
  if (t >= (long long)a.E * 16) return;
  const int c = (int)(t >> 4), m = (int)(t & 15);
  const long long cells = (long long)a.B * a.nc;
  const long long p0 = (long long)blockIdx.y * RSEG;
  float sA = 0.0f, sD = 0.0f, sb = 0.0f;
#pragma unroll 8
  for (int j = 0; j < RSEG; ++j) {
    const long long p = p0 + j;                 // p = b·nc + k
    if (p < cells) {
      const size_t ci = (size_t)p * a.E + c;
      sA += a.pA[ci * 16 + m];
      if (m == 0) {
        sD += a.pD[ci];
        sb += a.pb[ci];
      }
    }
  }
  const size_t o = ((size_t)blockIdx.y * a.E * 16 + t) * 3;
  seg[o] = sA;
  seg[o + 1] = sD;
  seg[o + 2] = sb;
}

__global__ void reduce_params_kernel(const Args a, const float* seg, int nseg) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // c·16 + m
  if (t >= (long long)a.E * 16) return;
  const int c = (int)(t >> 4), m = (int)(t & 15);
  float sA = 0.0f, sD = 0.0f, sb = 0.0f;
  for (int g = 0; g < nseg; ++g) {
    const size_t o = ((size_t)g * a.E * 16 + t) * 3;
    sA += seg[o];
    sD += seg[o + 1];
    sb += seg[o + 2];
  }
  a.dA_log[(size_t)c * 16 + m] = sA * -expf(a.A_log[(size_t)c * 16 + m]);
  if (m == 0) {
    a.dD[c] = sD;
    a.ddt_b[c] = sb;
  }
}

// 6b. dB | dC: sum of the per-block partials in a fixed order (four
// interleaved running sums over the blocks, cb ≡ 0, 1, 2, 3 mod 4, then
// combined pairwise), so four loads per thread are in flight.
__global__ void reduce_bc_kernel(const Args a) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // row·32 + col
  const long long M = (long long)a.B * a.L;
  if (t >= M * 32) return;
  const long long row = t >> 5;
  const int col = (int)(t & 31);
  const int nb = a.nbc;
  const float* p = a.pbc + row * 32 + col;
  const size_t stride = (size_t)M * 32;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  int cb = 0;
  for (; cb + 4 <= nb; cb += 4) {
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += p[(size_t)(cb + i) * stride];
  }
#pragma unroll
  for (int i = 0; i < 3; ++i)
    if (cb + i < nb) acc[i] += p[(size_t)(cb + i) * stride];
  a.dbc[row * a.ld_dbc + col] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

}  // namespace sbwd
}  // namespace r2l

#include "scan_bwd_seq.cuh"

namespace r2l {

// The walk along each sequence (scan_bwd_seq.cuh) runs when the chunk length
// is left to the library and one 32-channel block per (sequence, block) gives
// the GPU at least four blocks per SM; otherwise the chunked kernels above.
static bool use_seq(int B, int E, int chunk_tokens) {
  return chunk_tokens == 0 && (long long)B * (E / sbwd::QC) >= 4LL * 148;
}

bool scan_bwd_walks(int B, int E, int chunk_tokens) { return use_seq(B, E, chunk_tokens); }

int scan_bwd_chunk_tokens(int chunk_tokens) {
  if (chunk_tokens <= 0) return 16;
  return chunk_tokens > SCAN_BWD_MAX_CHUNK ? SCAN_BWD_MAX_CHUNK : chunk_tokens;
}

bool scan_bwd_supported(int B, int L, int E, int chunk_tokens) {
  if (use_seq(B, E, chunk_tokens)) return E % sbwd::QC == 0 && B <= 65535;
  const int T = scan_bwd_chunk_tokens(chunk_tokens);
  const long long nc = (L + T - 1) / T;
  const long long nseg = ((long long)B * nc + sbwd::RSEG - 1) / sbwd::RSEG;
  return E % sbwd::CPB == 0 && nc <= 65535 && B <= 65535 && nseg <= 65535;
}

size_t scan_bwd_scratch_bytes(int B, int L, int E, int chunk_tokens) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  if (use_seq(B, E, chunk_tokens)) {
    const size_t nc = (size_t)((L + sbwd::QS - 1) / sbwd::QS);
    return al((size_t)B * nc * E * 16 * 4) + al((size_t)B * E * 16 * 4) + 2 * al((size_t)B * E * 4) +
           al((size_t)(E / sbwd::QC) * B * L * 32 * 4);
  }
  const int T = scan_bwd_chunk_tokens(chunk_tokens);
  const size_t nc = (size_t)((L + T - 1) / T);
  const size_t cells = (size_t)B * nc * E;
  const size_t nseg = (cells / E + sbwd::RSEG - 1) / sbwd::RSEG;
  return al(cells * 16 * 4) * 3 + al(cells * 4) * 4 + al((size_t)(E / sbwd::CPB) * B * L * 32 * 4) +
         al(nseg * E * 16 * 3 * 4);
}

cudaError_t scan_bwd_f32(const ScanBwdArgs& g, void* scratch, cudaStream_t st) {
  using namespace sbwd;
  Args a{};
  a.u = g.u; a.z = g.z; a.u16 = g.u16; a.z16 = g.z16; a.ldz = g.ldz; a.dt = g.dt_raw; a.bc = g.bc; a.ldbc = g.ldbc;
  a.A_log = g.A_log; a.D = g.D; a.dt_b = g.dt_b; a.dy = g.dy;
  a.du = g.du; a.dz = g.dz; a.ld_dz = g.ld_dz; a.ddt = g.ddt_raw; a.dbc = g.dbc; a.ld_dbc = g.ld_dbc;
  a.dA_log = g.dA_log; a.dD = g.dD; a.ddt_b = g.ddt_b;
  a.B = g.B; a.L = g.L; a.E = g.E;
  a.T = scan_bwd_chunk_tokens(g.chunk_tokens);
  a.nc = (g.L + a.T - 1) / a.T;
  a.lengths = g.lengths;
  a.status = g.status;
  for (int m = 0; m < 16; ++m) {
    const float v = (float)std::log((double)(m + 1));
    std::memcpy(&a.lnbits[m], &v, sizeof(v));
  }
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  const long long M = (long long)g.B * g.L;
  if (use_seq(g.B, g.E, g.chunk_tokens)) {
    a.T = QS;
    a.nc = (g.L + QS - 1) / QS;
    char* p = (char*)scratch;
    a.ddt16 = g.ddt16; a.ld_ddt16 = g.ld_ddt16; a.dz16 = g.dz16; a.ld_dz16 = g.ld_dz16;
    a.hcar = g.hck ? g.hck : (float*)p;
    a.ckpt_ragged_only = g.hck ? 1 : 0;
    p += al((size_t)g.B * a.nc * g.E * 16 * 4);
    a.pA = (float*)p;   p += al((size_t)g.B * g.E * 16 * 4);
    a.pD = (float*)p;   p += al((size_t)g.B * g.E * 4);
    a.pb = (float*)p;   p += al((size_t)g.B * g.E * 4);
    a.pbc = (float*)p;
    a.nbc = g.E / QC;
    const dim3 grid(g.E / QC, g.B);
    seq_ckpt_kernel<<<grid, QT, 0, st>>>(a);
    seq_final_kernel<<<grid, QT, 0, st>>>(a);
    seq_reduce_params_kernel<<<(unsigned)((g.E * 16 + 255) / 256), 256, 0, st>>>(a);
    reduce_bc_kernel<<<(unsigned)((M * 32 + 255) / 256), 256, 0, st>>>(a);
    return cudaPeekAtLastError();
  }
  const size_t cells = (size_t)g.B * a.nc * g.E;
  char* p = (char*)scratch;
  a.hcar = (float*)p; p += al(cells * 16 * 4);
  a.gcar = (float*)p; p += al(cells * 16 * 4);
  a.pA = (float*)p;   p += al(cells * 16 * 4);
  a.hsd = (float*)p;  p += al(cells * 4);
  a.gsd = (float*)p;  p += al(cells * 4);
  a.pD = (float*)p;   p += al(cells * 4);
  a.pb = (float*)p;   p += al(cells * 4);
  a.pbc = (float*)p;  p += al((size_t)(g.E / CPB) * g.B * g.L * 32 * 4);
  a.nbc = g.E / CPB;
  float* seg = (float*)p;
  const int nseg = (int)(((size_t)g.B * a.nc + RSEG - 1) / RSEG);

  const dim3 grid(g.E / CPB, a.nc, g.B);
  const dim3 cgrid((unsigned)((g.E * 16 + 255) / 256), g.B, 2);
  const size_t ssmem = stage_floats(a.T) * sizeof(float);
  const size_t fsmem =
      (size_t)((a.T + 1) / 2) * THREADS * sizeof(float4) + (size_t)WARPS * a.T * 32 * sizeof(float) + ssmem;
  cudaError_t e = cudaFuncSetAttribute(final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsmem);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem)) !=
      cudaSuccess)
    return e;
  state_kernel<<<grid, THREADS, ssmem, st>>>(a);
  carry_kernel<<<cgrid, 256, 0, st>>>(a);
  final_kernel<<<grid, THREADS, fsmem, st>>>(a);
  reduce_params_seg_kernel<<<dim3((unsigned)((g.E * 16 + 255) / 256), nseg), 256, 0, st>>>(a, seg);
  reduce_params_kernel<<<(unsigned)((g.E * 16 + 255) / 256), 256, 0, st>>>(a, seg, nseg);
  reduce_bc_kernel<<<(unsigned)((M * 32 + 255) / 256), 256, 0, st>>>(a);
  return cudaPeekAtLastError();
}

}  // namespace r2l
