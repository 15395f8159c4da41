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

#include <type_traits>

#include "common.cuh"

namespace r2l {
namespace bwd {

constexpr int ROW_CHUNK = 64;      // positions per partial sum of a column reduction

__device__ __forceinline__ bool valid_row(const int* len, int L, long long m) {
  return len == nullptr || row_valid(len, L, m);
}

// Eight consecutive elements (16-byte aligned) widened to fp32, and eight
// fp32 values rounded to bf16 as one 16-byte vector.
__device__ __forceinline__ void load8(const bf16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  return q;
}

// One 64 × 64 tile of in[m, c] (rows m0 … m0+63, columns c0 … c0+63) rounded
// to bf16: to out[m, c] (when out is not null) and to its transpose outT[c, m]
// (when outT is not null).  Padding rows (m ≥ M, or position ≥ the sequence's
// length) are written as 0 in both; the grid runs over max(M, ldT) rows, so the
// columns M … ldT−1 of outT are zero too.  C, the leading dimensions and the
// base addresses are multiples of 8 elements: every access is a 16-byte vector
// (two for fp32 input), every row of a warp's accesses a whole 128-byte line.
template <typename TIn>
__global__ void __launch_bounds__(256) cvt_transpose_kernel(const TIn* __restrict__ in, long long ld_in, long long M,
                                                            int C, bf16* __restrict__ out, long long ld_out,
                                                            bf16* __restrict__ outT, long long ldT,
                                                            const int* __restrict__ len, int L) {
  __shared__ float tile[64][65];
  const long long m0 = (long long)blockIdx.y * 64;
  const int c0 = blockIdx.x * 64;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int g = threadIdx.x + 256 * k;
    const int r = g >> 3, cg = (g & 7) * 8;
    const long long m = m0 + r;
    const int c = c0 + cg;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (m < M && c < C && valid_row(len, L, m)) load8(in + m * ld_in + c, v);
    if (out != nullptr && m < M && c < C) *reinterpret_cast<uint4*>(out + m * ld_out + c) = pack8(v);
#pragma unroll
    for (int i = 0; i < 8; ++i) tile[r][cg + i] = v[i];
  }
  if (outT == nullptr) return;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int g = threadIdx.x + 256 * k;
    const int cc = g >> 3, rg = (g & 7) * 8;
    const int c = c0 + cc;
    const long long m = m0 + rg;
    if (c < C && m < ldT) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = tile[rg + i][cc];
      *reinterpret_cast<uint4*>(outT + (long long)c * ldT + m) = pack8(v);
    }
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

// Sequence and position of row m0, for walking rows m0, m0+1, … without a
// division per row.
struct RowWalk {
  long long b;
  int i, n, L;
  const int* len;
  long long m, M;
  __device__ __forceinline__ RowWalk(const int* len_, int L_, long long m0, long long M_)
      : len(len_), L(L_), m(m0), M(M_) {
    b = m0 >= 0 ? m0 / L_ : -((-m0 + L_ - 1) / L_);
    i = (int)(m0 - b * L_);
    n = (b >= 0 && m0 < M_) ? (len_ ? len_[b] : L_) : 0;
  }
  __device__ __forceinline__ bool valid() const { return b >= 0 && m < M && i < n; }
  __device__ __forceinline__ void next() {
    ++m;
    if (++i == L) {
      i = 0;
      ++b;
      n = m < M ? (len ? len[b] : L) : 0;
    }
  }
};

// The same with the row held in registers, for d = 256·NK: lane ℓ takes the
// 8-column groups 8ℓ + 256k (k < NK), read once as 16-byte vectors.
template <bool HAS_LN, int NK>
__global__ void __launch_bounds__(256) ln_gate_bwd_rows_reg_kernel(const bf16* __restrict__ o,
                                                                   const float* __restrict__ dh_out,
                                                                   const float* __restrict__ gamma,
                                                                   const float* __restrict__ beta, float g, int d,
                                                                   const int* __restrict__ len, int L, long long M,
                                                                   float2* __restrict__ stats,
                                                                   float* __restrict__ ds_row,
                                                                   bf16* __restrict__ dout) {
  const long long m = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  bf16* drow = dout + m * d;
  if (!valid_row(len, L, m)) {
#pragma unroll
    for (int k = 0; k < NK; ++k)
      *reinterpret_cast<uint4*>(drow + 8 * lane + 256 * k) = make_uint4(0u, 0u, 0u, 0u);
    if (lane == 0) {
      ds_row[m] = 0.0f;
      stats[m] = make_float2(0.0f, 0.0f);
    }
    return;
  }
  float ov[NK][8], gv[NK][8];
#pragma unroll
  for (int k = 0; k < NK; ++k) {
    const int j = 8 * lane + 256 * k;
    load8(o + m * d + j, ov[k]);
    load8(dh_out + m * d + j, gv[k]);
  }
  float mu = 0.0f, rstd = 1.0f;
  if (HAS_LN) {
    float sum = 0.0f;
#pragma unroll
    for (int k = 0; k < NK; ++k)
#pragma unroll
      for (int i = 0; i < 8; ++i) sum += ov[k][i];
#pragma unroll
    for (int x = 16; x; x >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, x);
    mu = sum / (float)d;
    float q = 0.0f;
#pragma unroll
    for (int k = 0; k < NK; ++k)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float t = ov[k][i] - mu;
        q += t * t;
      }
#pragma unroll
    for (int x = 16; x; x >>= 1) q += __shfl_xor_sync(0xffffffffu, q, x);
    rstd = rsqrtf(q / (float)d + 1e-5f);
  }
  float sh = 0.0f, s1 = 0.0f, s2 = 0.0f;
#pragma unroll
  for (int k = 0; k < NK; ++k) {
    const int j = 8 * lane + 256 * k;
    if (HAS_LN) {
      float gm[8], bt[8];
      load8(gamma + j, gm);
      load8(beta + j, bt);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float nh = (ov[k][i] - mu) * rstd;
        sh += gv[k][i] * (gm[i] * nh + bt[i]);
        const float gg = g * gv[k][i] * gm[i];
        s1 += gg;
        s2 += gg * nh;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) sh += gv[k][i] * ov[k][i];
    }
  }
#pragma unroll
  for (int x = 16; x; x >>= 1) {
    sh += __shfl_xor_sync(0xffffffffu, sh, x);
    s1 += __shfl_xor_sync(0xffffffffu, s1, x);
    s2 += __shfl_xor_sync(0xffffffffu, s2, x);
  }
  const float m1 = s1 / (float)d, m2 = s2 / (float)d;
#pragma unroll
  for (int k = 0; k < NK; ++k) {
    const int j = 8 * lane + 256 * k;
    float dv[8];
    if (HAS_LN) {
      float gm[8];
      load8(gamma + j, gm);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float nh = (ov[k][i] - mu) * rstd;
        dv[i] = rstd * (gm[i] * (g * gv[k][i]) - m1 - nh * m2);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) dv[i] = g * gv[k][i];
    }
    *reinterpret_cast<uint4*>(drow + j) = pack8(dv);
  }
  if (lane == 0) {
    ds_row[m] = sh;
    stats[m] = make_float2(mu, rstd);
  }
}

// ❸ column sums, chunk y of ROW_CHUNK rows: dγ and dβ partials
// part[y][0][j] = Σ ĝ ⊙ n̂, part[y][1][j] = Σ ĝ over the chunk's valid rows.
// Each thread takes four columns (one 16-byte load of dh⁺, one 8-byte load of o
// per row).
__global__ void __launch_bounds__(128) ln_bwd_cols_kernel(const bf16* __restrict__ o, const float* __restrict__ dh_out,
                                                          float g, int d, const int* __restrict__ len, int L,
                                                          long long M, const float2* __restrict__ stats,
                                                          float* __restrict__ part) {
  const int j = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (j >= d) return;
  const long long r0 = (long long)blockIdx.y * ROW_CHUNK;
  const long long r1 = r0 + ROW_CHUNK < M ? r0 + ROW_CHUNK : M;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bs = a;
  RowWalk w(len, L, r0, M);
  for (long long m = r0; m < r1; ++m, w.next()) {
    if (!w.valid()) continue;
    const float2 st = stats[m];
    const float4 gv = *reinterpret_cast<const float4*>(dh_out + m * d + j);
    const uint2 ov = *reinterpret_cast<const uint2*>(o + m * d + j);
    const float2 o01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov.x));
    const float2 o23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov.y));
    a.x += g * gv.x * ((o01.x - st.x) * st.y);
    a.y += g * gv.y * ((o01.y - st.x) * st.y);
    a.z += g * gv.z * ((o23.x - st.x) * st.y);
    a.w += g * gv.w * ((o23.y - st.x) * st.y);
    bs.x += g * gv.x;
    bs.y += g * gv.y;
    bs.z += g * gv.z;
    bs.w += g * gv.w;
  }
  *reinterpret_cast<float4*>(part + ((long long)blockIdx.y * 2 + 0) * d + j) = a;
  *reinterpret_cast<float4*>(part + ((long long)blockIdx.y * 2 + 1) * d + j) = bs;
}

// Column sums of chunk partials part[p][col] (p = 0 … nparts−1, C columns), in
// a fixed order: 256 threads = 32 columns × 8 interleaved subsets p ≡ s (mod 8),
// each summed in order, then the 8 subsets in order.  MODE 0: col < C0 → o0[col],
// else o1[col − C0].  MODE 1 (the conv's [5][E] layout, C0 = E): tap k < 4 →
// o0[c·4 + 3 − k], k = 4 → o1[c].
template <int MODE>
__global__ void __launch_bounds__(256) chunk_sum_kernel(const float* __restrict__ part, int nparts, int C, int C0,
                                                        float* __restrict__ o0, float* __restrict__ o1) {
  __shared__ float sh[8][33];
  const int cl = threadIdx.x & 31, sub = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + cl;
  float s = 0.0f;
  if (col < C)
    for (int p = sub; p < nparts; p += 8) s += part[(long long)p * C + col];
  sh[sub][cl] = s;
  __syncthreads();
  if (sub != 0 || col >= C) return;
  float t = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) t += sh[k][cl];
  if (MODE == 0) {
    if (col < C0) o0[col] = t; else o1[col - C0] = t;
  } else {
    const int k = col / C0, c = col - k * C0;
    if (k < 4) o0[c * 4 + 3 - k] = t; else o1[c] = t;
  }
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

// 16 bytes global → shared without registers (cp.async); zeros when !valid.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(sa), "l"(gmem), "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n" ::);
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

// conv + SiLU, over a tile of 32 rows × 128 channels.  With W = 4 taps,
// w_k = conv_w[c][W−1−k] multiplying x_{i+k}:
//   pre_i  = conv_b + Σ_k w_k·x_{i+k}   (x_j = 0 for j ≥ the sequence's length)
//   dpre_i = (du_s + du_x)_i · SiLU'(pre_i)   (0 on padding rows)
//   dx_j   = Σ_k w_k·dpre_{j−k}   (k ≤ j: the same sequence)
// The block first stages x (rows m0−3 … m0+34), du_s and du_x (rows m0−3 …
// m0+31) in shared memory by 16-byte asynchronous copies, all in flight at
// once, padding rows as zero.  Thread (p, grp) then takes the channel pair c,
// c+1 (c = 2p within the tile) and rows r0 = m0 + 16·grp … r0+15; dpre of the
// three rows above r0 is recomputed, so every tile is independent.  dx goes out
// as bf16 twice: into dxz (row-major) and into dxzT[c][r0 …] (its transpose, 16
// consecutive positions per channel: two 16-byte stores).  The chunk's
// parameter partials part[y][k][c] = Σ dpre_i·x_{i+k} (tap W−1−k) and
// part[y][4][c] = Σ dpre_i are summed over the row groups in order.
constexpr int CONV_ROWS = 32;
constexpr int CONV_GRP = CONV_ROWS / 16;          // 16-row groups: threads (p, grp)
constexpr int CONV_THREADS = 64 * CONV_GRP;
constexpr int CONV_CH = 128;
constexpr int CONV_XROWS = CONV_ROWS + 6;
constexpr int CONV_DROWS = CONV_ROWS + 3;
constexpr size_t CONV_SMEM = 2 * (size_t)CONV_DROWS * 64 * sizeof(float2) + (size_t)CONV_XROWS * 64 * 4;

__global__ void __launch_bounds__(CONV_THREADS) conv_bwd_kernel(
    const bf16* __restrict__ x, long long ldx, const float* __restrict__ conv_w, const float* __restrict__ conv_b,
    const float* __restrict__ du_s, const float* __restrict__ du_x, int E, const int* __restrict__ len, int L,
    long long M, bf16* __restrict__ dxz, long long lddxz, bf16* __restrict__ dxzT, long long ldT,
    float* __restrict__ part) {
  constexpr int NR = 16, HALO = 3, NQ = NR + 2 * HALO, ND = NR + HALO;
  extern __shared__ float4 conv_sm[];
  float2* gs = reinterpret_cast<float2*>(conv_sm);                          // du_s [CONV_DROWS][64 pairs]
  float2* gx = gs + CONV_DROWS * 64;                                          // du_x [CONV_DROWS][64 pairs]
  __nv_bfloat162* xs = reinterpret_cast<__nv_bfloat162*>(gx + CONV_DROWS * 64);   // x [CONV_XROWS][64 pairs]
  float2* red = gs;                                                          // [4][64][5], after the compute
  __shared__ unsigned char rowok[CONV_XROWS];
  const int c0 = blockIdx.x * CONV_CH;
  const int nch = min(CONV_CH, E - c0);                  // E is a multiple of 64, not always of 128
  const long long m0 = (long long)blockIdx.y * CONV_ROWS;

  // ---- staging
  if (threadIdx.x < CONV_XROWS) {
    const long long m = m0 - HALO + threadIdx.x;
    rowok[threadIdx.x] = m >= 0 && m < M && valid_row(len, L, m);
  }
  __syncthreads();
  for (int k = threadIdx.x; k < CONV_XROWS * 16; k += CONV_THREADS) {   // x: 16 × 16 B per row
    const int r = k >> 4, q = k & 15;
    const bool ok = rowok[r] && 8 * q < nch;
    const long long m = ok ? m0 - HALO + r : 0;
    cp_async16(xs + r * 64 + 4 * q, x + m * ldx + (ok ? c0 + 8 * q : 0), ok);
  }
  for (int k = threadIdx.x; k < CONV_DROWS * 32; k += CONV_THREADS) {   // du_s, du_x: 32 × 16 B per row
    const int r = k >> 5, q = k & 31;
    const bool ok = rowok[r] && 4 * q < nch;
    const long long off = ok ? (m0 - HALO + r) * E + c0 + 4 * q : 0;
    cp_async16(gs + r * 64 + 2 * q, du_s + off, ok);
    cp_async16(gx + r * 64 + 2 * q, du_x + off, ok);
  }
  cp_async_wait_all();
  __syncthreads();

  const int p = threadIdx.x & 63, grp = threadIdx.x >> 6;
  const int c = c0 + 2 * p;
  const bool live = 2 * p < nch;
  const int cw = live ? c : c0;
  const float4 wa = *reinterpret_cast<const float4*>(conv_w + (size_t)cw * 4);
  const float4 wb = *reinterpret_cast<const float4*>(conv_w + (size_t)(cw + 1) * 4);
  const float2 wk[4] = {make_float2(wa.w, wb.w), make_float2(wa.z, wb.z), make_float2(wa.y, wb.y),
                        make_float2(wa.x, wb.x)};
  const float2 bias = *reinterpret_cast<const float2*>(conv_b + cw);
  const long long r0 = m0 + NR * grp;
  const int rs = NR * grp;                               // the thread's first halo row in the staged tiles

  // per row t = 0 … NQ−1 (row r0 − 3 + t): valid and start-of-sequence bits
  unsigned vmask = 0, smask = 0;
  {
    RowWalk w(len, L, r0 - HALO, M);
#pragma unroll
    for (int t = 0; t < NQ; ++t, w.next()) {
      if (live && w.valid()) vmask |= 1u << t;
      if (w.i == 0) smask |= 1u << t;
    }
  }
  // rows t and t+k (k ≤ 3) are in the same sequence when no row in (t, t+k] starts one
  auto same = [&](int t, int k) { return ((smask >> (t + 1)) & ((1u << k) - 1u)) == 0u; };
  auto xv = [&](int t) { return __bfloat1622float2(xs[(rs + t) * 64 + p]); };

  float2 pw[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 pb = make_float2(0.f, 0.f);
  uint32_t packA[NR / 2], packB[NR / 2];                  // dx of channels c, c+1 as bf16 pairs of rows
  // SiLU'(v) = σ(v)·(1 + v·(1 − σ(v))), σ from the hardware exponential and reciprocal
  auto dsilu = [](float v) {
    const float sg = __fdividef(1.0f, 1.0f + __expf(-v));
    return sg * (1.0f + v * (1.0f - sg));
  };
  // CROSS: the window of rows crosses the start of a sequence, so every tap is
  // tested; otherwise all its rows belong to one sequence (padding rows are zero).
  auto rows = [&](auto cross_tag) {
    constexpr bool CROSS = decltype(cross_tag)::value;
    float2 dp[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                    make_float2(0.f, 0.f)};               // dpre at rows t, t−1, t−2, t−3
#pragma unroll
    for (int t = 0; t < ND; ++t) {
      float2 pre = bias;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (!CROSS || same(t, k)) {
          const float2 xx = xv(t + k);
          pre.x = fmaf(wk[k].x, xx.x, pre.x);
          pre.y = fmaf(wk[k].y, xx.y, pre.y);
        }
      float2 d = make_float2(0.f, 0.f);
      if (vmask & (1u << t)) {
        const float2 ga = gs[(rs + t) * 64 + p], gb = gx[(rs + t) * 64 + p];
        d.x = (ga.x + gb.x) * dsilu(pre.x);
        d.y = (ga.y + gb.y) * dsilu(pre.y);
      }
      dp[3] = dp[2];
      dp[2] = dp[1];
      dp[1] = dp[0];
      dp[0] = d;
      if (t >= HALO) {
        const int s = t - HALO;                           // output row r0 + s
        float2 dx = make_float2(0.f, 0.f);
        if (vmask & (1u << t)) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (!CROSS || k == 0 || same(t - k, k)) {
              dx.x = fmaf(wk[k].x, dp[k].x, dx.x);
              dx.y = fmaf(wk[k].y, dp[k].y, dx.y);
            }
          pb.x += d.x;
          pb.y += d.y;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (!CROSS || same(t, k)) {
              const float2 xx = xv(t + k);
              pw[k].x = fmaf(d.x, xx.x, pw[k].x);
              pw[k].y = fmaf(d.y, xx.y, pw[k].y);
            }
        }
        const long long row = r0 + s;
        if (live && row < M)
          *reinterpret_cast<__nv_bfloat162*>(dxz + row * lddxz + c) = __floats2bfloat162_rn(dx.x, dx.y);
        const uint32_t ux = __bfloat16_as_ushort(__float2bfloat16_rn(dx.x));
        const uint32_t uy = __bfloat16_as_ushort(__float2bfloat16_rn(dx.y));
        if (s & 1) {
          packA[s >> 1] |= ux << 16;
          packB[s >> 1] |= uy << 16;
        } else {
          packA[s >> 1] = ux;
          packB[s >> 1] = uy;
        }
      }
    }
  };
  if ((smask >> 1) & ((1u << (NQ - 1)) - 1u))
    rows(std::true_type{});
  else
    rows(std::false_type{});
  // the transpose (when asked for): rows r0 … r0+15 of channels c and c+1 (zero past M, up to ldT)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const long long m = r0 + 8 * h;
    if (dxzT != nullptr && live && m < ldT) {
      *reinterpret_cast<uint4*>(dxzT + (long long)c * ldT + m) =
          make_uint4(packA[4 * h], packA[4 * h + 1], packA[4 * h + 2], packA[4 * h + 3]);
      *reinterpret_cast<uint4*>(dxzT + (long long)(c + 1) * ldT + m) =
          make_uint4(packB[4 * h], packB[4 * h + 1], packB[4 * h + 2], packB[4 * h + 3]);
    }
  }
  __syncthreads();                                       // red overwrites the staged du
#pragma unroll
  for (int k = 0; k < 4; ++k) red[(grp * 64 + p) * 5 + k] = pw[k];
  red[(grp * 64 + p) * 5 + 4] = pb;
  __syncthreads();
  if (grp != 0 || !live) return;
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    float2 acc = red[p * 5 + k];
#pragma unroll
    for (int gq = 1; gq < CONV_GRP; ++gq) {
      acc.x += red[(gq * 64 + p) * 5 + k].x;
      acc.y += red[(gq * 64 + p) * 5 + k].y;
    }
    *reinterpret_cast<float2*>(part + ((long long)blockIdx.y * 5 + k) * E + c) = acc;
  }
}

// Rows i ≥ len_b of sequence b of a bf16 [B·L, cols] array (row stride ld)
// set to zero: one block per sequence, 16-byte stores (cols a multiple of 8).
// Activations the weight-gradient GEMMs read position-major must be finite
// on padding rows, where the gradient operand is zero.
__global__ void __launch_bounds__(256) zero_padding_rows_kernel(bf16* __restrict__ x, long long ld, int cols,
                                                                const int* __restrict__ len, int L) {
  const int b = blockIdx.x;
  const int n = len[b];
  const int c8 = cols / 8;
  const long long rows = (long long)(L - n) * c8;
  for (long long t = threadIdx.x; t < rows; t += blockDim.x) {
    const long long m = (long long)b * L + n + t / c8;
    *reinterpret_cast<uint4*>(x + m * ld + 8 * (t % c8)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// dh = dh⁺ + tmp on valid rows, dh⁺ on padding rows (the hook neither reads
// nor writes them); a block per row at a time, d a multiple of 4 (16-byte
// vectors).
__global__ void __launch_bounds__(256) add_rows_kernel(const float* __restrict__ dh_out, const float* __restrict__ tmp,
                                                       int d, const int* __restrict__ len, int L, long long M,
                                                       float* __restrict__ dh) {
  const int d4 = d / 4;
  for (long long m = blockIdx.x; m < M; m += gridDim.x) {
    const bool ok = valid_row(len, L, m);
    const float4* a = reinterpret_cast<const float4*>(dh_out + m * d);
    const float4* b = reinterpret_cast<const float4*>(tmp + m * d);
    float4* o = reinterpret_cast<float4*>(dh + m * d);
    for (int j = threadIdx.x; j < d4; j += blockDim.x) {
      float4 v = a[j];
      if (ok) {
        const float4 w = b[j];
        v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
      }
      o[j] = v;
    }
  }
}

}  // namespace bwd
}  // namespace r2l
