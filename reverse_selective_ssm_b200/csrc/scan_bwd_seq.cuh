// The reverse-scan gradient walked along each sequence (included by
// scan_bwd.cu; same Args, helpers and notation).  "Bifocal Diffusion Language
// Models" (arXiv 2606.27732v1), §3.4 step ❷, differentiated by the chain rule:
//
//   H_i = a_i ⊙ H_{i+1} + Δ_i u_i B_i   (right to left, H_n = 0)
//   G_i = a_{i−1} ⊙ G_{i−1} + dp_i C_i  (left to right, G_{−1} = 0)
//
// One block owns 32 channels of one sequence for its whole length, so G is
// carried from chunk to chunk in registers: no pass computes G's chunk
// states, and the parameter sums accumulate in registers over the sequence.
// Two launches do the work:
//   1. seq_ckpt_kernel walks H right to left and stores it at the right end of
//      every 16-position chunk (hck[b][k] = H_{16(k+1)}, zero past the end).
//      A training-mode forward (the two-thread scan with checkpoints) stores
//      the same states for every sequence whose length is a multiple of 16,
//      and then this launch only fills in the other sequences;
//   2. seq_final_kernel walks the chunks left to right.  Per chunk it stages
//      the per-(position, channel) scalars once and walks H from the
//      checkpoint (loaded with the chunk's inputs) over positions 15 … 4, keeping
//      the states at positions 12, 8 and 4 in shared memory.  Then per group of 4 positions, left to right,
//      it recomputes the group's H into registers from the state on its right
//      and walks G over it (28 H steps per 16 positions).  The G step needs
//      a_i ⊙ H_{i+1}, which is H_i − Δ_i u_i B_i, so only H_i is kept.
// Threads: two per channel, lanes j and j+16 of a warp, thread h holding the
// states 8h … 8h+7 as four f32x2 pairs.  Per position a channel's two halves
// of ⟨C, H⟩, Σ G ⊙ B and Σ gh ⊙ A meet by one xor-16 shuffle each; dB | dC
// over the warp's 16 channels goes through a per-warp shared-memory transpose
// (each lane sums one of the 32 columns over the channels in a fixed pairwise
// tree), and the block's two warps are summed in order.
//
// Padding positions (i ≥ the sequence's length) are staged as zeros: their
// decay is 1 and their input 0, so H stays 0 past the end and every gradient
// they produce is 0, and full chunks run the same unrolled code as any other.
//
// When every A_log of a block's 32 channels is bitwise log(1), …, log(16) (the
// S4D-real A = −(1 … 16)), the 8 decays of a thread are r^(8h+1) … r^(8h+8),
// r = e^{−Δ}: one exponential and seven products instead of eight
// exponentials.  The block decides this from its own A_log.

namespace r2l {
namespace sbwd {

constexpr int QC = 32;          // channels per block
constexpr int QT = 2 * QC;      // threads per block
constexpr int QS = 16;          // positions per chunk (the checkpoint spacing)
constexpr int QH = 4;           // positions of H held in registers
constexpr int QMINB = 7;        // resident blocks per SM the registers allow
// Slot of channel ch = 8a + b in a staged row: b rotated by a within its group
// of 8.  Both access patterns then hit 8 distinct 16-byte bank groups: the
// staging stores (one lane per 4-channel group, channels 4q + i for a fixed i)
// and the walk's reads (8 consecutive channels).
constexpr int QCP = QC;
__device__ __forceinline__ int qi(int ch) { return (ch & ~7) | ((ch + (ch >> 3)) & 7); }
// Row stride of the dB | dC transpose buffer: 36 words, so the eight 16-byte
// stores of a wavefront (channels j … j+7) start in distinct bank groups and a
// column read (one word per channel) touches 32 distinct banks.
constexpr int QXB = 36;

struct QLane {
  int w, j, h, cl, c, b, n, nck;
  float2 A[4];                  // A_m of states 8h … 8h+7, as pairs
};

// Lane setup and the block's power-path decision (every thread must call it).
__device__ __forceinline__ QLane qlane(const Args& a, bool& pow) {
  QLane l;
  const int lane = threadIdx.x & 31;
  l.w = threadIdx.x >> 5;
  l.j = lane & 15;
  l.h = lane >> 4;
  l.cl = l.w * 16 + l.j;
  l.c = blockIdx.x * QC + l.cl;
  l.b = blockIdx.y;
  l.n = seq_len(a, l.b);
  l.nck = (l.n + QS - 1) / QS;
  const float* al = a.A_log + (size_t)l.c * 16 + 8 * l.h;
  const float4 a0 = ld4(al), a1 = ld4(al + 4);
  const float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  int ok = 1;
#pragma unroll
  for (int i = 0; i < 8; ++i) ok &= __float_as_uint(v[i]) == a.lnbits[8 * l.h + i];
#pragma unroll
  for (int k = 0; k < 4; ++k) l.A[k] = make_float2(-expf(v[2 * k]), -expf(v[2 * k + 1]));
  pow = __syncthreads_and(ok) != 0;
  return l;
}

// The decays exp(Δ A_m) of the thread's 8 states.
template <bool POW>
__device__ __forceinline__ void qdecays(float delta, int h, const float2 (&A)[4], float2 (&ad)[4]) {
  if (POW) {
    const float r = exp2_mufu(-delta * kLog2e);
    const float2 p12 = make_float2(r, r * r);
    const float2 p34 = __fmul2_rn(p12, dup2(p12.y));
    const float2 p56 = __fmul2_rn(p12, dup2(p34.y));
    const float2 p78 = __fmul2_rn(p34, dup2(p34.y));
    const float2 base = dup2(h ? p78.y : 1.0f);        // r^8 for states 8 … 15
    ad[0] = __fmul2_rn(p12, base);
    ad[1] = __fmul2_rn(p34, base);
    ad[2] = __fmul2_rn(p56, base);
    ad[3] = __fmul2_rn(p78, base);
  } else {
    const float2 d2 = dup2(delta * kLog2e);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 t = __fmul2_rn(d2, A[k]);
      ad[k] = make_float2(exp2_mufu(t.x), exp2_mufu(t.y));
    }
  }
}

__device__ __forceinline__ size_t hck_idx(const Args& a, const QLane& l, int k) {
  return (((size_t)l.b * a.nc + k) * a.E + l.c) * 16 + 8 * l.h;
}

// ---- 1. checkpoints
// Chunks right to left; the raw inputs of the next chunk are loaded into
// registers while the current one is walked, and staged into the other of two
// shared buffers.
struct QRaw {
  float4 v[2], u[2], b;
};

__device__ __forceinline__ void qraw_load(const Args& a, const QLane& l, int s, QRaw& x) {
  const int c0 = blockIdx.x * QC;
  const int q4 = threadIdx.x & 7, rr = threadIdx.x >> 3;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int pos = s + rr + 8 * hf;
    x.v[hf] = x.u[hf] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (pos < l.n) {
      const size_t at = ((size_t)l.b * a.L + pos) * a.E + c0 + 4 * q4;
      x.v[hf] = ld4(a.dt + at);
      x.u[hf] = a.u16 ? ld4h(a.u16 + at) : ld4(a.u + at);
    }
  }
  const int pos = s + (threadIdx.x >> 2);
  x.b = pos < l.n ? ld4(a.bc + ((size_t)l.b * a.L + pos) * a.ldbc + 4 * (threadIdx.x & 3))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void __launch_bounds__(QT, QMINB) seq_ckpt_kernel(const Args a) {
  __shared__ float2 dd[2][QS][QCP];     // Δ, Δu
  __shared__ float4 bs[2][QS][4];       // B
  bool pow;
  const QLane l = qlane(a, pow);
  if (a.ckpt_ragged_only && l.n % QS == 0) return;    // stored by the training-mode forward
  const int c0 = blockIdx.x * QC;
  const int q4 = threadIdx.x & 7, rr = threadIdx.x >> 3;
  const float4 dtb = ld4(a.dt_b + c0 + 4 * q4);
  float2 H[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  QRaw x;
  if (l.nck > 0) qraw_load(a, l, (l.nck - 1) * QS, x);
  auto walk = [&](auto pow_tag) {
    constexpr bool POW = decltype(pow_tag)::value;
    for (int k = l.nck - 1; k >= 0; --k) {
      const int buf = k & 1;
      float* hp = a.hcar + hck_idx(a, l, k);
      st4(hp, make_float4(H[0].x, H[0].y, H[1].x, H[1].y));
      st4(hp + 4, make_float4(H[2].x, H[2].y, H[3].x, H[3].y));
      const int s = k * QS;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int row = rr + 8 * hf;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float2 o = make_float2(0.f, 0.f);
          if (s + row < l.n) {
            const float dl = softplus_fwd(get(x.v[hf], i) + get(dtb, i));
            o = make_float2(dl, dl * get(x.u[hf], i));
          }
          dd[buf][row][qi(4 * q4 + i)] = o;
        }
      }
      bs[buf][threadIdx.x >> 2][threadIdx.x & 3] = x.b;
      __syncthreads();
      if (k > 0) qraw_load(a, l, s - QS, x);
#pragma unroll
      for (int rr2 = 0; rr2 < QS; ++rr2) {
        const int r = QS - 1 - rr2;
        const float2 dv = dd[buf][r][qi(l.cl)];
        const float4 B0 = bs[buf][r][2 * l.h], B1 = bs[buf][r][2 * l.h + 1];
        float2 ad[4];
        qdecays<POW>(dv.x, l.h, l.A, ad);
        const float2 du = dup2(dv.y);
        H[0] = __ffma2_rn(ad[0], H[0], __fmul2_rn(du, lo2(B0)));
        H[1] = __ffma2_rn(ad[1], H[1], __fmul2_rn(du, hi2(B0)));
        H[2] = __ffma2_rn(ad[2], H[2], __fmul2_rn(du, lo2(B1)));
        H[3] = __ffma2_rn(ad[3], H[3], __fmul2_rn(du, hi2(B1)));
      }
    }
  };
  if (pow)
    walk(std::true_type{});
  else
    walk(std::false_type{});
}

// ---- 2. the gradient
struct QSmem {
  float4 sc[QS][QCP];     // u, Δ, Δu, dp; then du, ddt_raw, dz once the row is done
  float2 sc2[QS][QCP];    // dz factor dy·SiLU'(z), softplus'(v)
  float4 bc[QS][8];       // B | C
  float red[2][QS][32];   // dB | dC per warp
  float4 hb[QS / QH][2][QT];   // H at positions 4, 8, 12 of the chunk, and the checkpoint (16)
  float xb[2][16][QXB];   // per warp: one position's dB | dC by channel (row) and column
};

// Stage chunk k (rows s … s+15 of the block's 32 channels, zeros past the
// end): the per-element scalars, B | C, and the thread's checkpoint (loaded
// with the chunk's inputs, so the H walk starts from shared memory).
__device__ __forceinline__ void qstage(const Args& a, const QLane& l, QSmem& S, int k) {
  const int c0 = blockIdx.x * QC;
  const int s = k * QS;
  const int q4 = threadIdx.x & 7, rr = threadIdx.x >> 3;
  // the last chunk starts from H = 0 (nothing lies past the sequence's end);
  // a training-mode forward leaves that checkpoint unwritten
  const float* hp = a.hcar + hck_idx(a, l, k);
  const bool last = k == l.nck - 1;
  const float4 h0 = last ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(hp);
  const float4 h1 = last ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(hp + 4);
  const float4 dtb = ld4(a.dt_b + c0 + 4 * q4);
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int row = rr + 8 * hf, pos = s + row;
    float4 o[4];
    float2 o2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      o2[i] = make_float2(0.f, 0.f);
    }
    if (pos < l.n) {
      const size_t row_at = (size_t)l.b * a.L + pos;
      const size_t at = row_at * a.E + c0 + 4 * q4;
      const size_t atz = row_at * a.ldz + c0 + 4 * q4;
      const float4 v4 = ld4(a.dt + at);
      const float4 u4 = a.u16 ? ld4h(a.u16 + at) : ld4(a.u + at);
      const float4 z4 = a.z16 ? ld4h(a.z16 + atz) : ld4(a.z + atz);
      const float4 dy4 = ld4(a.dy + at);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float v = get(v4, i) + get(dtb, i);
        const float dl = softplus_fwd(v);
        const float uu = get(u4, i), zz = get(z4, i), dyy = get(dy4, i);
        const float sg = sigmoid_fast(zz);
        o[i] = make_float4(uu, dl, dl * uu, dyy * zz * sg);
        o2[i] = make_float2(dyy * sg * (1.0f + zz * (1.0f - sg)), softplus_grad(v));
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      S.sc[row][qi(4 * q4 + i)] = o[i];
      S.sc2[row][qi(4 * q4 + i)] = o2[i];
    }
  }
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int idx = threadIdx.x + QT * hf, row = idx >> 3, q = idx & 7, pos = s + row;
    S.bc[row][q] = pos < l.n ? ld4(a.bc + ((size_t)l.b * a.L + pos) * a.ldbc + 4 * q)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  S.hb[QS / QH - 1][0][threadIdx.x] = h0;
  S.hb[QS / QH - 1][1][threadIdx.x] = h1;
}

struct QAcc {
  float2 G[4], ap[4], dA[4];
  float dD, db;
};

template <bool POW>
__device__ __forceinline__ void qhstep(const QLane& l, const QSmem& S, int r, float2 (&H)[4]) {
  const float4 sc = S.sc[r][qi(l.cl)];
  const float4 B0 = S.bc[r][2 * l.h], B1 = S.bc[r][2 * l.h + 1];
  float2 ad[4];
  qdecays<POW>(sc.y, l.h, l.A, ad);
  const float2 du = dup2(sc.z);
  H[0] = __ffma2_rn(ad[0], H[0], __fmul2_rn(du, lo2(B0)));
  H[1] = __ffma2_rn(ad[1], H[1], __fmul2_rn(du, hi2(B0)));
  H[2] = __ffma2_rn(ad[2], H[2], __fmul2_rn(du, lo2(B1)));
  H[3] = __ffma2_rn(ad[3], H[3], __fmul2_rn(du, hi2(B1)));
}

// One position r of the chunk: G, the gradients, dB | dC into S.red.
template <bool POW>
__device__ __forceinline__ void qgstep(const QLane& l, QSmem& S, int r, const float2 (&Hr)[4], float Dc, QAcc& q) {
  const float4 sc = S.sc[r][qi(l.cl)];
  const float uu = sc.x, delta = sc.y, dlu = sc.z, dp = sc.w;
  const float4 B0 = S.bc[r][2 * l.h], B1 = S.bc[r][2 * l.h + 1];
  const float4 C0 = S.bc[r][4 + 2 * l.h], C1 = S.bc[r][5 + 2 * l.h];
  const float2 Bp[4] = {lo2(B0), hi2(B0), lo2(B1), hi2(B1)};
  const float2 Cp[4] = {lo2(C0), hi2(C0), lo2(C1), hi2(C1)};
  const float2 dp2 = dup2(dp), du2 = dup2(dlu), ndu2 = dup2(-dlu), dl2 = dup2(delta);
  float2 pc2 = make_float2(0.f, 0.f), sa2 = pc2, sb2 = pc2;
  float v[16];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    q.G[k] = __ffma2_rn(q.ap[k], q.G[k], __fmul2_rn(dp2, Cp[k]));
    pc2 = __ffma2_rn(Hr[k], Cp[k], pc2);
    sb2 = __ffma2_rn(q.G[k], Bp[k], sb2);
    const float2 gh = __fmul2_rn(q.G[k], __ffma2_rn(ndu2, Bp[k], Hr[k]));   // G ⊙ a ⊙ H_{r+1}
    sa2 = __ffma2_rn(gh, l.A[k], sa2);
    q.dA[k] = __ffma2_rn(dl2, gh, q.dA[k]);
    const float2 gb = __fmul2_rn(q.G[k], du2), hc = __fmul2_rn(dp2, Hr[k]);
    v[2 * k] = gb.x;
    v[2 * k + 1] = gb.y;
    v[8 + 2 * k] = hc.x;
    v[8 + 2 * k + 1] = hc.y;
  }
  float pc = pc2.x + pc2.y, sa = sa2.x + sa2.y, sb = sb2.x + sb2.y;
  pc += __shfl_xor_sync(0xffffffffu, pc, 16);
  sa += __shfl_xor_sync(0xffffffffu, sa, 16);
  sb += __shfl_xor_sync(0xffffffffu, sb, 16);
  // dB (columns 8h … 8h+7) and dC (16 + 8h …) over the warp's 16 channels:
  // the warp writes its 16 × 32 values by channel, then lane c sums column c
  // over the channels (a fixed tree: bitwise reproducible)
  float* xr = &S.xb[l.w][l.j][0];
  __syncwarp();
  *reinterpret_cast<float4*>(xr + 8 * l.h) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(xr + 8 * l.h + 4) = make_float4(v[4], v[5], v[6], v[7]);
  *reinterpret_cast<float4*>(xr + 16 + 8 * l.h) = make_float4(v[8], v[9], v[10], v[11]);
  *reinterpret_cast<float4*>(xr + 16 + 8 * l.h + 4) = make_float4(v[12], v[13], v[14], v[15]);
  __syncwarp();
  {
    const int col = l.j + 16 * l.h;                     // the lane index
    // a fixed pairwise tree, t[i] += t[i + w] for w = 8, 4, 2, 1, its adds
    // taken two at a time as packed f32x2 (the same additions, the same bits)
    float2 t[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) t[ch] = make_float2(S.xb[l.w][2 * ch][col], S.xb[l.w][2 * ch + 1][col]);
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) t[i] = __fadd2_rn(t[i], t[i + w]);
    S.red[l.w][r][col] = t[0].x + t[0].y;
  }
  // the gradients (both halves of a channel hold the same sums) go over the
  // row's staged scalars, which no later step reads
  const float p = fmaf(Dc, uu, pc);
  const float2 s2 = S.sc2[r][qi(l.cl)];
  const float ddt = fmaf(sb, uu, sa) * s2.y;
  float* o = reinterpret_cast<float*>(&S.sc[r][qi(l.cl)]);
  o[2 * l.h] = l.h ? p * s2.x : fmaf(Dc, dp, delta * sb);
  o[1] = ddt;
  q.dD = fmaf(dp, uu, q.dD);
  q.db += ddt;
  qdecays<POW>(delta, l.h, l.A, q.ap);                  // a_r, for G at r + 1
}

__global__ void __launch_bounds__(QT, QMINB) seq_final_kernel(const Args a) {
  __shared__ QSmem S;
  bool pow;
  const QLane l = qlane(a, pow);
  const int c0 = blockIdx.x * QC;
  const float Dc = a.D[l.c];
  QAcc q;
#pragma unroll
  for (int k = 0; k < 4; ++k) q.G[k] = q.ap[k] = q.dA[k] = make_float2(0.f, 0.f);
  q.dD = q.db = 0.0f;
  const size_t bl = (size_t)l.b * a.L;

  auto walk = [&](auto pow_tag) {
    constexpr bool POW = decltype(pow_tag)::value;
    for (int k = 0; k < l.nck; ++k) {
      const int s = k * QS;
      __syncthreads();                                    // the last chunk's epilogue is done with S
      qstage(a, l, S, k);
      __syncthreads();
      {
        const float4 h0 = S.hb[QS / QH - 1][0][threadIdx.x], h1 = S.hb[QS / QH - 1][1][threadIdx.x];
        float2 H[4] = {lo2(h0), hi2(h0), lo2(h1), hi2(h1)};
#pragma unroll
        for (int r = QS - 1; r >= QH; --r) {
          qhstep<POW>(l, S, r, H);
          if (r % QH == 0) {
            S.hb[r / QH - 1][0][threadIdx.x] = make_float4(H[0].x, H[0].y, H[1].x, H[1].y);
            S.hb[r / QH - 1][1][threadIdx.x] = make_float4(H[2].x, H[2].y, H[3].x, H[3].y);
          }
        }
      }
#pragma unroll 1
      for (int g = 0; g < QS / QH; ++g) {
        const float4 h0 = S.hb[g][0][threadIdx.x], h1 = S.hb[g][1][threadIdx.x];
        float2 H[4] = {lo2(h0), hi2(h0), lo2(h1), hi2(h1)};
        float2 Hs[QH][4];
#pragma unroll
        for (int r = QH - 1; r >= 0; --r) {
          qhstep<POW>(l, S, g * QH + r, H);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) Hs[r][kk] = H[kk];
        }
#pragma unroll
        for (int r = 0; r < QH; ++r) qgstep<POW>(l, S, g * QH + r, Hs[r], Dc, q);
      }
      __syncthreads();
      // rows s … s+15 of this sequence (the ones below L): du, ddt_raw, dz and
      // the block's partial dB | dC
      for (int i = threadIdx.x; i < 3 * QS * 8; i += QT) {
        const int arr = i / (QS * 8), r = (i / 8) % QS, qq = i & 7;
        if (s + r >= a.L) continue;
        const float* src = reinterpret_cast<const float*>(&S.sc[r][0]) + arr;
        const float4 v = make_float4(src[4 * qi(4 * qq)], src[4 * qi(4 * qq + 1)], src[4 * qi(4 * qq + 2)],
                                     src[4 * qi(4 * qq + 3)]);
        const size_t row = bl + s + r;
        bf16* d16 = arr == 1 ? a.ddt16 : arr == 2 ? a.dz16 : nullptr;
        if (d16) {
          const long long ld = arr == 1 ? a.ld_ddt16 : a.ld_dz16;
          const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
          *reinterpret_cast<uint2*>(d16 + row * ld + c0 + 4 * qq) =
              make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
        } else {
          float* dst = arr == 0 ? a.du + row * a.E : arr == 1 ? a.ddt + row * a.E : a.dz + row * a.ld_dz;
          st4(dst + c0 + 4 * qq, v);
        }
      }
      for (int i = threadIdx.x; i < QS * 8; i += QT) {
        const int r = i / 8, qq = i & 7;
        if (s + r >= a.L) continue;
        const float4 x = *reinterpret_cast<const float4*>(&S.red[0][r][4 * qq]);
        const float4 y = *reinterpret_cast<const float4*>(&S.red[1][r][4 * qq]);
        st4(a.pbc + ((size_t)blockIdx.x * a.B * a.L + bl + s + r) * 32 + 4 * qq,
            make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w));
      }
    }
  };
  if (pow)
    walk(std::true_type{});
  else
    walk(std::false_type{});

  // rows past the last chunk: zero gradients and partials
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long i = threadIdx.x; i < (long long)(a.L - l.nck * QS) * 8; i += QT) {
    const size_t row = bl + l.nck * QS + (size_t)(i / 8);
    const int qq = (int)(i & 7);
    st4(a.du + row * a.E + c0 + 4 * qq, zero);
    if (a.ddt16) *reinterpret_cast<uint2*>(a.ddt16 + row * a.ld_ddt16 + c0 + 4 * qq) = make_uint2(0u, 0u);
    else st4(a.ddt + row * a.E + c0 + 4 * qq, zero);
    if (a.dz16) *reinterpret_cast<uint2*>(a.dz16 + row * a.ld_dz16 + c0 + 4 * qq) = make_uint2(0u, 0u);
    else st4(a.dz + row * a.ld_dz + c0 + 4 * qq, zero);
    st4(a.pbc + ((size_t)blockIdx.x * a.B * a.L + row) * 32 + 4 * qq, zero);
  }
  float* pa = a.pA + ((size_t)l.b * a.E + l.c) * 16 + 8 * l.h;
  st4(pa, make_float4(q.dA[0].x, q.dA[0].y, q.dA[1].x, q.dA[1].y));
  st4(pa + 4, make_float4(q.dA[2].x, q.dA[2].y, q.dA[3].x, q.dA[3].y));
  if (l.h == 0) {
    a.pD[(size_t)l.b * a.E + l.c] = q.dD;
    a.pb[(size_t)l.b * a.E + l.c] = q.db;
  }
}

// dA_log, dD, ddt_b: the per-sequence partials summed over b in order.
__global__ void seq_reduce_params_kernel(const Args a) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // c·16 + m
  if (t >= (long long)a.E * 16) return;
  const int c = (int)(t >> 4), m = (int)(t & 15);
  float sA = 0.0f, sD = 0.0f, sb = 0.0f;
  for (int b = 0; b < a.B; ++b) {
    sA += a.pA[((size_t)b * a.E + c) * 16 + m];
    if (m == 0) {
      sD += a.pD[(size_t)b * a.E + c];
      sb += a.pb[(size_t)b * a.E + c];
    }
  }
  a.dA_log[t] = sA * -expf(a.A_log[t]);
  if (m == 0) {
    a.dD[c] = sD;
    a.ddt_b[c] = sb;
  }
}

}  // namespace sbwd
}  // namespace r2l
