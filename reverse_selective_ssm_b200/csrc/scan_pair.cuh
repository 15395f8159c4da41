// Reverse selective scan with two threads per channel ("Bifocal Diffusion
// Language Models", arXiv 2606.27732v1, §3.4 step ❷; the recurrence and its
// terms are those of scan_fast.cuh) with dt_proj fused (bf16, dt_rank 128):
// one pass over whole sequences, or, when sequences are split into chunks,
// the state-only first pass (FINAL = false) and the final pass from the
// carried states (FINAL = true).
//
// Why: at batch 8 a sequence-length scan has only B·E = 32,768 independent
// channel chains, about 7 warps per SM with one thread per channel, and each
// of those warps stalls on its own dependent arithmetic most of the time.
// Splitting each channel's 16 states over two threads doubles the warps at
// nearly the same instruction count:
//
//   * thread h ∈ {0, 1} of a channel holds the states m = 4k + 2e + h
//     (k = 0..3, e = 0..1) as four f32x2 pairs; their decays are
//     r^(m+1) = base·r^(4k)·(1, r²) with base = r^(1+h) on the power path;
//   * the state-independent terms of a token (decay base, Δu, D·u, SiLU(z))
//     are computed once, by the thread whose h is the token's parity, and
//     handed to the other with warp shuffles (the two threads of a channel are
//     lanes j and j + 16 of one warp);
//   * each thread's partial ⟨C, H⟩ over its 8 states goes to the token's
//     owner, which adds it, applies D·u and the gate, and writes y;
//   * the tensor core broadcasts B|C with a lane-dependent pattern: lanes
//     0–15 of each TMEM quarter receive B_{2n}, C_{2n} and lanes 16–31
//     B_{2n+1}, C_{2n+1} (n = 0..7), so a thread reads exactly its 16 values of
//     a token with one 16-column tcgen05.ld.
//
// A CTA covers 256 channels of one sequence: 16 compute warps, a TMA producer
// warp and an MMA warp (576 threads, one CTA per SM).  Warp w = 4p + q reads
// TMEM lane quarter q; its 16 channels are 128·(p/2) + 32q + 16·(p%2) + j.
// dt_proj runs as two MMAs per tile (channels 0–127 and 128–255, M = 128,
// N = 16 tokens, K = 128); a warp reads its quarter of the block it belongs
// to and moves each channel's dt_raw to the thread that needs it by shuffle.
#pragma once

#include "scan_fast.cuh"

namespace r2l {
namespace rscan {
namespace pair {

constexpr int CHP = 256;                          // channels per CTA
constexpr int PWARPS = 16;                        // compute warps
constexpr int PTHREADS = PWARPS * 32;
constexpr int GT = 4;                             // tokens per sub-tile (phase A, then phase B)
constexpr int GB = 8;                             // tokens per B|C group (one MMA, one handshake)
constexpr int NG = TS / GB;                       // groups per tile; TMEM region g serves group g
constexpr uint32_t P_ACT_TILE = TS * CHP * 2;     // one bf16 [TS × CHP] tile
constexpr uint32_t P_W_SLICE = CHP * DT_R * 2;    // bf16 W_dt [CHP × R]
constexpr uint32_t P_BC_COL0 = STAGES * 32;       // dt_raw: [stage][block] × 16 columns
constexpr uint32_t P_TMEM_COLS = 512;
constexpr uint32_t P_GROUP_COLS = GB * 16;        // 16 columns per token
constexpr uint32_t P_OPB_BYTES = GB * 16 * 32;    // GB·16 operand rows of 32 bytes
static_assert(P_BC_COL0 + NG * P_GROUP_COLS <= P_TMEM_COLS, "TMEM budget");
static_assert(GB * 16 <= 256 && GB % GT == 0, "one MMA (N = GB·16) per group");

struct SmemPair {
  static constexpr uint32_t W = 0;
  static constexpr uint32_t DR = P_W_SLICE;
  static constexpr uint32_t U = DR + STAGES * DR_TILE;
  static constexpr uint32_t DT = U;                               // unused (dt_proj fused)
  static constexpr uint32_t Z = U + STAGES * P_ACT_TILE;
  static constexpr uint32_t Y = Z;                                // y overwrites z in place
  static constexpr uint32_t BC = Z + STAGES * P_ACT_TILE;
  static constexpr uint32_t PAT = BC + STAGES * BC_TILE;          // lane-pattern operand
  static constexpr uint32_t OPB = PAT + ONES_BYTES;
  static constexpr uint32_t BAR = OPB + NG * P_OPB_BYTES;           // full, empty, dtready [STAGES], wfull, drain, bcready, bcfree [NG]
  static constexpr uint32_t SLOT = BAR + (3 * STAGES + 2 + 2 * NG) * 8;
  static constexpr size_t BYTES = 1024 + SLOT + 16;
  static constexpr int THREADS = PTHREADS + 64;
};

// The MMA warp: per tile, dt_raw for both 128-channel blocks, then the tile's
// four B|C groups in the order the compute warps take the tokens.
template <bool FWD>
__device__ __forceinline__ void run_mma_pair(uint8_t* smem, uint32_t tmem_base, uint64_t* full, uint64_t* dtready,
                                             uint64_t* wfull, uint64_t* drain, uint64_t* bcready, uint64_t* bcfree,
                                             int ntiles, unsigned* err) {
  using S = SmemPair;
  const int lane = threadIdx.x & 31;
  // pattern operand: row ℓ is (1, 1, 0, 0) for (ℓ mod 32) < 16, else (0, 0, 1, 1)
  for (int n = lane; n < 128; n += 32) {
    uint8_t* row = smem + S::PAT + opnd_row(n);
    const bool upper = (n & 31) >= 16;
    *reinterpret_cast<float4*>(row) = upper ? make_float4(0.0f, 0.0f, 1.0f, 1.0f) : make_float4(1.0f, 1.0f, 0.0f, 0.0f);
    *reinterpret_cast<float4*>(row + 128) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  for (int n = lane; n < NG * GB * 16; n += 32) {
    uint8_t* row = smem + S::OPB + (n / (GB * 16)) * P_OPB_BYTES + opnd_row(n % (GB * 16));
    *reinterpret_cast<float4*>(row) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    *reinterpret_cast<float4*>(row + 128) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  sm100::fence_proxy_async_smem();
  __syncwarp();
  constexpr uint32_t idt = sm100::idesc_bf16_f32(128, TS);
  constexpr uint32_t ibc = sm100::idesc_tf32_f32(128, GB * 16);
  const uint64_t a_pat = sm100::smem_desc_noswz(sm100::smem_u32(smem + S::PAT), 128, 256);
  const uint32_t w0 = sm100::smem_u32(smem + S::W);
  bool ok = sm100::mbar_wait(wfull, 0, err);
  for (int it = 0; it < ntiles && ok; ++it) {
    const int st = it % STAGES;
    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
    if (!sm100::mbar_wait(&full[st], ph, err)) break;
    sm100::tc_fence_after();
    if (lane == 0) {
      const uint32_t d0 = sm100::smem_u32(smem + S::DR + st * DR_TILE);
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
#pragma unroll
        for (int k = 0; k < DT_R / 16; ++k) {
          const uint32_t a_addr = w0 + (k / 4) * (CHP * 128) + blk * (128 * 128) + (k % 4) * 32;
          const uint32_t b_addr = d0 + (k / 4) * (TS * 128) + (k % 4) * 32;
          sm100::mma_bf16(tmem_base + (uint32_t)(st * 32 + blk * 16), sm100::smem_desc_k128(a_addr),
                          sm100::smem_desc_k128(b_addr), idt, k != 0);
        }
      }
      sm100::mma_commit(&dtready[st]);
    }
    __syncwarp();
    const float* bct = reinterpret_cast<const float*>(smem + S::BC + st * BC_TILE);
#pragma unroll 1
    for (int g = 0; g < NG; ++g) {
      if (!sm100::mbar_wait(&bcfree[g], ((uint32_t)it & 1u) ^ 1u, err)) { ok = false; break; }
      sm100::tc_fence_after();
      uint8_t* opb = smem + S::OPB + g * P_OPB_BYTES;
#pragma unroll
      for (int part = 0; part < GB / 2; ++part) {
        const int row = lane + 32 * part;            // 16·slot + n
        const int slot = row >> 4, n = row & 15;
        const int tok = FWD ? GB * g + slot : TS - 1 - GB * g - slot;
        const float v0 = bct[tok * 32 + 2 * n], v1 = bct[tok * 32 + 2 * n + 1];
        const float h0 = __uint_as_float(__float_as_uint(v0) & 0xFFFFE000u);
        const float h1 = __uint_as_float(__float_as_uint(v1) & 0xFFFFE000u);
        *reinterpret_cast<float4*>(opb + opnd_row(row)) = make_float4(h0, v0 - h0, h1, v1 - h1);
      }
      sm100::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        sm100::mma_tf32(tmem_base + P_BC_COL0 + (uint32_t)(g * P_GROUP_COLS), a_pat,
                        sm100::smem_desc_noswz(sm100::smem_u32(opb), 128, 256), ibc, 0u);
        sm100::mma_commit(&bcready[g]);
      }
      __syncwarp();
    }
  }
  if (lane == 0) {
    sm100::mma_commit(drain);
    sm100::mbar_wait(drain, 0, err, 1000000000ull);
  }
  __syncwarp();
}

// Per-thread constants of a (channel, half).
struct PCtx {
  float dtb, Dc;
  float A2[8];            // A_m · log2 e for the thread's states m = 4k + 2e + h, index 2k + e
  bool upper;             // h == 1
};

// The decays of the thread's 8 states for one token, as four pairs.
template <bool POW>
__device__ __forceinline__ void pair_decays(const PCtx& cx, float dec, float2 (&a)[4]) {
  if (POW) {
    const float r = dec;
    const float r2 = r * r;
    const float r4 = r2 * r2;
    const float r8 = r4 * r4;
    const float base = cx.upper ? r2 : r;
    a[0] = make_float2(base, base * r2);
    a[1] = __fmul2_rn(a[0], make_float2(r4, r4));
    a[2] = __fmul2_rn(a[0], make_float2(r8, r8));
    a[3] = __fmul2_rn(a[1], make_float2(r8, r8));
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = make_float2(ex2_approx(dec * cx.A2[2 * k]), ex2_approx(dec * cx.A2[2 * k + 1]));
  }
}

// One tile of 16 tokens as four sub-tiles of GT tokens; each pair of
// sub-tiles reads one B|C group (TMEM region g = sub-tile / 2).  Tokens
// outside [jlo, jhi) (a tile that crosses the chunk's start or end) leave the
// state untouched and write nothing.  Without FINAL (the chunked scheme's
// first pass) only the state and this thread's Σ Δ over its tokens advance.
template <bool FINAL, bool POW, bool FULL, bool FWD>
__device__ __forceinline__ void pair_tile(const PCtx& cx, float2 (&H)[4], float& sumd, const bf16* su, bf16* sz,
                                          bf16* yg, long long ldy, bool store_ok, int jlo, int jhi,
                                          const float (&dto)[8], uint32_t ph, uint64_t* bcready, uint64_t* bcfree,
                                          uint32_t t_bc, unsigned* err, bool& ok) {
  const int lane = threadIdx.x & 31;
  const int h = lane >> 4;
  // With FINAL, u and z of this thread's tokens are read one sub-tile ahead:
  // the y of a sub-tile is stored over its z rows, and a read placed after
  // those stores could not be moved above them (the compiler cannot tell the
  // rows apart).  The state-only pass stores nothing and reads in place.
  bf16 u_nx[GT / 2], z_nx[GT / 2];
  if (FINAL) {
#pragma unroll
    for (int i = 0; i < GT / 2; ++i) {
      const int j = (FWD ? 0 : TS - GT) + 2 * i + h;
      u_nx[i] = su[j * CHP];
      z_nx[i] = sz[j * CHP];
    }
  }
#pragma unroll
  for (int sb = 0; sb < TS / GT; ++sb) {
    const int g = sb / (GB / GT);                  // B|C group of this sub-tile
    const int gs = sb % (GB / GT);                 // sub-tile within the group
    const int j0 = FWD ? sb * GT : TS - GT - sb * GT;
    bf16 u_cur[GT / 2], z_cur[GT / 2];
#pragma unroll
    for (int i = 0; i < GT / 2; ++i) {
      u_cur[i] = FINAL ? u_nx[i] : su[(j0 + 2 * i + h) * CHP];
      if (FINAL) z_cur[i] = z_nx[i];
    }
    if (FINAL && sb + 1 < TS / GT) {
      const int jn = FWD ? (sb + 1) * GT : TS - GT - (sb + 1) * GT;
#pragma unroll
      for (int i = 0; i < GT / 2; ++i) {
        u_nx[i] = su[(jn + 2 * i + h) * CHP];
        z_nx[i] = sz[(jn + 2 * i + h) * CHP];
      }
    }
    // phase A for this thread's tokens t = 2i + h of the sub-tile
    float dec_o[GT / 2], du_o[GT / 2], Du_o[GT / 2], gz_o[GT / 2];
#pragma unroll
    for (int i = 0; i < GT / 2; ++i) {
      const int j = j0 + 2 * i + h;
      float delta, r;
      softplus_and_decay(dto[j0 / 2 + i] + cx.dtb, delta, r);
      const float uu = __bfloat162float(u_cur[i]);
      const bool valid = FULL || (j >= jlo && j < jhi);
      dec_o[i] = valid ? (POW ? r : delta) : (POW ? 1.0f : 0.0f);
      du_o[i] = valid ? delta * uu : 0.0f;
      if (FINAL) {
        Du_o[i] = cx.Dc * uu;
        gz_o[i] = silu_fast(__bfloat162float(z_cur[i]));
      } else {
        sumd += valid ? delta : 0.0f;
      }
    }
    // every thread needs the decay and Δu of all GT tokens: even tokens from
    // lane j, odd tokens from lane j + 16
    float dec_e[GT / 2], dec_d[GT / 2], du_e[GT / 2], du_d[GT / 2];
#pragma unroll
    for (int i = 0; i < GT / 2; ++i) {
      dec_e[i] = __shfl_sync(0xffffffffu, dec_o[i], lane & 15);
      dec_d[i] = __shfl_sync(0xffffffffu, dec_o[i], lane | 16);
      du_e[i] = __shfl_sync(0xffffffffu, du_o[i], lane & 15);
      du_d[i] = __shfl_sync(0xffffffffu, du_o[i], lane | 16);
    }
    float part[GT];     // this thread's half of ⟨C, H⟩ per token of the sub-tile
    if (gs == 0) {
      if (!sm100::mbar_wait(&bcready[g], ph, err)) { ok = false; return; }
      __syncwarp();
      sm100::tc_fence_after();
    }
#pragma unroll
    for (int slot = 0; slot < GT; ++slot) {
      const int t = FWD ? slot : GT - 1 - slot;
      const int j = j0 + t;
      float bv[16];
      sm100::tmem_ld16(t_bc + (uint32_t)(g * P_GROUP_COLS + (gs * GT + slot) * 16), bv);
      part[t] = 0.0f;
      if (FULL || (j >= jlo && j < jhi)) {
        const float dec = (t & 1) ? dec_d[t >> 1] : dec_e[t >> 1];
        const float du = (t & 1) ? du_d[t >> 1] : du_e[t >> 1];
        float2 a[4];
        pair_decays<POW>(cx, dec, a);
        const float2 du2 = make_float2(du, du);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          H[q] = __ffma2_rn(a[q], H[q], __fmul2_rn(du2, make_float2(bv[2 * q], bv[2 * q + 1])));
        if (FINAL) {
          float2 acc = __fmul2_rn(make_float2(bv[8], bv[9]), H[0]);
#pragma unroll
          for (int q = 1; q < 4; ++q) acc = __ffma2_rn(make_float2(bv[8 + 2 * q], bv[9 + 2 * q]), H[q], acc);
          part[t] = acc.x + acc.y;
        }
      }
    }
    if (gs == GB / GT - 1) {                       // the group's last token is read
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&bcfree[g]);
    }
    // y of this thread's tokens: its half of ⟨C, H⟩ plus the partner's
#pragma unroll
    for (int i = 0; i < (FINAL ? GT / 2 : 0); ++i) {
      const float give = h ? part[2 * i] : part[2 * i + 1];       // the partner's token
      const float mine = h ? part[2 * i + 1] : part[2 * i];
      const float other = __shfl_xor_sync(0xffffffffu, give, 16);
      const int j = j0 + 2 * i + h;
      const bool valid = FULL || (j >= jlo && j < jhi);
      const bf16 yv = __float2bfloat16_rn((mine + other + Du_o[i]) * gz_o[i]);
      if (store_ok && valid) {
        if (FULL) sz[j * CHP] = yv;
        else yg[(long long)j * ldy] = yv;
      }
    }
  }
}

template <bool FINAL, bool POW, bool FWD, bool CKPT>
__device__ __forceinline__ void pair_compute(const PCtx& cx, float2 (&H)[4], float& sumd, uint8_t* smem, uint64_t* full,
                                             uint64_t* empty, uint64_t* dtready, uint64_t* bcready, uint64_t* bcfree,
                                             uint32_t tmem_base, int ntiles, int s0, int e0, int b, int c, int cl,
                                             bool cvalid, const Params& p) {
  using S = SmemPair;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, pp = warp >> 2, blk = pp >> 1, s16 = pp & 1;
  const int h = lane >> 4;
  const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16);
  bool ok = true;
  for (int it = 0; it < ntiles && ok; ++it) {
    const int st = it % STAGES;
    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
    if (!sm100::mbar_wait(&full[st], ph, p.err)) break;
    if (!sm100::mbar_wait(&dtready[st], ph, p.err)) break;
    __syncwarp();
    sm100::tc_fence_after();
    float raw[16];
    sm100::tmem_ld16(t_lane + (uint32_t)(st * 32 + blk * 16), raw);
    // lane ℓ holds channel 128·blk + 32q + ℓ; this thread's channel sits in
    // lane 16·s16 + j, and it needs that channel's tokens 2i + h
    float dto[8];
    if (s16) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, raw[2 * i], 16);
        dto[i] = h ? raw[2 * i + 1] : other;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, raw[2 * i + 1], 16);
        dto[i] = h ? other : raw[2 * i];
      }
    }
    const int tbase = FWD ? s0 + it * TS : e0 - (it + 1) * TS;
    const int jlo = (!FWD && s0 > tbase) ? s0 - tbase : 0;
    const int jhi = (FWD && e0 - tbase < TS) ? e0 - tbase : TS;
    const bool full_tile = jlo == 0 && jhi == TS;
    const bf16* su = reinterpret_cast<const bf16*>(smem + S::U) + st * TS * CHP + cl;
    bf16* sz = reinterpret_cast<bf16*>(smem + S::Z) + st * TS * CHP + cl;
    bf16* yg = p.y + ((long long)b * p.L + tbase) * p.ldy + c;
    const uint32_t gph = (uint32_t)it & 1u;   // each group region is used once per tile
    if (full_tile)
      pair_tile<FINAL, POW, true, FWD>(cx, H, sumd, su, sz, yg, p.ldy, cvalid, 0, TS, dto, gph, bcready, bcfree,
                                       t_lane + P_BC_COL0, p.err, ok);
    else
      pair_tile<FINAL, POW, false, FWD>(cx, H, sumd, su, sz, yg, p.ldy, cvalid, jlo, jhi, dto, gph, bcready,
                                        bcfree, t_lane + P_BC_COL0, p.err, ok);
    // training mode: when the chunk ends at a multiple of 16 (the sequence's
    // length is one), every tile starts at one, and the state after the tile
    // is the scan gradient's checkpoint H_tbase.  Thread h holds the states
    // 4q + 2e + h; one exchange with the partner (lane ± 16) gives it the 8
    // consecutive states 8h … 8h+7, stored as two 16-byte vectors.
    if (CKPT && ok && (e0 % 16) == 0 && tbase >= 16) {
      const int h = lane >> 4;
      const float2 s0 = h ? H[0] : H[2], s1 = h ? H[1] : H[3];
      float r[4];
      r[0] = __shfl_xor_sync(0xffffffffu, s0.x, 16);
      r[1] = __shfl_xor_sync(0xffffffffu, s0.y, 16);
      r[2] = __shfl_xor_sync(0xffffffffu, s1.x, 16);
      r[3] = __shfl_xor_sync(0xffffffffu, s1.y, 16);
      if (cvalid) {
        const float2 k0 = h ? H[2] : H[0], k1 = h ? H[3] : H[1];
        float4* d4 = reinterpret_cast<float4*>(p.hck + (((long long)b * p.nc16 + (tbase / 16 - 1)) * p.E + c) * 16 +
                                               8 * h);
        d4[0] = h ? make_float4(r[0], k0.x, r[1], k0.y) : make_float4(k0.x, r[0], k0.y, r[1]);
        d4[1] = h ? make_float4(r[2], k1.x, r[3], k1.y) : make_float4(k1.x, r[2], k1.y, r[3]);
      }
    }
    if (!ok) break;
    if (FINAL && full_tile) sm100::fence_proxy_async_smem();   // y tile visible to the TMA store
    sm100::tc_fence_before();
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty[st]);
  }
}

// One pass over chunk blockIdx.y of T tokens of every sequence (p.T, p.nc).
// FINAL: y, starting from the carried state H_in(k) when sequences are split
// (zero with one chunk).  Otherwise the chunked scheme's first pass: the
// chunk's end state from a zero start and Σ Δ over it, into the carry buffer.
template <bool FINAL, bool FWD, bool CKPT = false>
__global__ void __launch_bounds__(SmemPair::THREADS, 1)
scan_pair_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_z,
                 const __grid_constant__ CUtensorMap tm_dr, const __grid_constant__ CUtensorMap tm_bc,
                 const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_w,
                 const Params p) {
  using S = SmemPair;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* dtready = empty + STAGES;
  uint64_t* wfull = dtready + STAGES;
  uint64_t* drain = wfull + 1;
  uint64_t* bcready = drain + 1;
  uint64_t* bcfree = bcready + NG;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::SLOT);

  grid_dep_wait();
  grid_dep_launch();
  const int cb = blockIdx.x, k = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n = p.len[b];
  const int s0 = k * p.T;
  const int e0 = min(s0 + p.T, n);
  if (s0 >= n) {                               // chunk entirely in the padding
    if (!FINAL && tid < PTHREADS) {
      const int q = warp & 3, pp = warp >> 2;
      const int c = cb * CHP + 128 * (pp >> 1) + 32 * q + 16 * (pp & 1) + (lane & 15);
      if (c < p.E) {
        float* dst = p.carry + (((long long)b * p.nc + k) * p.E + c) * 16;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          dst[4 * kk + (lane >> 4)] = 0.0f;
          dst[4 * kk + 2 + (lane >> 4)] = 0.0f;
        }
        if (lane < 16) p.carry_sum[((long long)b * p.nc + k) * p.E + c] = 0.0f;
      }
    }
    return;
  }
  const int ntiles = (e0 - s0 + TS - 1) / TS;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], PWARPS);
      sm100::mbar_init(&dtready[s], 1);
    }
    sm100::mbar_init(wfull, 1);
    sm100::mbar_init(drain, 1);
    for (int g = 0; g < NG; ++g) {
      sm100::mbar_init(&bcready[g], 1);
      sm100::mbar_init(&bcfree[g], PWARPS);
    }
    sm100::fence_barrier_init();
  }
  if (warp == PWARPS + 1) sm100::tmem_alloc(tmem_slot, P_TMEM_COLS);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == PWARPS) {
    if (lane == 0)
      run_producer<S, FINAL, true, FWD, CHP>(&tm_u, &tm_z, &tm_dr, &tm_bc, &tm_y, &tm_w, smem, full, empty, wfull, b,
                                            cb, s0, e0, ntiles, p);
    return;
  }
  if (warp == PWARPS + 1) {
    run_mma_pair<FWD>(smem, tmem_base, full, dtready, wfull, drain, bcready, bcfree, ntiles, p.err);
    sm100::named_bar_sync(1, PTHREADS + 32);   // every compute warp has finished reading TMEM
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, P_TMEM_COLS);
    return;
  }

  // compute warps: channel of this (warp, lane)
  const int q = warp & 3, pp = warp >> 2;
  const int cl = 128 * (pp >> 1) + 32 * q + 16 * (pp & 1) + (lane & 15);
  const int c = cb * CHP + cl;
  const bool cvalid = c < p.E;
  const int h = lane >> 4;
  PCtx cx;
  cx.upper = h != 0;
  cx.dtb = cvalid ? p.dt_b[c] : 0.0f;
  cx.Dc = cvalid ? p.D[c] : 0.0f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = 4 * kk + 2 * e + h;
      const float a = cvalid ? -expf(p.A_log[c * 16 + m]) : -(float)(m + 1);
      cx.A2[2 * kk + e] = a * LOG2E;
    }
  }
  const bool use_pow = !p.force_general && *p.a_general == 0u;
  // the thread's states m = 4kk + 2e + h sit at H[kk].x (e = 0) and H[kk].y (e = 1)
  float2 H[4];
  float* cst = (p.nc > 1 && cvalid) ? p.carry + (((long long)b * p.nc + k) * p.E + c) * 16 : nullptr;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    H[kk] = (FINAL && cst) ? make_float2(cst[4 * kk + h], cst[4 * kk + 2 + h]) : make_float2(0.0f, 0.0f);
  float sumd = 0.0f;
  if (use_pow)
    pair_compute<FINAL, true, FWD, CKPT>(cx, H, sumd, smem, full, empty, dtready, bcready, bcfree, tmem_base, ntiles,
                                         s0, e0, b, c, cl, cvalid, p);
  else
    pair_compute<FINAL, false, FWD, CKPT>(cx, H, sumd, smem, full, empty, dtready, bcready, bcfree, tmem_base,
                                          ntiles, s0, e0, b, c, cl, cvalid, p);
  if (!FINAL) {
    // chunk end state S_k and Σ Δ (each thread summed Δ over its own tokens)
    const float total = sumd + __shfl_xor_sync(0xffffffffu, sumd, 16);
    if (cst) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        cst[4 * kk + h] = H[kk].x;
        cst[4 * kk + 2 + h] = H[kk].y;
      }
      if (h == 0) p.carry_sum[((long long)b * p.nc + k) * p.E + c] = total;
    }
  }
  sm100::tc_fence_before();
  sm100::named_bar_sync(1, PTHREADS + 32);   // release TMEM to the dealloc
}

}  // namespace pair
}  // namespace rscan
}  // namespace r2l
