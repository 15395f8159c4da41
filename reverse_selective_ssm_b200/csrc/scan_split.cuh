// Reverse selective scan with the serial recurrence on warps of its own
// ("Bifocal Diffusion Language Models", arXiv 2606.27732v1, §3.4 step ❷: the
// Mamba-1 selective scan of the flipped sequence, run here from each
// sequence's last valid token to its first), dt_proj fused (bf16, dt_rank 128):
//
//   Δ_i = softplus(Δr_i·W_dtᵀ + dt_b),  H_i = e^{Δ_i A} ⊙ H_{i+1} + Δ_i u_i B_i,
//   y_i = (⟨C_i, H_i⟩ + D u_i) · SiLU(z_i).
//
// Only the state update is serial.  Everything else of a (token, channel) can
// be computed ahead of it (softplus, the decay base, Δu) or behind it (D·u,
// the SiLU(z) gate, the bf16 output), so a CTA (256 channels of one sequence)
// gives the two kinds of work to different warps:
//
//   * 8 recurrence warps, one thread per channel with its 16 states in
//     registers as eight f32x2 pairs (states 2k, 2k+1).  Per token a thread
//     reads (decay base r or Δ, Δu) from shared memory and its B|C from
//     tensor memory, forms the 16 decays (r, r², …, r¹⁶ on the power path),
//     updates the state and writes p = ⟨C, H⟩ back to shared memory.
//   * 4 phase-A warps, one thread per pair of adjacent channels.  Per tile
//     they read dt_raw (the dt_proj MMA result) from tensor memory and u from
//     the stage, and write (r or Δ, Δu) ahead of the recurrence; one tile
//     behind it they read p, u and z and write y = (p + D u)·SiLU(z).
//   * A TMA producer warp: the CTA's W_dt slice once, then u, z, Δr and B|C
//     tiles of 16 tokens into a 4-stage ring, and each finished y tile back
//     out with a bulk tensor store.
//   * A dt_proj warp: per pair of tiles dt_raw = W_dt slice · Δr tilesᵀ
//     (M = 128 channels × N = 32 tokens, bf16, into TMEM), issued as soon as
//     the tiles land.
//   * An MMA warp: per group of 4 tokens the broadcast of B|C into TMEM
//     columns that every lane holds alike: one tf32 MMA (N = 128) of an
//     all-ones operand with a row (hi, mid, lo) per value, exact in fp32.
//     Few, wide MMAs: the issue of small tcgen05.mma instructions, not their
//     arithmetic, is what costs.
//
// The recurrence threads thus run about 42 instructions per (token, channel)
// and no transcendental on the power path; the handoffs cost shared-memory
// traffic, not issue slots of the serial warps.
//
// Tensor-memory lanes: the W_dt slice is loaded with its even rows in
// operand rows 0–127 and its odd rows in 128–255 (a 3-D tensor map that
// steps over every second row), so the dt_proj result for channels 2ℓ and
// 2ℓ + 1 sits in lane ℓ of the two accumulator blocks, and phase-A warp q
// in lane quarter q (warp index mod 4) owns channels 2ℓ, 2ℓ + 1 with
// ℓ = 32q + lane.
//
// Synchronisation (mbarriers, every wait bounded by %globaltimer):
//   full / empty [4 stages]   producer → {phase-A, MMA};   {phase-A ×4, MMA} → producer
//   dtready [4 stages]        dt_proj MMA commit → phase-A
//   hfull / pready [4 slots]  phase-A ×4 → recurrence;     recurrence ×8 → phase-A
//   bcready / bcfree [3]      B|C MMA commit → recurrence;  recurrence ×8 → MMA
// A token outside the chunk (a tile that crosses its edge) gets r = 1 (Δ = 0),
// Δu = 0 and B = C = 0, so the recurrence runs unchanged and leaves the state
// exactly as it was; its y is not written.
//
// FINAL = false is the chunked scheme's state-only first pass: no C·H, no y;
// the end state goes to the carry buffer and the phase-A warps sum Δ.
#pragma once

#include "scan_fast.cuh"

namespace r2l {
namespace rscan {
namespace split {

constexpr int CHS = 256;                          // channels per CTA
// Warp roles, in this order: warps that feed the recurrence come first, so
// that a scheduler preferring lower warp indices serves them before the
// recurrence warps that wait on them.
constexpr int PROD_WARP = 0;                      // TMA producer
constexpr int MMA_WARP = 1;                       // B|C broadcast MMAs, TMEM owner
constexpr int DT_WARP = 2;                        // dt_proj MMAs
constexpr int AWARPS = 4;                         // phase-A warps
constexpr int AWARP0 = 3;
constexpr int RWARPS = 8;                         // recurrence warps
constexpr int RWARP0 = AWARP0 + AWARPS;
constexpr int THREADS = (RWARP0 + RWARPS) * 32;
constexpr int TEARDOWN_THREADS = THREADS - 32;    // every TMEM user (all but the producer)
constexpr int SIN = 4;                            // input stages
constexpr int GT = 4;                             // tokens per group
constexpr int GPT = TS / GT;                      // groups per tile
constexpr int HS = GPT;                           // handoff slots: the phase-A warps run one tile ahead
constexpr int NB = 3;                             // B|C slots in tensor memory
constexpr uint32_t ACT = TS * CHS * 2;            // bf16 [16 × 256] tile
constexpr uint32_t W_BYTES = CHS * DT_R * 2;      // bf16 W_dt slice [256 × 128]
constexpr uint32_t RD_SLOT = GT * CHS * 8;        // float2 (r or Δ, Δu) per (token, channel)
constexpr uint32_t P_SLOT = GT * CHS * 4;         // float p per (token, channel)
constexpr uint32_t OPB_SLOT = GT * 32 * 32;       // 32 operand rows of 32 bytes per token
constexpr uint32_t DR_ATOM = SIN * TS * 128;      // one K half of the Δr ring: [SIN stages][16 rows][128 B]
// TMEM columns: dt_raw of stage pair q = st / 2 at [64q, 64q + 64) (block 0
// then block 1, 32 tokens each: the pair's first tile, then its second), then
// NB slots of GT·32 columns of B|C.
constexpr uint32_t TM_DT = 0;
constexpr uint32_t TM_BC = SIN * 32;
constexpr uint32_t TM_COLS = 512;
static_assert(TM_BC + NB * GT * 32 <= TM_COLS, "TMEM budget");
static_assert(TS % GT == 0 && HS == GPT, "one handoff slot per group of a tile");
static_assert(SIN % 2 == 0, "dt_proj runs on pairs of stages");

struct Smem {
  static constexpr uint32_t W = 0;                       // [K atom][256 rows][128 B]: rows 0–127 even channels
  static constexpr uint32_t U = W + W_BYTES;             // [SIN] u tiles
  static constexpr uint32_t Z = U + SIN * ACT;           // [SIN] z tiles; y is written over z
  static constexpr uint32_t DR = Z + SIN * ACT;          // Δr ring: [K half][SIN][16 rows × 128 B], swizzled
  static constexpr uint32_t BC = DR + SIN * DR_TILE;     // [SIN] B|C tiles [16 × 32] fp32
  static constexpr uint32_t RD = BC + SIN * BC_TILE;     // [HS] (r or Δ, Δu)   [GT][CHS] float2
  static constexpr uint32_t P = RD + HS * RD_SLOT;       // [HS] p              [GT][CHS] float
  static constexpr uint32_t OPB = P + HS * P_SLOT;       // [NB] B|C operand rows
  static constexpr uint32_t ONE = OPB + NB * OPB_SLOT;   // the all-ones operand
  static constexpr uint32_t BAR = ONE + ONES_BYTES;
  static constexpr uint32_t NBAR = 3 * SIN + 3 + 2 * HS + 2 * NB;
  static constexpr uint32_t SLOT = BAR + NBAR * 8;
  static constexpr size_t BYTES = 1024 + SLOT + 16;
};
static_assert(Smem::BYTES <= 232448, "shared memory budget of one CTA");
static_assert(Smem::DR % 1024 == 0 && Smem::W % 1024 == 0, "swizzled tiles need 1024-byte alignment");

struct Bars {
  uint64_t *full, *empty, *dtready, *wfull, *drain, *dtdrain, *hfull, *pready, *bcready, *bcfree;
  __device__ explicit Bars(uint8_t* smem) {
    full = reinterpret_cast<uint64_t*>(smem + Smem::BAR);
    empty = full + SIN;
    dtready = empty + SIN;
    wfull = dtready + SIN;
    drain = wfull + 1;
    dtdrain = drain + 1;
    hfull = dtdrain + 1;
    pready = hfull + HS;
    bcready = pready + HS;
    bcfree = bcready + NB;
  }
};

// Tokens of a tile: row j of the tile is sequence position tbase + j; rows
// [jlo, jhi) lie in the chunk.  Tiles are taken from the chunk's right end
// (left end with FWD), and the tokens of a tile in the scan's order: the
// t-th token taken is row j = TS − 1 − t (t with FWD).
struct TileSpan {
  int tbase, jlo, jhi;
  __device__ TileSpan(int it, int s0, int e0, bool fwd) {
    tbase = fwd ? s0 + it * TS : e0 - (it + 1) * TS;
    jlo = (!fwd && s0 > tbase) ? s0 - tbase : 0;
    jhi = (fwd && e0 - tbase < TS) ? e0 - tbase : TS;
  }
  __device__ bool full() const { return jlo == 0 && jhi == TS; }
};

template <bool FWD>
__device__ __forceinline__ constexpr int tile_row(int t) { return FWD ? t : TS - 1 - t; }

// v = hi + mid + lo with each part exactly representable in tf32 (the top 11
// significant bits, the next 11, the last 2), so a tf32 MMA that adds the
// three reproduces v exactly.
__device__ __forceinline__ void split3(float v, float& hi, float& mid, float& lo) {
  hi = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
  const float r = v - hi;
  mid = __uint_as_float(__float_as_uint(r) & 0xFFFFE000u);
  lo = r - mid;
}

// ---------------------------------------------------------------- producer
template <bool FINAL, bool FWD>
__device__ __forceinline__ void run_producer(const CUtensorMap* tm_u, const CUtensorMap* tm_z,
                                             const CUtensorMap* tm_dr, const CUtensorMap* tm_bc,
                                             const CUtensorMap* tm_y, const CUtensorMap* tm_w, uint8_t* smem,
                                             const Bars& bar, int b, int cb, int s0, int e0, int ntiles,
                                             const Params& p) {
  using S = Smem;
  sm100::prefetch_tmap(tm_u);
  sm100::prefetch_tmap(tm_dr);
  sm100::prefetch_tmap(tm_bc);
  sm100::prefetch_tmap(tm_w);
  if (FINAL) {
    sm100::prefetch_tmap(tm_z);
    sm100::prefetch_tmap(tm_y);
  }
  // W_dt slice: K atoms a = 0, 1 of the even rows (block 0) and odd rows (block 1)
  sm100::mbar_arrive_expect_tx(bar.wfull, W_BYTES);
#pragma unroll
  for (int a = 0; a < DT_R / 64; ++a)
#pragma unroll
    for (int blk = 0; blk < 2; ++blk)
      sm100::tma_load_3d(smem + S::W + a * (CHS * 128) + blk * (128 * 128), tm_w, a * 64, blk, cb * (CHS / 2),
                         bar.wfull);
  constexpr uint32_t bytes = (FINAL ? 2 : 1) * ACT + BC_TILE + DR_TILE;
  int issued = 0;
  bool ok = true;
  const int iters = ntiles + (FINAL ? SIN : 0);
  for (int it = 0; it < iters; ++it) {
    const int st = it % SIN;
    const uint32_t ph = (uint32_t)(it / SIN) & 1u;
    if (!sm100::mbar_wait(&bar.empty[st], ph ^ 1u, p.err)) { ok = false; break; }
    if (FINAL && it >= SIN) {
      const TileSpan sp(it - SIN, s0, e0, FWD);   // the tile just finished in this stage
      if (sp.full()) {                             // its y sits over its z tile
        sm100::tma_store_2d(tm_y, smem + S::Z + st * ACT, cb * CHS, b * p.L + sp.tbase);
        sm100::bulk_commit();
        sm100::bulk_wait_read_all();               // the z slot is reloaded below
      }
    }
    if (it < ntiles) {
      // may start before row 0 (reverse, b = 0) or run past the last row (FWD): reads zeros
      const int row0 = b * p.L + TileSpan(it, s0, e0, FWD).tbase;
      sm100::mbar_arrive_expect_tx(&bar.full[st], bytes);
      sm100::tma_load_2d(smem + S::U + st * ACT, tm_u, cb * CHS, row0, &bar.full[st]);
      if (FINAL) sm100::tma_load_2d(smem + S::Z + st * ACT, tm_z, cb * CHS, row0, &bar.full[st]);
#pragma unroll
      for (int a = 0; a < DT_R / 64; ++a)
        sm100::tma_load_2d(smem + S::DR + a * DR_ATOM + st * (TS * 128), tm_dr, a * 64, row0, &bar.full[st]);
      sm100::tma_load_2d(smem + S::BC + st * BC_TILE, tm_bc, 0, row0, &bar.full[st]);
      ++issued;
    }
  }
  if (FINAL) sm100::bulk_wait_all();
  if (!ok) {  // let the loads still in flight land before the CTA can exit
    for (int it = issued - 1; it >= 0 && it >= issued - SIN; --it)
      sm100::mbar_wait(&bar.full[it % SIN], (uint32_t)(it / SIN) & 1u, nullptr, 1000000000ull);
    sm100::mbar_wait(bar.wfull, 0, nullptr, 1000000000ull);
  }
}

// ---------------------------------------------------------------- dt_proj warp
// One thread: per pair of tiles (stages st, st + 1, adjacent in the Δr ring)
// dt_raw = W_dt slice · Δr tilesᵀ into the pair's TMEM columns, as soon as
// both tiles have landed (for the last tile of an odd count the second half
// reads stale rows whose results nobody reads).
__device__ __forceinline__ void run_dt(uint8_t* smem, uint32_t tmem, const Bars& bar, int ntiles, unsigned* err) {
  using S = Smem;
  constexpr uint32_t idt = sm100::idesc_bf16_f32(128, 2 * TS);
  const uint32_t w0 = sm100::smem_u32(smem + S::W);
  bool ok = sm100::mbar_wait(bar.wfull, 0, err);
  for (int it = 0; it < ntiles && ok; it += 2) {
    const int st = it % SIN;
    const uint32_t ph = (uint32_t)(it / SIN) & 1u;
    if (!sm100::mbar_wait(&bar.full[st], ph, err)) break;
    if (it + 1 < ntiles && !sm100::mbar_wait(&bar.full[st + 1], ph, err)) break;
    sm100::tc_fence_after();
    const uint32_t d0 = sm100::smem_u32(smem + S::DR + st * (TS * 128));
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
#pragma unroll
      for (int k = 0; k < DT_R / 16; ++k) {
        const uint32_t a_addr = w0 + (k / 4) * (CHS * 128) + blk * (128 * 128) + (k % 4) * 32;
        const uint32_t b_addr = d0 + (k / 4) * DR_ATOM + (k % 4) * 32;
        sm100::mma_bf16(tmem + TM_DT + (uint32_t)((st / 2) * 64 + blk * 32), sm100::smem_desc_k128(a_addr),
                        sm100::smem_desc_k128(b_addr), idt, k != 0);
      }
    }
    sm100::mma_commit(&bar.dtready[st]);
    sm100::mma_commit(&bar.dtready[st + 1]);
  }
  sm100::mma_commit(bar.dtdrain);
  sm100::mbar_wait(bar.dtdrain, 0, err, 1000000000ull);
}

// ---------------------------------------------------------------- MMA warp
// Per group of 4 tokens: the B|C operand rows, then one tf32 MMA that
// broadcasts them into a TMEM slot.
template <bool FWD>
__device__ __forceinline__ void run_mma(uint8_t* smem, uint32_t tmem, const Bars& bar, int ntiles, int s0, int e0,
                                        unsigned* err) {
  using S = Smem;
  const int lane = threadIdx.x & 31;
  // the all-ones operand: rows (1, 1, 1, 0 | 0, 0, 0, 0) add a row's slots
  // 0–2; B|C operand rows hold (hi, mid, lo, 0) of one value and zeros in
  // slots 4–7, which are written here once and never again
  for (int n = lane; n < 128; n += 32) {
    uint8_t* r0 = smem + S::ONE + opnd_row(n);
    *reinterpret_cast<float4*>(r0) = make_float4(1.0f, 1.0f, 1.0f, 0.0f);
    *reinterpret_cast<float4*>(r0 + 128) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  for (int n = lane; n < NB * GT * 32; n += 32)
    *reinterpret_cast<float4*>(smem + S::OPB + (n / (GT * 32)) * OPB_SLOT + opnd_row(n % (GT * 32)) + 128) =
        make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  sm100::fence_proxy_async_smem();
  __syncwarp();
  constexpr uint32_t ibc = sm100::idesc_tf32_f32(128, GT * 32);
  const uint64_t a_ones = sm100::smem_desc_noswz(sm100::smem_u32(smem + S::ONE), 128, 256);
  bool ok = true;
  int G = 0;
  for (int it = 0; it < ntiles && ok; ++it) {
    const int st = it % SIN;
    const uint32_t ph = (uint32_t)(it / SIN) & 1u;
    if (!sm100::mbar_wait(&bar.full[st], ph, err)) break;
    const TileSpan sp(it, s0, e0, FWD);
    const float* bct = reinterpret_cast<const float*>(smem + S::BC + st * BC_TILE);
#pragma unroll 1
    for (int g = 0; g < GPT; ++g, ++G) {
      const int bs = G % NB;
      if (!sm100::mbar_wait(&bar.bcfree[bs], ((uint32_t)(G / NB) & 1u) ^ 1u, err)) { ok = false; break; }
      sm100::tc_fence_after();
      uint8_t* opb = smem + S::OPB + bs * OPB_SLOT;
      float v[GT];
#pragma unroll
      for (int t = 0; t < GT; ++t) {               // row 32·t + lane: value `lane` of the group's t-th token
        const int j = FWD ? g * GT + t : TS - 1 - g * GT - t;
        v[t] = (j >= sp.jlo && j < sp.jhi) ? bct[j * 32 + lane] : 0.0f;
      }
#pragma unroll
      for (int t = 0; t < GT; ++t) {
        float hi, mid, lo;
        split3(v[t], hi, mid, lo);
        *reinterpret_cast<float4*>(opb + opnd_row(32 * t + lane)) = make_float4(hi, mid, lo, 0.0f);
      }
      sm100::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {        // columns 32·t + n of the slot: value n (B_0..15, C_0..15) of token t
        sm100::mma_tf32(tmem + TM_BC + (uint32_t)(bs * GT * 32), a_ones,
                        sm100::smem_desc_noswz(sm100::smem_u32(opb), 128, 256), ibc, 0u);
        sm100::mma_commit(&bar.bcready[bs]);
      }
      __syncwarp();
    }
    if (!ok) break;
    if (lane == 0) sm100::mbar_arrive(&bar.empty[st]);   // done with the tile's B|C
  }
  if (lane == 0) {
    sm100::mma_commit(bar.drain);
    sm100::mbar_wait(bar.drain, 0, err, 1000000000ull);
  }
  __syncwarp();
}

// ---------------------------------------------------------------- recurrence
// One token of one channel: the 16 decays, the state update and (FINAL)
// p = ⟨C, H⟩.  bc: the token's B_0..15, then (FINAL) C_0..15; rd: (r, Δu) on
// the power path, (Δ, Δu) otherwise.
template <bool FINAL, bool POW>
__device__ __forceinline__ float rec_token(float2 (&H)[8], const uint32_t (&bc)[FINAL ? 32 : 16], float2 rd,
                                           const float (&A2)[16]) {
  float2 a[8];
  if (POW) {
    const float r = rd.x;
    const float r2 = r * r;
    a[0] = make_float2(r, r2);
    a[1] = __fmul2_rn(a[0], make_float2(r2, r2));              // r³ r⁴
    const float r4 = a[1].y;
    a[2] = __fmul2_rn(a[0], make_float2(r4, r4));              // r⁵ r⁶
    a[3] = __fmul2_rn(a[1], make_float2(r4, r4));              // r⁷ r⁸
    const float r8 = a[3].y;
#pragma unroll
    for (int q = 0; q < 4; ++q) a[4 + q] = __fmul2_rn(a[q], make_float2(r8, r8));   // r⁹ … r¹⁶
  } else {
    const float2 d2 = make_float2(rd.x, rd.x);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 e = __fmul2_rn(d2, make_float2(A2[2 * k], A2[2 * k + 1]));
      a[k] = make_float2(ex2_approx(e.x), ex2_approx(e.y));
    }
  }
  const float2 du2 = make_float2(rd.y, rd.y);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    H[k] = __ffma2_rn(a[k], H[k],
                      __fmul2_rn(du2, make_float2(__uint_as_float(bc[2 * k]), __uint_as_float(bc[2 * k + 1]))));
  if constexpr (!FINAL) {
    return 0.0f;
  } else {
  float2 acc0 = __fmul2_rn(make_float2(__uint_as_float(bc[16]), __uint_as_float(bc[17])), H[0]);
  float2 acc1 = __fmul2_rn(make_float2(__uint_as_float(bc[18]), __uint_as_float(bc[19])), H[1]);
#pragma unroll
  for (int k = 2; k < 8; k += 2) {
    acc0 = __ffma2_rn(make_float2(__uint_as_float(bc[16 + 2 * k]), __uint_as_float(bc[17 + 2 * k])), H[k], acc0);
    acc1 = __ffma2_rn(make_float2(__uint_as_float(bc[18 + 2 * k]), __uint_as_float(bc[19 + 2 * k])), H[k + 1],
                      acc1);
  }
  const float2 s = __fadd2_rn(acc0, acc1);
  return s.x + s.y;
  }
}

template <bool FINAL, bool POW>
__device__ __forceinline__ void run_rec(uint8_t* smem, uint32_t tmem, const Bars& bar, int ntiles, int b, int cb,
                                        int k, const Params& p) {
  using S = Smem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cl = (warp - RWARP0) * 32 + lane;
  const int c = cb * CHS + cl;
  const bool cvalid = c < p.E;
  float A2[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) A2[m] = (!POW && cvalid) ? -expf(p.A_log[c * 16 + m]) * LOG2E : 0.0f;
  float2 H[8];
  const float* cin = (FINAL && p.nc > 1 && cvalid) ? p.carry + (((long long)b * p.nc + k) * p.E + c) * 16 : nullptr;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 v = cin ? reinterpret_cast<const float4*>(cin)[q] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    H[2 * q] = make_float2(v.x, v.y);
    H[2 * q + 1] = make_float2(v.z, v.w);
  }
  // every lane of the broadcast holds the same B|C; read this warp's quarter
  const uint32_t t_bc = tmem + ((uint32_t)((warp & 3) * 32) << 16) + TM_BC;
  const float2* rd_base = reinterpret_cast<const float2*>(smem + S::RD) + cl;
  float* p_base = reinterpret_cast<float*>(smem + S::P) + cl;
  const int ngroups = ntiles * GPT;
  for (int G = 0; G < ngroups; ++G) {
    const int slot = G % HS, bs = G % NB;
    if (!sm100::mbar_wait(&bar.hfull[slot], (uint32_t)(G / HS) & 1u, p.err)) break;
    if (!sm100::mbar_wait(&bar.bcready[bs], (uint32_t)(G / NB) & 1u, p.err)) break;
    sm100::tc_fence_after();
    float2 rd[GT];
#pragma unroll
    for (int t = 0; t < GT; ++t) rd[t] = rd_base[(slot * GT + t) * CHS];
    const uint32_t tb = t_bc + (uint32_t)(bs * GT * 32);
    uint32_t b0[FINAL ? 32 : 16], b1[FINAL ? 32 : 16];   // without FINAL only B is read
    float pv[GT];
    sm100::tmem_ld_nowait(tb, b0);
    sm100::tmem_wait_ld_bind(b0);
    sm100::tmem_ld_nowait(tb + 32, b1);             // token 1 in flight during token 0
    pv[0] = rec_token<FINAL, POW>(H, b0, rd[0], A2);
    sm100::tmem_wait_ld_bind(b1);
    sm100::tmem_ld_nowait(tb + 64, b0);
    pv[1] = rec_token<FINAL, POW>(H, b1, rd[1], A2);
    sm100::tmem_wait_ld_bind(b0);
    sm100::tmem_ld_nowait(tb + 96, b1);
    pv[2] = rec_token<FINAL, POW>(H, b0, rd[2], A2);
    sm100::tmem_wait_ld_bind(b1);
    pv[3] = rec_token<FINAL, POW>(H, b1, rd[3], A2);
    if (FINAL) {
#pragma unroll
      for (int t = 0; t < GT; ++t) p_base[(slot * GT + t) * CHS] = pv[t];
    }
    sm100::tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      sm100::mbar_arrive(&bar.bcfree[bs]);
      sm100::mbar_arrive(&bar.pready[slot]);
    }
  }
  if (!FINAL && cvalid) {   // the chunk's end state S_k
    float4* dst = reinterpret_cast<float4*>(p.carry + (((long long)b * p.nc + k) * p.E + c) * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_float4(H[2 * q].x, H[2 * q].y, H[2 * q + 1].x, H[2 * q + 1].y);
  }
}

// ---------------------------------------------------------------- phase-A warps
struct AuxCtx {
  int cl0;               // first of the thread's two channels (within the CTA)
  bool cval;             // the pair lies inside d_inner (d_inner is even)
  float2 dtb, Dv;
  uint32_t t_dt;         // TMEM address of this warp's lane quarter
};

// One group of GT tokens for the thread's two channels: the epilogue of group
// g of the previous tile (EPI; stage pst, span psp) and phase A of group g of
// this tile (stage st, span sp), both through handoff slot g.  All shared-
// memory reads come first, then the arithmetic, then all writes: the compiler
// cannot tell the buffers apart, so a read placed after a write would wait
// for it and the tokens' latency chains would run one after another.
//
// Epilogue: y = (p + D u)·SiLU(z) into the z slot for a whole tile (stored
// by TMA), else straight to global memory for the rows inside the chunk.
// Phase A: (r or Δ, Δu) into the slot; dtr holds the tile's dt_raw, columns
// 0–15 channel cl0 and 16–31 channel cl0 + 1, in tile-row order.
template <bool FINAL, bool POW, bool FWD, bool EPI>
__device__ __forceinline__ void aux_group(uint8_t* smem, const AuxCtx& ax, int g, int st, const TileSpan& sp,
                                          int pst, const TileSpan& psp, const uint32_t (&dtr)[32], float2& sumd,
                                          int b, int cb, const Params& p) {
  using S = Smem;
  const float* pv = reinterpret_cast<const float*>(smem + S::P) + g * GT * CHS + ax.cl0;
  const bf16* pu = reinterpret_cast<const bf16*>(smem + S::U + pst * ACT) + ax.cl0;
  bf16* pz = reinterpret_cast<bf16*>(smem + S::Z + pst * ACT) + ax.cl0;
  const bf16* su = reinterpret_cast<const bf16*>(smem + S::U + st * ACT) + ax.cl0;
  float4* rd = reinterpret_cast<float4*>(reinterpret_cast<float2*>(smem + S::RD) + g * GT * CHS + ax.cl0);
  // ---- reads
  float2 ep[GT], eu[GT], ez[GT], au[GT];
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    const int j = tile_row<FWD>(g * GT + t);
    if (EPI) {
      ep[t] = *reinterpret_cast<const float2*>(pv + t * CHS);
      eu[t] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(pu + j * CHS));
      ez[t] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(pz + j * CHS));
    }
    au[t] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(su + j * CHS));
  }
  // ---- arithmetic
  __nv_bfloat162 yv[GT];
  float4 hv[GT];
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    const int j = tile_row<FWD>(g * GT + t);
    if (EPI) {
      const float2 sv = __ffma2_rn(ax.Dv, eu[t], ep[t]);
      yv[t] = __floats2bfloat162_rn(sv.x * silu_fast(ez[t].x), sv.y * silu_fast(ez[t].y));
    }
    const bool valid = j >= sp.jlo && j < sp.jhi;
    float d0, r0, d1, r1;
    softplus_and_decay(__uint_as_float(dtr[j]) + ax.dtb.x, d0, r0);
    softplus_and_decay(__uint_as_float(dtr[16 + j]) + ax.dtb.y, d1, r1);
    const float2 du = __fmul2_rn(make_float2(d0, d1), au[t]);
    if (valid) {
      hv[t] = make_float4(POW ? r0 : d0, du.x, POW ? r1 : d1, du.y);
      if (!FINAL) sumd = __fadd2_rn(sumd, make_float2(d0, d1));
    } else {
      hv[t] = make_float4(POW ? 1.0f : 0.0f, 0.0f, POW ? 1.0f : 0.0f, 0.0f);
    }
  }
  // ---- writes
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    rd[(t * CHS) / 2] = hv[t];
    if (EPI) {
      const int j = tile_row<FWD>(g * GT + t);
      if (psp.full()) {
        *reinterpret_cast<__nv_bfloat162*>(pz + j * CHS) = yv[t];
      } else if (j >= psp.jlo && j < psp.jhi && ax.cval) {
        *reinterpret_cast<__nv_bfloat162*>(p.y + ((long long)b * p.L + psp.tbase + j) * p.ldy + cb * CHS +
                                           ax.cl0) = yv[t];
      }
    }
  }
}

// The last tile's epilogue, group g (nothing follows it to overlap with).
template <bool FWD>
__device__ __forceinline__ void aux_epilogue_last(uint8_t* smem, const AuxCtx& ax, int g, int pst,
                                                  const TileSpan& psp, int b, int cb, const Params& p) {
  using S = Smem;
  const float* pv = reinterpret_cast<const float*>(smem + S::P) + g * GT * CHS + ax.cl0;
  const bf16* pu = reinterpret_cast<const bf16*>(smem + S::U + pst * ACT) + ax.cl0;
  bf16* pz = reinterpret_cast<bf16*>(smem + S::Z + pst * ACT) + ax.cl0;
  float2 ep[GT], eu[GT], ez[GT];
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    const int j = tile_row<FWD>(g * GT + t);
    ep[t] = *reinterpret_cast<const float2*>(pv + t * CHS);
    eu[t] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(pu + j * CHS));
    ez[t] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(pz + j * CHS));
  }
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    const int j = tile_row<FWD>(g * GT + t);
    const float2 sv = __ffma2_rn(ax.Dv, eu[t], ep[t]);
    const __nv_bfloat162 yv = __floats2bfloat162_rn(sv.x * silu_fast(ez[t].x), sv.y * silu_fast(ez[t].y));
    if (psp.full()) {
      *reinterpret_cast<__nv_bfloat162*>(pz + j * CHS) = yv;
    } else if (j >= psp.jlo && j < psp.jhi && ax.cval) {
      *reinterpret_cast<__nv_bfloat162*>(p.y + ((long long)b * p.L + psp.tbase + j) * p.ldy + cb * CHS + ax.cl0) =
          yv;
    }
  }
}

template <bool FINAL, bool POW, bool FWD>
__device__ __forceinline__ void run_aux(uint8_t* smem, uint32_t tmem, const Bars& bar, int ntiles, int s0, int e0,
                                        int b, int cb, int k, const Params& p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;                      // TMEM lane quarter (warp index mod 4)
  AuxCtx ax;
  ax.cl0 = 2 * (32 * q + lane);
  const int c0 = cb * CHS + ax.cl0;
  ax.cval = c0 < p.E;
  ax.dtb = ax.cval ? make_float2(p.dt_b[c0], p.dt_b[c0 + 1]) : make_float2(0.0f, 0.0f);
  ax.Dv = ax.cval ? make_float2(p.D[c0], p.D[c0 + 1]) : make_float2(0.0f, 0.0f);
  ax.t_dt = tmem + ((uint32_t)(q * 32) << 16) + TM_DT;
  float2 sumd = make_float2(0.0f, 0.0f);
  bool ok = true;
  for (int it = 0; it < ntiles && ok; ++it) {
    const int st = it % SIN;
    const uint32_t ph = (uint32_t)(it / SIN) & 1u;
    if (!sm100::mbar_wait(&bar.full[st], ph, p.err)) break;
    if (!sm100::mbar_wait(&bar.dtready[st], ph, p.err)) break;
    sm100::tc_fence_after();
    uint32_t dtr[32], dlo[16], dhi[16];              // channel cl0 (block 0), cl0 + 1 (block 1)
    const uint32_t dcol = ax.t_dt + (uint32_t)((st / 2) * 64 + (st & 1) * TS);
    sm100::tmem_ld16_nowait(dcol, dlo);
    sm100::tmem_ld16_nowait(dcol + 32, dhi);
    sm100::tmem_wait_ld_bind(dlo);
    sm100::tmem_wait_ld_bind(dhi);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      dtr[i] = dlo[i];
      dtr[16 + i] = dhi[i];
    }
    const TileSpan sp(it, s0, e0, FWD);
    const int pst = (it + SIN - 1) % SIN;                  // the previous tile's stage
    const TileSpan psp(it - 1, s0, e0, FWD);
#pragma unroll
    for (int g = 0; g < GPT; ++g) {
      const int G = it * GPT + g;
      // slot g was last used by group G − HS (the previous tile's group g)
      if (!sm100::mbar_wait(&bar.pready[g], ((uint32_t)(G / HS) & 1u) ^ 1u, p.err)) { ok = false; break; }
      if (FINAL && it > 0)
        aux_group<FINAL, POW, FWD, true>(smem, ax, g, st, sp, pst, psp, dtr, sumd, b, cb, p);
      else
        aux_group<FINAL, POW, FWD, false>(smem, ax, g, st, sp, pst, psp, dtr, sumd, b, cb, p);
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&bar.hfull[g]);
    }
    if (!ok) break;
    // the stage is released once nothing reads it any more: after phase A
    // without FINAL, after the epilogue (one tile later) with it
    const int rel = FINAL ? it - 1 : it;
    if (rel >= 0) {
      if (FINAL) sm100::fence_proxy_async_smem();          // y tile visible to the TMA store
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&bar.empty[rel % SIN]);
    }
  }
  if (FINAL && ok && ntiles > 0) {
    const int it = ntiles;                                 // the last tile's epilogues
    const int pst = (it - 1) % SIN;
    const TileSpan psp(it - 1, s0, e0, FWD);
#pragma unroll
    for (int g = 0; g < GPT; ++g) {
      const int G = it * GPT + g;
      if (!sm100::mbar_wait(&bar.pready[g], ((uint32_t)(G / HS) & 1u) ^ 1u, p.err)) { ok = false; break; }
      aux_epilogue_last<FWD>(smem, ax, g, pst, psp, b, cb, p);
    }
    if (ok) {
      sm100::fence_proxy_async_smem();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&bar.empty[pst]);
    }
  }
  if (!FINAL && ax.cval) {                                 // Σ Δ over the chunk
    float* dst = p.carry_sum + ((long long)b * p.nc + k) * p.E + c0;
    dst[0] = sumd.x;
    dst[1] = sumd.y;
  }
}

// ---------------------------------------------------------------- kernel
// One CTA: channels [256·blockIdx.x, +256) of sequence blockIdx.z over chunk
// blockIdx.y of p.T tokens.
// 15 warps at up to 128 registers: each of the SM's four 16K-register
// partitions holds up to four of the block's warps.
template <bool FINAL, bool FWD>
__global__ void __launch_bounds__(THREADS, 1)
scan_split_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_z,
                  const __grid_constant__ CUtensorMap tm_dr, const __grid_constant__ CUtensorMap tm_bc,
                  const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_w,
                  const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Bars bar(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::SLOT);
  const int cb = blockIdx.x, k = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = p.len[b];
  const int s0 = k * p.T;
  const int e0 = min(s0 + p.T, n);
  if (s0 >= n) {                               // chunk entirely in the padding
    if (!FINAL && tid < CHS) {
      const int c = cb * CHS + tid;
      if (c < p.E) {
        float4* dst = reinterpret_cast<float4*>(p.carry + (((long long)b * p.nc + k) * p.E + c) * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        p.carry_sum[((long long)b * p.nc + k) * p.E + c] = 0.0f;
      }
    }
    return;
  }
  const int ntiles = (e0 - s0 + TS - 1) / TS;
  if (tid == 0) {
    for (int s = 0; s < SIN; ++s) {
      sm100::mbar_init(&bar.full[s], 1);
      sm100::mbar_init(&bar.empty[s], AWARPS + 1);
      sm100::mbar_init(&bar.dtready[s], 1);
    }
    sm100::mbar_init(bar.wfull, 1);
    sm100::mbar_init(bar.drain, 1);
    sm100::mbar_init(bar.dtdrain, 1);
    for (int h = 0; h < HS; ++h) {
      sm100::mbar_init(&bar.hfull[h], AWARPS);
      sm100::mbar_init(&bar.pready[h], RWARPS);
    }
    for (int s = 0; s < NB; ++s) {
      sm100::mbar_init(&bar.bcready[s], 1);
      sm100::mbar_init(&bar.bcfree[s], RWARPS);
    }
    sm100::fence_barrier_init();
  }
  if (warp == MMA_WARP) sm100::tmem_alloc(tmem_slot, TM_COLS);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the power path is decided once per call (a_log_check_kernel)
  const bool use_pow = !p.force_general && *p.a_general == 0u;

  if (warp == PROD_WARP) {
    if ((tid & 31) == 0)
      run_producer<FINAL, FWD>(&tm_u, &tm_z, &tm_dr, &tm_bc, &tm_y, &tm_w, smem, bar, b, cb, s0, e0, ntiles, p);
    return;                                    // takes no part in the teardown
  }
  if (warp == DT_WARP) {
    if ((tid & 31) == 0) run_dt(smem, tmem, bar, ntiles, p.err);
    __syncwarp();
    sm100::tc_fence_before();
    sm100::named_bar_sync(1, TEARDOWN_THREADS);
    return;
  }
  if (warp == MMA_WARP) {
    run_mma<FWD>(smem, tmem, bar, ntiles, s0, e0, p.err);
    sm100::named_bar_sync(1, TEARDOWN_THREADS);   // every TMEM reader is done
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, TM_COLS);
    return;
  }
  if (warp >= RWARP0) {
    if (use_pow) run_rec<FINAL, true>(smem, tmem, bar, ntiles, b, cb, k, p);
    else run_rec<FINAL, false>(smem, tmem, bar, ntiles, b, cb, k, p);
  } else {
    if (use_pow) run_aux<FINAL, true, FWD>(smem, tmem, bar, ntiles, s0, e0, b, cb, k, p);
    else run_aux<FINAL, false, FWD>(smem, tmem, bar, ntiles, s0, e0, b, cb, k, p);
  }
  sm100::tc_fence_before();
  sm100::named_bar_sync(1, TEARDOWN_THREADS);
}

}  // namespace split
}  // namespace rscan
}  // namespace r2l
