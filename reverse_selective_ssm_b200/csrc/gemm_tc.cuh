// Persistent warp-specialised bf16 GEMM on the 5th-generation tensor cores
// (tcgen05 + TMEM), fed by TMA:
//
//     C[m, n] = Σ_k A[m, k] · B[n, k]        (A [M, K], B [N, K], both K-major)
//
// which is y = x Wᵀ for an nn.Linear weight W [out, in].  Used for the four
// projections of the Mamba-1 block in the R2L sidecar (in_proj, x_proj,
// dt_proj, out_proj; "Bifocal Diffusion Language Models", arXiv 2606.27732v1,
// §3.4 step ❷).
//
// One CTA per SM (192 threads) loops over 128 × BN output tiles:
//   warp 0     TMA producer: 64-wide K slices of A and B into a STAGES-deep
//              shared-memory ring (128-byte swizzle), one mbarrier per slot.
//   warp 1     allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN,
//              K=16) into one of two TMEM accumulators and commits the slot
//              back to the producer when its MMAs retire.
//   warps 2-5  epilogue: tcgen05.ld the accumulator (warp w reads TMEM lanes
//              32·(w%4) …), round, store rows of C; then release the
//              accumulator so the next tile's MMAs overlap this epilogue.
// Rows of padding (position ≥ the sequence's length) are not stored, and
// 128-row tiles with no valid row are skipped by every role alike.
// Every mbarrier wait is bounded; on a timeout the kernel raises a flag in the
// workspace status word, drains what it issued and returns.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace r2l {

// True if rows [r0, r1) of a right-padded [B, L] batch contain a valid row.
__device__ __forceinline__ bool rows_have_valid(const int* __restrict__ len, int L, long long r0,
                                                long long r1) {
  long long b = r0 / L;
  long long start = b * L;
  while (start < r1) {
    const long long lo = r0 > start ? r0 : start;
    if ((int)(lo - start) < len[b]) return true;
    ++b;
    start += L;
  }
  return false;
}

// MB: 128-row MMA blocks per tile.  MB = 1 keeps two accumulators so one
// tile's epilogue overlaps the next tile's MMAs; MB = 2 (BN = 256) fills all
// 512 TMEM columns with one 256 × 256 tile, reading a third fewer operand
// bytes per flop; its epilogue copies the accumulator into registers and
// hands it back before staging and storing, so the next tile's MMAs wait
// only for the TMEM reads.
template <int BN, typename TOut, int MB = 1>
struct TcGemmCfg {
  static constexpr int BM = 128 * MB;
  static constexpr int NACC = MB == 1 ? 2 : 1;        // accumulator buffers
  static constexpr int EPI_WARPS = 4 * MB;             // one warpgroup per 128-row block
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int BK = 64;                       // 128 bytes of bf16: one swizzle row
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  // epilogue staging: per epilogue warp two [32 rows × 32 cols] buffers
  static constexpr uint32_t STG_BYTES = 32 * 32 * sizeof(TOut);
  static constexpr int STG_SWIZZLE = 32 * sizeof(TOut);   // 64 (bf16 rows) or 128 (fp32 rows)
  static constexpr size_t BUDGET = 227 * 1024 - 1024 - 256 - 2 * EPI_WARPS * STG_BYTES;
  static constexpr int STAGES_FIT = (int)(BUDGET / STAGE_BYTES);
  static constexpr int STAGES = STAGES_FIT < 6 ? STAGES_FIT : 6;
  static constexpr uint32_t TMEM_COLS = 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
  static_assert(MB == 1 || (MB == 2 && BN == 256), "two M blocks only with 256-column tiles");
  static constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + STAGES * (size_t)STAGE_BYTES + 2 * EPI_WARPS * STG_BYTES + 256;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "UMMA N for M=128 is a multiple of 16 up to 256");
  static_assert(B_BYTES % 1024 == 0, "B tile must keep 1024-byte swizzle-atom alignment");
  static_assert(STAGES >= 3, "shared memory too small for the pipeline");
};

// Write one thread's row of 32 values into a [32 × 32] staging buffer laid
// out for a TMA store with STG_SWIZZLE: the 16-byte chunk k of row r sits at
// chunk k ^ ((r >> 1) & 3) for 64-byte rows, k ^ (r & 7) for 128-byte rows,
// so the 32 rows written by a warp hit distinct banks.
template <typename TOut>
__device__ __forceinline__ void stage_row32(uint8_t* buf, int r, const float (&v)[32]);

template <>
__device__ __forceinline__ void stage_row32<bf16>(uint8_t* buf, int r, const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 p = __floats2bfloat162_rn(v[k * 8 + 2 * j], v[k * 8 + 2 * j + 1]);
      w[j] = *reinterpret_cast<uint32_t*>(&p);
    }
    const int pk = k ^ ((r >> 1) & 3);
    *reinterpret_cast<uint4*>(buf + r * 64 + pk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <>
__device__ __forceinline__ void stage_row32<float>(uint8_t* buf, int r, const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int pk = k ^ (r & 7);
    *reinterpret_cast<float4*>(buf + r * 128 + pk * 16) = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  }
}

template <typename TOut>
__device__ __forceinline__ void store_row32(TOut* dst, const float (&v)[32]);

template <>
__device__ __forceinline__ void store_row32<bf16>(bf16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 p = __floats2bfloat162_rn(v[q * 8 + 2 * j], v[q * 8 + 2 * j + 1]);
      w[j] = *reinterpret_cast<uint32_t*>(&p);
    }
    d4[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <>
__device__ __forceinline__ void store_row32<float>(float* dst, const float (&v)[32]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// C2 (optional): columns n < c2_cols are also written, rounded to bf16, into
// C2[m, n] (row stride ldc2).  x_proj uses it to hand Δr to dt_proj in bf16.
// splits > 1 (fp32 C only; C2 unused): each tile's K range is cut into
// `splits` parts computed by different CTAs; the part s of a tile is stored
// at rows s·Mp + row of the tensor tmC describes (a partial-sum buffer of
// `splits` slices of Mp rows, Mp = M rounded up to whole tiles), and a
// separate kernel adds the slices in a fixed order.  For short, wide-K GEMMs
// with fewer tiles than SMs.
// AMN / BMN: A (B) is stored MN-major, as [K, M] ([K, N]) with the M (N)
// index contiguous; it is loaded in boxes of 64 MN elements × 64 K rows and
// read through the MN-major descriptor.  The weight gradients of the
// projections contract over positions, and their operands are activations
// and gradients stored position-major, i.e. MN-major.
template <int BN, typename TOut, int MB = 1, int AMN = 0, int BMN = 0>
__global__ void __launch_bounds__(TcGemmCfg<BN, TOut, MB>::THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC, bf16* __restrict__ C2, int ldc2, int c2_cols,
               int M, int N, int K, const int* __restrict__ len, int L, unsigned* __restrict__ err,
               int splits) {
  using Cfg = TcGemmCfg<BN, TOut, MB>;
  constexpr int BM = Cfg::BM, BK = Cfg::BK, STAGES = Cfg::STAGES, NACC = Cfg::NACC;
  static_assert(!BMN || BN % 64 == 0, "an MN-major B tile is whole 64-column boxes");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* sStg = sB + STAGES * Cfg::B_BYTES;          // 2 staging buffers per epilogue warp (1024-byte aligned)
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + 2 * Cfg::EPI_WARPS * Cfg::STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_k = (K + BK - 1) / BK;
  const int kps = (num_k + splits - 1) / splits;       // K blocks per split
  const long long total = (long long)num_m * num_n * splits;   // work units: (tile, split)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      sm100::mbar_init(&tfull[a], 1);
      sm100::mbar_init(&tempty[a], 32 * Cfg::EPI_WARPS);
    }
    sm100::mbar_init(drain, 1);
    sm100::fence_barrier_init();
    sm100::prefetch_tmap(&tmA);
    sm100::prefetch_tmap(&tmB);
    sm100::prefetch_tmap(&tmC);
  }
  grid_dep_wait();
  if (warp == 1) sm100::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_launch();

  auto tile_live = [&](long long t) -> bool {
    if (!len) return true;
    const long long r0 = (t / splits / num_n) * BM;
    const long long r1 = r0 + BM < M ? r0 + BM : M;
    return rows_have_valid(len, L, r0, r1);
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
        const long long tile = t / splits;
        const int mb = (int)(tile / num_n), nb = (int)(tile % num_n);
        const int kb0 = (int)(t % splits) * kps, kb1 = kb0 + kps < num_k ? kb0 + kps : num_k;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!sm100::mbar_wait(&empty[stage], phase ^ 1u, err)) { ok = false; break; }
          sm100::mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
          if (AMN) {
#pragma unroll
            for (int i = 0; i < BM / 64; ++i)
              sm100::tma_load_2d(sA + stage * Cfg::A_BYTES + i * 8192, &tmA, mb * BM + 64 * i, kb * BK, &full[stage]);
          } else {
            sm100::tma_load_2d(sA + stage * Cfg::A_BYTES, &tmA, kb * BK, mb * BM, &full[stage]);
          }
          if (BMN) {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i)
              sm100::tma_load_2d(sB + stage * Cfg::B_BYTES + i * 8192, &tmB, nb * BN + 64 * i, kb * BK, &full[stage]);
          } else {
            sm100::tma_load_2d(sB + stage * Cfg::B_BYTES, &tmB, kb * BK, nb * BN, &full[stage]);
          }
          ++issued[stage];
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {  // drain the loads still in flight before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) sm100::mbar_wait(&full[s], (uint32_t)(issued[s] - 1) & 1u, nullptr, 1000000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = sm100::idesc_bf16_f32_mn(128, BN, AMN != 0, BMN != 0);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (long long t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!tile_live(t)) continue;
        if (!sm100::mbar_wait(&tempty[acc], aphase ^ 1u, err)) { ok = false; break; }
        sm100::tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        const int kb0 = (int)(t % splits) * kps, kb1 = kb0 + kps < num_k ? kb0 + kps : num_k;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!sm100::mbar_wait(&full[stage], phase, err)) { ok = false; break; }
          sm100::tc_fence_after();
          const uint32_t a0 = sm100::smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b0 = sm100::smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {  // rows 128·mb …: accumulator columns [BN·mb, BN·mb + BN)
              // K-major: 16 K elements are 32 bytes along a 128-byte row; MN-major:
              // 16 K rows are two 1024-byte atoms, and 128 M rows are two 8 KB boxes
              const uint64_t da = AMN ? sm100::smem_desc_mn128(a0 + mb * (2 * 8192) + k * 2048)
                                      : sm100::smem_desc_k128(a0 + mb * (128 * 128) + k * 32);
              const uint64_t db = BMN ? sm100::smem_desc_mn128(b0 + k * 2048) : sm100::smem_desc_k128(b0 + k * 32);
              sm100::mma_bf16(d_tmem + (uint32_t)(mb * BN), da, db, idesc, (kb != kb0) | (k != 0));
            }
          }
          sm100::mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        sm100::mma_commit(&tfull[acc]);
        if (++acc == NACC) { acc = 0; aphase ^= 1u; }
      }
      // all MMAs issued by this thread have retired once `drain` completes
      sm100::mma_commit(drain);
      sm100::mbar_wait(drain, 0, err, 1000000000ull);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each 32 × 32 block goes TMEM -> registers -> swizzled staging buffer ->
    // TMA store (rows past M or columns past N are clipped by the store).
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;   // the 128-row M block this warp drains
    uint8_t* stg = sStg + (warp - 2) * 2 * Cfg::STG_BYTES;
    int acc = 0;
    uint32_t aphase = 0;
    int chunk = 0;
    if constexpr (MB == 2) {
      // One accumulator: read the thread's whole row (256 columns) out of
      // TMEM as packed bf16 pairs, hand the accumulator back at once so the
      // next tile's MMAs start, then stage and store the row from registers
      // while they run.
      static_assert(std::is_same<TOut, bf16>::value, "256 x 256 tiles store bf16");
      for (long long t = blockIdx.x; t < total; t += gridDim.x) {
        if (!tile_live(t)) continue;
        if (!sm100::mbar_wait(&tfull[0], aphase, err)) break;
        sm100::tc_fence_after();
        const long long tile = t / splits;
        const int mb = (int)(tile / num_n), nb = (int)(tile % num_n);
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 32) {
          float v[32];
          sm100::tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * BN + c0), v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            pk[c0 / 2 + j] = *reinterpret_cast<uint32_t*>(&b2);
          }
        }
        sm100::tc_fence_before();
        sm100::mbar_arrive(&tempty[0]);
        aphase ^= 1u;
        const int row0 = mb * BM + h * 128 + q * 32;
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 32, ++chunk) {
          uint8_t* buf = stg + (chunk & 1) * Cfg::STG_BYTES;
          if (lane == 0) sm100::bulk_wait_read_le1();
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int pkk = k ^ ((lane >> 1) & 3);
            *reinterpret_cast<uint4*>(buf + lane * 64 + pkk * 16) =
                make_uint4(pk[c0 / 2 + 4 * k], pk[c0 / 2 + 4 * k + 1], pk[c0 / 2 + 4 * k + 2], pk[c0 / 2 + 4 * k + 3]);
          }
          sm100::fence_proxy_async_smem();
          __syncwarp();
          const int col = nb * BN + c0;
          if (lane == 0 && col < N && row0 < M) {
            sm100::tma_store_2d(&tmC, buf, col, row0);
            sm100::bulk_commit();
          }
        }
      }
      if (lane == 0) sm100::bulk_wait_all();
    } else
    for (long long t = blockIdx.x; t < total; t += gridDim.x) {
      if (!tile_live(t)) continue;
      if (!sm100::mbar_wait(&tfull[acc], aphase, err)) break;
      sm100::tc_fence_after();
      const long long tile = t / splits;
      const int mb = (int)(tile / num_n), nb = (int)(tile % num_n);
      {
        const int row0 = mb * BM + h * 128 + q * 32;     // this warp's 32 rows of M block h
        const long long row = (long long)row0 + lane;
        const bool row_ok = row < M && (!len || row_valid(len, L, row));
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32, ++chunk) {
          float v[32];
          sm100::tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + h * BN + c0), v);
          const int col = nb * BN + c0;
          uint8_t* buf = stg + (chunk & 1) * Cfg::STG_BYTES;
          if (lane == 0) sm100::bulk_wait_read_le1();   // the store that used `buf` has read it
          __syncwarp();
          stage_row32<TOut>(buf, lane, v);
          sm100::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && col < N && row0 < M) {
            const int prow = splits > 1 ? (int)(t % splits) * (num_m * BM) + row0 : row0;
            sm100::tma_store_2d(&tmC, buf, col, prow);
            sm100::bulk_commit();
          }
          if (C2 && splits == 1 && row_ok && col < c2_cols) {
            bf16* d2 = C2 + row * (long long)ldc2 + col;
            if (col + 32 <= c2_cols) {
              store_row32<bf16>(d2, v);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < c2_cols - col) d2[j] = __float2bfloat16_rn(v[j]);
            }
          }
        }
      }
      sm100::tc_fence_before();
      sm100::mbar_arrive(&tempty[acc]);
      if (++acc == NACC) { acc = 0; aphase ^= 1u; }
    }
    if (MB == 1 && lane == 0) sm100::bulk_wait_all();
  }

  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 1) sm100::tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
}

}  // namespace r2l
