// Host launcher of the bf16 reverse selective scan: chunk choice, TMA
// descriptors for the u / z / dt_raw / B|C tiles, and the launch sequence.
#include <cuda.h>

#include "launch_pdl.h"
#include "scan_fast.cuh"
#include "scan_fast.h"
#include "scan_pair.cuh"
#include "scan_split.cuh"
#include "tmap.h"

namespace r2l {

int scan_auto_chunk_tokens(int B, int L, int E, bool pair) {
  using namespace rscan;
  if (pair) {
    // two threads per channel, one 256-channel CTA per SM: split sequences
    // only when one pass leaves most SMs idle, into as many chunks as one wave
    // of CTAs holds (each chunk costs a second, state-only pass)
    const long long ctas1 = (long long)B * ((E + rscan::pair::CHP - 1) / rscan::pair::CHP);
    const int whole = (L + TS - 1) / TS * TS;
    if (ctas1 * 3 >= 148LL * 2) return whole;
    long long nc = 148 / ctas1;
    if (nc < 2) return whole;
    long long T = (L + nc - 1) / nc;
    T = (T + TS - 1) / TS * TS;
    if (T < 4 * TS) T = 4 * TS;
    return (int)(T < whole ? T : whole);
  }
  // Compute warps with one chunk per sequence; below ~6 per SM of a 148-SM
  // part the sequence is split so that about 24 per SM are in flight.
  const long long warps1 = (long long)B * ((E + CTHREADS - 1) / CTHREADS) * CWARPS;
  const long long target = 148LL * 24;
  const int whole = (L + TS - 1) / TS * TS;
  if (warps1 >= 148LL * 6) return whole;
  long long nc = (target + warps1 - 1) / warps1;
  long long T = (L + nc - 1) / nc;
  T = (T + TS - 1) / TS * TS;
  if (T < 4 * TS) T = 4 * TS;
  return (int)(T < whole ? T : whole);
}

int scan_resolve_chunk_tokens(int B, int L, int E, int chunk_tokens, bool pair) {
  using namespace rscan;
  if (chunk_tokens <= 0) return scan_auto_chunk_tokens(B, L, E, pair);
  const int T = (chunk_tokens + TS - 1) / TS * TS;
  const int whole = (L + TS - 1) / TS * TS;
  return T < whole ? T : whole;
}

size_t scan_carry_bytes(int B, int L, int E, int chunk_tokens, bool pair) {
  const int T = scan_resolve_chunk_tokens(B, L, E, chunk_tokens, pair);
  const long long nc = (L + T - 1) / T;
  if (nc <= 1) return 0;
  return (size_t)B * nc * E * 17 * sizeof(float);
}

namespace {

// The kernel behind scans with dt_proj fused: 2 = the recurrence on warps of
// its own (scan_split.cuh), 1 = two threads per channel (scan_pair.cuh),
// 0 = one thread per channel with B|C read from shared memory.
#ifndef R2L_SCAN_IMPL
#define R2L_SCAN_IMPL 1
#endif

template <bool FWD>
cudaError_t launch_split(const ScanArgs& a, const rscan::Params& p, int nc, cudaStream_t st, int* launches) {
  using namespace rscan;
  namespace sp = rscan::split;
  constexpr int CHS = sp::CHS;
  const long long M = (long long)a.B * a.L;
  CUtensorMap tu, tz, tdr, tbc, ty, tw;
  if (!make_tmap_2d(&tu, a.u, 2, a.E, M, a.ldu * 2, CHS, TS, 0) ||
      !make_tmap_2d(&tz, a.z, 2, a.E, M, a.ldz * 2, CHS, TS, 0) ||
      !make_tmap_2d(&tbc, a.bc, 4, 32, M, a.ldbc * 4, 32, TS, 0) ||
      !make_tmap_2d(&ty, a.y, 2, a.E, M, a.ldy * 2, CHS, TS, 0) ||
      !make_tmap_2d(&tdr, a.dr, 2, DT_R, M, a.lddr * 2, 64, TS, 128) ||
      !make_tmap_rows_by_parity(&tw, a.wdt, 2, DT_R, a.E, (long long)DT_R * 2, 64, CHS / 2, 128))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sp::scan_split_kernel<true, FWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sp::Smem::BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.E + CHS - 1) / CHS, nc, a.B);
  if (nc > 1) {
    if ((e = cudaFuncSetAttribute(sp::scan_split_kernel<false, FWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sp::Smem::BYTES)) != cudaSuccess)
      return e;
    sp::scan_split_kernel<false, FWD><<<grid, sp::THREADS, sp::Smem::BYTES, st>>>(tu, tz, tdr, tbc, ty, tw, p);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    chunk_carry_kernel<<<dim3((a.E + 127) / 128, a.B), 128, 0, st>>>(p);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    if (launches) *launches += 2;
  }
  sp::scan_split_kernel<true, FWD><<<grid, sp::THREADS, sp::Smem::BYTES, st>>>(tu, tz, tdr, tbc, ty, tw, p);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaSuccess;
}

template <bool FWD>
cudaError_t launch_pair(const ScanArgs& a, const rscan::Params& p, int nc, cudaStream_t st, int* launches) {
  using namespace rscan;
  using Sp = pair::SmemPair;
  constexpr int CHP = pair::CHP;
  const long long M = (long long)a.B * a.L;
  CUtensorMap tu, tz, tdr, tbc, ty, tw;
  if (!make_tmap_2d(&tu, a.u, 2, a.E, M, a.ldu * 2, CHP, TS, 0) ||
      !make_tmap_2d(&tz, a.z, 2, a.E, M, a.ldz * 2, CHP, TS, 0) ||
      !make_tmap_2d(&tbc, a.bc, 4, 32, M, a.ldbc * 4, 32, TS, 0) ||
      !make_tmap_2d(&ty, a.y, 2, a.E, M, a.ldy * 2, CHP, TS, 0) ||
      !make_tmap_2d(&tdr, a.dr, 2, DT_R, M, a.lddr * 2, 64, TS, 128) ||
      !make_tmap_2d(&tw, a.wdt, 2, DT_R, a.E, (long long)DT_R * 2, 64, CHP, 128))
    return cudaErrorInvalidValue;
  // training mode (p.hck): the final pass also stores the scan gradient's checkpoints
  const bool ckpt = !FWD && p.hck != nullptr;
  cudaError_t e = cudaFuncSetAttribute(pair::scan_pair_kernel<true, FWD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sp::BYTES);
  if (e != cudaSuccess) return e;
  if (ckpt && (e = cudaFuncSetAttribute(pair::scan_pair_kernel<true, false, true>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sp::BYTES)) != cudaSuccess)
    return e;
  const dim3 grid((a.E + CHP - 1) / CHP, nc, a.B);
  if (nc > 1) {
    if ((e = cudaFuncSetAttribute(pair::scan_pair_kernel<false, FWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)Sp::BYTES)) != cudaSuccess)
      return e;
    if ((e = launch_pdl(pair::scan_pair_kernel<false, FWD>, grid, dim3(Sp::THREADS), Sp::BYTES, st, tu, tz, tdr,
                        tbc, ty, tw, p)) != cudaSuccess)
      return e;
    if ((e = launch_pdl(chunk_carry_kernel, dim3((a.E + 127) / 128, a.B), dim3(128), 0, st, p)) != cudaSuccess)
      return e;
    if (launches) *launches += 2;
  }
  if (ckpt)
    e = launch_pdl(pair::scan_pair_kernel<true, false, true>, grid, dim3(Sp::THREADS), Sp::BYTES, st, tu, tz, tdr,
                   tbc, ty, tw, p);
  else
    e = launch_pdl(pair::scan_pair_kernel<true, FWD>, grid, dim3(Sp::THREADS), Sp::BYTES, st, tu, tz, tdr, tbc, ty,
                   tw, p);
  if (e != cudaSuccess) return e;
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaSuccess;
}

template <bool FINAL, bool DTMMA, bool FWD>
cudaError_t prep_kernel() {
  return cudaFuncSetAttribute(rscan::chunk_scan_kernel<FINAL, DTMMA, FWD>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rscan::Smem<DTMMA>::BYTES);
}

template <bool DTMMA, bool FWD>
cudaError_t launch(const ScanArgs& a, const rscan::Params& p, int nc, cudaStream_t st, int* launches) {
  using namespace rscan;
  using Sm = Smem<DTMMA>;
  const long long M = (long long)a.B * a.L;
  CUtensorMap tu, tz, tdt, tbc, ty, tw;
  if (!make_tmap_2d(&tu, a.u, 2, a.E, M, a.ldu * 2, CH, TS, 0) ||
      !make_tmap_2d(&tz, a.z, 2, a.E, M, a.ldz * 2, CH, TS, 0) ||
      !make_tmap_2d(&tbc, a.bc, 4, 32, M, a.ldbc * 4, 32, TS, 0) ||
      !make_tmap_2d(&ty, a.y, 2, a.E, M, a.ldy * 2, CH, TS, 0))
    return cudaErrorInvalidValue;
  if (DTMMA) {
    if (!make_tmap_2d(&tdt, a.dr, 2, DT_R, M, a.lddr * 2, 64, TS, 128) ||
        !make_tmap_2d(&tw, a.wdt, 2, DT_R, a.E, (long long)DT_R * 2, 64, CH, 128))
      return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_2d(&tdt, a.dt, 2, a.E, M, a.ldt * 2, CH, TS, 0)) return cudaErrorInvalidValue;
    tw = tdt;
  }
  cudaError_t e;
  const dim3 grid((a.E + CH - 1) / CH, nc, a.B);
  if (DTMMA && R2L_SCAN_IMPL == 2) return launch_split<FWD>(a, p, nc, st, launches);
  if (DTMMA && R2L_SCAN_IMPL == 1) return launch_pair<FWD>(a, p, nc, st, launches);
  if ((e = prep_kernel<true, DTMMA, FWD>()) != cudaSuccess) return e;
  if (nc > 1) {
    if ((e = prep_kernel<false, DTMMA, FWD>()) != cudaSuccess) return e;
    chunk_scan_kernel<false, DTMMA, FWD><<<grid, Sm::THREADS, Sm::BYTES, st>>>(tu, tz, tdt, tbc, ty, tw, p);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    chunk_carry_kernel<<<dim3((a.E + 127) / 128, a.B), 128, 0, st>>>(p);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    if (launches) *launches += 2;
  }
  chunk_scan_kernel<true, DTMMA, FWD><<<grid, Sm::THREADS, Sm::BYTES, st>>>(tu, tz, tdt, tbc, ty, tw, p);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaSuccess;
}

}  // namespace

bool scan_writes_checkpoints(int dt_rank, bool forward) {
  return dt_rank == kScanFusedDtRank && !forward && R2L_SCAN_IMPL == 1;
}

cudaError_t scan_bf16(const ScanArgs& a, cudaStream_t st, int* launches) {
  using namespace rscan;
  if (launches) *launches = 0;
  const long long M = (long long)a.B * a.L;
  if (M <= 0 || a.E <= 0) return cudaSuccess;
  const int T = a.chunk_tokens;
  if (T <= 0 || T % TS) return cudaErrorInvalidValue;
  const int nc = (a.L + T - 1) / T;
  if (nc > 1 && !a.carry) return cudaErrorInvalidValue;

  Params p;
  p.A_log = a.A_log;
  p.D = a.D;
  p.dt_b = a.dt_b;
  p.y = a.y;
  p.ldy = a.ldy;
  p.E = a.E;
  p.L = a.L;
  p.T = T;
  p.nc = nc;
  p.len = a.len;
  p.carry = a.carry;
  p.carry_sum = a.carry ? a.carry + (size_t)a.B * nc * a.E * 16 : nullptr;
  p.err = a.err;
  p.force_general = a.force_general;
  p.a_general = a.a_general;
  if (!a.force_general && !a.a_general) return cudaErrorInvalidValue;
  p.fwd = a.forward;
  p.hck = nullptr;
  p.nc16 = (a.L + 15) / 16;
  if (a.hck_written) *a.hck_written = 0;
  if (a.hck && a.dt_mma && scan_writes_checkpoints(kScanFusedDtRank, a.forward != 0)) {   // the two-thread kernel
    p.hck = a.hck;
    if (a.hck_written) *a.hck_written = 1;
  }
  if (a.dt_mma) {
    if (!a.dr || !a.wdt || (a.lddr % 8)) return cudaErrorInvalidValue;
    return a.forward ? launch<true, true>(a, p, nc, st, launches) : launch<true, false>(a, p, nc, st, launches);
  }
  return a.forward ? launch<false, true>(a, p, nc, st, launches) : launch<false, false>(a, p, nc, st, launches);
}

}  // namespace r2l
