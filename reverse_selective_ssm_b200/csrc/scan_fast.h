// Host interface of the bf16 reverse selective scan (scan_fast.cuh).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stddef.h>

namespace r2l {

// dt_rank for which the scan computes dt_proj itself on the tensor cores.
constexpr int kScanFusedDtRank = 128;

struct ScanArgs {
  const __nv_bfloat16* u;   long long ldu;    // [B·L, E]
  const __nv_bfloat16* z;   long long ldz;    // [B·L, E] (row stride ldz)
  const __nv_bfloat16* dt;  long long ldt;    // dt_raw [B·L, E] (before bias and softplus); unused with dt_mma
  const __nv_bfloat16* dr;  long long lddr;   // dt_mma: Δr [B·L, 128] (x_proj output)
  const __nv_bfloat16* wdt;                    // dt_mma: W_dt [E, 128]
  const float* bc;          long long ldbc;   // [B·L, 32]: B in columns 0..15, C in 16..31
  const float* A_log;                          // [E, 16]
  const float* D;                              // [E]
  const float* dt_b;                           // [E]
  __nv_bfloat16* y;         long long ldy;    // [B·L, E]
  int B, L, E;
  const int* len;                              // device [B], clamped to [0, L]
  int chunk_tokens;                            // tokens per chunk (resolved, > 0)
  float* carry;                                // scan_carry_bytes() of device scratch (may be null if 1 chunk)
  unsigned* err;                               // device status word
  int force_general;                           // never use the A = -(1..16) power path
  const unsigned* a_general;                   // device flag of a_log_check_kernel (0: power path); read
                                               // unless force_general
  int dt_mma;                                  // compute dt_raw = Δr·W_dtᵀ inside the scan (dt_rank 128)
  int forward;                                 // left-to-right block
  // training mode: H at every position 16(k+1) < len into hck[B][⌈L/16⌉][E][16]
  // (the scan gradient's checkpoints), for every sequence whose length is a
  // multiple of 16.  Only the two-thread kernel (right to left, dt_proj fused)
  // writes them; *hck_written (when set) says whether it did.
  float* hck;
  int* hck_written;
};

// Tokens per chunk chosen from the shape alone (deterministic, no device
// query).  `pair`: the scan runs with dt_proj fused (two threads per channel).
int scan_auto_chunk_tokens(int B, int L, int E, bool pair = false);
// Chunk length actually used for a request (0 = automatic), a multiple of 16.
int scan_resolve_chunk_tokens(int B, int L, int E, int chunk_tokens, bool pair = false);
// Bytes of carry scratch the scan needs for this shape and chunk length.
size_t scan_carry_bytes(int B, int L, int E, int chunk_tokens, bool pair = false);
// Whether a bf16 scan with this dt_rank and direction stores the scan
// gradient's checkpoints when given a buffer (ScanArgs::hck).
bool scan_writes_checkpoints(int dt_rank, bool forward);
// Enqueue the scan (1 or 3 launches).  Returns the number of kernels launched
// through *launches when not null.
cudaError_t scan_bf16(const ScanArgs& a, cudaStream_t st, int* launches);

}  // namespace r2l
