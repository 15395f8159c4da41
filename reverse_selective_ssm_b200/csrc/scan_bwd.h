// Host interface of the fp32 reverse-scan gradient (scan_bwd.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <cuda_bf16.h>

namespace r2l {

constexpr int SCAN_BWD_MAX_CHUNK = 32;   // positions per chunk (shared memory: 5 KB each)

struct ScanBwdArgs {
  const float *u, *z, *dt_raw, *bc, *A_log, *D, *dt_b, *dy;
  // bf16 u and z (what the bf16 forward writes) in place of u and z when set
  const __nv_bfloat16 *u16, *z16;
  int ldz, ldbc;
  float *du, *dz, *ddt_raw, *dbc, *dA_log, *dD, *ddt_b;
  int ld_dz, ld_dbc;
  int B, L, E, chunk_tokens;
  const int* lengths;   // device [B] or null
  unsigned* status;     // device status word (R2L_DEVFLAG_* bits)
  // [B][⌈L/16⌉][E][16]: H at every position 16(k+1) < len, which a
  // training-mode forward has stored for every sequence whose length is a
  // multiple of 16; the gradient computes the other sequences' into it (null:
  // it computes all of them in its own scratch).  Used by the walk along each
  // sequence only.
  float* hck;
  // bf16 copies of ddt_raw and dz written instead of the fp32 arrays (rows of
  // stride ld_ddt16 / ld_dz16), by the walk along each sequence only
  // (scan_bwd_walks); null: fp32
  __nv_bfloat16* ddt16;
  long long ld_ddt16;
  __nv_bfloat16* dz16;
  long long ld_dz16;
};

// Whether a call of this shape takes the walk along each sequence.
bool scan_bwd_walks(int B, int E, int chunk_tokens);

int scan_bwd_chunk_tokens(int chunk_tokens);
bool scan_bwd_supported(int B, int L, int E, int chunk_tokens);   // grid limits of the launches
size_t scan_bwd_scratch_bytes(int B, int L, int E, int chunk_tokens);
cudaError_t scan_bwd_f32(const ScanBwdArgs& a, void* scratch, cudaStream_t st);

}  // namespace r2l
