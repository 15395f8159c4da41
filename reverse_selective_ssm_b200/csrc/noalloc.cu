// r2l_reverse_scan_noalloc: the reverse selective scan with its scratch (the
// device status word, the clamped lengths and the chunk carries) held in a
// fixed-size array that is part of the library's device image, for callers
// that must not allocate device memory at run time.
#include "r2l.h"

namespace {

// The scratch.  One copy exists on every device that loads the library, for
// as long as the library stays loaded.  In host code the name only denotes a
// host-side stand-in: kernels must be given the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_scan_scratch[R2L_NOALLOC_SCRATCH_BYTES];

// Device address of g_scan_scratch in the current device's context, looked up
// on every call.  The lookup allocates nothing; not caching it means a call
// after cudaDeviceReset (or after the primary context was destroyed and made
// again) gets the array's address in the new context instead of a dangling
// one.  The very first lookup on a device loads the library's device image
// into that context.
r2l_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scan_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return R2L_ERR_CUDA;
  }
  *out = p;
  return R2L_OK;
}

}  // namespace

extern "C" r2l_status r2l_reverse_scan_noalloc(const void* u, const void* z, int ldz, const void* dt_raw,
                                               const float* bc, int ldbc, const float* A_log, const float* D,
                                               const float* dt_b, void* y, const r2l_dims* dims, int B, int L,
                                               const int32_t* lengths, int chunk_tokens, void* stream) {
  if (!dims || B <= 0 || L <= 0) return R2L_ERR_INVALID_ARG;
  const size_t need = r2l_reverse_scan_workspace_size(dims, B, L, chunk_tokens);
  if (need == 0) return R2L_ERR_INVALID_ARG;
  if (need > (size_t)R2L_NOALLOC_SCRATCH_BYTES) return R2L_ERR_WORKSPACE;
  void* scratch = nullptr;
  const r2l_status s = scratch_address(&scratch);
  if (s != R2L_OK) return s;
  // The scan zeroes the status word itself and writes the lengths and every
  // carry slot it later reads, so the previous call's contents never leak in.
  return r2l_reverse_scan(u, z, ldz, dt_raw, bc, ldbc, A_log, D, dt_b, y, dims, B, L, lengths, chunk_tokens,
                          scratch, (size_t)R2L_NOALLOC_SCRATCH_BYTES, stream);
}
