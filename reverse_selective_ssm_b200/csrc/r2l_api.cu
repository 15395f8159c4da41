// libr2l: host side of the C ABI declared in include/r2l.h — argument checks,
// workspace carve-up and the launch sequence of the R2L sidecar forward
// ("Bifocal Diffusion Language Models", arXiv 2606.27732v1, §3.4 steps ❶–❹).
//
// Launch sequence for one hook (all on the caller's stream, no host sync):
//   prep lengths → in_proj GEMM → conv+SiLU → x_proj GEMM → dt_proj GEMM
//   → reverse selective scan (+SiLU(z) gate) → out_proj GEMM
//   → LayerNorm + tanh(s)-gated residual (valid rows only)
#include <cmath>
#include <cstdint>
#include <cstring>

#include "r2l.h"
#include "common.cuh"
#include "simt_kernels.cuh"
#include "scan_simple.cuh"
#include "launch_pdl.h"
#include "tc_gemm.h"
#include "scan_fast.h"
#include "scan_bwd.h"
#include "conv_fast.cuh"
#include "bwd_kernels.cuh"

// conv + SiLU fused into the x_proj GEMM on the bf16 path (0: separate kernels).
#ifndef R2L_CONVX
#define R2L_CONVX 1
#endif

#include <algorithm>
#include <type_traits>

using r2l::bf16;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Byte offsets of the workspace regions for a [B, L] batch.
struct Plan {
  size_t status, len, aflags, xz, u, dbc, dr, dt, y, o, carry, xsplit, xsplit_bytes, osplit, osplit_bytes, total;
  int chunk_tokens;  // scan chunk length (bf16 path)
  int osplits;       // out_proj K splits left to the LayerNorm kernel (0: o stored by the GEMM)
  bool ragged = false;  // the caller gave per-sequence lengths (set by the entry point)
  long long M;
  int E, d, R, N, ldd;
  size_t act;
  unsigned flags;
};

bool make_plan(const r2l_dims* dm, int B, int L, Plan* p) {
  if (!dm || B <= 0 || L <= 0) return false;
  if (dm->d_model <= 0 || dm->d_inner <= 0 || dm->dt_rank <= 0 || dm->d_state <= 0) return false;
  if (dm->dtype != R2L_BF16 && dm->dtype != R2L_FP32) return false;
  p->M = (long long)B * L;
  p->E = dm->d_inner;
  p->d = dm->d_model;
  p->R = dm->dt_rank;
  p->N = dm->d_state;
  p->ldd = p->R + 2 * p->N;
  p->act = dm->dtype == R2L_BF16 ? 2 : 4;
  p->flags = dm->flags;
  const size_t M = (size_t)p->M;
  size_t off = 0;
  p->status = off; off = align_up(off + 16, kAlign);
  p->len = off;    off = align_up(off + sizeof(int) * (size_t)B, kAlign);
  p->aflags = off; off = align_up(off + sizeof(unsigned) * r2l::kMaxCheckedHooks, kAlign);   // per-hook power-path flags
  p->xz = off;     off = align_up(off + M * 2 * p->E * p->act, kAlign);
  p->u = off;      off = align_up(off + M * p->E * p->act, kAlign);
  p->dbc = off;    off = align_up(off + M * p->ldd * sizeof(float), kAlign);
  p->dr = off;     off = align_up(off + M * p->R * 2, kAlign);   // Δr in bf16 (tensor-core path)
  // the bf16 layer with dt_rank 128 runs dt_proj inside the scan: dt_raw never
  // reaches memory, so its region is only reserved for the other paths
  const bool pair = dm->dtype == R2L_BF16 && p->R == r2l::kScanFusedDtRank;
  p->dt = off;     if (!pair) off = align_up(off + M * p->E * p->act, kAlign);
  p->y = off;      off = align_up(off + M * p->E * p->act, kAlign);
  p->o = off;      off = align_up(off + M * p->d * p->act, kAlign);
  p->chunk_tokens = r2l::scan_resolve_chunk_tokens(B, L, p->E, 0, pair);
  p->carry = off;
  if (dm->dtype == R2L_BF16) off = align_up(off + r2l::scan_carry_bytes(B, L, p->E, p->chunk_tokens, pair), kAlign);
  // x_proj split-K partial sums (bf16 path, few 128-row tiles)
  p->xsplit = off;
  p->xsplit_bytes = dm->dtype == R2L_BF16 ? r2l::tc_gemm_partial_bytes(p->M, p->ldd, p->E) : 0;
  off = align_up(off + p->xsplit_bytes, kAlign);
  // out_proj of a batch whose 128 × 256 tiles do not fill the SMs (bf16 path,
  // d ≤ 2048): K-split fp32 partial sums that the LayerNorm kernel adds
  p->osplits = dm->dtype == R2L_BF16 && p->d <= 2048 ? r2l::tc_gemm_kept_splits(p->M, p->d, p->E) : 0;
  p->osplit = off;
  p->osplit_bytes = (size_t)p->osplits * (size_t)((p->M + 127) / 128 * 128) * p->d * sizeof(float);
  off = align_up(off + p->osplit_bytes, kAlign);
  p->total = off;
  return true;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }


r2l_status check_weights(const r2l_weights* w) {
  if (!w) return R2L_ERR_INVALID_ARG;
  const void* ptrs[] = {w->in_proj_w, w->conv_w, w->conv_b, w->x_proj_w, w->dt_proj_w,
                        w->dt_proj_b, w->A_log, w->D, w->out_proj_w};
  for (const void* q : ptrs) {
    if (!q) return R2L_ERR_INVALID_ARG;
    if (!aligned16(q)) return R2L_ERR_ALIGNMENT;
  }
  if ((w->ln_w == nullptr) != (w->ln_b == nullptr)) return R2L_ERR_INVALID_ARG;
  if (w->ln_w && (!aligned16(w->ln_w) || !aligned16(w->ln_b))) return R2L_ERR_ALIGNMENT;
  return R2L_OK;
}

r2l_status check_call(void* hidden, const r2l_dims* dm, int B, int L, void* ws, size_t ws_bytes,
                      Plan* plan) {
  if (!hidden || !dm) return R2L_ERR_INVALID_ARG;
  if (!make_plan(dm, B, L, plan)) return R2L_ERR_INVALID_ARG;
  if (dm->d_state != 16 || dm->d_conv != 4) return R2L_ERR_UNSUPPORTED;
  // bf16 path: TMA needs 16-byte row strides for every GEMM operand
  if (dm->dtype == R2L_BF16 && ((dm->d_model % 8) || (dm->d_inner % 8) || (dm->dt_rank % 8)))
    return R2L_ERR_UNSUPPORTED;
  // grid limits of the launches below
  if (L > 65535 || B > 65535 || (plan->M + 63) / 64 > 65535) return R2L_ERR_UNSUPPORTED;
  if (!aligned16(hidden)) return R2L_ERR_ALIGNMENT;
  if (!ws || ws_bytes < plan->total) return R2L_ERR_WORKSPACE;
  if (!aligned16(ws)) return R2L_ERR_ALIGNMENT;
  return R2L_OK;
}

#define R2L_LAUNCH_CHECK()                                   \
  do {                                                       \
    if (cudaPeekAtLastError() != cudaSuccess) {              \
      (void)cudaGetLastError();                              \
      return R2L_ERR_CUDA;                                   \
    }                                                        \
  } while (0)

// Optional stage-boundary events and launch counting (profiled entry point).
struct Prof {
  cudaEvent_t* ev = nullptr;
  int launches = 0;
  r2l_status mark(int k, cudaStream_t st) {
    if (ev && cudaEventRecord(ev[k], st) != cudaSuccess) return R2L_ERR_CUDA;
    return R2L_OK;
  }
};

template <typename TA, typename TW, typename TC>
r2l_status gemm(const TA* A, int lda, const TW* W, int ldw, TC* C, int ldc, long long M, int N,
                int K, const int* len, int L, cudaStream_t st) {
  dim3 grid((N + 63) / 64, (unsigned)((M + 63) / 64));
  r2l::gemm_simt_kernel<TA, TW, TC><<<grid, 256, 0, st>>>(A, lda, W, ldw, C, ldc, (int)M, N, K, len, L);
  R2L_LAUNCH_CHECK();
  return R2L_OK;
}

r2l_status prep(const Plan& p, char* ws, const int32_t* lengths, int B, int L, cudaStream_t st,
                Prof* prof = nullptr) {
  if (prof) prof->launches++;
  if (cudaMemsetAsync(ws + p.status, 0, 16, st) != cudaSuccess) return R2L_ERR_CUDA;
  r2l::prep_lengths_kernel<<<(B + 127) / 128, 128, 0, st>>>(
      lengths, (int*)(ws + p.len), B, L, (unsigned*)(ws + p.status));
  R2L_LAUNCH_CHECK();
  return R2L_OK;
}

// The float nearest ln(m+1) for m = 0..15: the A_log of the S4D-real
// initialisation A = −(1..16), against which a_log_check_kernel compares.
r2l::LnTable ln_table() {
  r2l::LnTable t;
  for (int m = 0; m < 16; ++m) {
    const float v = (float)std::log((double)(m + 1));
    std::memcpy(&t.bits[m], &v, sizeof(v));
  }
  return t;
}

// Decide the scan's power path for this call (see a_log_check_kernel): writes
// 0 or 1 into the second word of the status region.  With force_general the
// scan never reads it.
r2l_status check_a_log(const float* A_log, int E, unsigned* status, bool force_general, cudaStream_t st,
                       Prof* prof) {
  if (force_general) return R2L_OK;
  if (prof) prof->launches++;
  r2l::ALogSet set{};
  set.a[0] = A_log;
  r2l::a_log_check_kernel<<<1, 1024, 0, st>>>(set, E, ln_table(), status + 1);
  R2L_LAUNCH_CHECK();
  return R2L_OK;
}

// The same decision for the n hooks of a stack (n ≤ kMaxCheckedHooks), in one
// launch: flags[k] for hook k.
r2l_status check_a_log_hooks(const r2l_weights* w, int n, int E, unsigned* flags, cudaStream_t st) {
  r2l::ALogSet set{};
  for (int k = 0; k < n; ++k) set.a[k] = w[k].A_log;
  r2l::a_log_check_kernel<<<n, 1024, 0, st>>>(set, E, ln_table(), flags);
  R2L_LAUNCH_CHECK();
  return R2L_OK;
}

#define R2L_TRY(expr)                  \
  do {                                 \
    r2l_status _s = (expr);            \
    if (_s != R2L_OK) return _s;       \
  } while (0)

// One projection y = x Wᵀ: tensor cores (tcgen05) for bf16, SIMT fp32 otherwise.
// c2 (bf16 path only): columns < c2_cols also stored in bf16 (Δr for dt_proj).
template <typename T, typename TC>
r2l_status proj(const T* A, int lda, const T* W, int ldw, TC* C, int ldc, long long M, int N, int K,
                const int* len, int L, unsigned* err, cudaStream_t st, bf16* c2 = nullptr, int ldc2 = 0,
                int c2_cols = 0, float* partial = nullptr, size_t partial_bytes = 0, bool ragged = false) {
  if constexpr (std::is_same<T, bf16>::value) {
    r2l::TcGemm g{};
    g.ragged = ragged;
    g.A = A; g.lda = lda; g.B = W; g.ldb = ldw; g.C = C; g.ldc = ldc;
    g.c_fp32 = std::is_same<TC, float>::value;
    g.C2 = c2; g.ldc2 = ldc2; g.c2_cols = c2_cols;
    g.M = (int)M; g.N = N; g.K = K; g.len = len; g.L = L; g.err = err;
    g.partial = partial; g.partial_bytes = partial_bytes;
    return r2l::tc_gemm(g, st) == cudaSuccess ? R2L_OK : R2L_ERR_CUDA;
  } else {
    return gemm(A, lda, W, ldw, C, ldc, M, N, K, len, L, st);
  }
}

// LayerNorm + gated residual for bf16 rows of d <= 2048 (nv = ceil(d / 256)).
// With ps (the out_proj partial sums of a small batch, `splits` slices of
// `slice` floats) o is added up from them, and written to `o` when o_keep is
// set (the layer always sets it: the gradient of a training forward and the
// debug entry point read o back).
template <int NV>
r2l_status ln_bf16_nv(bool has_ln, unsigned blocks, cudaStream_t st, bf16* h, const bf16* o, const float* lw,
                      const float* lb, float g, int d, const int* len, int L, long long M, float* hhat,
                      const float* ps, int splits, long long slice, bool o_keep) {
  cudaError_t e;
  const dim3 grid(blocks), block(128);
  bf16* o_out = o_keep ? const_cast<bf16*>(o) : nullptr;
  if (ps)
    e = has_ln ? r2l::launch_pdl(r2l::ln_residual_bf16_kernel<NV, true, true>, grid, block, 0, st, h, o, lw, lb, g, d,
                                 len, L, M, hhat, ps, splits, slice, o_out)
               : r2l::launch_pdl(r2l::ln_residual_bf16_kernel<NV, false, true>, grid, block, 0, st, h, o, lw, lb, g, d,
                                 len, L, M, hhat, ps, splits, slice, o_out);
  else
    e = has_ln ? r2l::launch_pdl(r2l::ln_residual_bf16_kernel<NV, true>, grid, block, 0, st, h, o, lw, lb, g, d, len,
                                 L, M, hhat, (const float*)nullptr, 0, 0LL, (bf16*)nullptr)
               : r2l::launch_pdl(r2l::ln_residual_bf16_kernel<NV, false>, grid, block, 0, st, h, o, lw, lb, g, d, len,
                                 L, M, hhat, (const float*)nullptr, 0, 0LL, (bf16*)nullptr);
  if (e != cudaSuccess) return R2L_ERR_CUDA;
  R2L_LAUNCH_CHECK();
  return R2L_OK;
}

r2l_status launch_ln_bf16(int nv, bool has_ln, unsigned blocks, cudaStream_t st, bf16* h, const bf16* o,
                          const float* lw, const float* lb, float g, int d, const int* len, int L, long long M,
                          float* hhat, const float* ps = nullptr, int splits = 0, long long slice = 0,
                          bool o_keep = false) {
  switch (nv) {
    case 1: return ln_bf16_nv<1>(has_ln, blocks, st, h, o, lw, lb, g, d, len, L, M, hhat, ps, splits, slice, o_keep);
    case 2: return ln_bf16_nv<2>(has_ln, blocks, st, h, o, lw, lb, g, d, len, L, M, hhat, ps, splits, slice, o_keep);
    case 3: return ln_bf16_nv<3>(has_ln, blocks, st, h, o, lw, lb, g, d, len, L, M, hhat, ps, splits, slice, o_keep);
    case 4: return ln_bf16_nv<4>(has_ln, blocks, st, h, o, lw, lb, g, d, len, L, M, hhat, ps, splits, slice, o_keep);
    case 5: return ln_bf16_nv<5>(has_ln, blocks, st, h, o, lw, lb, g, d, len, L, M, hhat, ps, splits, slice, o_keep);
    case 6: return ln_bf16_nv<6>(has_ln, blocks, st, h, o, lw, lb, g, d, len, L, M, hhat, ps, splits, slice, o_keep);
    case 7: return ln_bf16_nv<7>(has_ln, blocks, st, h, o, lw, lb, g, d, len, L, M, hhat, ps, splits, slice, o_keep);
    default: return ln_bf16_nv<8>(has_ln, blocks, st, h, o, lw, lb, g, d, len, L, M, hhat, ps, splits, slice, o_keep);
  }
}

template <typename T>
r2l_status run_layer(T* hidden, const r2l_weights* w, const Plan& p, float g, int B, int L,
                     char* ws, cudaStream_t st, const r2l_debug_out* dbg, Prof* prof, bool residual = true,
                     const unsigned* a_flag = nullptr, float* hck = nullptr, int* hck_written = nullptr) {
  Prof dummy;
  if (!prof) prof = &dummy;
  const long long M = p.M;
  const int E = p.E, d = p.d, R = p.R;
  const int* len = (const int*)(ws + p.len);
  T* xz = (T*)(ws + p.xz);
  T* u = (T*)(ws + p.u);
  float* dbc = (float*)(ws + p.dbc);
  T* dt = (T*)(ws + p.dt);
  T* y = (T*)(ws + p.y);
  T* o = (T*)(ws + p.o);
  bf16* dr = (bf16*)(ws + p.dr);
  unsigned* err = (unsigned*)(ws + p.status);
  const size_t es = sizeof(T);
  constexpr bool kTC = std::is_same<T, bf16>::value;
  const bool fwd = (p.flags & R2L_FLAG_FORWARD_SCAN) != 0;   // left-to-right block

  // a1: [x | z] = h · W_inᵀ
  R2L_TRY(prof->mark(R2L_STAGE_IN_PROJ, st));
  prof->launches++;
  R2L_TRY(proj(hidden, d, (const T*)w->in_proj_w, d, xz, 2 * E, M, 2 * E, d, len, L, err, st, nullptr, 0, 0, nullptr,
               0, p.ragged));
  // a2: u = SiLU(anti-causal conv(x)); a3: [Δr | B | C] = u · W_xᵀ (fp32 out).
  // bf16 with an x_proj of 160 columns and at least one 128-row tile per SM:
  // one kernel does both (the conv runs in x_proj's operand producer and u
  // is written once, for the scan).
  R2L_TRY(prof->mark(R2L_STAGE_CONV, st));
  bool convx_done = false;
  if constexpr (kTC) {
    if (R2L_CONVX && r2l::convx_supported(p.ldd, E) && r2l::convx_worthwhile(M)) {
      R2L_TRY(prof->mark(R2L_STAGE_X_PROJ, st));
      prof->launches++;
      r2l::ConvX c{};
      c.x = (const bf16*)xz; c.ldx = 2LL * E; c.conv_w = w->conv_w; c.conv_b = w->conv_b;
      c.u = (bf16*)u; c.ldu = E; c.W = (const bf16*)w->x_proj_w; c.C = dbc; c.ldc = p.ldd;
      c.C2 = dr; c.ldc2 = R; c.c2_cols = R; c.M = (int)M; c.E = E; c.len = len; c.L = L; c.err = err; c.fwd = fwd;
      if (r2l::convx_gemm(c, st) != cudaSuccess) return R2L_ERR_CUDA;
      convx_done = true;
    }
  }
  if (!convx_done) {
    prof->launches++;
    if constexpr (kTC) {
      namespace cv = r2l::conv;
      const int nt = cv::tokens_per_thread(B, L, E, r2l::sm_count());
      const dim3 grid((E / 8 + cv::THREADS - 1) / cv::THREADS, (L + nt - 1) / nt, B);
      auto kern = fwd ? (nt == 8 ? cv::conv_silu_bf16_kernel<true, 8> : cv::conv_silu_bf16_kernel<true, 16>)
                      : (nt == 8 ? cv::conv_silu_bf16_kernel<false, 8> : cv::conv_silu_bf16_kernel<false, 16>);
      const cudaError_t e = r2l::launch_pdl(kern, grid, dim3(cv::THREADS), 0, st, (const bf16*)xz, 2 * E, u, E,
                                            (const float*)w->conv_w, (const float*)w->conv_b, (const int*)len, L);
      if (e != cudaSuccess) return R2L_ERR_CUDA;
      R2L_LAUNCH_CHECK();
    } else {
      dim3 grid((E + 127) / 128, L, B);
      r2l::conv_silu_kernel<T><<<grid, 128, 0, st>>>(xz, 2 * E, u, E, w->conv_w, w->conv_b, len, L, fwd);
      R2L_LAUNCH_CHECK();
    }
    R2L_TRY(prof->mark(R2L_STAGE_X_PROJ, st));
    prof->launches++;
    R2L_TRY(proj(u, E, (const T*)w->x_proj_w, E, dbc, p.ldd, M, p.ldd, E, len, L, err, st, dr, R, R,
                 (float*)(ws + p.xsplit), p.xsplit_bytes));
  }
  // a4: dt_raw = Δr · W_dtᵀ  (bias + softplus applied in the scan)
  R2L_TRY(prof->mark(R2L_STAGE_DT_PROJ, st));
  prof->launches++;
  // bf16 with dt_rank 128: dt_proj runs on the tensor cores inside the scan
  const bool dt_fused = kTC && R == r2l::kScanFusedDtRank;
  if constexpr (kTC) {
    if (!dt_fused) R2L_TRY(proj((const T*)dr, R, (const T*)w->dt_proj_w, R, dt, E, M, E, R, len, L, err, st));
    else prof->launches--;
  } else {
    R2L_TRY(gemm((const float*)dbc, p.ldd, (const T*)w->dt_proj_w, R, dt, E, M, E, R, len, L, st));
  }
  // a5: reverse selective scan, y = (C·H + D u) · SiLU(z)
  R2L_TRY(prof->mark(R2L_STAGE_SCAN, st));
  prof->launches++;
  if constexpr (kTC) {
    // the power-path decision: this hook's flag from the stack's one check, or its own
    if (!a_flag) R2L_TRY(check_a_log(w->A_log, E, err, (p.flags & R2L_FLAG_GENERAL_A) != 0, st, prof));
    r2l::ScanArgs sa{};
    sa.u = u; sa.ldu = E;
    sa.z = xz + E; sa.ldz = 2 * E;
    sa.dt = dt; sa.ldt = E;
    sa.bc = dbc + R; sa.ldbc = p.ldd;
    sa.A_log = w->A_log; sa.D = w->D; sa.dt_b = w->dt_proj_b;
    sa.y = y; sa.ldy = E;
    sa.B = B; sa.L = L; sa.E = E; sa.len = len;
    sa.chunk_tokens = p.chunk_tokens;
    sa.carry = (float*)(ws + p.carry);
    sa.err = err;
    sa.force_general = (int)(p.flags & R2L_FLAG_GENERAL_A);
    sa.a_general = a_flag ? a_flag : err + 1;
    sa.dt_mma = dt_fused ? 1 : 0;
    sa.forward = fwd ? 1 : 0;
    sa.dr = dr; sa.lddr = R;
    sa.wdt = (const bf16*)w->dt_proj_w;
    sa.hck = hck;
    sa.hck_written = hck_written;
    int nl = 0;
    if (r2l::scan_bf16(sa, st, &nl) != cudaSuccess) return R2L_ERR_CUDA;
    prof->launches += nl - 1;
  } else {
    dim3 grid((E + 127) / 128, B);
    r2l::scan_simple_kernel<T><<<grid, 128, 0, st>>>(u, xz + E, 2 * E, dt, dbc, p.ldd, R, w->A_log,
                                                     w->D, w->dt_proj_b, y, E, len, L, fwd);
    R2L_LAUNCH_CHECK();
  }
  // a6: o = y · W_outᵀ.  A small batch (few 128 × 256 tiles) splits K and
  // leaves fp32 partial sums, which the LayerNorm kernel adds (and stores o
  // from); without the LayerNorm step (the gradient's recomputed forward) the
  // split-K sum kernel stores o, with the same additions in the same order.
  R2L_TRY(prof->mark(R2L_STAGE_OUT_PROJ, st));
  prof->launches++;
  const bool osplit = kTC && p.osplits > 0 && d <= 2048;
  const long long Mp = (M + 127) / 128 * 128;
  if (osplit) {
    r2l::TcGemm gm{};
    gm.A = (const bf16*)y; gm.lda = E; gm.B = (const bf16*)w->out_proj_w; gm.ldb = E;
    gm.C = nullptr; gm.ldc = d; gm.c_fp32 = true; gm.keep_partials = true; gm.kept_splits = p.osplits;
    gm.M = (int)M; gm.N = d; gm.K = E; gm.len = len; gm.L = L; gm.err = err;
    gm.partial = (float*)(ws + p.osplit); gm.partial_bytes = p.osplit_bytes;
    if (r2l::tc_gemm(gm, st) != cudaSuccess) return R2L_ERR_CUDA;
    if (!residual) {
      prof->launches++;
      float* ps = (float*)(ws + p.osplit);
      if (r2l::tc_gemm_add_partials(ps, p.osplits, Mp, d, ps, d, (bf16*)o, d, d, (int)M, len, L, st) != cudaSuccess)
        return R2L_ERR_CUDA;
    }
  } else {
    R2L_TRY(proj(y, E, (const T*)w->out_proj_w, E, o, d, M, d, E, len, L, err, st, nullptr, 0, 0, nullptr, 0,
                 p.ragged));
  }

  if (dbg) {
    const size_t rowsE = (size_t)M;
    if (dbg->x && cudaMemcpy2DAsync(dbg->x, E * es, xz, 2 * E * es, E * es, rowsE, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return R2L_ERR_CUDA;
    if (dbg->z && cudaMemcpy2DAsync(dbg->z, E * es, xz + E, 2 * E * es, E * es, rowsE, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return R2L_ERR_CUDA;
    if (dbg->u && cudaMemcpyAsync(dbg->u, u, rowsE * E * es, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return R2L_ERR_CUDA;
    if (dbg->dbc && cudaMemcpyAsync(dbg->dbc, dbc, rowsE * p.ldd * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess) return R2L_ERR_CUDA;
    if (dbg->y && cudaMemcpyAsync(dbg->y, y, rowsE * E * es, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return R2L_ERR_CUDA;
    // with the split out_proj and the LayerNorm step, o is copied once that has stored it
    if (dbg->o && !(osplit && residual) &&
        cudaMemcpyAsync(dbg->o, o, rowsE * d * es, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return R2L_ERR_CUDA;
  }
  // stop here when only the intermediates are wanted (the hook's gradient)
  if (!residual) return R2L_OK;
  // a7 + a8: LayerNorm (optional) and h += g · ĥ on valid rows
  float* hhat = dbg ? dbg->hhat : nullptr;
  R2L_TRY(prof->mark(R2L_STAGE_LN_RESIDUAL, st));
  prof->launches++;
  if (kTC && d <= 2048) {
    const unsigned blocks = (unsigned)((M + 3) / 4);
    const int nv = (d + 255) / 256;
    R2L_TRY(launch_ln_bf16(nv, w->ln_w != nullptr, blocks, st, (bf16*)hidden, (const bf16*)o, w->ln_w, w->ln_b,
                           g, d, len, L, M, hhat, osplit ? (const float*)(ws + p.osplit) : nullptr, p.osplits,
                           Mp * d, osplit));
    if (osplit && dbg && dbg->o &&
        cudaMemcpyAsync(dbg->o, o, (size_t)M * d * sizeof(T), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return R2L_ERR_CUDA;
  } else if (w->ln_w) {
    r2l::ln_gate_residual_kernel<T, true><<<(unsigned)M, 256, 0, st>>>(hidden, o, w->ln_w, w->ln_b, g, d, len, L, hhat);
    R2L_LAUNCH_CHECK();
  } else {
    r2l::ln_gate_residual_kernel<T, false><<<(unsigned)M, 256, 0, st>>>(hidden, o, nullptr, nullptr, g, d, len, L, hhat);
    R2L_LAUNCH_CHECK();
  }
  R2L_TRY(prof->mark(R2L_NUM_STAGES, st));
  return R2L_OK;
}

r2l_status forward_impl(void* hidden, const r2l_weights* weights, const r2l_dims* dims, float s,
                        int B, int L, const int32_t* lengths, void* workspace,
                        size_t workspace_bytes, void* stream, const r2l_debug_out* dbg,
                        Prof* prof = nullptr) {
  Plan p;
  R2L_TRY(check_call(hidden, dims, B, L, workspace, workspace_bytes, &p));
  p.ragged = lengths != nullptr;
  R2L_TRY(check_weights(weights));
  if (lengths && ((uintptr_t)lengths & 3u)) return R2L_ERR_ALIGNMENT;
  const float g = (float)std::tanh((double)s);
  if (g == 0.0f && !dbg) return R2L_OK;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  R2L_TRY(prep(p, ws, lengths, B, L, st, prof));
  if (dims->dtype == R2L_BF16)
    return run_layer<bf16>((bf16*)hidden, weights, p, g, B, L, ws, st, dbg, prof);
  return run_layer<float>((float*)hidden, weights, p, g, B, L, ws, st, dbg, prof);
}

}  // namespace

extern "C" {

int r2l_abi_version(void) { return R2L_ABI_VERSION; }

const char* r2l_status_string(r2l_status s) {
  switch (s) {
    case R2L_OK: return "R2L_OK";
    case R2L_ERR_INVALID_ARG: return "R2L_ERR_INVALID_ARG: null pointer, bad size or bad enum";
    case R2L_ERR_UNSUPPORTED: return "R2L_ERR_UNSUPPORTED: shape outside what the kernels implement";
    case R2L_ERR_ALIGNMENT: return "R2L_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case R2L_ERR_WORKSPACE: return "R2L_ERR_WORKSPACE: workspace missing or too small";
    case R2L_ERR_CUDA: return "R2L_ERR_CUDA: a CUDA call or kernel launch failed";
    case R2L_ERR_DEVICE_CHECK: return "R2L_ERR_DEVICE_CHECK: a device-side check raised a flag";
  }
  return "R2L_ERR_UNKNOWN";
}

size_t r2l_workspace_size(const r2l_dims* dims, int B, int L) {
  Plan p;
  if (!make_plan(dims, B, L, &p)) return 0;
  return p.total;
}

r2l_status r2l_sidecar_forward(void* hidden, const r2l_weights* weights, const r2l_dims* dims,
                               float s, int B, int L, const int32_t* lengths, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return forward_impl(hidden, weights, dims, s, B, L, lengths, workspace, workspace_bytes, stream,
                      nullptr);
}

r2l_status r2l_sidecar_forward_debug(void* hidden, const r2l_weights* weights, const r2l_dims* dims,
                                     float s, int B, int L, const int32_t* lengths,
                                     void* workspace, size_t workspace_bytes, void* stream,
                                     const r2l_debug_out* debug) {
  if (!debug) return R2L_ERR_INVALID_ARG;
  return forward_impl(hidden, weights, dims, s, B, L, lengths, workspace, workspace_bytes, stream,
                      debug);
}

r2l_status r2l_sidecar_forward_profiled(void* hidden, const r2l_weights* weights,
                                        const r2l_dims* dims, float s, int B, int L,
                                        const int32_t* lengths, void* workspace,
                                        size_t workspace_bytes, void* stream,
                                        void* const* events, int n_events, int* launches) {
  if (!events || n_events != R2L_NUM_STAGES + 1) return R2L_ERR_INVALID_ARG;
  for (int k = 0; k < n_events; ++k)
    if (!events[k]) return R2L_ERR_INVALID_ARG;
  Prof prof;
  prof.ev = (cudaEvent_t*)events;
  const r2l_status st = forward_impl(hidden, weights, dims, s, B, L, lengths, workspace,
                                     workspace_bytes, stream, nullptr, &prof);
  if (launches) *launches = prof.launches;
  return st;
}

r2l_status r2l_sidecar_stack(void* hidden, const r2l_weights* weights, const float* s, int n_hooks,
                             const r2l_dims* dims, int B, int L, const int32_t* lengths,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (!weights || !s || n_hooks <= 0) return R2L_ERR_INVALID_ARG;
  Plan p;
  R2L_TRY(check_call(hidden, dims, B, L, workspace, workspace_bytes, &p));
  p.ragged = lengths != nullptr;
  for (int k = 0; k < n_hooks; ++k) R2L_TRY(check_weights(&weights[k]));
  if (lengths && ((uintptr_t)lengths & 3u)) return R2L_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  bool prepared = false;
  // one launch decides the scan's power path for every hook (bf16 path)
  const bool one_check = dims->dtype == R2L_BF16 && !(dims->flags & R2L_FLAG_GENERAL_A) &&
                         n_hooks <= r2l::kMaxCheckedHooks;
  unsigned* aflags = (unsigned*)(ws + p.aflags);
  for (int k = 0; k < n_hooks; ++k) {
    const float g = (float)std::tanh((double)s[k]);
    if (g == 0.0f) continue;
    if (!prepared) {
      R2L_TRY(prep(p, ws, lengths, B, L, st));
      if (one_check) R2L_TRY(check_a_log_hooks(weights, n_hooks, p.E, aflags, st));
      prepared = true;
    }
    if (dims->dtype == R2L_BF16)
      R2L_TRY(run_layer<bf16>((bf16*)hidden, &weights[k], p, g, B, L, ws, st, nullptr, nullptr, true,
                              one_check ? aflags + k : nullptr));
    else
      R2L_TRY(run_layer<float>((float*)hidden, &weights[k], p, g, B, L, ws, st, nullptr, nullptr));
  }
  return R2L_OK;
}

size_t r2l_reverse_scan_workspace_size(const r2l_dims* dims, int B, int L, int chunk_tokens) {
  if (!dims || B <= 0 || L <= 0 || dims->d_inner <= 0) return 0;
  if (dims->dtype != R2L_BF16 && dims->dtype != R2L_FP32) return 0;
  size_t off = align_up(16, kAlign);
  off = align_up(off + sizeof(int) * (size_t)B, kAlign);
  if (dims->dtype == R2L_BF16) off = align_up(off + r2l::scan_carry_bytes(B, L, dims->d_inner, chunk_tokens), kAlign);
  return off;
}

r2l_status r2l_reverse_scan(const void* u, const void* z, int ldz, const void* dt_raw, const float* bc,
                            int ldbc, const float* A_log, const float* D, const float* dt_b, void* y,
                            const r2l_dims* dims, int B, int L, const int32_t* lengths, int chunk_tokens,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!u || !z || !dt_raw || !bc || !A_log || !D || !dt_b || !y || !dims) return R2L_ERR_INVALID_ARG;
  if (B <= 0 || L <= 0 || dims->d_inner <= 0) return R2L_ERR_INVALID_ARG;
  if (dims->dtype != R2L_BF16 && dims->dtype != R2L_FP32) return R2L_ERR_INVALID_ARG;
  if (dims->d_state != 16) return R2L_ERR_UNSUPPORTED;
  const int E = dims->d_inner;
  if (ldz < E || ldbc < 32) return R2L_ERR_INVALID_ARG;
  if (L > 65535 || B > 65535) return R2L_ERR_UNSUPPORTED;
  for (const void* q : {u, z, dt_raw, (const void*)bc, (const void*)A_log, (const void*)D, (const void*)dt_b, (const void*)y})
    if (!aligned16(q)) return R2L_ERR_ALIGNMENT;
  if (dims->dtype == R2L_BF16 && ((ldz % 8) || (E % 8) || (ldbc % 4))) return R2L_ERR_ALIGNMENT;
  if (lengths && ((uintptr_t)lengths & 3u)) return R2L_ERR_ALIGNMENT;
  const size_t need = r2l_reverse_scan_workspace_size(dims, B, L, chunk_tokens);
  if (!workspace || workspace_bytes < need) return R2L_ERR_WORKSPACE;
  if (!aligned16(workspace)) return R2L_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  unsigned* status = (unsigned*)ws;
  int* len = (int*)(ws + align_up(16, kAlign));
  float* carry = (float*)(ws + align_up(align_up(16, kAlign) + sizeof(int) * (size_t)B, kAlign));
  if (cudaMemsetAsync(status, 0, 16, st) != cudaSuccess) return R2L_ERR_CUDA;
  r2l::prep_lengths_kernel<<<(B + 127) / 128, 128, 0, st>>>(lengths, len, B, L, status);
  R2L_LAUNCH_CHECK();
  if (dims->dtype == R2L_BF16) {
    const bool force_general = (dims->flags & R2L_FLAG_GENERAL_A) != 0;
    R2L_TRY(check_a_log(A_log, E, status, force_general, st, nullptr));
    r2l::ScanArgs sa{};
    sa.u = (const bf16*)u; sa.ldu = E;
    sa.z = (const bf16*)z; sa.ldz = ldz;
    sa.dt = (const bf16*)dt_raw; sa.ldt = E;
    sa.bc = bc; sa.ldbc = ldbc;
    sa.A_log = A_log; sa.D = D; sa.dt_b = dt_b;
    sa.y = (bf16*)y; sa.ldy = E;
    sa.B = B; sa.L = L; sa.E = E; sa.len = len;
    sa.chunk_tokens = r2l::scan_resolve_chunk_tokens(B, L, E, chunk_tokens);
    sa.carry = carry;
    sa.err = status;
    sa.force_general = force_general ? 1 : 0;
    sa.a_general = status + 1;
    sa.forward = (dims->flags & R2L_FLAG_FORWARD_SCAN) ? 1 : 0;
    if (r2l::scan_bf16(sa, st, nullptr) != cudaSuccess) return R2L_ERR_CUDA;
  } else {
    dim3 grid((E + 127) / 128, B);
    r2l::scan_simple_kernel<float><<<grid, 128, 0, st>>>((const float*)u, (const float*)z, ldz,
                                                         (const float*)dt_raw, bc, ldbc, 0, A_log, D, dt_b,
                                                         (float*)y, E, len, L,
                                                         (dims->flags & R2L_FLAG_FORWARD_SCAN) != 0);
    R2L_LAUNCH_CHECK();
  }
  return R2L_OK;
}

size_t r2l_reverse_scan_backward_workspace_size(const r2l_dims* dims, int B, int L, int chunk_tokens) {
  if (!dims || B <= 0 || L <= 0 || dims->d_inner <= 0 || chunk_tokens < 0) return 0;
  if ((dims->dtype != R2L_FP32 && dims->dtype != R2L_BF16) || dims->d_state != 16 || dims->d_inner % 64) return 0;
  if (!r2l::scan_bwd_supported(B, L, dims->d_inner, chunk_tokens)) return 0;
  return align_up(16, kAlign) + align_up(r2l::scan_bwd_scratch_bytes(B, L, dims->d_inner, chunk_tokens), kAlign);
}

r2l_status r2l_reverse_scan_backward(const void* u, const void* z, int ldz, const void* dt_raw, const float* bc,
                                     int ldbc, const float* A_log, const float* D, const float* dt_b,
                                     const void* dy, void* du, void* dz, int ld_dz, void* ddt_raw, float* dbc,
                                     int ld_dbc, float* dA_log, float* dD, float* ddt_b, const r2l_dims* dims,
                                     int B, int L, const int32_t* lengths, int chunk_tokens, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (!u || !z || !dt_raw || !bc || !A_log || !D || !dt_b || !dy || !du || !dz || !ddt_raw || !dbc || !dA_log ||
      !dD || !ddt_b || !dims)
    return R2L_ERR_INVALID_ARG;
  if (B <= 0 || L <= 0 || dims->d_inner <= 0 || chunk_tokens < 0) return R2L_ERR_INVALID_ARG;
  if (dims->dtype != R2L_BF16 && dims->dtype != R2L_FP32) return R2L_ERR_INVALID_ARG;
  if (dims->d_state != 16 || (dims->flags & R2L_FLAG_FORWARD_SCAN)) return R2L_ERR_UNSUPPORTED;
  const bool act16 = dims->dtype == R2L_BF16;   // u and z in bf16, everything else fp32
  const int E = dims->d_inner;
  if (E % 64) return R2L_ERR_UNSUPPORTED;
  if (ldz < E || ld_dz < E || ldbc < 32 || ld_dbc < 32) return R2L_ERR_INVALID_ARG;
  if ((ldbc % 4) || (ldz % 4) || (ld_dz % 4)) return R2L_ERR_ALIGNMENT;
  if (L > 65535 || B > 65535 || !r2l::scan_bwd_supported(B, L, E, chunk_tokens)) return R2L_ERR_UNSUPPORTED;
  for (const void* q : {u, z, dt_raw, (const void*)bc, (const void*)A_log, (const void*)D, (const void*)dt_b, dy,
                        (const void*)du, (const void*)dz, (const void*)ddt_raw, (const void*)dbc,
                        (const void*)dA_log, (const void*)dD, (const void*)ddt_b})
    if (!aligned16(q)) return R2L_ERR_ALIGNMENT;
  if (lengths && ((uintptr_t)lengths & 3u)) return R2L_ERR_ALIGNMENT;
  const size_t need = r2l_reverse_scan_backward_workspace_size(dims, B, L, chunk_tokens);
  if (!workspace || workspace_bytes < need) return R2L_ERR_WORKSPACE;
  if (!aligned16(workspace)) return R2L_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  if (cudaMemsetAsync(ws, 0, 16, st) != cudaSuccess) return R2L_ERR_CUDA;
  r2l::ScanBwdArgs a{};
  a.u = act16 ? nullptr : (const float*)u; a.z = act16 ? nullptr : (const float*)z;
  a.u16 = act16 ? (const bf16*)u : nullptr; a.z16 = act16 ? (const bf16*)z : nullptr;
  a.ldz = ldz; a.dt_raw = (const float*)dt_raw;
  a.bc = bc; a.ldbc = ldbc; a.A_log = A_log; a.D = D; a.dt_b = dt_b; a.dy = (const float*)dy;
  a.du = (float*)du; a.dz = (float*)dz; a.ld_dz = ld_dz; a.ddt_raw = (float*)ddt_raw;
  a.dbc = dbc; a.ld_dbc = ld_dbc; a.dA_log = dA_log; a.dD = dD; a.ddt_b = ddt_b;
  a.B = B; a.L = L; a.E = E; a.chunk_tokens = chunk_tokens;
  a.lengths = lengths;
  a.status = (unsigned*)ws;
  if (r2l::scan_bwd_f32(a, ws + align_up(16, kAlign), st) != cudaSuccess) return R2L_ERR_CUDA;
  return R2L_OK;
}

r2l_status r2l_get_device_status(const void* workspace, void* stream, uint32_t* flags_out) {
  if (!workspace || !flags_out) return R2L_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return R2L_ERR_CUDA;
  uint32_t f = 0;
  if (cudaMemcpy(&f, workspace, sizeof(f), cudaMemcpyDeviceToHost) != cudaSuccess) return R2L_ERR_CUDA;
  *flags_out = f;
  return f ? R2L_ERR_DEVICE_CHECK : R2L_OK;
}

}  // extern "C"

// ============================================================================
// The gradient of one hook (r2l_sidecar_backward).  The forward is recomputed
// into the workspace (as r2l_sidecar_forward computes it, without the final
// residual), then the chain rule runs in reverse: gate and LayerNorm, out_proj,
// the scan, dt_proj, x_proj, conv + SiLU, in_proj.  Input gradients are
// tcgen05 GEMMs against transposed weights; weight gradients are tcgen05 GEMMs
// of transposed (position-major) activations, with padding positions zeroed so
// that they contribute nothing.
// ============================================================================
namespace {

struct BwdPlan {
  Plan f;                                        // the forward's regions
  long long Mp;                                  // positions rounded up to 8 (K of the weight gradients)
  size_t dt32, winT, woutT, wxT, wdtT, stats, dsrow, do16, lnpart, dy, doT, yT, dus, dz, ddt, dbcs, sbwd, sbwd_bytes,
      ddt16, ddr, ddbc16, dux, cpart, dxz16, hT, dhtmp, gpart, gpart_bytes, hck, total;
};

long long row_chunks(long long M) { return (M + r2l::bwd::ROW_CHUNK - 1) / r2l::bwd::ROW_CHUNK; }

bool make_bwd_plan(const r2l_dims* dm, int B, int L, BwdPlan* q) {
  if (!make_plan(dm, B, L, &q->f)) return false;
  const Plan& p = q->f;
  const size_t M = (size_t)p.M, E = p.E, d = p.d, R = p.R, N2 = 2 * p.N, ldd = p.ldd;
  q->Mp = (p.M + 7) / 8 * 8;
  const size_t Mp = (size_t)q->Mp;
  size_t off = p.total;
  auto take = [&](size_t bytes) { const size_t at = off; off = align_up(off + bytes, kAlign); return at; };
  q->dt32 = take(M * E * 4);
  q->hck = take((size_t)B * ((L + 15) / 16) * E * 16 * 4);   // the forward's H checkpoints
  q->winT = take(d * 2 * E * 2);
  q->woutT = take(E * d * 2);
  q->wxT = take(E * ldd * 2);
  q->wdtT = take(R * E * 2);
  q->stats = take(M * 8);
  q->dsrow = take(M * 4);
  q->do16 = take(M * d * 2);
  q->lnpart = take((size_t)row_chunks(p.M) * 2 * d * 4);
  q->dy = take(M * E * 4);
  q->dus = take(M * E * 4);
  q->dz = take(M * E * 4);
  q->ddt = take(M * E * 4);
  q->dbcs = take(M * N2 * 4);
  r2l_dims sd = *dm;
  sd.dtype = R2L_BF16;
  q->sbwd_bytes = r2l_reverse_scan_backward_workspace_size(&sd, B, L, 0);
  if (q->sbwd_bytes == 0) return false;
  q->sbwd = take(q->sbwd_bytes);
  q->ddt16 = take(M * E * 2);
  q->ddr = take(M * R * 4);
  q->ddbc16 = take(M * ldd * 2);
  q->dux = take(M * E * 4);
  q->cpart = take((size_t)((q->Mp + r2l::bwd::CONV_ROWS - 1) / r2l::bwd::CONV_ROWS) * 5 * E * 4);
  q->dxz16 = take(M * 2 * E * 2);
  q->hT = take(d * Mp * 2);
  q->dhtmp = take(M * d * 4);
  // split-K scratch: the largest any fp32-output GEMM below asks for
  size_t gp = 0;
  auto need = [&](long long m, int n, int k) { gp = std::max(gp, r2l::tc_gemm_partial_bytes(m, n, k)); };
  need(p.M, p.E, p.R);                 // dt_raw
  need(p.M, p.E, p.d);                 // dy
  need(p.d, p.E, (int)p.M);            // dW_out
  need(p.M, p.R, p.E);                 // dΔr
  need(p.E, p.R, (int)p.M);            // dW_dt
  need(p.M, p.E, p.ldd);               // du_x
  need(p.ldd, p.E, (int)p.M);          // dW_x
  need(p.M, p.d, 2 * p.E);             // dh
  need(2LL * p.E, p.d, (int)p.M);      // dW_in
  q->gpart_bytes = gp;
  q->gpart = take(gp);
  q->total = off;
  return true;
}

// in[m, c] (M rows, C columns) rounded to bf16 into out[m, c] (when out is not
// null, ld_out) and into its transpose outT[c, m] (when outT is not null, ldT ≥
// M; columns M … ldT−1 zero).  Padding rows are zero in both.
template <typename TIn>
r2l_status cvt_transpose(const TIn* in, long long ld_in, long long M, int C, bf16* out, long long ld_out, bf16* outT,
                         long long ldT, const int* len, int L, cudaStream_t st) {
  if (M <= 0 || C <= 0) return R2L_OK;
  const long long rows = outT ? std::max(M, ldT) : M;
  const dim3 grid((unsigned)((C + 63) / 64), (unsigned)((rows + 63) / 64));
  r2l::bwd::cvt_transpose_kernel<TIn><<<grid, 256, 0, st>>>(in, ld_in, M, C, out, ld_out, outT, ldT, len, L);
  R2L_LAUNCH_CHECK();
  return R2L_OK;
}

template <typename TIn>
r2l_status transpose(const TIn* in, long long ld_in, long long M, int C, bf16* outT, long long ldT, const int* len,
                     int L, cudaStream_t st) {
  return cvt_transpose<TIn>(in, ld_in, M, C, nullptr, 0, outT, ldT, len, L, st);
}

// C[m, n] = Σ_k A[m, k]·B[n, k], bf16 operands, fp32 result.  a_mn / b_mn: A
// stored [K, M] / B stored [K, N] (position-major operands of a weight gradient).
r2l_status gemm_f32(const bf16* A, int lda, const bf16* Bm, int ldb, float* C, int ldc, long long M, int N, int K,
                    const int* len, int L, unsigned* err, float* partial, size_t partial_bytes, cudaStream_t st,
                    bool a_mn = false, bool b_mn = false) {
  r2l::TcGemm g{};
  g.A = A; g.lda = lda; g.B = Bm; g.ldb = ldb; g.C = C; g.ldc = ldc; g.c_fp32 = true;
  g.a_mn = a_mn; g.b_mn = b_mn;
  g.M = (int)M; g.N = N; g.K = K; g.len = len; g.L = L; g.err = err;
  g.partial = partial; g.partial_bytes = partial_bytes;
  return r2l::tc_gemm(g, st) == cudaSuccess ? R2L_OK : R2L_ERR_CUDA;
}

r2l_status check_grads(const r2l_grads* gr, const r2l_weights* w) {
  if (!gr) return R2L_ERR_INVALID_ARG;
  const void* ptrs[] = {gr->in_proj_w, gr->conv_w, gr->conv_b, gr->x_proj_w, gr->dt_proj_w,
                        gr->dt_proj_b, gr->A_log, gr->D, gr->out_proj_w};
  for (const void* q : ptrs) {
    if (!q) return R2L_ERR_INVALID_ARG;
    if (!aligned16(q)) return R2L_ERR_ALIGNMENT;
  }
  if (w->ln_w && (!gr->ln_w || !gr->ln_b)) return R2L_ERR_INVALID_ARG;
  if (gr->ln_w && (!aligned16(gr->ln_w) || !aligned16(gr->ln_b))) return R2L_ERR_ALIGNMENT;
  return R2L_OK;
}

// The forward as the gradient needs it, into the backward's workspace: the
// layer on `target` (in place with the residual, or reading it only), its
// scan storing the scan gradient's checkpoints where it can (*hck_written),
// and dt_raw = Δr·W_dtᵀ in fp32.
r2l_status forward_for_backward(bf16* target, bool residual, const r2l_weights* w, const BwdPlan& q, float g, int B,
                                int L, const int32_t* lengths, char* ws, cudaStream_t st, int* hck_written) {
  const Plan& p = q.f;
  R2L_TRY(prep(p, ws, lengths, B, L, st));
  R2L_TRY(run_layer<bf16>(target, w, p, g, B, L, ws, st, nullptr, nullptr, residual, nullptr, (float*)(ws + q.hck),
                          hck_written));
  return gemm_f32((const bf16*)(ws + p.dr), p.R, (const bf16*)w->dt_proj_w, p.R, (float*)(ws + q.dt32), p.E, p.M,
                  p.E, p.R, (const int*)(ws + p.len), L, (unsigned*)(ws + p.status), (float*)(ws + q.gpart),
                  q.gpart_bytes, st);
}

r2l_status backward_impl(const void* hidden, const r2l_weights* w, const r2l_dims* dims, float s, int B, int L,
                         const int32_t* lengths, const float* dh_out, float* dh, float* ds, const r2l_grads* gr,
                         void* workspace, size_t workspace_bytes, cudaStream_t st) {
  namespace K = r2l::bwd;
  BwdPlan q;
  if (!make_bwd_plan(dims, B, L, &q)) return R2L_ERR_INVALID_ARG;
  q.f.ragged = lengths != nullptr;
  const Plan& p = q.f;
  char* ws = (char*)workspace;
  const long long M = p.M, Mp = q.Mp;
  const int E = p.E, d = p.d, R = p.R, ldd = p.ldd;
  const int* len = (const int*)(ws + p.len);
  unsigned* err = (unsigned*)(ws + p.status);
  float* gpart = (float*)(ws + q.gpart);
  const size_t gpb = q.gpart_bytes;
  const double gd = std::tanh((double)s);
  const float g = (float)gd;
  const float dgate = (float)(1.0 - gd * gd);   // d tanh(s) / ds

  // ---- the forward's intermediates: xz, u, Δr|B|C, Δr (bf16), y, o; dt_raw in
  // fp32; the scan gradient's checkpoints.  Recomputed here, or left in the
  // workspace by r2l_sidecar_forward_train (R2L_FLAG_SAVED_FORWARD).
  float* hck = (float*)(ws + q.hck);
  int hck_written = 0;
  if (dims->flags & R2L_FLAG_SAVED_FORWARD) {
    R2L_TRY(prep(p, ws, lengths, B, L, st));
    hck_written = r2l::scan_writes_checkpoints(R, false) ? 1 : 0;
  } else {
    // hidden is only read (no residual)
    R2L_TRY(forward_for_backward((bf16*)const_cast<void*>(hidden), false, w, q, g, B, L, lengths, ws, st,
                                 &hck_written));
  }
  const bf16* xz = (const bf16*)(ws + p.xz);
  const bf16* u = (const bf16*)(ws + p.u);
  const float* dbc = (const float*)(ws + p.dbc);
  const bf16* dr = (const bf16*)(ws + p.dr);
  const bf16* y = (const bf16*)(ws + p.y);
  const bf16* o = (const bf16*)(ws + p.o);
  const float* dt32 = (const float*)(ws + q.dt32);

  // ---- weights transposed once: W_outᵀ [E, d], W_dtᵀ [R, E], W_xᵀ [E, R+2N], W_inᵀ [d, 2E]
  bf16* woutT = (bf16*)(ws + q.woutT);
  bf16* wdtT = (bf16*)(ws + q.wdtT);
  bf16* wxT = (bf16*)(ws + q.wxT);
  bf16* winT = (bf16*)(ws + q.winT);
  R2L_TRY(transpose((const bf16*)w->out_proj_w, E, d, E, woutT, d, nullptr, d, st));
  R2L_TRY(transpose((const bf16*)w->dt_proj_w, R, E, R, wdtT, E, nullptr, E, st));
  R2L_TRY(transpose((const bf16*)w->x_proj_w, E, ldd, E, wxT, ldd, nullptr, ldd, st));
  R2L_TRY(transpose((const bf16*)w->in_proj_w, d, 2LL * E, d, winT, 2LL * E, nullptr, 2 * E, st));

  // ---- ❹ gate and ❸ LayerNorm
  float2* stats = (float2*)(ws + q.stats);
  float* dsrow = (float*)(ws + q.dsrow);
  bf16* do16 = (bf16*)(ws + q.do16);
  const bool has_ln = w->ln_w != nullptr;
  const unsigned rblocks = (unsigned)((M + 7) / 8);
  if (d == 2048 && has_ln)   // the row in registers (16-byte loads, one pass over memory)
    K::ln_gate_bwd_rows_reg_kernel<true, 8><<<rblocks, 256, 0, st>>>(o, dh_out, w->ln_w, w->ln_b, g, d, len, L, M,
                                                                     stats, dsrow, do16);
  else if (d == 2048)
    K::ln_gate_bwd_rows_reg_kernel<false, 8><<<rblocks, 256, 0, st>>>(o, dh_out, nullptr, nullptr, g, d, len, L, M,
                                                                      stats, dsrow, do16);
  else if (has_ln)
    K::ln_gate_bwd_rows_kernel<true><<<rblocks, 256, 0, st>>>(o, dh_out, w->ln_w, w->ln_b, g, d, len, L, M, stats,
                                                              dsrow, do16);
  else
    K::ln_gate_bwd_rows_kernel<false><<<rblocks, 256, 0, st>>>(o, dh_out, nullptr, nullptr, g, d, len, L, M, stats,
                                                               dsrow, do16);
  R2L_LAUNCH_CHECK();
  K::sum_kernel<<<1, 1024, 0, st>>>(dsrow, M, dgate, ds);
  R2L_LAUNCH_CHECK();
  const long long nrc = row_chunks(M);
  if (has_ln) {
    float* lnpart = (float*)(ws + q.lnpart);
    K::ln_bwd_cols_kernel<<<dim3((unsigned)((d + 511) / 512), (unsigned)nrc), 128, 0, st>>>(o, dh_out, g, d, len, L,
                                                                                            M, stats, lnpart);
    R2L_LAUNCH_CHECK();
    K::chunk_sum_kernel<0><<<(2 * d + 31) / 32, 256, 0, st>>>(lnpart, (int)nrc, 2 * d, d, gr->ln_w, gr->ln_b);
    R2L_LAUNCH_CHECK();
  }

  // ---- out_proj: dy = do·W_out, dW_out = doᵀ·y
  float* dy = (float*)(ws + q.dy);
  R2L_TRY(gemm_f32(do16, d, woutT, d, dy, E, M, E, d, len, L, err, gpart, gpb, st));
  // the weight gradients read their operands position-major (MN-major); the
  // gradient side is zero on padding rows, the activation side is zeroed there
  K::zero_padding_rows_kernel<<<B, 256, 0, st>>>(const_cast<bf16*>(y), E, E, len, L);
  K::zero_padding_rows_kernel<<<B, 256, 0, st>>>(const_cast<bf16*>(u), E, E, len, L);
  K::zero_padding_rows_kernel<<<B, 256, 0, st>>>(const_cast<bf16*>(dr), R, R, len, L);
  R2L_LAUNCH_CHECK();
  R2L_TRY(gemm_f32(do16, d, y, E, gr->out_proj_w, E, d, E, (int)M, nullptr, d, err, gpart, gpb, st, true, true));

  // ---- ❷ the scan (bf16 u and z, fp32 dt_raw, B|C and dy); on the walk along
  // each sequence it writes ddt_raw and dz in bf16 itself
  const bool walks = r2l::scan_bwd_walks(B, E, 0);
  bf16* ddt16 = (bf16*)(ws + q.ddt16);
  bf16* dxz16 = (bf16*)(ws + q.dxz16);
  float* dus = (float*)(ws + q.dus);
  float* dz = (float*)(ws + q.dz);
  float* ddt = (float*)(ws + q.ddt);
  float* dbcs = (float*)(ws + q.dbcs);
  {
    r2l::ScanBwdArgs a{};
    a.u16 = u; a.z16 = xz + E; a.ldz = 2 * E; a.dt_raw = dt32; a.bc = dbc + R; a.ldbc = ldd;
    a.A_log = w->A_log; a.D = w->D; a.dt_b = w->dt_proj_b; a.dy = dy;
    a.du = dus; a.dz = dz; a.ld_dz = E; a.ddt_raw = ddt; a.dbc = dbcs; a.ld_dbc = 2 * p.N;
    a.dA_log = gr->A_log; a.dD = gr->D; a.ddt_b = gr->dt_proj_b;
    a.B = B; a.L = L; a.E = E; a.chunk_tokens = 0; a.lengths = len;
    a.status = err;
    a.hck = hck_written ? hck : nullptr;
    if (walks) {   // ddt_raw and dz straight to the bf16 GEMM operands
      a.ddt16 = ddt16; a.ld_ddt16 = E;
      a.dz16 = dxz16 + E; a.ld_dz16 = 2LL * E;
    }
    char* sw = ws + q.sbwd;
    if (cudaMemsetAsync(sw, 0, 16, st) != cudaSuccess) return R2L_ERR_CUDA;
    if (r2l::scan_bwd_f32(a, sw + align_up(16, kAlign), st) != cudaSuccess) return R2L_ERR_CUDA;
  }

  // ---- dt_proj: dΔr = ddt_raw·W_dt, dW_dt = ddt_rawᵀ·Δr
  if (!walks) R2L_TRY(cvt_transpose(ddt, E, M, E, ddt16, E, (bf16*)nullptr, 0, len, L, st));
  float* ddr = (float*)(ws + q.ddr);
  R2L_TRY(gemm_f32(ddt16, E, wdtT, E, ddr, R, M, R, E, len, L, err, gpart, gpb, st));
  R2L_TRY(gemm_f32(ddt16, E, dr, R, gr->dt_proj_w, R, E, R, (int)M, nullptr, E, err, gpart, gpb, st, true, true));

  // ---- x_proj: d[Δr|B|C] → du_x = d[Δr|B|C]·W_x, dW_x = d[Δr|B|C]ᵀ·u
  bf16* ddbc16 = (bf16*)(ws + q.ddbc16);
  R2L_TRY(cvt_transpose(ddr, R, M, R, ddbc16, ldd, (bf16*)nullptr, 0, len, L, st));
  R2L_TRY(cvt_transpose(dbcs, 2LL * p.N, M, 2 * p.N, ddbc16 + R, ldd, (bf16*)nullptr, 0, len, L, st));
  float* dux = (float*)(ws + q.dux);
  R2L_TRY(gemm_f32(ddbc16, ldd, wxT, ldd, dux, E, M, E, ldd, len, L, err, gpart, gpb, st));
  R2L_TRY(gemm_f32(ddbc16, ldd, u, E, gr->x_proj_w, E, ldd, E, (int)M, nullptr, ldd, err, gpart, gpb, st, true,
                   true));

  // ---- conv + SiLU: dx (into dxz), dconv_w, dconv_b; dz into dxz
  float* cpart = (float*)(ws + q.cpart);
  if (cudaFuncSetAttribute(K::conv_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::CONV_SMEM) !=
      cudaSuccess)
    return R2L_ERR_CUDA;
  K::conv_bwd_kernel<<<dim3((unsigned)((E + K::CONV_CH - 1) / K::CONV_CH), (unsigned)((Mp + K::CONV_ROWS - 1) / K::CONV_ROWS)),
                       K::CONV_THREADS, K::CONV_SMEM, st>>>(xz, 2LL * E, w->conv_w, w->conv_b, dus, dux, E, len, L, M, dxz16, 2LL * E, nullptr, Mp,
                                     cpart);
  R2L_LAUNCH_CHECK();
  K::chunk_sum_kernel<1><<<(5 * E + 31) / 32, 256, 0, st>>>(cpart, (int)((Mp + K::CONV_ROWS - 1) / K::CONV_ROWS), 5 * E,
                                                            E, gr->conv_w, gr->conv_b);
  R2L_LAUNCH_CHECK();
  if (!walks) R2L_TRY(cvt_transpose(dz, E, M, E, dxz16 + E, 2LL * E, (bf16*)nullptr, 0, len, L, st));

  // ---- in_proj: dh = dh⁺ + [dx | dz]·W_in, dW_in = [dx | dz]ᵀ·h
  float* dhtmp = (float*)(ws + q.dhtmp);
  R2L_TRY(gemm_f32(dxz16, 2 * E, winT, 2 * E, dhtmp, d, M, d, 2 * E, len, L, err, gpart, gpb, st));
  K::add_rows_kernel<<<(unsigned)std::min<long long>(M, 148 * 8), 256, 0, st>>>(dh_out, dhtmp, d, len, L, M, dh);
  R2L_LAUNCH_CHECK();
  // h is the caller's (its padding rows may hold anything): transposed with
  // padding zeroed, and read K-major
  bf16* hT = (bf16*)(ws + q.hT);
  R2L_TRY(transpose((const bf16*)hidden, d, M, d, hT, Mp, len, L, st));
  R2L_TRY(gemm_f32(dxz16, 2 * E, hT, (int)Mp, gr->in_proj_w, d, 2LL * E, d, (int)M, nullptr, 2 * E, err, gpart, gpb,
                   st, true, false));
  return R2L_OK;
}

}  // namespace

extern "C" {

size_t r2l_sidecar_backward_workspace_size(const r2l_dims* dims, int B, int L) {
  if (!dims || dims->dtype != R2L_BF16) return 0;
  BwdPlan q;
  if (!make_bwd_plan(dims, B, L, &q)) return 0;
  return q.total;
}

namespace {
// The checks r2l_sidecar_backward and r2l_sidecar_forward_train share.
r2l_status check_train_call(const void* hidden, const r2l_weights* weights, const r2l_dims* dims, int B, int L,
                            const int32_t* lengths, void* workspace, size_t workspace_bytes) {
  if (!hidden || !dims) return R2L_ERR_INVALID_ARG;
  Plan p;
  if (!make_plan(dims, B, L, &p)) return R2L_ERR_INVALID_ARG;
  if (dims->d_state != 16 || dims->d_conv != 4) return R2L_ERR_UNSUPPORTED;
  if (dims->dtype != R2L_BF16 || (dims->flags & R2L_FLAG_FORWARD_SCAN)) return R2L_ERR_UNSUPPORTED;
  if ((dims->d_model % 8) || (dims->d_inner % 64) || (dims->dt_rank % 8)) return R2L_ERR_UNSUPPORTED;
  if (L > 65535 || B > 65535 || (p.M + 63) / 64 > 65535) return R2L_ERR_UNSUPPORTED;
  R2L_TRY(check_weights(weights));
  if (!aligned16(hidden)) return R2L_ERR_ALIGNMENT;
  if (lengths && ((uintptr_t)lengths & 3u)) return R2L_ERR_ALIGNMENT;
  BwdPlan q;
  if (!make_bwd_plan(dims, B, L, &q)) return R2L_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < q.total) return R2L_ERR_WORKSPACE;
  if (!aligned16(workspace)) return R2L_ERR_ALIGNMENT;
  return R2L_OK;
}
}  // namespace

r2l_status r2l_sidecar_forward_train(const void* hidden, void* out, const r2l_weights* weights, const r2l_dims* dims,
                                     float s, int B, int L, const int32_t* lengths, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (!out || out == hidden) return R2L_ERR_INVALID_ARG;
  R2L_TRY(check_train_call(hidden, weights, dims, B, L, lengths, workspace, workspace_bytes));
  if (!aligned16(out)) return R2L_ERR_ALIGNMENT;
  BwdPlan q;
  make_bwd_plan(dims, B, L, &q);
  q.f.ragged = lengths != nullptr;
  cudaStream_t st = (cudaStream_t)stream;
  // h⁺ is formed in `out` (a copy of h, updated in place on valid rows); h,
  // which the gradient reads again, stays as it is
  if (cudaMemcpyAsync(out, hidden, (size_t)q.f.M * q.f.d * sizeof(bf16), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return R2L_ERR_CUDA;
  int hck_written = 0;
  return forward_for_backward((bf16*)out, true, weights, q, (float)std::tanh((double)s), B, L, lengths,
                              (char*)workspace, st, &hck_written);
}

r2l_status r2l_sidecar_backward(const void* hidden, const r2l_weights* weights, const r2l_dims* dims, float s, int B,
                                int L, const int32_t* lengths, const float* dh_out, float* dh, float* ds,
                                const r2l_grads* grads, void* workspace, size_t workspace_bytes, void* stream) {
  if (!dh_out || !dh || !ds) return R2L_ERR_INVALID_ARG;
  R2L_TRY(check_train_call(hidden, weights, dims, B, L, lengths, workspace, workspace_bytes));
  R2L_TRY(check_grads(grads, weights));
  for (const void* q : {(const void*)dh_out, (const void*)dh})
    if (!aligned16(q)) return R2L_ERR_ALIGNMENT;
  if ((uintptr_t)ds & 3u) return R2L_ERR_ALIGNMENT;
  return backward_impl(hidden, weights, dims, s, B, L, lengths, dh_out, dh, ds, grads, workspace, workspace_bytes,
                       (cudaStream_t)stream);
}

}  // extern "C"
