/*
 * r2l.h — C ABI of libr2l, the B200 (sm_100a) R2L sidecar forward.
 *
 * The operation is the reverse-direction Mamba stream of "Bifocal Diffusion
 * Language Models: Asymmetric Bidirectional Context for Parallel Generation"
 * (arXiv 2606.27732v1), §3.4 "R2LM Architecture", steps ❶–❹: for hidden
 * states h ∈ R^{B×L×d},
 *
 *     h⁺ = h + tanh(s) · LN( flip( Mamba( flip(h) ) ) )
 *
 * where Mamba is the Mamba-1 selective-scan block (step ❷; d_state = 16,
 * d_conv = 4, expand 2 per §4.1) and LN is a LayerNorm local to the stream
 * (step ❸).  With flip applied per sequence to its valid prefix, the block
 * runs from each sequence's last valid token to its first:
 *
 *     [x | z] = h·W_inᵀ
 *     u_i     = SiLU(conv_b + Σ_{k=0..3} conv_w[:, 3-k] ⊙ x_{i+k})   (x_j = 0, j ≥ len)
 *     [Δr | B | C]_i = u_i·W_xᵀ
 *     Δ_i     = softplus(Δr_i·W_dtᵀ + dt_b)
 *     H_i     = exp(Δ_i ⊗ A) ⊙ H_{i+1} + (Δ_i ⊙ u_i) ⊗ B_i,   H_len = 0,  A = -exp(A_log)
 *     y_i     = (H_i·C_i + D ⊙ u_i) ⊙ SiLU(z_i)
 *     o_i     = y_i·W_outᵀ
 *     h_i    += tanh(s) · (γ ⊙ (o_i − mean) / sqrt(var + 1e-5) + β)      (0 ≤ i < len)
 *
 * Conventions (all entry points):
 *   - Every pointer in a forward call is a DEVICE pointer owned by the caller,
 *     except the r2l_dims / r2l_weights / r2l_debug_out structs themselves,
 *     which are host memory read during the call only.  The library never
 *     allocates, frees or synchronises on the forward path.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream) and runs asynchronously.  Errors found on the
 *     host are returned as r2l_status before anything is enqueued; nothing is
 *     thrown and nothing is printed.
 *   - Matrices are row-major, nn.Linear convention W[out][in].
 *   - The library holds no mutable global state; calls on different streams
 *     with different workspaces may run concurrently.  Two calls that share a
 *     workspace must be ordered by the caller.
 */
#ifndef R2L_H
#define R2L_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define R2L_ABI_VERSION 1

#if defined(__GNUC__)
#define R2L_API __attribute__((visibility("default")))
#else
#define R2L_API
#endif

typedef enum {
  R2L_OK = 0,
  R2L_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad enum */
  R2L_ERR_UNSUPPORTED = 2,   /* d_state != 16, d_conv != 4, or a size the kernels do not tile */
  R2L_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
  R2L_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than r2l_workspace_size() */
  R2L_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
  R2L_ERR_DEVICE_CHECK = 6   /* r2l_get_device_status found a device-side flag */
} r2l_status;

typedef enum {
  R2L_BF16 = 0,   /* bf16 activations and GEMM weights, fp32 accumulation and state */
  R2L_FP32 = 1    /* fp32 everywhere, true fp32 arithmetic (no TF32) */
} r2l_dtype;

/* r2l_dims.flags
 *
 * The scan's power path (bf16 path only).  When A is the S4D-real
 * initialisation A[c][m] = -(m+1), the 16 decays exp(Δ·A[c][m]) of a (position,
 * channel) are the powers r, r², …, r¹⁶ of r = exp(-Δ), so the scan needs one
 * reciprocal instead of 16 exponentials.  The choice is made once per call
 * (per hook of r2l_sidecar_stack), on the device, by an exact test: the power
 * path is taken when every A_log[c][m] equals, bit for bit, the float nearest
 * ln(m+1), and the scan then uses A[c][m] = -(m+1) exactly (it differs from
 * -exp(A_log[c][m]) by less than 2e-7 relative).  Any other A_log, even one
 * entry, sends the whole call down the general path (one exponential per
 * state).  R2L_FLAG_GENERAL_A skips the test and always takes the general
 * path.  The fp32 path always evaluates exp(Δ·A) directly.                   */
#define R2L_FLAG_GENERAL_A 0x1u     /* never take the A = -(1..16) power fast path of the scan    */
#define R2L_FLAG_FORWARD_SCAN 0x2u  /* run the block left to right instead: causal conv and a
                                       forward scan (the "L2R Mamba" control of Table 4); every
                                       other step is unchanged                                    */
#define R2L_FLAG_SAVED_FORWARD 0x4u /* r2l_sidecar_backward only: the workspace holds this hook's
                                       forward from r2l_sidecar_forward_train, so the forward is
                                       not recomputed                                             */
/* Device status bits, reported by r2l_get_device_status(). */
#define R2L_DEVFLAG_LENGTH_CLAMPED 0x1u   /* a lengths[b] was outside [0, L] and was clamped */
#define R2L_DEVFLAG_TIMEOUT 0x2u          /* a kernel gave up waiting on a pipeline barrier (results invalid) */

typedef struct {
  int d_model;       /* d: hidden width of the backbone                             */
  int d_inner;       /* E: expanded width (2·d_model in the paper's setup)         */
  int d_state;       /* N: SSM state size; must be 16                              */
  int dt_rank;       /* R: rank of the Δ projection                                */
  int d_conv;        /* W: depthwise conv width; must be 4                         */
  r2l_dtype dtype;   /* activation / GEMM-weight storage type                      */
  unsigned flags;    /* R2L_FLAG_* bits, 0 by default                              */
} r2l_dims;

/* One hook's parameters.  Device pointers, read-only, 16-byte aligned.
 * "act" = bf16 for R2L_BF16, fp32 for R2L_FP32.                               */
typedef struct {
  const void  *in_proj_w;   /* act  [2E, d]   rows 0..E-1 produce x, rows E..2E-1 produce z */
  const float *conv_w;      /* fp32 [E, W]    tap W-1 multiplies the current token          */
  const float *conv_b;      /* fp32 [E]                                                      */
  const void  *x_proj_w;    /* act  [R+2N, E] output rows ordered Δr | B | C                 */
  const void  *dt_proj_w;   /* act  [E, R]                                                   */
  const float *dt_proj_b;   /* fp32 [E]                                                      */
  const float *A_log;       /* fp32 [E, N]    A = -exp(A_log)                                */
  const float *D;           /* fp32 [E]                                                      */
  const void  *out_proj_w;  /* act  [d, E]                                                   */
  const float *ln_w;        /* fp32 [d]  LayerNorm γ; ln_w = ln_b = NULL: no LayerNorm       */
  const float *ln_b;        /* fp32 [d]  LayerNorm β                                         */
} r2l_weights;

/* Optional intermediates for testing (device pointers, NULL = not wanted).
 * Row b·L + i holds position i of sequence b; rows with i ≥ len_b hold
 * unspecified values, except in hhat where they are not written.             */
typedef struct {
  void  *x;        /* act  [B·L, E]      in_proj, first half                  */
  void  *z;        /* act  [B·L, E]      in_proj, second half                 */
  void  *u;        /* act  [B·L, E]      conv + SiLU                          */
  float *dbc;      /* fp32 [B·L, R+2N]   x_proj output Δr | B | C             */
  void  *y;        /* act  [B·L, E]      scan output after the SiLU(z) gate   */
  void  *o;        /* act  [B·L, d]      out_proj output                      */
  float *hhat;     /* fp32 [B·L, d]      LayerNorm output (pre-gate)          */
} r2l_debug_out;

/* ABI version of the loaded library (R2L_ABI_VERSION at build time). */
R2L_API int r2l_abi_version(void);

/* Human-readable name of a status code; never NULL, static storage. */
R2L_API const char *r2l_status_string(r2l_status status);

/* Bytes of device workspace a forward call on a [B, L] batch needs.  Returns 0
 * for invalid dims or sizes.  The size depends only on (dims, B, L).          */
R2L_API size_t r2l_workspace_size(const r2l_dims *dims, int B, int L);

/* The sidecar forward of §3.4 on hidden [B, L, d_model] (act dtype), updated in
 * place: rows i < len_b become h⁺, rows i ≥ len_b are neither read nor written.
 *
 *   lengths   device int32 [B] of valid lengths, or NULL for all L.  Values
 *             outside [0, L] are clamped on the device and flagged
 *             (R2L_DEVFLAG_LENGTH_CLAMPED, see r2l_get_device_status).
 *   s         the hook's scalar gate; g = tanh(s) is formed in double on the
 *             host and rounded to float.  If g == 0 the call returns R2L_OK
 *             without enqueuing anything (the identity at initialisation, §3.4 ❹).
 *   workspace device scratch of at least r2l_workspace_size(dims, B, L) bytes,
 *             16-byte aligned, caller-owned; its contents on entry do not
 *             matter and on return are unspecified (the device status word
 *             lives at its start).
 * Checks on the host: non-null pointers, positive sizes, d_state == 16,
 * d_conv == 4, 16-byte alignment, workspace size, supported tiling.  On any
 * error nothing is enqueued.                                                   */
R2L_API r2l_status r2l_sidecar_forward(void *hidden, const r2l_weights *weights, const r2l_dims *dims,
                               float s, int B, int L, const int32_t *lengths,
                               void *workspace, size_t workspace_bytes, void *stream);

/* Same as r2l_sidecar_forward, and also copies the intermediates requested in
 * *debug (non-NULL fields) into the caller's buffers.  For tests.  Unlike the
 * forward call it runs the layer even when tanh(s) == 0.                       */
R2L_API r2l_status r2l_sidecar_forward_debug(void *hidden, const r2l_weights *weights, const r2l_dims *dims,
                                     float s, int B, int L, const int32_t *lengths,
                                     void *workspace, size_t workspace_bytes, void *stream,
                                     const r2l_debug_out *debug);

/* n_hooks sidecar layers applied one after another to the same hidden tensor
 * (§4.1: a hook after every 4th decoder layer; here the backbone between hooks
 * is whatever the caller does between calls, i.e. nothing).  weights and s are
 * host arrays of n_hooks entries.  Same contract as r2l_sidecar_forward.      */
R2L_API r2l_status r2l_sidecar_stack(void *hidden, const r2l_weights *weights, const float *s, int n_hooks,
                             const r2l_dims *dims, int B, int L, const int32_t *lengths,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Stages of one hook, in launch order, for r2l_sidecar_forward_profiled. */
typedef enum {
  R2L_STAGE_IN_PROJ = 0,      /* [x | z] = h·W_inᵀ                              */
  R2L_STAGE_CONV = 1,         /* u = SiLU(anti-causal conv(x))                  */
  R2L_STAGE_X_PROJ = 2,       /* [Δr | B | C] = u·W_xᵀ                          */
  R2L_STAGE_DT_PROJ = 3,      /* Δr·W_dtᵀ                                       */
  R2L_STAGE_SCAN = 4,         /* reverse selective scan and SiLU(z) gate        */
  R2L_STAGE_OUT_PROJ = 5,     /* o = y·W_outᵀ                                   */
  R2L_STAGE_LN_RESIDUAL = 6,  /* LayerNorm and tanh(s)-gated residual           */
  R2L_NUM_STAGES = 7
} r2l_stage;

/* Same as r2l_sidecar_forward, and also records events[k] on `stream` just
 * before stage k starts and events[R2L_NUM_STAGES] after the last stage.
 * events: host array of n_events cudaEvent_t handles (passed as void*),
 * created and owned by the caller; n_events must be R2L_NUM_STAGES + 1.  A
 * stage that is fused into its neighbour shows zero time.  *launches (if not
 * NULL) receives the number of kernels the call enqueued.  For measurement.  */
R2L_API r2l_status r2l_sidecar_forward_profiled(void *hidden, const r2l_weights *weights,
                                        const r2l_dims *dims, float s, int B, int L,
                                        const int32_t *lengths, void *workspace,
                                        size_t workspace_bytes, void *stream,
                                        void *const *events, int n_events, int *launches);

/* Bytes of device workspace r2l_reverse_scan needs for a [B, L] batch split
 * into chunks of chunk_tokens tokens (0 = automatic).  0 for invalid input. */
R2L_API size_t r2l_reverse_scan_workspace_size(const r2l_dims *dims, int B, int L, int chunk_tokens);

/* The selective scan of §3.4 step ❷ on its own (the Mamba-1 scan, run from
 * each sequence's last valid token to its first) followed by the SiLU(z) gate:
 *
 *     Δ_i = softplus(dt_raw_i + dt_b);  H_i = exp(Δ_i ⊗ A) ⊙ H_{i+1} + (Δ_i ⊙ u_i) ⊗ B_i;
 *     y_i = (H_i·C_i + D ⊙ u_i) ⊙ SiLU(z_i),   H entering position len_b − 1 is 0.
 *
 *   u        act  [B·L, E]     (row stride E)
 *   z        act  [B·L, ldz]   first E columns are z
 *   dt_raw   act  [B·L, E]     Δr·W_dtᵀ, before bias and softplus
 *   bc       fp32 [B·L, ldbc]  B in columns 0..15, C in columns 16..31
 *   A_log    fp32 [E, 16],  D, dt_b  fp32 [E]
 *   y        act  [B·L, E]     output; rows i ≥ len_b are not written
 *   lengths  as for r2l_sidecar_forward
 *   chunk_tokens  bf16 path: tokens per chunk when sequences are split for
 *            parallelism (rounded up to a multiple of 16; 0 = automatic).
 *            Ignored by the fp32 path, which scans each sequence whole.
 *   workspace  ≥ r2l_reverse_scan_workspace_size(dims, B, L, chunk_tokens) bytes,
 *            16-byte aligned (chunk carries and the device status word).
 * Device pointers, 16-byte aligned; ldz a multiple of 8 and ldbc of 4.        */
R2L_API r2l_status r2l_reverse_scan(const void *u, const void *z, int ldz, const void *dt_raw,
                                    const float *bc, int ldbc, const float *A_log, const float *D,
                                    const float *dt_b, void *y, const r2l_dims *dims, int B, int L,
                                    const int32_t *lengths, int chunk_tokens, void *workspace,
                                    size_t workspace_bytes, void *stream);

/* Capacity, in bytes, of the scratch array behind r2l_reverse_scan_noalloc. */
#define R2L_NOALLOC_SCRATCH_BYTES (16u << 20)

/* r2l_reverse_scan without a workspace argument, for callers that cannot
 * allocate device memory while they run: for example a serving runtime that
 * reserves all device memory when it starts and forbids allocation while it
 * handles requests, or a plug-in whose host program owns the CUDA context and
 * its allocator.  It computes exactly what r2l_reverse_scan computes.  (The
 * paper has no counterpart; this entry point exists for such callers only.)
 *
 * Its scratch (status word, clamped lengths, chunk carries) is a fixed array
 * of R2L_NOALLOC_SCRATCH_BYTES that the library's device code declares; every
 * device that loads the library holds it until the process exits.  The entry
 * point calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Every call looks up the array's device address in the current device's
 *     context (cudaGetSymbolAddress; nothing is allocated), so the address
 *     stays right after cudaDeviceReset.  The first call on a device also
 *     loads the library's device image into that context; make that first
 *     call before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents
 *     (each call rewrites what it reads).  Calls whose work overlaps on the
 *     GPU (for instance on two streams) race on it; order them.
 *   - A request that needs more scratch than the array holds
 *     (r2l_reverse_scan_workspace_size() > R2L_NOALLOC_SCRATCH_BYTES) returns
 *     R2L_ERR_WORKSPACE and enqueues nothing.  A smaller chunk count (larger
 *     chunk_tokens) needs less scratch; one chunk per sequence needs almost none.
 * r2l_get_device_status cannot read this scratch; use r2l_reverse_scan when
 * device-side flags matter.  Other arguments and errors as r2l_reverse_scan. */
R2L_API r2l_status r2l_reverse_scan_noalloc(const void *u, const void *z, int ldz, const void *dt_raw,
                                            const float *bc, int ldbc, const float *A_log, const float *D,
                                            const float *dt_b, void *y, const r2l_dims *dims, int B, int L,
                                            const int32_t *lengths, int chunk_tokens, void *stream);

/* Bytes of device workspace r2l_reverse_scan_backward needs for a [B, L]
 * batch split into chunks of chunk_tokens positions (0 = automatic, 16).
 * 0 for invalid or unsupported input (see r2l_reverse_scan_backward).       */
R2L_API size_t r2l_reverse_scan_backward_workspace_size(const r2l_dims *dims, int B, int L, int chunk_tokens);

/* Gradient of r2l_reverse_scan (the scan of §3.4 step ❷ with its softplus(Δ)
 * input and SiLU(z) gate), the step that training the sidecar alone
 * back-propagates through.  For dy = ∂L/∂y it returns, with the forward's
 * notation (a_i = exp(Δ_i A), G_i = ∂L/∂H_i = a_{i-1} ⊙ G_{i-1} + dp_i C_i,
 * dp_i = dy_i ⊙ SiLU(z_i)):
 *
 *   du      [B·L, E]   D ⊙ dp_i + Δ_i ⊙ Σ_m G_i[:,m] B_i[m]
 *   ddt_raw [B·L, E]   (Σ_m G_i ⊙ H_{i+1} ⊙ a_i ⊙ A + u_i ⊙ Σ_m G_i B_i) ⊙ softplus'(dt_raw_i + dt_b)
 *   dz      [B·L, ld_dz] first E columns: dy_i ⊙ p_i ⊙ SiLU'(z_i), p_i = H_i·C_i + D ⊙ u_i
 *   dbc     [B·L, ld_dbc] columns 0..15 dB_i = Σ_e G_i Δ_i u_i, 16..31 dC_i = Σ_e dp_i H_i
 *   dA_log  [E, 16]    A ⊙ Σ_i Δ_i ⊙ G_i ⊙ H_{i+1} ⊙ a_i   (summed over the batch)
 *   dD, ddt_b [E]      Σ_i dp_i ⊙ u_i,  Σ_i ddt_raw_i        (summed over the batch)
 *
 * Rows i ≥ len_b of du, ddt_raw, dz and dbc are written with zeros.  Inputs
 * are those of r2l_reverse_scan (u, z, dt_raw, bc, A_log, D, dt_b, lengths)
 * plus dy [B·L, E].  Every reduction runs in a fixed order: the results are
 * bitwise reproducible for a given chunk_tokens.
 *
 * Supported: dims->dtype R2L_FP32 (every array fp32) or R2L_BF16 (u and z
 * bf16 as the bf16 forward stores them, every other array fp32), d_state == 16, d_inner a multiple of 64, B and L up to 65535 with
 * B·⌈L / chunk⌉ ≤ 2,097,120 (grid limits), the right-to-left block (the
 * R2L_FLAG_FORWARD_SCAN flag returns R2L_ERR_UNSUPPORTED); ldz, ld_dz and
 * ldbc multiples of 4.  chunk_tokens: positions per chunk (1 … 32; larger values are
 * clamped to 32; 0 = 16).  workspace ≥
 * r2l_reverse_scan_backward_workspace_size(dims, B, L, chunk_tokens) bytes,
 * 16-byte aligned; its first 16 bytes are the device status word that
 * r2l_get_device_status reads.  Device pointers, 16-byte aligned.          */
R2L_API r2l_status r2l_reverse_scan_backward(const void *u, const void *z, int ldz, const void *dt_raw,
                                             const float *bc, int ldbc, const float *A_log, const float *D,
                                             const float *dt_b, const void *dy, void *du, void *dz, int ld_dz,
                                             void *ddt_raw, float *dbc, int ld_dbc, float *dA_log, float *dD,
                                             float *ddt_b, const r2l_dims *dims, int B, int L,
                                             const int32_t *lengths, int chunk_tokens, void *workspace,
                                             size_t workspace_bytes, void *stream);

/* Gradients of one hook's parameters: fp32 device arrays, 16-byte aligned,
 * caller-owned, each shaped like the matching field of r2l_weights (in_proj_w
 * [2E, d], conv_w [E, W], conv_b [E], x_proj_w [R+2N, E], dt_proj_w [E, R],
 * dt_proj_b [E], A_log [E, N], D [E], out_proj_w [d, E], ln_w and ln_b [d]).
 * ln_w / ln_b may be NULL when the hook has no LayerNorm.  Every array is
 * written in full (not accumulated into).                                    */
typedef struct {
  float *in_proj_w, *conv_w, *conv_b, *x_proj_w, *dt_proj_w, *dt_proj_b, *A_log, *D, *out_proj_w, *ln_w, *ln_b;
} r2l_grads;

/* Bytes of device workspace r2l_sidecar_backward needs for a [B, L] batch;
 * 0 for invalid or unsupported input.                                        */
R2L_API size_t r2l_sidecar_backward_workspace_size(const r2l_dims *dims, int B, int L);

/* The gradient of one hook (§3.4 steps ❶–❹), the step that training the
 * sidecar alone (the paper's R2LM-PI setting, §3.4 and §4.1) back-propagates
 * through.  For the hook's input hidden [B, L, d] (act dtype, as given to
 * r2l_sidecar_forward) and dh_out = ∂L/∂h⁺ (fp32 [B, L, d]) it writes
 *
 *   dh    fp32 [B, L, d]  ∂L/∂h: dh_out on padding rows (the hook neither reads
 *                          nor writes them), dh_out + ∂L/∂h through the sidecar
 *                          on valid rows
 *   *ds   fp32 scalar     ∂L/∂s = (1 − tanh²(s)) Σ dh_out ⊙ ĥ (device pointer)
 *   grads                 ∂L/∂(every parameter), summed over the batch
 *
 * The forward is recomputed into the workspace (unless R2L_FLAG_SAVED_FORWARD
 * says r2l_sidecar_forward_train left it there), then the chain rule runs in
 * reverse: gate, LayerNorm, out_proj, the scan (bf16 u and z, fp32 state),
 * dt_proj, x_proj, conv + SiLU, in_proj.  GEMM operands are bf16 (gradients
 * rounded once to bf16 where they feed a GEMM), accumulation fp32; every
 * reduction over positions runs in a fixed order, so results are bitwise
 * reproducible.
 *
 * Supported: dims->dtype R2L_BF16, d_state 16, d_conv 4, d_model and dt_rank
 * multiples of 8, d_inner a multiple of 64, the right-to-left block
 * (R2L_FLAG_FORWARD_SCAN returns R2L_ERR_UNSUPPORTED).  workspace ≥
 * r2l_sidecar_backward_workspace_size(dims, B, L) bytes, 16-byte aligned; its
 * first 16 bytes are the status word r2l_get_device_status reads.  Other
 * arguments, conventions and errors as r2l_sidecar_forward; hidden is not
 * written.                                                                     */
R2L_API r2l_status r2l_sidecar_backward(const void *hidden, const r2l_weights *weights, const r2l_dims *dims,
                                        float s, int B, int L, const int32_t *lengths, const float *dh_out,
                                        float *dh, float *ds, const r2l_grads *grads, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* The hook's forward for training (the R2LM-PI setting, §3.4 and §4.1):
 * out = h⁺ = h + tanh(s)·ĥ as r2l_sidecar_forward computes it, written to
 * `out` (act dtype [B, L, d], 16-byte aligned, not aliasing hidden: padding
 * rows are copied from hidden; hidden is not written, since the gradient reads
 * it again), and everything r2l_sidecar_backward needs left in `workspace`
 * (≥ r2l_sidecar_backward_workspace_size(dims, B, L) bytes): the forward's
 * intermediates, dt_raw in fp32, and the H checkpoints of its scan gradient
 * (every 16 positions, for sequences whose length is a multiple of 16, with
 * dt_rank 128).  A later r2l_sidecar_backward with R2L_FLAG_SAVED_FORWARD in
 * dims->flags and the same hidden, weights, other dims, s, B, L, lengths and
 * workspace (untouched in between) skips its recomputation of the forward.
 * Supported shapes and errors as r2l_sidecar_backward; out == hidden returns
 * R2L_ERR_INVALID_ARG.  Runs the layer even when tanh(s) == 0 (the gradient
 * needs ĥ for ds).                                                            */
R2L_API r2l_status r2l_sidecar_forward_train(const void *hidden, void *out, const r2l_weights *weights,
                                             const r2l_dims *dims, float s, int B, int L, const int32_t *lengths,
                                             void *workspace, size_t workspace_bytes, void *stream);

/* Synchronises `stream`, then reads the device status word that the last
 * forward call on `workspace` wrote.  *flags_out receives the R2L_DEVFLAG_*
 * bits.  Returns R2L_ERR_DEVICE_CHECK if any bit is set, R2L_ERR_CUDA if the
 * stream reported an error, R2L_OK otherwise.  Not for the hot path.          */
R2L_API r2l_status r2l_get_device_status(const void *workspace, void *stream, uint32_t *flags_out);

#ifdef __cplusplus
}
#endif

#endif /* R2L_H */
