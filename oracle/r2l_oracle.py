"""Reference oracle for the R2L sidecar forward (the ``ReverseMambaLayer``).

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously-correct CPU
statement of what the CUDA library computes.  Only ``tests/``, the package's
``smoke()`` entry and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it; the library itself never does, and it shares no
code with the GPU path (it imports numpy and nothing else).

Arithmetic is float64 throughout.  Inputs arrive as numpy arrays holding the
exact values of the stored tensors (bf16 or fp32, widened without rounding).
Matrix products use ``numpy.matmul`` as a library primitive; everything else
is written out step by step in the order of the source below, with no blocking,
fusion or reordering.

Source: "Bifocal Diffusion Language Models: Asymmetric Bidirectional Context
for Parallel Generation" (arXiv 2606.27732v1), §3.4 "R2LM Architecture",
steps ❶–❹, and §4.1 "Experimental Setup" (d_state=16, d_conv=4, expand 2,
a hook after every 4th of 28 decoder layers).  Step ❷ names the Mamba-1
selective-scan block (Gu & Dao, "Mamba: Linear-Time Sequence Modeling with
Selective State Spaces", 2023, §3 and Algorithm 2); the block's internals
below are that block: in_proj -> depthwise conv of width d_conv -> SiLU ->
data-dependent (Δ, B, C) projections -> softplus(Δ) -> selective scan with
Ā = exp(ΔA), B̄u = ΔBu -> + D·u -> ·SiLU(z) -> out_proj.

Readings taken where the pages are silent:
  * the flip of step ❶ and the un-flip of step ❸ are applied per sequence to
    its valid prefix [0, len_b) of a right-padded row; in original coordinates
    the block therefore runs from position len_b-1 down to 0 with a zero
    initial state, and its depthwise conv reads positions i..i+d_conv-1 with
    the last tap (the "current token" tap of the forward block) on position i;
    positions >= len_b are zero for the conv and are never read or written;
  * LN of step ❸ is a standard affine LayerNorm over d_model, biased variance,
    eps = 1e-5; passing ``ln_w = ln_b = None`` selects the variant without it;
  * no bias on in_proj, x_proj, out_proj; conv and dt_proj carry biases;
  * softplus(v) = log1p(exp(v)), and v for v > 20;
  * the x_proj output is split in the order [Δ_r | B | C].

Parity status: every function below is pinned by tests in
``tests/test_oracle_pins.py`` against closed forms, library routines,
brute force and the invariants the pages state (s = 0 identity, right-context
only, flip equivalence, parameter count).  The absolute values of a full layer
have no printed worked example on the pages; beyond the pins the oracle is the
only numeric reference.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "silu",
    "softplus",
    "in_proj",
    "anticausal_conv_silu",
    "x_proj",
    "dt_softplus",
    "reverse_selective_scan",
    "out_proj",
    "layer_norm",
    "gated_residual",
    "round_to_bf16",
    "sidecar_sequence",
    "sidecar_forward",
    "sidecar_stack",
    "flip_valid",
]

SOFTPLUS_THRESHOLD = 20.0
LN_EPS = 1e-5


def silu(v: np.ndarray) -> np.ndarray:
    """SiLU(v) = v * sigmoid(v) = v / (1 + exp(-v))  (Mamba-1 block activation)."""
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def softplus(v: np.ndarray) -> np.ndarray:
    """softplus(v) = log(1 + exp(v)); returns v itself above the threshold 20.

    The Mamba-1 block parameterises the step size as Δ = softplus(·).
    """
    v = np.asarray(v, dtype=np.float64)
    big = v > SOFTPLUS_THRESHOLD
    safe = np.where(big, 0.0, v)
    return np.where(big, v, np.log1p(np.exp(safe)))


def in_proj(h: np.ndarray, W_in: np.ndarray):
    """Mamba-1 input projection: [x | z] = h · W_inᵀ (no bias).

    h: [n, d_model];  W_in: [2·d_inner, d_model] (nn.Linear convention).
    Rows 0..d_inner-1 of W_in give x, rows d_inner..2·d_inner-1 give z.
    """
    xz = np.matmul(h, W_in.T)
    E = W_in.shape[0] // 2
    return xz[:, :E], xz[:, E:]


def anticausal_conv_silu(x: np.ndarray, conv_w: np.ndarray, conv_b: np.ndarray) -> np.ndarray:
    """Depthwise conv of width W in reversed order, then SiLU.

    In flipped coordinates the Mamba-1 conv is causal: its last tap multiplies
    the current token and tap W-1-k multiplies the token k steps earlier.  Back
    in original coordinates "k steps earlier" is position i+k, so

        u[i, c] = SiLU( conv_b[c] + Σ_{k=0..W-1} conv_w[c, W-1-k] · x[i+k, c] ),

    with x[j, ·] = 0 for j >= n (the sequence's own end; §3.4 steps ❶–❷).

    x: [n, E];  conv_w: [E, W];  conv_b: [E]  ->  u: [n, E]
    """
    n, E = x.shape
    W = conv_w.shape[1]
    pre = np.empty((n, E), dtype=np.float64)
    pre[:] = conv_b
    for k in range(W):
        if k >= n:
            break
        # x shifted up by k rows: row i holds x[i+k] (zero past the end)
        pre[: n - k] += conv_w[:, W - 1 - k] * x[k:]
    return silu(pre)


def x_proj(u: np.ndarray, W_x: np.ndarray, dt_rank: int, d_state: int):
    """Data-dependent projections [Δ_r | B | C] = u · W_xᵀ (no bias).

    u: [n, E];  W_x: [dt_rank + 2·d_state, E].
    Returns dr [n, dt_rank], B [n, d_state], C [n, d_state].
    """
    dbc = np.matmul(u, W_x.T)
    R, N = dt_rank, d_state
    return dbc[:, :R], dbc[:, R : R + N], dbc[:, R + N : R + 2 * N]


def dt_softplus(dr: np.ndarray, W_dt: np.ndarray, b_dt: np.ndarray) -> np.ndarray:
    """Step size Δ = softplus(dr · W_dtᵀ + b_dt).

    dr: [n, R];  W_dt: [E, R];  b_dt: [E]  ->  Δ: [n, E]
    """
    return softplus(np.matmul(dr, W_dt.T) + b_dt)


def reverse_selective_scan(u, delta, A, B, C, D, z):
    """The selective scan of §3.4 step ❷, run from the last position to the first.

    With state H ∈ R^{E×N} starting at zero past the sequence end:

        for i = n-1 down to 0:
            H      = exp(Δ[i] ⊗ A) ⊙ H + (Δ[i] · u[i]) ⊗ B[i]
            y[i]   = H · C[i] + D ⊙ u[i]
        y = y ⊙ SiLU(z)

    (Ā = exp(ΔA) and B̄u = ΔBu, the discretisation of the Mamba-1 block.)
    Running the recurrence from i = n-1 down to 0 is the same as flipping the
    sequence, scanning forward and flipping back (steps ❶–❸).

    u, delta, z: [n, E];  A: [E, N] (negative);  B, C: [n, N];  D: [E]
    Returns y: [n, E].
    """
    n, E = u.shape
    N = A.shape[1]
    H = np.zeros((E, N), dtype=np.float64)
    y = np.empty((n, E), dtype=np.float64)
    for i in range(n - 1, -1, -1):
        dA = np.exp(delta[i][:, None] * A)                 # [E, N]
        dBu = (delta[i] * u[i])[:, None] * B[i][None, :]   # [E, N]
        H = dA * H + dBu
        y[i] = np.matmul(H, C[i]) + D * u[i]
    return y * silu(z)


def out_proj(y: np.ndarray, W_out: np.ndarray) -> np.ndarray:
    """Mamba-1 output projection o = y · W_outᵀ (no bias).  W_out: [d_model, E]."""
    return np.matmul(y, W_out.T)


def layer_norm(o: np.ndarray, ln_w, ln_b, eps: float = LN_EPS) -> np.ndarray:
    """Stream-local LayerNorm of §3.4 step ❸ over the last axis (d_model).

    ĥ = γ ⊙ (o − mean) / sqrt(var + eps) + β, biased variance.  With
    ``ln_w is None and ln_b is None`` the step is skipped and ĥ = o.
    """
    if ln_w is None and ln_b is None:
        return o
    mu = o.mean(axis=-1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=-1, keepdims=True)
    return (o - mu) / np.sqrt(var + eps) * ln_w + ln_b


def gated_residual(h: np.ndarray, h_r2l: np.ndarray, s: float) -> np.ndarray:
    """§3.4 step ❹: h⁺ = h + tanh(s) · h_R2L."""
    return h + np.tanh(np.float64(s)) * h_r2l


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), in one step.

    bfloat16 keeps 8 significant bits.  v = m·2^e with m in [0.5, 1) (frexp);
    rounding m·2^8 to an integer with ``numpy.rint`` (ties to even) and scaling
    back gives the nearest representable value.  The values this project
    rounds are far from bf16's overflow and subnormal ranges, which this
    helper does not treat specially; NaN and ±inf pass through.
    """
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    out = np.ldexp(np.rint(m * 256.0), e - 8)
    return np.where(np.isfinite(v), out, v)


def sidecar_sequence(h, w, s, length=None, return_intermediates=False):
    """One sequence through one hook: §3.4 steps ❶–❹ on rows [0, length).

    h: [L, d_model] float64 (exact stored values).  w: dict of float64 arrays
    with keys W_in, conv_w, conv_b, W_x, W_dt, b_dt, A_log, D, W_out, ln_w,
    ln_b (ln_* may be None).  Returns h⁺ (float64, unrounded); rows >= length
    are returned unchanged.
    """
    L = h.shape[0]
    n = L if length is None else int(length)
    out = np.array(h, dtype=np.float64, copy=True)
    inter = {}
    if n <= 0:
        return (out, inter) if return_intermediates else out
    E = w["W_in"].shape[0] // 2
    N = w["A_log"].shape[1]
    R = w["W_dt"].shape[1]
    hv = out[:n]
    x, z = in_proj(hv, w["W_in"])
    u = anticausal_conv_silu(x, w["conv_w"], w["conv_b"])
    dr, Bm, Cm = x_proj(u, w["W_x"], R, N)
    delta = dt_softplus(dr, w["W_dt"], w["b_dt"])
    A = -np.exp(w["A_log"])
    y = reverse_selective_scan(u, delta, A, Bm, Cm, w["D"], z)
    o = out_proj(y, w["W_out"])
    hhat = layer_norm(o, w.get("ln_w"), w.get("ln_b"))
    out[:n] = gated_residual(hv, hhat, s)
    if return_intermediates:
        inter = dict(x=x, z=z, u=u, dr=dr, B=Bm, C=Cm, delta=delta, y=y, o=o, hhat=hhat)
        return out, inter
    return out


def flip_valid(h, lengths=None):
    """Reverse each sequence's valid prefix [0, len_b) of a right-padded batch
    along the sequence axis (§3.4 step ❶'s flip, per sequence); padding stays."""
    h = np.array(h, copy=True)
    L = h.shape[1]
    for b in range(h.shape[0]):
        n = L if lengths is None else int(lengths[b])
        n = min(max(n, 0), L)
        h[b, :n] = h[b, :n][::-1]
    return h


def sidecar_forward(h, w, s, lengths=None, out_dtype="f64", batch_indices=None,
                    return_intermediates=False, direction="r2l"):
    """The hook on a right-padded batch h [B, L, d_model] (float64 values).

    Sequences are independent; ``batch_indices`` restricts the work to a subset
    of them (the rest of the returned array is a copy of the input).  Rows at or
    beyond a sequence's length are left as they were.  ``out_dtype`` "bf16"
    rounds h⁺ once to bfloat16; "f32" rounds once to float32; "f64" keeps it.
    """
    h = np.asarray(h, dtype=np.float64)
    if direction == "l2r":
        # The same block scanning left to right (the "L2R Mamba" control of
        # Table 4): since the reverse block is flip ∘ Mamba ∘ flip (§3.4
        # steps ❶–❸), the forward block on h is flip(R2L(flip(h))).
        if return_intermediates:
            raise ValueError("intermediates are reported for direction='r2l' only")
        hf = flip_valid(h, lengths)
        return flip_valid(sidecar_forward(hf, w, s, lengths, out_dtype, batch_indices), lengths)
    if direction != "r2l":
        raise ValueError(direction)
    Bsz, L, _ = h.shape
    out = np.array(h, copy=True)
    inters = {}
    idx = range(Bsz) if batch_indices is None else batch_indices
    for b in idx:
        n = L if lengths is None else int(lengths[b])
        if return_intermediates:
            out[b], inters[b] = sidecar_sequence(h[b], w, s, n, True)
        else:
            out[b] = sidecar_sequence(h[b], w, s, n)
        nv = min(max(n, 0), L)
        if out_dtype == "bf16":
            out[b, :nv] = round_to_bf16(out[b, :nv])
        elif out_dtype == "f32":
            out[b, :nv] = out[b, :nv].astype(np.float32).astype(np.float64)
    return (out, inters) if return_intermediates else out


def sidecar_stack(h, weights_list, s_list, lengths=None, out_dtype="f64", batch_indices=None):
    """Hooks applied one after another to the same hidden tensor (§4.1: after
    every 4th decoder layer; with an identity backbone between hooks the hooks
    compose directly).  The hidden tensor is stored in ``out_dtype`` between
    hooks, so each hook's output is rounded before the next hook reads it.
    """
    cur = np.asarray(h, dtype=np.float64)
    for w, s in zip(weights_list, s_list):
        cur = sidecar_forward(cur, w, s, lengths, out_dtype, batch_indices)
    return cur
