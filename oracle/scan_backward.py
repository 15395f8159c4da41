"""Reference oracle for the gradient of the reverse selective scan.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: imported by
``tests/`` and by the CPU legs of ``bench.py``, never by the library.  It
imports numpy and nothing else.

What it differentiates: the scan of "Bifocal Diffusion Language Models"
(arXiv 2606.27732v1) §3.4 step ❷ (the Mamba-1 selective scan, run on the
flipped sequence, i.e. from each sequence's last valid position to its first)
with its softplus(Δ) input and its SiLU(z) gate, exactly as the forward entry
point ``r2l_reverse_scan`` computes it:

    v_i  = dt_raw_i + dt_b,     Δ_i = softplus(v_i)      (v > 20: Δ = v)
    A    = -exp(A_log)
    a_i  = exp(Δ_i ⊗ A)                                   [E, N]
    H_n  = 0,   H_i = a_i ⊙ H_{i+1} + (Δ_i u_i) ⊗ B_i     (i = n-1 … 0)
    p_i  = H_i · C_i + D ⊙ u_i
    y_i  = p_i ⊙ SiLU(z_i)

Training the sidecar alone (the R2LM-PI setting of the paper's §3.4 and
§4.1) back-propagates through this step.  The gradients below are the chain
rule written out for it, for an upstream gradient dy = ∂L/∂y:

    dp_i   = dy_i ⊙ SiLU(z_i)
    dz_i   = dy_i ⊙ p_i ⊙ SiLU'(z_i),   SiLU'(z) = σ(z)·(1 + z·(1 − σ(z)))
    G_i    = ∂L/∂H_i  (through p_i and through H_{i-1} = a_{i-1} ⊙ H_i + …)
           = dp_i ⊗ C_i + a_{i-1} ⊙ G_{i-1},   G_{-1} = 0  (i = 0 … n-1,
             the opposite direction to the scan)
    dC_i   = Σ_e dp_i[e] · H_i[e, :]
    dB_i   = Σ_e G_i[e, :] · Δ_i[e] · u_i[e]
    ∂a_i   = G_i ⊙ H_{i+1}
    dΔ_i   = Σ_m ∂a_i[:, m] · a_i[:, m] · A[:, m]  +  u_i ⊙ Σ_m G_i[:, m] · B_i[m]
    du_i   = D ⊙ dp_i  +  Δ_i ⊙ Σ_m G_i[:, m] · B_i[m]
    dA     = Σ_i Δ_i ⊗ 1 ⊙ ∂a_i ⊙ a_i,      dA_log = dA ⊙ A
    dD     = Σ_i dp_i ⊙ u_i
    ddt_raw_i = dΔ_i ⊙ softplus'(v_i)  (σ(v), and 1 for v > 20)
    ddt_b  = Σ_i ddt_raw_i

Parity status: pinned in ``tests/test_oracle_scan_backward.py`` by central
finite differences of the forward oracle (``reverse_selective_scan``, itself
pinned), one input at a time, and by the adjoint's closed form at n = 1.
"""
from __future__ import annotations

import numpy as np

from .r2l_oracle import SOFTPLUS_THRESHOLD, silu, softplus

__all__ = ["sigmoid", "reverse_scan_backward", "reverse_scan_backward_batch", "reverse_scan_forward_from_raw"]


def sigmoid(v: np.ndarray) -> np.ndarray:
    """σ(v) = 1 / (1 + e^{-v})."""
    return 1.0 / (1.0 + np.exp(-v))


def reverse_scan_forward_from_raw(u, dt_raw, dt_b, A_log, B, C, D, z):
    """y of the scan step as ``r2l_reverse_scan`` takes its inputs (Δ before
    its bias and softplus, A as A_log), composed from the pinned forward
    oracle: Δ = softplus(dt_raw + dt_b), A = -exp(A_log), then the scan."""
    from .r2l_oracle import reverse_selective_scan
    return reverse_selective_scan(u, softplus(dt_raw + dt_b), -np.exp(A_log), B, C, D, z)


def reverse_scan_backward(u, dt_raw, dt_b, A_log, B, C, D, z, dy):
    """Gradients of Σ dy ⊙ y for one sequence of n positions.

    u, dt_raw, z, dy: [n, E];  B, C: [n, N];  A_log: [E, N];  D, dt_b: [E].
    Returns a dict with du, ddt_raw, dz [n, E], dB, dC [n, N], dA_log [E, N],
    dD, ddt_b [E].
    """
    n, E = u.shape
    N = A_log.shape[1]
    A = -np.exp(A_log)
    v = dt_raw + dt_b
    delta = softplus(v)
    dsoft = np.where(v > SOFTPLUS_THRESHOLD, 1.0, sigmoid(v))

    # the scan itself, keeping every state: H[i] is H_i, H[n] = 0
    a = np.exp(delta[:, :, None] * A[None, :, :])             # [n, E, N]
    H = np.zeros((n + 1, E, N))
    for i in range(n - 1, -1, -1):
        H[i] = a[i] * H[i + 1] + (delta[i] * u[i])[:, None] * B[i][None, :]
    p = np.einsum("ien,in->ie", H[:n], C) + D[None, :] * u

    sz = silu(z)
    sg = sigmoid(z)
    dp = dy * sz
    dz = dy * p * sg * (1.0 + z * (1.0 - sg))

    du = np.empty((n, E))
    ddelta = np.empty((n, E))
    dB = np.empty((n, N))
    dC = np.empty((n, N))
    dA = np.zeros((E, N))
    G = np.zeros((E, N))
    for i in range(n):                                         # the adjoint runs left to right
        if i > 0:
            G = a[i - 1] * G
        G = G + dp[i][:, None] * C[i][None, :]
        dC[i] = np.einsum("e,en->n", dp[i], H[i])
        dB[i] = np.einsum("en,e->n", G, delta[i] * u[i])
        da = G * H[i + 1]
        gB = np.matmul(G, B[i])                                # Σ_m G[:, m] B_i[m]
        ddelta[i] = np.sum(da * a[i] * A, axis=1) + u[i] * gB
        du[i] = D * dp[i] + delta[i] * gB
        dA += delta[i][:, None] * da * a[i]
    dD = np.sum(dp * u, axis=0)
    ddt_raw = ddelta * dsoft
    return {"du": du, "ddt_raw": ddt_raw, "dz": dz, "dB": dB, "dC": dC,
            "dA_log": dA * A, "dD": dD, "ddt_b": np.sum(ddt_raw, axis=0)}


def reverse_scan_backward_batch(u, dt_raw, dt_b, A_log, B, C, D, z, dy, lengths=None):
    """The same over a right-padded batch: u, dt_raw, z, dy [Bt, L, E]; B, C
    [Bt, L, N].  Each sequence b uses its first lengths[b] positions; the
    per-position gradients of padding positions are zero, and the parameter
    gradients (dA_log, dD, ddt_b) are summed over the sequences."""
    Bt, L, E = u.shape
    N = A_log.shape[1]
    lens = [L] * Bt if lengths is None else [int(x) for x in lengths]
    out = {"du": np.zeros((Bt, L, E)), "ddt_raw": np.zeros((Bt, L, E)), "dz": np.zeros((Bt, L, E)),
           "dB": np.zeros((Bt, L, N)), "dC": np.zeros((Bt, L, N)),
           "dA_log": np.zeros((E, N)), "dD": np.zeros(E), "ddt_b": np.zeros(E)}
    for b in range(Bt):
        n = lens[b]
        if n <= 0:
            continue
        g = reverse_scan_backward(u[b, :n], dt_raw[b, :n], dt_b, A_log, B[b, :n], C[b, :n], D, z[b, :n],
                                  dy[b, :n])
        for k in ("du", "ddt_raw", "dz", "dB", "dC"):
            out[k][b, :n] = g[k]
        for k in ("dA_log", "dD", "ddt_b"):
            out[k] += g[k]
    return out
