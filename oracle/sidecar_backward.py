"""Reference oracle for the gradient of one whole sidecar hook.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: imported by
``tests/`` and never by the library.  It imports numpy and the other oracle
modules, nothing else.

What it differentiates: one hook of "Bifocal Diffusion Language Models"
(arXiv 2606.27732v1), §3.4 steps ❶–❹, on one sequence of n valid positions,
as ``r2l_oracle.sidecar_sequence`` computes it:

    [x | z] = h W_inᵀ
    pre_i   = conv_b + Σ_k conv_w[:, W-1-k] ⊙ x_{i+k}   (x_j = 0 for j ≥ n),   u = SiLU(pre)
    [Δr | B | C] = u W_xᵀ,   v = Δr W_dtᵀ + b_dt
    y       = the reverse scan (u, softplus(v), A = -exp(A_log), B, C, D, z)   (§3.4 ❷)
    o       = y W_outᵀ,   ĥ = LN(o) (γ, β; or ĥ = o without LN)   (❸)
    h⁺      = h + tanh(s) ĥ   (❹)

Training the sidecar alone (the paper's R2LM-PI setting, §3.4 and §4.1)
needs ∂L/∂(every parameter) and ∂L/∂h (the gradient passed on to the frozen
layers before the hook) from ∂L/∂h⁺.  The pages print no gradient; this is the
chain rule written out, step by step in reverse order:

    ĝ      = tanh(s) dh⁺;   ds = (1 - tanh²(s)) Σ dh⁺ ⊙ ĥ
    LN:      n̂ = (o - μ)/σ,  dγ = Σ ĝ ⊙ n̂,  dβ = Σ ĝ,
             do = (γ ĝ - mean(γ ĝ) - n̂ mean(γ ĝ ⊙ n̂)) / σ        (per row)
    out_proj: dy = do W_out,  dW_out = doᵀ y
    scan:    scan_backward.reverse_scan_backward (du_s, ddt_raw, dz, dB, dC, dA_log, dD, db_dt)
    dt_proj: dΔr = ddt_raw W_dt,  dW_dt = ddt_rawᵀ Δr
    x_proj:  d[Δr|B|C] → du_x = d[Δr|B|C] W_x,  dW_x = d[Δr|B|C]ᵀ u;  du = du_s + du_x
    SiLU:    dpre = du ⊙ SiLU'(pre)
    conv:    dx_{i+k} += conv_w[:, W-1-k] ⊙ dpre_i,  dconv_w[:, W-1-k] = Σ_i dpre_i ⊙ x_{i+k},
             dconv_b = Σ_i dpre_i
    in_proj: dh = dh⁺ + [dx | dz] W_in,  dW_in = [dx | dz]ᵀ h

Matrix products use ``numpy.matmul`` as a library primitive.

Parity status: pinned in ``tests/test_oracle_sidecar_backward.py`` by central
finite differences of the forward oracle for h, s and every parameter, and by
the s = 0 closed form (dh = dh⁺, every other gradient zero except ds).
"""
from __future__ import annotations

import numpy as np

from .r2l_oracle import LN_EPS, silu, sidecar_sequence
from .scan_backward import reverse_scan_backward, sigmoid

__all__ = ["sidecar_sequence_backward", "sidecar_backward_batch"]


def _silu_grad(v):
    """SiLU'(v) = σ(v) (1 + v (1 - σ(v)))."""
    sg = sigmoid(v)
    return sg * (1.0 + v * (1.0 - sg))


def sidecar_sequence_backward(h, w, s, dh_out, length=None):
    """Gradients of Σ dh_out ⊙ sidecar_sequence(h, w, s, length).

    h, dh_out: [L, d_model] float64; w as for ``sidecar_sequence``.  Rows at
    or past ``length`` pass their gradient straight through (they are not
    read).  Returns a dict: dh [L, d_model], ds (float) and d<name> for every
    entry of w (dln_w / dln_b are None without the LayerNorm).
    """
    L, d = h.shape
    n = L if length is None else int(length)
    g = float(np.tanh(np.float64(s)))
    out = {"dh": np.array(dh_out, dtype=np.float64, copy=True), "ds": 0.0}
    for k, v in w.items():
        out["d" + k] = None if v is None else np.zeros_like(v, dtype=np.float64)
    if n <= 0:
        return out
    E = w["W_in"].shape[0] // 2
    W = w["conv_w"].shape[1]
    _, it = sidecar_sequence(h, w, s, n, return_intermediates=True)
    hv = h[:n]
    x, z, u, dr, y, o, hhat = it["x"], it["z"], it["u"], it["dr"], it["y"], it["o"], it["hhat"]
    dho = dh_out[:n]

    # ❹ gated residual
    out["ds"] = float((1.0 - g * g) * np.sum(dho * hhat))
    ghat = g * dho

    # ❸ LayerNorm
    if w.get("ln_w") is None and w.get("ln_b") is None:
        do = ghat
    else:
        mu = o.mean(axis=-1, keepdims=True)
        var = ((o - mu) ** 2).mean(axis=-1, keepdims=True)
        sig = np.sqrt(var + LN_EPS)
        nh = (o - mu) / sig
        out["dln_w"] = np.sum(ghat * nh, axis=0)
        out["dln_b"] = np.sum(ghat, axis=0)
        gg = ghat * w["ln_w"]
        do = (gg - gg.mean(axis=-1, keepdims=True) - nh * (gg * nh).mean(axis=-1, keepdims=True)) / sig

    # out_proj
    dy = np.matmul(do, w["W_out"])
    out["dW_out"] = np.matmul(do.T, y)

    # ❷ the scan, with dt_raw = Δr W_dtᵀ
    dt_raw = np.matmul(dr, w["W_dt"].T)
    N = w["A_log"].shape[1]
    R = w["W_dt"].shape[1]
    Bm, Cm = it["B"], it["C"]
    gs = reverse_scan_backward(u, dt_raw, w["b_dt"], w["A_log"], Bm, Cm, w["D"], z, dy)
    out["dA_log"] = gs["dA_log"]
    out["dD"] = gs["dD"]
    out["db_dt"] = gs["ddt_b"]

    # dt_proj
    ddr = np.matmul(gs["ddt_raw"], w["W_dt"])
    out["dW_dt"] = np.matmul(gs["ddt_raw"].T, dr)

    # x_proj
    ddbc = np.concatenate([ddr, gs["dB"], gs["dC"]], axis=1)          # [n, R + 2N]
    assert ddbc.shape[1] == R + 2 * N
    du = gs["du"] + np.matmul(ddbc, w["W_x"])
    out["dW_x"] = np.matmul(ddbc.T, u)

    # conv + SiLU (anti-causal taps, zero past the sequence's end)
    pre = np.empty((n, E))
    pre[:] = w["conv_b"]
    for k in range(min(W, n)):
        pre[: n - k] += w["conv_w"][:, W - 1 - k] * x[k:]
    dpre = du * _silu_grad(pre)
    dx = np.zeros((n, E))
    for k in range(min(W, n)):
        dx[k:] += w["conv_w"][:, W - 1 - k] * dpre[: n - k]
        out["dconv_w"][:, W - 1 - k] = np.sum(dpre[: n - k] * x[k:], axis=0)
    out["dconv_b"] = np.sum(dpre, axis=0)

    # in_proj
    dxz = np.concatenate([dx, gs["dz"]], axis=1)                      # [n, 2E]
    out["dh"][:n] += np.matmul(dxz, w["W_in"])
    out["dW_in"] = np.matmul(dxz.T, hv)
    assert np.allclose(silu(pre), u)
    return out


def sidecar_backward_batch(h, w, s, dh_out, lengths=None):
    """The same over a right-padded batch: h, dh_out [B, L, d_model].  Each
    sequence b uses its first lengths[b] positions; padding rows pass dh_out
    through unchanged (the hook neither reads nor writes them), and the
    parameter gradients and ds are summed over the sequences."""
    Bt, L, _ = h.shape
    lens = [L] * Bt if lengths is None else [int(x) for x in lengths]
    total = None
    dh = np.empty_like(np.asarray(dh_out, dtype=np.float64))
    for b in range(Bt):
        g = sidecar_sequence_backward(h[b], w, s, dh_out[b], lens[b])
        dh[b] = g.pop("dh")
        if total is None:
            total = g
        else:
            for k, v in g.items():
                if v is not None:
                    total[k] = total[k] + v
    total["dh"] = dh
    return total
