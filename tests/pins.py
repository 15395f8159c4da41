"""Checks that pin the CPU oracle to facts outside itself.

Each ``pin_*`` function takes the oracle namespace ``O`` (the real module, or a
deliberately broken copy in the mutation tests) and raises AssertionError when
the oracle disagrees with a closed form, a library routine, a brute-force
computation or an invariant stated in "Bifocal Diffusion Language Models"
(arXiv 2606.27732v1), §3.4 steps ❶–❹.

None of these checks retypes the oracle's formula: they use torch's own
functional ops, a different algorithm (the O(n²) unrolled sum), a different
direction (a forward block on the flipped sequence) or a property that holds
for any correct implementation.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

RNG = np.random.default_rng


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b)))) if b.size else 1.0
    assert err <= tol * scale, f"{what}: max err {err:.3e} > {tol:.1e}·{scale:.3g}"


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def tiny_weights(rng, d=12, E=24, N=16, R=3, W=4, scale=0.3, ln="seeded"):
    """O(1)-scale random weights so every term of the layer is visible."""
    w = dict(
        W_in=rng.normal(0, scale, (2 * E, d)),
        conv_w=rng.normal(0, 0.5, (E, W)),
        conv_b=rng.normal(0, 0.2, (E,)),
        W_x=rng.normal(0, scale, (R + 2 * N, E)),
        W_dt=rng.normal(0, scale, (E, R)),
        b_dt=rng.normal(-1.0, 0.5, (E,)),
        A_log=np.log(rng.uniform(0.5, 4.0, (E, N))),
        D=rng.normal(1.0, 0.3, (E,)),
        W_out=rng.normal(0, scale, (d, E)),
    )
    if ln == "seeded":
        w["ln_w"] = rng.normal(1.0, 0.2, (d,))
        w["ln_b"] = rng.normal(0.0, 0.2, (d,))
    else:
        w["ln_w"] = None
        w["ln_b"] = None
    return w


# ---------------------------------------------------------------- pointwise ops

def pin_activations(O):
    """SiLU and softplus against torch's library routines (threshold 20)."""
    v = np.concatenate([np.linspace(-40, 40, 2001), [-1e-300, 0.0, 19.999, 20.0, 20.001, 30.0]])
    _close(O.silu(v), F.silu(_t(v)).numpy(), 1e-15, "silu")
    _close(O.softplus(v), F.softplus(_t(v), beta=1.0, threshold=20.0).numpy(), 1e-15, "softplus")


def pin_round_bf16(O):
    """One-step RNE to bf16 against torch's fp32->bf16 conversion on fp32-exact
    inputs (no double rounding possible), plus hand-made ties."""
    rng = RNG(7)
    f32 = rng.normal(0, 3, 20000).astype(np.float32)
    ref = torch.from_numpy(f32).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_to_bf16(f32.astype(np.float64))
    assert np.array_equal(got, ref), "round_to_bf16 disagrees with torch on fp32-exact values"
    # 1 + 2^-8 is the tie between 1 and 1 + 2^-7: ties to even -> 1.0
    # 1 + 3·2^-8 is the tie between 1+2^-7 and 1+2^-6: -> 1 + 2^-6
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)])
    want = np.array([1.0, 1 + 2.0 ** -6, -1.0])
    assert np.array_equal(O.round_to_bf16(ties), want), "round_to_bf16 ties"


# ---------------------------------------------------------------- projections

def pin_in_proj_split(O):
    """[x | z] = h·W_inᵀ: structured weights fix the split order and the
    orientation of W_in (an nn.Linear [out, in] matrix)."""
    rng = RNG(1)
    n, d, E = 5, 3, 4
    h = rng.normal(size=(n, d))
    W = np.zeros((2 * E, d))
    W[0, 0] = 1.0      # x[:,0] = h[:,0]
    W[1, 2] = 2.0      # x[:,1] = 2 h[:,2]
    W[E, 1] = -3.0     # z[:,0] = -3 h[:,1]
    W[2 * E - 1, 0] = 5.0
    x, z = O.in_proj(h, W)
    assert x.shape == (n, E) and z.shape == (n, E)
    _close(x[:, 0], h[:, 0], 0, "in_proj x0")
    _close(x[:, 1], 2 * h[:, 2], 0, "in_proj x1")
    _close(z[:, 0], -3 * h[:, 1], 0, "in_proj z0")
    _close(z[:, E - 1], 5 * h[:, 0], 0, "in_proj z_last")
    Wr = rng.normal(size=(2 * E, d))
    x, z = O.in_proj(h, Wr)
    ref = F.linear(_t(h), _t(Wr)).numpy()
    _close(np.concatenate([x, z], axis=1), ref, 1e-14, "in_proj vs F.linear")


def pin_x_proj_split(O):
    """[Δ_r | B | C] split order and orientation."""
    rng = RNG(2)
    n, E, R, N = 4, 6, 2, 3
    u = rng.normal(size=(n, E))
    W = np.zeros((R + 2 * N, E))
    W[0, 1] = 1.0          # dr[:,0] = u[:,1]
    W[R, 2] = 2.0          # B[:,0]  = 2 u[:,2]
    W[R + N, 3] = 3.0      # C[:,0]  = 3 u[:,3]
    W[R + 2 * N - 1, 5] = -1.0
    dr, Bm, Cm = O.x_proj(u, W, R, N)
    assert dr.shape == (n, R) and Bm.shape == (n, N) and Cm.shape == (n, N)
    _close(dr[:, 0], u[:, 1], 0, "x_proj dr")
    _close(Bm[:, 0], 2 * u[:, 2], 0, "x_proj B")
    _close(Cm[:, 0], 3 * u[:, 3], 0, "x_proj C")
    _close(Cm[:, N - 1], -u[:, 5], 0, "x_proj C last")


def pin_dt(O):
    """Δ = softplus(dr·W_dtᵀ + b_dt) against torch's linear + softplus."""
    rng = RNG(3)
    dr = rng.normal(size=(7, 3)) * 4
    W = rng.normal(size=(5, 3)) * 3
    b = rng.normal(size=(5,)) * 5
    ref = F.softplus(F.linear(_t(dr), _t(W), _t(b)), threshold=20.0).numpy()
    _close(O.dt_softplus(dr, W, b), ref, 1e-14, "dt_softplus")


def pin_conv(O):
    """The anti-causal conv equals flip ∘ (torch causal depthwise conv1d) ∘ flip,
    and an impulse picks out the taps in the stated order."""
    rng = RNG(4)
    for n in (1, 2, 3, 7, 16):
        E, W = 5, 4
        x = rng.normal(size=(n, E))
        w = rng.normal(size=(E, W))
        b = rng.normal(size=(E,))
        xf = _t(x[::-1].copy()).T[None]                     # [1, E, n] flipped
        pre_f = F.conv1d(xf, _t(w)[:, None, :], _t(b), padding=W - 1, groups=E)[0, :, :n]
        ref = F.silu(pre_f).T.numpy()[::-1]                 # un-flip
        _close(O.anticausal_conv_silu(x, w, b), ref, 1e-14, f"conv n={n}")
    # impulse at position j: pre-activation at i is w[W-1-(j-i)] for i<=j<=i+W-1
    n, E, W = 9, 1, 4
    w = np.array([[10.0, 20.0, 30.0, 40.0]])
    for j in range(n):
        x = np.zeros((n, E))
        x[j, 0] = 1.0
        u = O.anticausal_conv_silu(x, w, np.zeros(E))
        pre = np.zeros(n)
        for i in range(n):
            k = j - i
            if 0 <= k < W:
                pre[i] = w[0, W - 1 - k]
        _close(u[:, 0], F.silu(_t(pre)).numpy(), 1e-15, f"conv impulse j={j}")


# ---------------------------------------------------------------- the scan

def brute_force_scan(u, delta, A, B, C, D, z):
    """O(n²) unrolled form of the reverse recurrence (an independent algorithm):

        y_i = SiLU(z_i) · ( Σ_{j=i}^{n-1} Σ_m C_i[m] · exp(A[:,m] · Σ_{k=i}^{j-1} Δ_k) · B_j[m] · Δ_j u_j
                            + D u_i )
    """
    n, E = u.shape
    y = np.zeros((n, E))
    for i in range(n):
        acc = D * u[i]
        cum = np.zeros(E)
        for j in range(i, n):
            decay = np.exp(cum[:, None] * A)                          # [E, N]
            acc = acc + (decay * B[j][None, :] * C[i][None, :]).sum(axis=1) * delta[j] * u[j]
            cum = cum + delta[j]
        y[i] = acc * (z[i] / (1.0 + np.exp(-z[i])))
    return y


def _scan_inputs(rng, n, E=6, N=5):
    u = rng.normal(size=(n, E))
    delta = rng.uniform(0.01, 0.8, size=(n, E))
    A = -rng.uniform(0.1, 3.0, size=(E, N))
    B = rng.normal(size=(n, N))
    C = rng.normal(size=(n, N))
    D = rng.normal(size=(E,))
    z = rng.normal(size=(n, E))
    return u, delta, A, B, C, D, z


def pin_scan_bruteforce(O):
    rng = RNG(5)
    for n in (1, 2, 5, 17, 40):
        args = _scan_inputs(rng, n)
        _close(O.reverse_selective_scan(*args), brute_force_scan(*args), 1e-12, f"scan n={n}")


def pin_scan_special_cases(O):
    rng = RNG(6)
    n = 12
    u, delta, A, B, C, D, z = _scan_inputs(rng, n)
    g = z / (1.0 + np.exp(-z))
    # A = 0: no decay, H_i is the suffix sum of Δ u B (reverse cumulative sum)
    A0 = np.zeros_like(A)
    terms = (delta * u)[:, :, None] * B[:, None, :]                  # [n, E, N]
    Hs = np.flip(np.cumsum(np.flip(terms, 0), 0), 0)
    want = ((Hs * C[:, None, :]).sum(-1) + D * u) * g
    _close(O.reverse_selective_scan(u, delta, A0, B, C, D, z), want, 1e-12, "scan A=0")
    # A -> -inf: no memory, H_i = Δ_i u_i B_i
    Ainf = np.full_like(A, -1e30)
    want = ((delta * u) * (B * C).sum(-1)[:, None] + D * u) * g
    _close(O.reverse_selective_scan(u, delta, Ainf, B, C, D, z), want, 1e-12, "scan A=-inf")
    # linearity in u for fixed Δ, B, C, z
    u2 = rng.normal(size=u.shape)
    lhs = O.reverse_selective_scan(2.0 * u - 3.0 * u2, delta, A, B, C, D, z)
    rhs = 2.0 * O.reverse_selective_scan(u, delta, A, B, C, D, z) - 3.0 * O.reverse_selective_scan(u2, delta, A, B, C, D, z)
    _close(lhs, rhs, 1e-12, "scan linearity")
    # last position sees only itself: y_{n-1} = (⟨C,B⟩ Δ u + D u)·SiLU(z)
    y = O.reverse_selective_scan(u, delta, A, B, C, D, z)
    want_last = ((B[-1] * C[-1]).sum() * delta[-1] * u[-1] + D * u[-1]) * g[-1]
    _close(y[-1], want_last, 1e-13, "scan last position")


# ---------------------------------------------------------------- norm / residual

def pin_layer_norm(O):
    rng = RNG(8)
    o = rng.normal(size=(6, 10)) * 3 + 1
    gw = rng.normal(size=10)
    gb = rng.normal(size=10)
    ref = F.layer_norm(_t(o), (10,), _t(gw), _t(gb), eps=1e-5).numpy()
    _close(O.layer_norm(o, gw, gb), ref, 1e-13, "layer_norm vs F.layer_norm")
    # LN(0) = β exactly (mean 0, variance 0)
    _close(O.layer_norm(np.zeros((3, 10)), gw, gb), np.tile(gb, (3, 1)), 0, "LN(0)=beta")
    # no-LN variant is the identity
    assert np.array_equal(O.layer_norm(o, None, None), o)


def pin_gate(O):
    rng = RNG(9)
    h = rng.normal(size=(4, 5))
    r = rng.normal(size=(4, 5))
    assert np.array_equal(O.gated_residual(h, r, 0.0), h), "tanh(0) gate must be the identity"
    _close(O.gated_residual(h, r, 0.7), h + np.tanh(0.7) * r, 1e-15, "gate")
    _close(O.gated_residual(h, r, 50.0), h + r, 1e-15, "gate saturates at tanh -> 1")


# ---------------------------------------------------------------- whole layer

def forward_mamba_block_l2r(hs, w):
    """A left-to-right Mamba-1 block + LN written with torch functional ops
    (causal conv1d with left padding, forward scan).  Used only on a flipped
    sequence to check the flip definition of §3.4 steps ❶–❸."""
    h = _t(hs)
    n = h.shape[0]
    E = w["W_in"].shape[0] // 2
    Wc = w["conv_w"].shape[1]
    N = w["A_log"].shape[1]
    R = w["W_dt"].shape[1]
    xz = F.linear(h, _t(w["W_in"]))
    x, z = xz[:, :E], xz[:, E:]
    xc = F.conv1d(x.T[None], _t(w["conv_w"])[:, None, :], _t(w["conv_b"]), padding=Wc - 1, groups=E)[0, :, :n].T
    u = F.silu(xc)
    dbc = F.linear(u, _t(w["W_x"]))
    dr, Bm, Cm = dbc[:, :R], dbc[:, R:R + N], dbc[:, R + N:]
    delta = F.softplus(F.linear(dr, _t(w["W_dt"]), _t(w["b_dt"])), threshold=20.0)
    A = -torch.exp(_t(w["A_log"]))
    H = torch.zeros(E, N, dtype=torch.float64)
    ys = []
    for t in range(n):
        H = torch.exp(delta[t][:, None] * A) * H + (delta[t] * u[t])[:, None] * Bm[t][None, :]
        ys.append(H @ Cm[t] + _t(w["D"]) * u[t])
    y = torch.stack(ys) * F.silu(z)
    o = F.linear(y, _t(w["W_out"]))
    if w.get("ln_w") is None:
        return o.numpy()
    return F.layer_norm(o, (o.shape[-1],), _t(w["ln_w"]), _t(w["ln_b"]), eps=1e-5).numpy()


def pin_flip_equivalence(O):
    """h⁺ = h + tanh(s)·LN(flip(Mamba(flip(h)))) with a forward block (C3)."""
    rng = RNG(10)
    for ln in ("seeded", "none"):
        w = tiny_weights(rng, ln=ln)
        for n in (1, 3, 9, 20):
            h = rng.normal(size=(n, w["W_in"].shape[1]))
            s = 0.8
            hhat = forward_mamba_block_l2r(h[::-1].copy(), w)[::-1]
            want = h + np.tanh(s) * hhat
            got = O.sidecar_sequence(h, w, s)
            _close(got, want, 1e-11, f"flip equivalence n={n} ln={ln}")


def pin_s_zero_identity(O):
    rng = RNG(11)
    w = tiny_weights(rng)
    h = rng.normal(size=(2, 9, w["W_in"].shape[1]))
    out = O.sidecar_forward(h, w, 0.0)
    assert np.array_equal(out, h), "s=0 must return the input bit for bit"


def pin_right_context_only(O):
    """Output at position i depends only on inputs at j >= i (exact)."""
    rng = RNG(12)
    w = tiny_weights(rng)
    n, d = 14, w["W_in"].shape[1]
    h = rng.normal(size=(n, d))
    base = O.sidecar_sequence(h, w, 0.6)
    for i in (1, 5, 13):
        h2 = h.copy()
        h2[:i] = rng.normal(size=(i, d)) * 10
        out2 = O.sidecar_sequence(h2, w, 0.6)
        assert np.array_equal(out2[i:], base[i:]), f"positions >= {i} changed"
        assert not np.allclose(out2[i - 1], base[i - 1]), "the perturbed row itself must change"
    # and a change at position j does reach positions < j
    h3 = h.copy()
    h3[n - 1] += 1.0
    out3 = O.sidecar_sequence(h3, w, 0.6)
    assert not np.allclose(out3[0], base[0]), "right context must reach position 0"


def pin_ragged_isolation(O):
    """A sequence in a right-padded batch equals the same sequence alone, and
    equals the independently written forward block through the flip (C3, C7);
    the padding (NaN) is never read and is returned unchanged."""
    rng = RNG(13)
    w = tiny_weights(rng)
    B, L, d = 3, 10, w["W_in"].shape[1]
    lengths = [10, 4, 0]
    h = rng.normal(size=(B, L, d))
    for b, n in enumerate(lengths):
        h[b, n:] = np.nan
    out = O.sidecar_forward(h, w, 0.9, lengths=lengths)
    for b, n in enumerate(lengths):
        alone = O.sidecar_sequence(h[b, :n], w, 0.9) if n > 0 else h[b, :0]
        assert np.array_equal(out[b, :n], alone), f"sequence {b} differs from running alone"
        if n > 0:
            want = h[b, :n] + np.tanh(0.9) * forward_mamba_block_l2r(h[b, :n][::-1].copy(), w)[::-1]
            _close(out[b, :n], want, 1e-11, f"sequence {b} against the forward block through the flip")
        assert np.all(np.isnan(out[b, n:])), f"padding of sequence {b} was written"
        assert np.all(np.isfinite(out[b, :n]))


def pin_stack_composition(O):
    """Hooks compose in order, each with its own weights and gate: the stack
    (fp64 between hooks) on a ragged batch equals the hooks applied one after
    another through the independently written forward block and the flip (C3);
    and with bf16 storage each hook's output is rounded before the next hook
    reads it."""
    rng = RNG(14)
    ws = [tiny_weights(rng) for _ in range(3)]
    ss = [0.3, -0.7, 0.5]
    lengths = [6, 4]
    h = rng.normal(size=(2, 6, ws[0]["W_in"].shape[1]))
    h[1, 4:] = np.nan
    got = O.sidecar_stack(h, ws, ss, lengths=lengths)
    for b, n in enumerate(lengths):
        cur = h[b, :n].copy()
        for w, s in zip(ws, ss):
            cur = cur + np.tanh(s) * forward_mamba_block_l2r(cur[::-1].copy(), w)[::-1]
        _close(got[b, :n], cur, 1e-10, f"stack of 3 hooks, sequence {b}")
        assert np.all(np.isnan(got[b, n:])), f"padding of sequence {b} was written"
    hb = O.round_to_bf16(rng.normal(size=(2, 6, ws[0]["W_in"].shape[1])))
    cur = hb
    for w, s in zip(ws, ss):
        cur = O.round_to_bf16(O.sidecar_forward(cur, w, s))
    assert np.array_equal(O.sidecar_stack(hb, ws, ss, out_dtype="bf16"), cur)


def pin_l2r_direction(O):
    """The left-to-right control equals a forward Mamba block written with
    torch ops (no flip involved), and a change at position j reaches only
    positions >= j."""
    rng = RNG(15)
    w = tiny_weights(rng)
    B, L, d = 2, 9, w["W_in"].shape[1]
    lengths = [9, 5]
    h = rng.normal(size=(B, L, d))
    got = O.sidecar_forward(h, w, 0.6, lengths=lengths, direction="l2r")
    for b, n in enumerate(lengths):
        want = h[b, :n] + np.tanh(0.6) * forward_mamba_block_l2r(h[b, :n], w)
        _close(got[b, :n], want, 1e-11, f"l2r b={b}")
        assert np.array_equal(got[b, n:], h[b, n:])
    h2 = h.copy()
    h2[0, 6:] += 1.0
    out2 = O.sidecar_forward(h2, w, 0.6, lengths=lengths, direction="l2r")
    assert np.array_equal(out2[0, :6], got[0, :6]), "left-to-right: positions < 6 must not change"


ALL_PINS = [
    pin_activations, pin_round_bf16, pin_in_proj_split, pin_x_proj_split, pin_dt,
    pin_conv, pin_scan_bruteforce, pin_scan_special_cases, pin_layer_norm, pin_gate,
    pin_flip_equivalence, pin_s_zero_identity, pin_right_context_only,
    pin_ragged_isolation, pin_stack_composition, pin_l2r_direction,
]
