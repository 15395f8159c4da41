"""Pins of the scan-gradient oracle (oracle/scan_backward.py): the gradient of
the reverse selective scan of "Bifocal Diffusion Language Models" (arXiv
2606.27732v1, §3.4 step ❷), checked against things other than itself:

  * central finite differences of the forward oracle, input by input (the
    forward oracle is pinned on its own in test_oracle_pins.py);
  * the closed form at n = 1, where H_0 = Δ u B and nothing decays;
  * batch wrapper: padding positions get zero gradients, parameter gradients
    are the sum over sequences;
  * planted mistakes (wrong adjoint direction, a decay index off by one, a
    dropped term) are caught by the finite-difference pin.
"""
import numpy as np
import pytest

import oracle as O
import oracle.r2l_oracle as R

N = 16


def _inputs(n, E, seed, big_v=False):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((n, E))
    dt_raw = rng.standard_normal((n, E)) * 0.5
    dt_b = rng.uniform(-3.0, 0.0, E)
    if big_v:
        dt_raw[0, 0] = 25.0                     # softplus(v) = v branch, far from the threshold
    A_log = np.log(np.tile(np.arange(1, N + 1, dtype=np.float64), (E, 1))) + rng.uniform(-0.3, 0.3, (E, N))
    B = rng.standard_normal((n, N))
    C = rng.standard_normal((n, N))
    D = rng.standard_normal(E)
    z = rng.standard_normal((n, E))
    dy = rng.standard_normal((n, E))
    return dict(u=u, dt_raw=dt_raw, dt_b=dt_b, A_log=A_log, B=B, C=C, D=D, z=z), dy


def _loss(args, dy):
    y = O.reverse_scan_forward_from_raw(args["u"], args["dt_raw"], args["dt_b"], args["A_log"], args["B"],
                                        args["C"], args["D"], args["z"])
    return float(np.sum(dy * y))


def _fd(args, dy, name, eps=1e-6):
    x = args[name]
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        old = x[idx]
        x[idx] = old + eps
        lp = _loss(args, dy)
        x[idx] = old - eps
        lm = _loss(args, dy)
        x[idx] = old
        g[idx] = (lp - lm) / (2 * eps)
    return g


GRAD_OF = {"u": "du", "dt_raw": "ddt_raw", "z": "dz", "B": "dB", "C": "dC", "A_log": "dA_log", "D": "dD",
           "dt_b": "ddt_b"}


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-12))


def _oracle_grads(args, dy, fn=None):
    fn = fn or O.reverse_scan_backward
    return fn(args["u"], args["dt_raw"], args["dt_b"], args["A_log"], args["B"], args["C"], args["D"],
              args["z"], dy)


@pytest.mark.parametrize("n,E,seed,big_v", [(6, 3, 1, False), (9, 2, 2, True), (1, 4, 3, False)])
def test_scan_backward_matches_finite_differences(n, E, seed, big_v):
    args, dy = _inputs(n, E, seed, big_v)
    g = _oracle_grads(args, dy)
    for name, gname in GRAD_OF.items():
        fd = _fd(args, dy, name)
        assert _rel(g[gname], fd) < 1e-6, f"{gname}: rel err {_rel(g[gname], fd):.2e}"


def test_scan_backward_closed_form_single_position():
    args, dy = _inputs(1, 5, 7)
    u, z, D = args["u"][0], args["z"][0], args["D"]
    v = args["dt_raw"][0] + args["dt_b"]
    delta = np.log1p(np.exp(v))
    Bv, Cv = args["B"][0], args["C"][0]
    sz = z / (1.0 + np.exp(-z))
    dp = dy[0] * sz
    bc = float(Bv @ Cv)
    g = _oracle_grads(args, dy)
    sig_v = 1.0 / (1.0 + np.exp(-v))
    assert np.allclose(g["du"][0], dp * (delta * bc + D), rtol=1e-12, atol=1e-14)
    assert np.allclose(g["ddt_raw"][0], dp * u * bc * sig_v, rtol=1e-12, atol=1e-14)
    assert np.allclose(g["dB"][0], np.sum(dp * delta * u) * Cv, rtol=1e-12, atol=1e-14)
    assert np.allclose(g["dC"][0], np.sum(dp * delta * u) * Bv, rtol=1e-12, atol=1e-14)
    assert np.allclose(g["dA_log"], 0.0)              # nothing decays at n = 1
    assert np.allclose(g["dD"], dp * u, rtol=1e-12, atol=1e-14)


def test_scan_backward_batch_padding_and_sums():
    Bt, L, E = 3, 7, 4
    lens = [7, 0, 4]
    parts = [_inputs(L, E, 20 + b) for b in range(Bt)]
    shared = parts[0][0]
    u = np.stack([p[0]["u"] for p in parts]); dt = np.stack([p[0]["dt_raw"] for p in parts])
    Bm = np.stack([p[0]["B"] for p in parts]); Cm = np.stack([p[0]["C"] for p in parts])
    z = np.stack([p[0]["z"] for p in parts]); dy = np.stack([p[1] for p in parts])
    out = O.reverse_scan_backward_batch(u, dt, shared["dt_b"], shared["A_log"], Bm, Cm, shared["D"], z, dy, lens)
    tot = {k: 0.0 for k in ("dA_log", "dD", "ddt_b")}
    for b, n in enumerate(lens):
        for k in ("du", "ddt_raw", "dz", "dB", "dC"):
            assert np.all(out[k][b, n:] == 0.0)
        if n == 0:
            continue
        g = O.reverse_scan_backward(u[b, :n], dt[b, :n], shared["dt_b"], shared["A_log"], Bm[b, :n], Cm[b, :n],
                                    shared["D"], z[b, :n], dy[b, :n])
        assert np.array_equal(out["du"][b, :n], g["du"])
        for k in tot:
            tot[k] = tot[k] + g[k]
    for k in tot:
        assert np.allclose(out[k], tot[k], rtol=1e-13, atol=1e-15)


# ---- planted mistakes: each must fail the finite-difference pin ----

def _mutant(kind):
    def bwd(u, dt_raw, dt_b, A_log, B, C, D, z, dy):
        n, E = u.shape
        A = -np.exp(A_log)
        v = dt_raw + dt_b
        delta = O.softplus(v)
        dsoft = np.where(v > R.SOFTPLUS_THRESHOLD, 1.0, O.sigmoid(v))
        a = np.exp(delta[:, :, None] * A[None])
        H = np.zeros((n + 1, E, A.shape[1]))
        for i in range(n - 1, -1, -1):
            H[i] = a[i] * H[i + 1] + (delta[i] * u[i])[:, None] * B[i][None, :]
        p = np.einsum("ien,in->ie", H[:n], C) + D * u
        sg = O.sigmoid(z)
        dp = dy * O.silu(z)
        dz = dy * p * sg * (1 + z * (1 - sg))
        du = np.empty((n, E)); dd = np.empty((n, E)); dB = np.empty((n, A.shape[1])); dC = np.empty_like(dB)
        dA = np.zeros_like(A)
        G = np.zeros_like(A)
        order = range(n - 1, -1, -1) if kind == "adjoint_direction" else range(n)
        prev = None
        for i in order:
            if prev is not None:
                G = (a[i] if kind == "decay_index" else a[prev]) * G
            G = G + dp[i][:, None] * C[i][None, :]
            dC[i] = dp[i] @ H[i]
            dB[i] = (delta[i] * u[i]) @ G
            da = G * H[i + 1]
            gB = G @ B[i]
            dd[i] = np.sum(da * a[i] * A, 1) + u[i] * gB
            du[i] = (0.0 if kind == "drop_D" else D * dp[i]) + delta[i] * gB
            dA += delta[i][:, None] * da * a[i]
            prev = i
        ddt = dd * dsoft
        return {"du": du, "ddt_raw": ddt, "dz": dz, "dB": dB, "dC": dC, "dA_log": dA * A,
                "dD": np.sum(dp * u, 0), "ddt_b": ddt.sum(0)}
    return bwd


@pytest.mark.parametrize("kind", ["adjoint_direction", "decay_index", "drop_D"])
def test_finite_difference_pin_catches_planted_mistake(kind):
    args, dy = _inputs(6, 3, 5)
    g = _oracle_grads(args, dy, _mutant(kind))
    worst = 0.0
    for name, gname in GRAD_OF.items():
        worst = max(worst, _rel(g[gname], _fd(args, dy, name)))
    assert worst > 1e-3, f"planted mistake {kind} not caught (worst rel err {worst:.2e})"


def test_unplanted_mutant_template_is_the_oracle():
    """The mutant template with no mistake reproduces the oracle (so the
    planted mistakes above differ from it in one place each)."""
    args, dy = _inputs(6, 3, 5)
    a = _oracle_grads(args, dy, _mutant("none"))
    b = _oracle_grads(args, dy)
    for k in a:
        assert np.allclose(a[k], b[k], rtol=1e-12, atol=1e-14)
