"""Pins of the whole-hook gradient oracle (oracle/sidecar_backward.py): the
gradient of one sidecar hook of "Bifocal Diffusion Language Models" (arXiv
2606.27732v1, §3.4 steps ❶–❹), checked against things other than itself:

  * central finite differences of the pinned forward oracle
    (``sidecar_sequence``) for h, s and every parameter, with and without
    the LayerNorm, on a full-length and a shorter valid prefix;
  * the s = 0 closed form: the hook is the identity, so dh = dh⁺ and every
    parameter gradient is zero, while ds = Σ dh⁺ ⊙ ĥ.
"""
import numpy as np
import pytest

import oracle as O
from oracle.sidecar_backward import sidecar_sequence_backward

D_MODEL, E, N, R, W = 4, 6, 16, 2, 4


def _weights(seed, ln=True):
    rng = np.random.default_rng(seed)
    w = {
        "W_in": rng.standard_normal((2 * E, D_MODEL)) * 0.5,
        "conv_w": rng.standard_normal((E, W)) * 0.5,
        "conv_b": rng.standard_normal(E) * 0.1,
        "W_x": rng.standard_normal((R + 2 * N, E)) * 0.5,
        "W_dt": rng.standard_normal((E, R)) * 0.5,
        "b_dt": rng.uniform(-3.0, -1.0, E),
        "A_log": np.log(np.tile(np.arange(1, N + 1, dtype=np.float64), (E, 1))) + rng.uniform(-0.2, 0.2, (E, N)),
        "D": rng.standard_normal(E),
        "W_out": rng.standard_normal((D_MODEL, E)) * 0.5,
        "ln_w": 1.0 + rng.standard_normal(D_MODEL) * 0.2 if ln else None,
        "ln_b": rng.standard_normal(D_MODEL) * 0.2 if ln else None,
    }
    return w


def _loss(h, w, s, dh, n):
    return float(np.sum(dh * O.sidecar_sequence(h, w, s, n)))


def _fd_array(f, x, eps=1e-6):
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        old = x[idx]
        x[idx] = old + eps
        lp = f()
        x[idx] = old - eps
        lm = f()
        x[idx] = old
        g[idx] = (lp - lm) / (2 * eps)
    return g


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-12))


@pytest.mark.parametrize("ln,L,n,seed", [(True, 7, 7, 1), (True, 9, 6, 2), (False, 5, 5, 3)])
def test_sidecar_backward_matches_finite_differences(ln, L, n, seed):
    rng = np.random.default_rng(100 + seed)
    h = rng.standard_normal((L, D_MODEL))
    dh = rng.standard_normal((L, D_MODEL))
    w = _weights(seed, ln)
    s = 0.7
    g = sidecar_sequence_backward(h, w, s, dh, n)
    fd_h = _fd_array(lambda: _loss(h, w, s, dh, n), h)
    assert _rel(g["dh"], fd_h) < 1e-6, f"dh: {_rel(g['dh'], fd_h):.2e}"
    sv = np.array([s])
    fd_s = _fd_array(lambda: _loss(h, w, sv[0], dh, n), sv)[0]
    assert abs(g["ds"] - fd_s) <= 1e-6 * max(1.0, abs(fd_s))
    for k, v in w.items():
        if v is None:
            assert g["d" + k] is None
            continue
        fd = _fd_array(lambda: _loss(h, w, s, dh, n), v)
        assert _rel(g["d" + k], fd) < 1e-6, f"d{k}: rel err {_rel(g['d' + k], fd):.2e}"


def test_sidecar_backward_zero_gate_is_identity():
    rng = np.random.default_rng(7)
    h = rng.standard_normal((6, D_MODEL))
    dh = rng.standard_normal((6, D_MODEL))
    w = _weights(4)
    g = sidecar_sequence_backward(h, w, 0.0, dh)
    assert np.array_equal(g["dh"], dh)
    for k, v in w.items():
        assert np.all(g["d" + k] == 0.0), k
    _, it = O.sidecar_sequence(h, w, 0.0, return_intermediates=True)
    assert np.isclose(g["ds"], np.sum(dh * it["hhat"]), rtol=1e-12)


def test_finite_difference_pin_catches_planted_mistake(monkeypatch):
    """A plausible mistake planted in the oracle (SiLU' taken as σ alone)
    must fail the finite-difference pin."""
    import oracle.sidecar_backward as SB
    monkeypatch.setattr(SB, "_silu_grad", lambda v: O.sigmoid(v))
    rng = np.random.default_rng(11)
    h = rng.standard_normal((6, D_MODEL))
    dh = rng.standard_normal((6, D_MODEL))
    w = _weights(5)
    g = SB.sidecar_sequence_backward(h, w, 0.7, dh)
    fd = _fd_array(lambda: _loss(h, w, 0.7, dh, 6), w["conv_b"])
    assert _rel(g["dconv_b"], fd) > 1e-3


def test_batched_backward_padding_and_sums():
    """Ragged batch: each sequence's gradient is the single-sequence one on its
    valid prefix, padding rows pass dh⁺ through, parameter gradients add up;
    and a whole batch still matches finite differences of the batched forward."""
    from oracle.sidecar_backward import sidecar_backward_batch
    rng = np.random.default_rng(21)
    Bt, L = 3, 6
    lens = [6, 0, 3]
    h = rng.standard_normal((Bt, L, D_MODEL))
    dh = rng.standard_normal((Bt, L, D_MODEL))
    w = _weights(6)
    s = -0.4
    g = sidecar_backward_batch(h, w, s, dh, lens)
    for b, n in enumerate(lens):
        one = sidecar_sequence_backward(h[b], w, s, dh[b], n)
        assert np.array_equal(g["dh"][b], one["dh"])
        assert np.array_equal(g["dh"][b, n:], dh[b, n:])
    fd = _fd_array(lambda: float(np.sum(dh * O.sidecar_forward(h, w, s, np.array(lens)))), w["W_x"])
    assert _rel(g["dW_x"], fd) < 1e-6
    sv = np.array([s])
    fds = _fd_array(lambda: float(np.sum(dh * O.sidecar_forward(h, w, sv[0], np.array(lens)))), sv)[0]
    assert abs(g["ds"] - fds) <= 1e-6 * max(1.0, abs(fds))
