"""Plant a plausible mistake in the oracle (on the CPU) and check that at least
one pin catches it.  Shows the pins constrain every step, not only the whole."""
import numpy as np
import pytest

import oracle.r2l_oracle as R

from . import pins


def _conv_taps_reversed(x, conv_w, conv_b):
    n, E = x.shape
    W = conv_w.shape[1]
    pre = np.empty((n, E)); pre[:] = conv_b
    for k in range(min(W, n)):
        pre[: n - k] += conv_w[:, k] * x[k:]
    return R.silu(pre)


def _conv_causal(x, conv_w, conv_b):
    n, E = x.shape
    W = conv_w.shape[1]
    pre = np.empty((n, E)); pre[:] = conv_b
    for k in range(min(W, n)):
        pre[k:] += conv_w[:, W - 1 - k] * x[: n - k]
    return R.silu(pre)


def _scan_variant(direction=-1, use_D=True, sign=1.0, use_delta_in=True, swap_bc=False, gate=True):
    def scan(u, delta, A, B, C, D, z):
        if swap_bc:
            B, C = C, B
        n, E = u.shape
        H = np.zeros((E, A.shape[1]))
        y = np.empty((n, E))
        rng = range(n - 1, -1, -1) if direction < 0 else range(n)
        for i in rng:
            inp = (delta[i] * u[i]) if use_delta_in else u[i]
            H = np.exp(sign * delta[i][:, None] * A) * H + inp[:, None] * B[i][None, :]
            y[i] = H @ C[i] + (D * u[i] if use_D else 0.0)
        return y * R.silu(z) if gate else y
    return scan


def _in_proj_swapped(h, W_in):
    x, z = np.matmul(h, W_in.T)[:, : W_in.shape[0] // 2], np.matmul(h, W_in.T)[:, W_in.shape[0] // 2:]
    return z, x


def _xp(u, W_x, R_, N):
    dbc = u @ W_x.T
    return dbc[:, :R_], dbc[:, R_:R_ + N], dbc[:, R_ + N:]


def _ln_unbiased(o, ln_w, ln_b, eps=1e-5):
    if ln_w is None and ln_b is None:
        return o
    mu = o.mean(-1, keepdims=True)
    var = o.var(-1, ddof=1, keepdims=True)
    return (o - mu) / np.sqrt(var + eps) * ln_w + ln_b


def _ln_no_beta(o, ln_w, ln_b, eps=1e-5):
    if ln_w is None and ln_b is None:
        return o
    mu = o.mean(-1, keepdims=True)
    var = ((o - mu) ** 2).mean(-1, keepdims=True)
    return (o - mu) / np.sqrt(var + eps) * ln_w


def _gate_linear(h, r, s):
    return h + s * r


def _dt_no_bias(dr, W_dt, b_dt):
    return R.softplus(dr @ W_dt.T)


def _softplus_as_exp(v):
    return np.exp(np.asarray(v, dtype=np.float64))


def _silu_as_sigmoid(v):
    v = np.asarray(v, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-v))


def _stack_reversed(h, weights_list, s_list, lengths=None, out_dtype="f64", batch_indices=None):
    cur = np.asarray(h, dtype=np.float64)
    for w, s in zip(reversed(weights_list), reversed(s_list)):
        cur = R.sidecar_forward(cur, w, s, lengths, out_dtype, batch_indices)
    return cur


def _stack_gates_rotated(h, weights_list, s_list, lengths=None, out_dtype="f64", batch_indices=None):
    cur = np.asarray(h, dtype=np.float64)
    for w, s in zip(weights_list, list(s_list[1:]) + list(s_list[:1])):
        cur = R.sidecar_forward(cur, w, s, lengths, out_dtype, batch_indices)
    return cur


MUTANTS = {
    "conv taps reversed": ("anticausal_conv_silu", _conv_taps_reversed),
    "conv causal direction": ("anticausal_conv_silu", _conv_causal),
    "scan forward direction": ("reverse_selective_scan", _scan_variant(direction=+1)),
    "scan drops D": ("reverse_selective_scan", _scan_variant(use_D=False)),
    "scan A sign flipped": ("reverse_selective_scan", _scan_variant(sign=-1.0)),
    "scan drops delta on input": ("reverse_selective_scan", _scan_variant(use_delta_in=False)),
    "scan swaps B and C": ("reverse_selective_scan", _scan_variant(swap_bc=True)),
    "scan drops SiLU(z) gate": ("reverse_selective_scan", _scan_variant(gate=False)),
    "in_proj x/z swapped": ("in_proj", _in_proj_swapped),
    "x_proj B/C swapped": ("x_proj", lambda u, W, r, n: (lambda t: (t[0], t[2], t[1]))(_xp(u, W, r, n))),
    "LN unbiased variance": ("layer_norm", _ln_unbiased),
    "LN drops beta": ("layer_norm", _ln_no_beta),
    "gate without tanh": ("gated_residual", _gate_linear),
    "dt drops bias": ("dt_softplus", _dt_no_bias),
    "softplus replaced by exp": ("softplus", _softplus_as_exp),
    "silu replaced by sigmoid": ("silu", _silu_as_sigmoid),
    "stack applies the hooks in reverse order": ("sidecar_stack", _stack_reversed),
    "stack pairs the gates with the wrong hooks": ("sidecar_stack", _stack_gates_rotated),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(R, attr, fn)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(R)
        except (AssertionError, ValueError, IndexError, FloatingPointError) as e:  # noqa: PERF203
            caught.append((pin.__name__, str(e)[:80]))
    assert caught, f"mutant '{name}' passed every pin"
