"""Helpers shared by the GPU parity tests: run a synthetic case through the C
ABI and through the CPU oracle, and the tolerance measures the tests use.

Tolerances (the layer's contract):
  fp32 path, output h⁺:               max_i |a_i − b_i| / max(|b_i|, 1e-3·rms(b))  ≤ 1e-4
  fp32 path, ĥ and intermediates:     max |a − b| / max |b|                         ≤ 1e-4
  bf16 path, everything:              max |a − b| / max |b|                         ≤ 2e-2
The per-element form is used only where it is well conditioned (h⁺ is
dominated by h ~ N(0, 1)); GEMM outputs and the LayerNorm output have
elements near zero by cancellation, where a per-element ratio measures
nothing but fp32 rounding of the cancelled terms.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

TOL_FP32 = 1e-4
TOL_BF16 = 2e-2


def err_fp32(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    rms = float(np.sqrt(np.mean(b * b))) if b.size else 0.0
    den = np.maximum(np.abs(b), 1e-3 * rms)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(a - b) / den)) if a.size else 0.0


def err_bf16(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if not a.size:
        return 0.0
    m = float(np.max(np.abs(b)))
    return float(np.max(np.abs(a - b))) / (m if m > 0 else 1.0)


def err_for(dtype):
    """Metric for the final output h⁺."""
    return err_fp32 if dtype == torch.float32 else err_bf16


def err_norm(a, b) -> float:
    """max |a − b| / max |b| (intermediates, ĥ)."""
    return err_bf16(a, b)


def tol_for(dtype):
    return TOL_FP32 if dtype == torch.float32 else TOL_BF16


def device_weights(case):
    return [bd.weights_to_device(w) for w in case.weights]


DEBUG_KEYS = ("x", "z", "u", "dbc", "y", "o", "hhat")


def _debug_buffers(case, keys, dev):
    M, E, d = case.B * case.L, case.dims.d_inner, case.dims.d_model
    ldd = case.dims.dt_rank + 2 * case.dims.d_state
    shapes = {"x": ((M, E), case.dtype), "z": ((M, E), case.dtype), "u": ((M, E), case.dtype),
              "y": ((M, E), case.dtype), "o": ((M, d), case.dtype), "dbc": ((M, ldd), torch.float32),
              "hhat": ((M, d), torch.float32)}
    return {k: torch.full(shapes[k][0], float("nan"), dtype=shapes[k][1], device=dev) for k in keys}


def run_gpu(case, debug=False, flags=0, s=None, keys=DEBUG_KEYS):
    """Run ``case`` through libr2l.  Returns (h⁺ on CPU, debug dict on CPU,
    device flags).  With ``debug`` (one hook) the intermediates named in
    ``keys`` are returned too."""
    dev = "cuda"
    dims = bd.dims_of(case.dims, case.dtype, flags)
    h = case.h.to(dev).contiguous()
    lengths = None if case.lengths is None else case.lengths.to(dev)
    ws = bd.alloc_workspace(dims, case.B, case.L)
    wdev = device_weights(case)
    outs = {}
    if debug:
        assert len(wdev) == 1
        outs = _debug_buffers(case, keys, dev)
        bd.sidecar_forward_debug(h, wdev[0], dims, case.s[0] if s is None else s, lengths, ws,
                                 outputs=outs)
    elif len(wdev) == 1:
        bd.sidecar_forward(h, wdev[0], dims, case.s[0] if s is None else s, lengths, ws)
    else:
        bd.sidecar_stack(h, wdev, dims, case.s, lengths, ws)
    torch.cuda.synchronize()
    st, flags_out = bd.get_device_status(ws)
    return h.cpu(), {k: v.cpu() for k, v in outs.items()}, flags_out


def run_gpu_stack_last_debug(case, keys=("y", "hhat")):
    """A multi-hook case with its last hook run through the debug entry point:
    hooks 0 … H−2 through r2l_sidecar_stack, then hook H−1 alone.  Returns
    (hidden entering the last hook, final h⁺, the last hook's intermediates),
    all on the CPU."""
    dev = "cuda"
    dims = bd.dims_of(case.dims, case.dtype)
    h = case.h.to(dev).contiguous()
    lengths = None if case.lengths is None else case.lengths.to(dev)
    ws = bd.alloc_workspace(dims, case.B, case.L)
    wdev = device_weights(case)
    bd.sidecar_stack(h, wdev[:-1], dims, case.s[:-1], lengths, ws)
    torch.cuda.synchronize()
    before = h.cpu()
    outs = _debug_buffers(case, keys, dev)
    bd.sidecar_forward_debug(h, wdev[-1], dims, case.s[-1], lengths, ws, outputs=outs)
    torch.cuda.synchronize()
    st, flags_out = bd.get_device_status(ws)
    assert flags_out == 0, flags_out
    return before, h.cpu(), {k: v.cpu() for k, v in outs.items()}


def oracle_hook_rows(h_seq, w, s, lo, n, out_dtype):
    """The oracle's intermediates and rounded h⁺ for one hook on rows [lo, n)
    of one sequence h_seq [L, d] (float64), run on that span alone: exact for
    those rows, since the output at i depends on rows ≥ i only (up to n)."""
    out, inter = O.sidecar_sequence(h_seq[lo:n], w, s, n - lo, return_intermediates=True)
    if out_dtype == "bf16":
        out = O.round_to_bf16(out)
    elif out_dtype == "f32":
        out = out.astype(np.float32).astype(np.float64)
    return out, inter


def out_dtype_name(dtype):
    return "f32" if dtype == torch.float32 else "bf16"


def run_oracle(case, batch_indices, intermediates=False, suffix=None):
    """Oracle h⁺ for the listed sequences (float64 array [B, L, d]).  With
    ``suffix`` = S, each listed sequence is run on its last S valid positions
    only (exact for those positions: the output at i depends on j ≥ i only)."""
    h = S.to_f64(case.h)
    ws = [S.weights_f64(w) for w in case.weights]
    lengths = None if case.lengths is None else case.lengths.numpy()
    od = out_dtype_name(case.dtype)
    if suffix is None:
        if len(ws) == 1:
            return O.sidecar_forward(h, ws[0], case.s[0], lengths, od, batch_indices,
                                     return_intermediates=intermediates)
        return O.sidecar_stack(h, ws, case.s, lengths, od, batch_indices)
    out = np.array(h, copy=True)
    for b in batch_indices:
        n = case.L if lengths is None else int(lengths[b])
        lo = max(0, n - suffix)
        sub = h[b:b + 1, lo:n]
        if len(ws) == 1:
            r = O.sidecar_forward(sub, ws[0], case.s[0], None, od)
        else:
            r = O.sidecar_stack(sub, ws, case.s, None, od)
        out[b, lo:n] = r[0]
    return out


def valid_rows(case, b):
    n = case.L if case.lengths is None else int(case.lengths[b])
    return n


def check_sampled_rows(case, got, dbg, full=(), suffix=None, hook=0, h_in=None, keys=("y", "hhat")):
    """Compare one hook's GPU results with the oracle on sampled rows: the
    sequences in ``full`` over all their valid rows, every other sequence over
    its last ``suffix`` valid rows (none if suffix is None).  Checked: h⁺ with
    the output metric, and each intermediate in ``keys`` (the scan output y,
    the pre-gate ĥ, …) with max|a−b|/max|b|.  ``h_in`` is the hidden state the
    hook read (default: the case's input); ``hook`` picks its weights and
    gate.  Returns the largest error seen per quantity."""
    tol = tol_for(case.dtype)
    h = S.to_f64(case.h if h_in is None else h_in)
    w = S.weights_f64(case.weights[hook])
    s = case.s[hook]
    od = out_dtype_name(case.dtype)
    L = case.L
    worst = {}
    for b in range(case.B):
        n = valid_rows(case, b)
        if b in full:
            lo = 0
        elif suffix is not None:
            lo = max(0, n - suffix)
        else:
            continue
        if n <= lo:
            continue
        want, inter = oracle_hook_rows(h[b], w, s, lo, n, od)
        e = err_for(case.dtype)(S.to_f64(got[b, lo:n]), want)
        assert e <= tol, f"{case.name} hook {hook} h+ b={b} rows [{lo},{n}): err {e:.3e}"
        worst["h+"] = max(worst.get("h+", 0.0), e)
        for k in keys:
            g = S.to_f64(dbg[k][b * L + lo: b * L + n])
            e = err_norm(g, inter[k])
            assert e <= tol, f"{case.name} hook {hook} {k} b={b} rows [{lo},{n}): err {e:.3e}"
            worst[k] = max(worst.get(k, 0.0), e)
    return worst
