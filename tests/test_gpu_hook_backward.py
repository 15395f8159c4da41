"""The gradient of one whole hook (r2l_sidecar_backward) against the oracle of
oracle/sidecar_backward.py: the chain rule through §3.4 steps ❶–❹ of "Bifocal
Diffusion Language Models" (arXiv 2606.27732v1), the step that training the
sidecar alone (R2LM-PI, §3.4 and §4.1) back-propagates through.

Every output is checked: dh (and, bit for bit, that padding rows pass dh⁺
through), ds, and the gradient of every parameter.  Widths are those of
workload 1 (d_model 2048, d_inner 4096, dt_rank 128).  Tolerance: the bf16
path's max |a − b| / max |b| ≤ 2e-2, per output; the GPU's forward
intermediates are stored in bf16 and the gradients that feed a GEMM are
rounded once to bf16, where the oracle keeps float64 throughout.
"""
import numpy as np
import pytest
import torch

import oracle as O
from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

from . import gpu_util as G

pytestmark = pytest.mark.gpu

TOL = 2e-2
PARAMS = ("W_in", "conv_w", "conv_b", "W_x", "W_dt", "b_dt", "A_log", "D", "W_out", "ln_w", "ln_b")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bd.load()


def make(B, L, seed, lengths=None, ln="seeded", x_proj_std=0.8, D_value=0.5, dims=S.BIG):
    h = S.make_hidden(B, L, dims.d_model, torch.bfloat16, seed=seed)
    if lengths is not None:
        h = S.poison_padding(h, lengths)
    w = S.make_weights(dims, torch.bfloat16, seed=seed + 1000, x_proj_std=x_proj_std, D_value=D_value, ln=ln)
    g = torch.Generator().manual_seed(seed + 2000)
    dh_out = torch.randn((B, L, dims.d_model), generator=g, dtype=torch.float32)
    return dims, h, w, dh_out


def run_gpu(dims, h, w, s, dh_out, lengths=None):
    dev = "cuda"
    B, L = h.shape[0], h.shape[1]
    bdims = bd.dims_of(dims, torch.bfloat16)
    wdev = bd.weights_to_device(w, dev)
    grads = bd.alloc_grads(wdev, dev)
    for v in grads.values():
        if v is not None:
            v.fill_(float("nan"))                # every gradient must be written
    ws = torch.empty(bd.sidecar_backward_workspace_size(bdims, B, L), dtype=torch.uint8, device=dev)
    ln = None if lengths is None else lengths.to(dev)
    dh, ds = bd.sidecar_backward(h.to(dev), wdev, bdims, s, dh_out.to(dev), grads, ln, workspace=ws)
    torch.cuda.synchronize()
    st, flags = bd.get_device_status(ws)
    assert st == 0 and flags == 0, (st, flags)
    return dh.cpu(), float(ds.cpu()[0]), {k: None if v is None else v.cpu() for k, v in grads.items()}


def run_oracle(h, w, s, dh_out, lengths=None):
    return O.sidecar_backward_batch(S.to_f64(h), S.weights_f64(w), s, S.to_f64(dh_out),
                                    None if lengths is None else lengths.tolist())


def hhat_pair(dims, h, w, s, lengths):
    """ĥ (the pre-gate output) of the GPU forward and of the oracle, valid rows
    only, float64 [rows, d] each."""
    case = S.Case("backward", dims, torch.bfloat16, h.shape[0], h.shape[1], h, [w], [s], lengths=lengths)
    _, dbg, _ = G.run_gpu(case, debug=True, keys=("hhat",))
    lens = [case.L] * case.B if lengths is None else lengths.tolist()
    got = np.concatenate([S.to_f64(dbg["hhat"][b * case.L: b * case.L + n]) for b, n in enumerate(lens)])
    _, inter = O.sidecar_forward(S.to_f64(h), S.weights_f64(w), s, None if lengths is None else lengths.numpy(),
                                 batch_indices=range(case.B), return_intermediates=True)
    want = np.concatenate([inter[b]["hhat"] for b, n in enumerate(lens) if n > 0])
    return got, want


def check_ds(ds, ds_ref, s, dh_out, lengths, hh_gpu, hh_ref):
    """ds = (1 − tanh²(s))·Σ dh⁺ ⊙ ĥ is a dot product of many terms of both
    signs, so a relative error measures cancellation, not accuracy.  Checked
    instead: (a) the reduction, against the same sum taken over the GPU
    forward's own ĥ, within fp32 rounding of the sum of |terms|; (b) the
    oracle's ds, within the bound the forward's measured error in ĥ implies,
    |Σ dh⁺ ⊙ (ĥ_gpu − ĥ_ref)| ≤ Σ |dh⁺| · max |ĥ_gpu − ĥ_ref|."""
    L = dh_out.shape[1]
    lens = [L] * dh_out.shape[0] if lengths is None else lengths.tolist()
    g = np.concatenate([S.to_f64(dh_out[b, :n]) for b, n in enumerate(lens)])
    gate = 1.0 - np.tanh(np.float64(s)) ** 2
    own = gate * np.sum(g * hh_gpu)
    assert abs(ds - own) <= 1e-4 * gate * np.sum(np.abs(g * hh_gpu)) + 1e-30, (ds, own)
    bound = gate * np.sum(np.abs(g)) * np.max(np.abs(hh_gpu - hh_ref))
    assert abs(ds - ds_ref) <= bound + 1e-4 * abs(ds_ref), (ds, ds_ref, bound)


def compare(got, want, h, dh_out, lengths, tol=TOL, ds_check=None):
    dh, ds, grads = got
    B, L = h.shape[0], h.shape[1]
    lens = [L] * B if lengths is None else lengths.tolist()
    errs = {}
    valid = np.concatenate([S.to_f64(dh[b, :n]).ravel() for b, n in enumerate(lens)])
    ref = np.concatenate([want["dh"][b, :n].ravel() for b, n in enumerate(lens)])
    errs["dh"] = G.err_norm(valid, ref)
    for b, n in enumerate(lens):              # padding rows: dh⁺ passed through, bit for bit
        assert torch.equal(dh[b, n:].view(torch.int32), dh_out[b, n:].view(torch.int32)), f"padding of {b}"
    if ds_check is not None:
        check_ds(ds, want["ds"], *ds_check)
    for k in PARAMS:
        wk = want.get("d" + k)
        if wk is None:
            assert grads.get(k) is None
            continue
        gk = grads[k]
        assert torch.isfinite(gk).all(), f"d{k} not written"
        errs["d" + k] = G.err_norm(S.to_f64(gk), wk)
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"errors above {tol}: {bad} (all: {errs})"
    return errs


def test_hook_backward_ragged_against_oracle():
    """B = 2 × L = 160, one sequence ragged (97), NaN padding, seeded LayerNorm,
    a visible scan (x_proj std 0.8), s = 0.7."""
    lengths = torch.tensor([160, 97], dtype=torch.int32)
    dims, h, w, dh_out = make(2, 160, seed=81, lengths=lengths)
    got = run_gpu(dims, h, w, 0.7, dh_out, lengths)
    hh = hhat_pair(dims, h, w, 0.7, lengths)
    compare(got, run_oracle(h, w, 0.7, dh_out, lengths), h, dh_out, lengths,
            ds_check=(0.7, dh_out, lengths) + hh)


def test_hook_backward_odd_sizes():
    """d_inner 192 (the conv gradient's 128-channel tiles end part-way), d_model
    136, dt_rank 8, and B·L = 2 × 75 positions (not a multiple of 8: the
    transposed operands carry zero columns past the last position), ragged."""
    dims = S.Dims(d_model=136, d_inner=192, d_state=16, dt_rank=8, d_conv=4)
    lengths = torch.tensor([75, 38], dtype=torch.int32)
    _, h, w, dh_out = make(2, 75, seed=86, lengths=lengths, dims=dims)
    got = run_gpu(dims, h, w, 0.9, dh_out, lengths)
    hh = hhat_pair(dims, h, w, 0.9, lengths)
    compare(got, run_oracle(h, w, 0.9, dh_out, lengths), h, dh_out, lengths,
            ds_check=(0.9, dh_out, lengths) + hh)


def test_hook_backward_batch_of_eight():
    """B = 8 × L = 96 at workload-1 widths: at batch 8 the scan gradient walks
    each sequence in one block, from the H checkpoints that the recomputed
    forward scan stores every 16 positions.  Ragged lengths end checkpoint
    chunks part-way; one sequence has a single position."""
    lengths = torch.tensor([96, 17, 64, 1, 80, 33, 96, 48], dtype=torch.int32)
    dims, h, w, dh_out = make(8, 96, seed=87, lengths=lengths)
    got = run_gpu(dims, h, w, 0.6, dh_out, lengths)
    hh = hhat_pair(dims, h, w, 0.6, lengths)
    compare(got, run_oracle(h, w, 0.6, dh_out, lengths), h, dh_out, lengths,
            ds_check=(0.6, dh_out, lengths) + hh)


def test_hook_backward_without_layernorm():
    """No LayerNorm (ĥ = o), s = −1.2, one sequence of 128."""
    dims, h, w, dh_out = make(1, 128, seed=82, ln="none")
    got = run_gpu(dims, h, w, -1.2, dh_out)
    hh = hhat_pair(dims, h, w, -1.2, None)
    compare(got, run_oracle(h, w, -1.2, dh_out), h, dh_out, None, ds_check=(-1.2, dh_out, None) + hh)


def test_hook_backward_workload_1():
    """Workload 1 as it stands (B = 1, L = 2048, the configs' N(0, 0.02)
    weights and D = 1, s = 1.0)."""
    case = S.make_case(1)
    g = torch.Generator().manual_seed(83)
    dh_out = torch.randn(case.h.shape, generator=g, dtype=torch.float32)
    got = run_gpu(case.dims, case.h, case.weights[0], case.s[0], dh_out)
    hh = hhat_pair(case.dims, case.h, case.weights[0], case.s[0], None)
    compare(got, run_oracle(case.h, case.weights[0], case.s[0], dh_out), case.h, dh_out, None,
            ds_check=(case.s[0], dh_out, None) + hh)


def test_hook_backward_reproducible():
    lengths = torch.tensor([96, 45], dtype=torch.int32)
    dims, h, w, dh_out = make(2, 96, seed=84, lengths=lengths)
    a = run_gpu(dims, h, w, 0.4, dh_out, lengths)
    b = run_gpu(dims, h, w, 0.4, dh_out, lengths)
    assert torch.equal(a[0].view(torch.int32), b[0].view(torch.int32))
    assert a[1] == b[1]
    for k in PARAMS:
        assert torch.equal(a[2][k].view(torch.int32), b[2][k].view(torch.int32)), k


def test_hook_backward_zero_gate():
    """s = 0: the hook is the identity, so dh = dh⁺ bit for bit and every
    parameter's gradient is zero; only ds = Σ dh⁺ ⊙ ĥ is not."""
    dims, h, w, dh_out = make(1, 64, seed=85)
    dh, ds, grads = run_gpu(dims, h, w, 0.0, dh_out)
    assert torch.equal(dh.view(torch.int32), dh_out.view(torch.int32))
    for k in PARAMS:
        assert torch.count_nonzero(grads[k]) == 0, k
    want = run_oracle(h, w, 0.0, dh_out)
    check_ds(ds, want["ds"], 0.0, dh_out, None, *hhat_pair(dims, h, w, 0.0, None))


@pytest.mark.parametrize("B,L,lens,seed", [(8, 96, [96, 17, 64, 1, 80, 33, 96, 48], 88), (2, 160, [160, 97], 89)])
def test_saved_forward_matches_recompute(B, L, lens, seed):
    """r2l_sidecar_forward_train followed by r2l_sidecar_backward with
    R2L_FLAG_SAVED_FORWARD gives, bit for bit, what r2l_sidecar_backward alone
    gives (it recomputes the same forward); the training forward's output is
    r2l_sidecar_forward's, and the input is left untouched.  B = 8: the walk
    along each sequence, from the training forward's checkpoints where the
    length is a multiple of 16; B = 2: the chunked scan gradient."""
    dev = "cuda"
    lengths = torch.tensor(lens, dtype=torch.int32)
    dims, h, w, dh_out = make(B, L, seed=seed, lengths=lengths)
    bdims = bd.dims_of(dims, torch.bfloat16)
    wdev = bd.weights_to_device(w, dev)
    hd, ln, gd = h.to(dev), lengths.to(dev), dh_out.to(dev)
    h_before = hd.clone()
    g1 = bd.alloc_grads(wdev, dev)
    dh1, ds1 = bd.sidecar_backward(hd, wdev, bdims, 0.6, gd, g1, ln)
    out, ws = bd.sidecar_forward_train(hd, wdev, bdims, 0.6, ln)
    g2 = bd.alloc_grads(wdev, dev)
    for v in g2.values():
        if v is not None:
            v.fill_(float("nan"))
    sdims = bd.dims_of(dims, torch.bfloat16, bd.R2L_FLAG_SAVED_FORWARD)
    dh2, ds2 = bd.sidecar_backward(hd, wdev, sdims, 0.6, gd, g2, ln, workspace=ws)
    torch.cuda.synchronize()
    st, flags = bd.get_device_status(ws)
    assert st == 0 and flags == 0, (st, flags)
    assert torch.equal(hd.view(torch.int16), h_before.view(torch.int16)), "input written"
    assert torch.equal(dh1.view(torch.int32), dh2.view(torch.int32))
    assert torch.equal(ds1.view(torch.int32), ds2.view(torch.int32))
    for k in PARAMS:
        assert torch.equal(g1[k].view(torch.int32), g2[k].view(torch.int32)), k
    h_fwd = hd.clone()
    bd.sidecar_forward(h_fwd, wdev, bdims, 0.6, ln)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), h_fwd.view(torch.int16))
