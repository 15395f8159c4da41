"""The fp32 reverse-scan gradient (r2l_reverse_scan_backward) against the
oracle of oracle/scan_backward.py: the chain rule through the scan of
"Bifocal Diffusion Language Models" (arXiv 2606.27732v1, §3.4 step ❷) with
its softplus(Δ) input and SiLU(z) gate.

Covered: ragged lengths that end chunks part-way and an empty sequence (with
NaN in every padding row of every input), chunk lengths 1, 7, 16 and 32,
bitwise reproducibility, the full d_inner of 4096 (64 channel blocks in the
dB | dC reduction), and the B = 8 × L = 4096 batch on sampled channels.  At
B = 8 × d_inner 4096 the library walks each sequence in one block
(scan_bwd_seq.cuh): that path is covered with ragged lengths, the power and
the general decays in one call, bf16 inputs and reproducibility.
Tolerance: max |a − b| / max |b| ≤ 1e-4 per output (fp32 against fp64).
"""
import numpy as np
import pytest
import torch

import oracle as O
from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

from . import gpu_util as G

pytestmark = pytest.mark.gpu

OUTS = ("du", "ddt_raw", "dz", "dB", "dC", "dA_log", "dD", "ddt_b")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bd.load()


def run_gpu(c, B, L, E, lengths=None, chunk=0, act=torch.float32):
    """act = torch.bfloat16: u and z are passed in bf16 (what the bf16 forward
    stores), every other array in fp32."""
    dev = "cuda"
    d = {k: v.to(dev).contiguous() for k, v in c.items()}
    if act == torch.bfloat16:
        d["u"] = d["u"].to(torch.bfloat16)
        d["z"] = d["z"].to(torch.bfloat16)
    M = B * L
    o = {k: torch.full((M, E), 7.0, device=dev) for k in ("du", "ddt_raw", "dz")}
    o["dbc"] = torch.full((M, 32), 7.0, device=dev)
    o["dA_log"] = torch.empty((E, 16), device=dev)
    o["dD"] = torch.empty(E, device=dev)
    o["ddt_b"] = torch.empty(E, device=dev)
    dims = bd.make_dims(64, E, dtype=act)
    ln = None if lengths is None else lengths.to(dev)
    n = bd.reverse_scan_backward_workspace_size(dims, B, L, chunk)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    bd.reverse_scan_backward(d["u"], d["z"], d["dt_raw"], d["bc"], d["A_log"], d["D"], d["dt_b"], d["dy"],
                             o["du"], o["dz"], o["ddt_raw"], o["dbc"], o["dA_log"], o["dD"], o["ddt_b"], dims,
                             B, L, lengths=ln, chunk_tokens=chunk, workspace=ws)
    st, flags = bd.get_device_status(ws)
    assert st == 0 and flags == 0, (st, flags)
    out = {k: v.cpu() for k, v in o.items()}
    out["dB"] = out["dbc"][:, :16]
    out["dC"] = out["dbc"][:, 16:]
    return out


def oracle(c, B, L, E, lengths, channels=None):
    """Oracle gradients; with ``channels`` only those channels (valid for the
    per-channel outputs: channels interact only through dB and dC)."""
    sel = slice(None) if channels is None else channels
    f = lambda k: S.to_f64(c[k]).reshape(B, L, -1)
    u, z, dt, dy = f("u")[:, :, sel], f("z")[:, :, sel], f("dt_raw")[:, :, sel], f("dy")[:, :, sel]
    bc = f("bc")
    return O.reverse_scan_backward_batch(u, dt, S.to_f64(c["dt_b"])[sel], S.to_f64(c["A_log"])[sel], bc[:, :, :16],
                                         bc[:, :, 16:], S.to_f64(c["D"])[sel], z, dy,
                                         None if lengths is None else lengths.tolist())


def compare(got, want, B, L, E, lengths, names=OUTS, channels=None):
    lens = [L] * B if lengths is None else lengths.tolist()
    sel = slice(None) if channels is None else channels
    for k in names:
        g = S.to_f64(got[k])
        w = want[k]
        if k in ("du", "ddt_raw", "dz", "dB", "dC"):
            g = g.reshape(B, L, -1)
            if k in ("du", "ddt_raw", "dz"):
                g = g[:, :, sel]
            for b, n in enumerate(lens):
                assert np.all(g[b, n:] == 0.0), f"{k}: padding of sequence {b} not zero"
            valid = np.concatenate([g[b, :n].ravel() for b, n in enumerate(lens)])
            ref = np.concatenate([w[b, :n].ravel() for b, n in enumerate(lens)])
        else:
            valid, ref = g[sel].ravel(), w.ravel()
        e = G.err_norm(valid, ref)
        assert e <= G.TOL_FP32, f"{k}: err {e:.3e}"


@pytest.mark.parametrize("chunk", [0, 1, 7, 32])
def test_scan_backward_ragged(chunk):
    B, L, E = 3, 70, 128
    lengths = torch.tensor([70, 33, 0], dtype=torch.int32)
    c = S.make_scan_bwd_case(B, L, E, seed=61, lengths=lengths)
    got = run_gpu(c, B, L, E, lengths, chunk)
    compare(got, oracle(c, B, L, E, lengths), B, L, E, lengths)


def test_scan_backward_reproducible():
    B, L, E = 2, 100, 192
    lengths = torch.tensor([100, 61], dtype=torch.int32)
    c = S.make_scan_bwd_case(B, L, E, seed=62, lengths=lengths)
    a = run_gpu(c, B, L, E, lengths)
    b = run_gpu(c, B, L, E, lengths)
    for k in ("du", "ddt_raw", "dz", "dbc", "dA_log", "dD", "ddt_b"):
        assert torch.equal(a[k].view(torch.int32), b[k].view(torch.int32)), k


def test_scan_backward_full_width():
    B, L, E = 2, 1024, 4096
    lengths = torch.tensor([1024, 777], dtype=torch.int32)
    c = S.make_scan_bwd_case(B, L, E, seed=63, lengths=lengths)
    got = run_gpu(c, B, L, E, lengths)
    compare(got, oracle(c, B, L, E, lengths), B, L, E, lengths)


def test_scan_backward_serving_size_sampled_channels():
    """B = 8 × L = 4096 × d_inner 4096 (the serving batch, all lengths full):
    per-channel outputs of 128 sampled channels (two blocks of 64, one at each
    end) against the oracle run on those channels alone."""
    B, L, E = 8, 4096, 4096
    c = S.make_scan_bwd_case(B, L, E, seed=64)
    got = run_gpu(c, B, L, E)
    ch = np.r_[0:64, 4032:4096]
    want = oracle(c, B, L, E, None, channels=ch)
    compare(got, want, B, L, E, None, names=("du", "ddt_raw", "dz", "dA_log", "dD", "ddt_b"), channels=ch)
    assert torch.isfinite(got["dbc"]).all()


@pytest.mark.parametrize("chunk", [0, 7])
def test_scan_backward_bf16_inputs(chunk):
    """u and z in bf16, as the bf16 forward writes them (dims dtype R2L_BF16),
    against the oracle on those same bf16 values widened exactly: the only
    differences left are the kernel's fp32 arithmetic, so the fp32 tolerance
    holds.  Ragged lengths, an empty sequence, NaN padding."""
    B, L, E = 3, 70, 128
    lengths = torch.tensor([70, 33, 0], dtype=torch.int32)
    c = S.make_scan_bwd_case(B, L, E, seed=65, lengths=lengths)
    c["u"] = c["u"].to(torch.bfloat16).float()
    c["z"] = c["z"].to(torch.bfloat16).float()
    got = run_gpu(c, B, L, E, lengths, chunk, act=torch.bfloat16)
    compare(got, oracle(c, B, L, E, lengths), B, L, E, lengths)


def walk_case(seed, mixed_A):
    """B = 8 × d_inner 4096: 1024 blocks of 32 channels, enough for the walk
    along each sequence.  Lengths end chunks part-way, one sequence is empty,
    one has a single position, one fills L = 70 (its last chunk runs past L).
    With mixed_A every other 32-channel block gets a random A, so one call
    runs blocks on the power path and blocks on the general path."""
    B, L, E = 8, 70, 4096
    lengths = torch.tensor([70, 33, 0, 1, 16, 17, 64, 50], dtype=torch.int32)
    c = S.make_scan_bwd_case(B, L, E, seed=seed, lengths=lengths)
    if mixed_A:
        g = torch.Generator().manual_seed(seed + 1)
        rnd = torch.log(torch.rand((E, 16), generator=g) * 15.0 + 0.5)
        blk = (torch.arange(E) // 32) % 2 == 1
        c["A_log"][blk] = rnd[blk]
    return c, B, L, E, lengths


@pytest.mark.parametrize("mixed_A", [False, True])
def test_scan_backward_walk_along_sequences(mixed_A):
    c, B, L, E, lengths = walk_case(67, mixed_A)
    got = run_gpu(c, B, L, E, lengths)
    compare(got, oracle(c, B, L, E, lengths), B, L, E, lengths)


def test_scan_backward_walk_bf16_inputs():
    c, B, L, E, lengths = walk_case(68, True)
    for k in ("u", "z"):
        c[k] = c[k].to(torch.bfloat16).to(torch.float32)
    got = run_gpu(c, B, L, E, lengths, act=torch.bfloat16)
    compare(got, oracle(c, B, L, E, lengths), B, L, E, lengths)


def test_scan_backward_walk_reproducible():
    c, B, L, E, lengths = walk_case(69, True)
    a = run_gpu(c, B, L, E, lengths)
    b = run_gpu(c, B, L, E, lengths)
    for k in OUTS:
        assert torch.equal(a[k].view(torch.int32), b[k].view(torch.int32)), k
