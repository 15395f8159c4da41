"""The reverse selective scan on its own (r2l_reverse_scan) against the
oracle's scan, on O(1)-scale inputs where every term of the recurrence is
visible: several chunk lengths (one chunk, chunks splitting the sequence
mid-tile, chunks of one pipeline stage), ragged lengths including 0 and 1, a
partial 128-channel block, the A = -(1..16) power path and random A.
"Bifocal Diffusion Language Models" (arXiv 2606.27732v1), §3.4 step ❷."""
import numpy as np
import pytest
import torch

import oracle as O
from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

from . import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bd.load()


def make_scan_inputs(B, L, E, seed, structured_A=True, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    M = B * L
    u = torch.randn((M, E), generator=g).to(dtype)
    z = torch.randn((M, 2 * E), generator=g).to(dtype)           # z in the first E columns
    dt_raw = (torch.randn((M, E), generator=g) * 0.5).to(dtype)
    bc = torch.randn((M, 40), generator=g, dtype=torch.float32)  # B | C | 8 unused columns
    if structured_A:
        A_log = torch.log(torch.arange(1, 17, dtype=torch.float32)).repeat(E, 1).contiguous()
    else:
        A_log = torch.log(torch.rand((E, 16), generator=g) * 6 + 0.2)
    D = torch.randn((E,), generator=g)
    dt_b = torch.log(torch.expm1(torch.rand((E,), generator=g) * 0.3 + 0.01))   # Δ ≈ 0.01..0.3
    return dict(u=u, z=z, dt_raw=dt_raw, bc=bc, A_log=A_log.contiguous(), D=D, dt_b=dt_b.float())


def oracle_scan(inp, B, L, E, lengths):
    f = S.to_f64
    u, z, dt_raw, bc = f(inp["u"]), f(inp["z"])[:, :E], f(inp["dt_raw"]), f(inp["bc"])
    A = -np.exp(f(inp["A_log"]))
    delta_all = O.softplus(dt_raw + f(inp["dt_b"]))
    out = np.full((B * L, E), np.nan)
    for b in range(B):
        n = L if lengths is None else int(lengths[b])
        if n == 0:
            continue
        r = slice(b * L, b * L + n)
        out[r] = O.reverse_selective_scan(u[r], delta_all[r], A, bc[r, :16], bc[r, 16:32], f(inp["D"]), z[r])
    return out


def run_scan(inp, B, L, E, lengths, chunk_tokens, dtype=torch.bfloat16, flags=0):
    dev = "cuda"
    d = {k: v.to(dev).contiguous() for k, v in inp.items()}
    y = torch.full((B * L, E), float("nan"), dtype=dtype, device=dev)
    dims = bd.make_dims(64, E, dt_rank=8, dtype=dtype, flags=flags)
    lens = None if lengths is None else torch.tensor(lengths, dtype=torch.int32, device=dev)
    bd.reverse_scan(d["u"], d["z"], d["dt_raw"], d["bc"], d["A_log"], d["D"], d["dt_b"], y, dims, B, L,
                    lens, chunk_tokens)
    torch.cuda.synchronize()
    return y.cpu()


def check(got, want, B, L, lengths, tol):
    for b in range(B):
        n = L if lengths is None else int(lengths[b])
        g = S.to_f64(got[b * L: b * L + n])
        w = want[b * L: b * L + n]
        e = G.err_norm(g, w)
        assert e <= tol, f"sequence {b} (len {n}): err {e:.3e}"
        if n < L:
            assert torch.isnan(got[b * L + n: (b + 1) * L].float()).all(), f"padding of sequence {b} written"


@pytest.mark.parametrize("chunk_tokens", [0, 16, 48, 96, 100000])
@pytest.mark.parametrize("structured", [True, False])
def test_scan_bf16_chunks(chunk_tokens, structured):
    B, L, E = 3, 301, 384
    lengths = [301, 1, 170]
    inp = make_scan_inputs(B, L, E, seed=11 + structured, structured_A=structured)
    got = run_scan(inp, B, L, E, lengths, chunk_tokens)
    want = oracle_scan(inp, B, L, E, lengths)
    check(got, want, B, L, lengths, 5e-3)


def test_scan_bf16_partial_channel_block_and_empty():
    B, L, E = 4, 130, 200            # 200 = full 128- or 64-channel blocks + a partial one
    lengths = [0, 130, 64, 17]
    inp = make_scan_inputs(B, L, E, seed=21)
    want = oracle_scan(inp, B, L, E, lengths)
    for T in (0, 32):
        got = run_scan(inp, B, L, E, lengths, T)
        check(got, want, B, L, lengths, 5e-3)


def test_scan_bf16_forced_general_path():
    B, L, E = 2, 257, 256
    inp = make_scan_inputs(B, L, E, seed=31, structured_A=True)
    want = oracle_scan(inp, B, L, E, None)
    a = run_scan(inp, B, L, E, None, 64)
    b = run_scan(inp, B, L, E, None, 64, flags=bd.R2L_FLAG_GENERAL_A)
    check(a, want, B, L, None, 5e-3)
    check(b, want, B, L, None, 5e-3)


def test_scan_fp32():
    B, L, E = 2, 77, 136
    lengths = [77, 40]
    inp = make_scan_inputs(B, L, E, seed=41, structured_A=False, dtype=torch.float32)
    got = run_scan(inp, B, L, E, lengths, 0, dtype=torch.float32)
    want = oracle_scan(inp, B, L, E, lengths)
    check(got, want, B, L, lengths, 1e-5)


def test_scan_long_sequence_many_chunks():
    """One sequence of 4096 tokens over the full 4096 channels, automatic
    chunking (splits the sequence) against one chunk."""
    B, L, E = 1, 4096, 4096
    inp = make_scan_inputs(B, L, E, seed=51)
    want = oracle_scan(inp, B, L, E, None)
    auto = run_scan(inp, B, L, E, None, 0)
    whole = run_scan(inp, B, L, E, None, 1 << 20)
    check(auto, want, B, L, None, 5e-3)
    check(whole, want, B, L, None, 5e-3)


def oracle_scan_forward(inp, B, L, E, lengths):
    """The left-to-right scan through the reverse oracle on flipped data."""
    f = S.to_f64
    u, z, dt_raw, bc = f(inp["u"]), f(inp["z"])[:, :E], f(inp["dt_raw"]), f(inp["bc"])
    A = -np.exp(f(inp["A_log"]))
    delta_all = O.softplus(dt_raw + f(inp["dt_b"]))
    out = np.full((B * L, E), np.nan)
    for b in range(B):
        n = L if lengths is None else int(lengths[b])
        if n == 0:
            continue
        r = slice(b * L, b * L + n)
        fl = lambda a: a[r][::-1]
        yf = O.reverse_selective_scan(fl(u), fl(delta_all), A, fl(bc[:, :16]), fl(bc[:, 16:32]), f(inp["D"]), fl(z))
        out[r] = yf[::-1]
    return out


@pytest.mark.parametrize("chunk_tokens", [0, 48, 100000])
@pytest.mark.parametrize("structured", [True, False])
def test_scan_forward_direction(chunk_tokens, structured):
    """R2L_FLAG_FORWARD_SCAN: the left-to-right scan (Table 4's control)."""
    B, L, E = 3, 301, 384
    lengths = [301, 1, 170]
    inp = make_scan_inputs(B, L, E, seed=71 + structured, structured_A=structured)
    got = run_scan(inp, B, L, E, lengths, chunk_tokens, flags=bd.R2L_FLAG_FORWARD_SCAN)
    want = oracle_scan_forward(inp, B, L, E, lengths)
    check(got, want, B, L, lengths, 5e-3)


def test_scan_forward_fp32():
    B, L, E = 2, 77, 136
    lengths = [77, 40]
    inp = make_scan_inputs(B, L, E, seed=81, structured_A=False, dtype=torch.float32)
    got = run_scan(inp, B, L, E, lengths, 0, dtype=torch.float32, flags=bd.R2L_FLAG_FORWARD_SCAN)
    want = oracle_scan_forward(inp, B, L, E, lengths)
    check(got, want, B, L, lengths, 1e-5)
