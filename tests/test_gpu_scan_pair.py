"""The scan's two-threads-per-channel kernel (used when every sequence is scanned
in one pass: batches of 8 and more at d_inner 4096) against the oracle of
"Bifocal Diffusion Language Models" (arXiv 2606.27732v1, §3.4 steps ❶–❹).

The scan is made visible (D = 0, O(1) B and C), lengths start and end tiles
part-way (1, 17, 100, 143, 159) or are empty, the padding is NaN, and both
directions and the general-A path are covered.  y, ĥ and h⁺ are compared."""
import numpy as np
import pytest
import torch

import oracle as O
from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

from . import gpu_util as G

pytestmark = pytest.mark.gpu

LENS = [160, 1, 17, 100, 159, 64, 0, 143]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bd.load()


def _case(seed, A_log=None):
    case = S.make_case(1, B=8, L=160)            # config-1 widths, 8 sequences of up to 160 tokens
    case.lengths = torch.tensor(LENS, dtype=torch.int32)
    case.h = S.poison_padding(case.h, case.lengths)
    case.weights = [S.make_weights(case.dims, torch.bfloat16, seed=seed, x_proj_std=0.8, D_value=0.0,
                                   ln="seeded", A_log=A_log)]
    return case


def _flip_rows(a, n):
    out = np.array(a, copy=True)
    out[:n] = a[:n][::-1]
    return out


def _check(case, got, dbg, direction):
    lengths = case.lengths.numpy()
    h64 = S.to_f64(case.h)
    w64 = S.weights_f64(case.weights[0])
    src = O.flip_valid(h64, lengths) if direction == "l2r" else h64
    _, inter = O.sidecar_forward(src, w64, case.s[0], lengths, "bf16", return_intermediates=True)
    want = O.sidecar_forward(h64, w64, case.s[0], lengths, "bf16", direction=direction)
    L = case.L
    for b, n in enumerate(LENS):
        if n == 0:
            assert torch.equal(got[b].view(torch.int16), case.h[b].view(torch.int16))
            continue
        for k in ("y", "hhat"):
            w = inter[b][k]
            if direction == "l2r":
                w = _flip_rows(w, n)
            e = G.err_norm(S.to_f64(dbg[k][b * L: b * L + n]), w)
            assert e <= G.TOL_BF16, f"{direction} {k} b={b} (len {n}): err {e:.3e}"
        e = G.err_bf16(S.to_f64(got[b, :n]), want[b, :n])
        assert e <= G.TOL_BF16, f"{direction} h+ b={b} (len {n}): err {e:.3e}"
        assert torch.equal(got[b, n:].view(torch.int16), case.h[b, n:].view(torch.int16)), \
            f"padding of sequence {b} was written"


@pytest.mark.parametrize("direction", ["r2l", "l2r"])
def test_pair_scan_visible_ragged(direction):
    case = _case(231)
    flags = bd.R2L_FLAG_FORWARD_SCAN if direction == "l2r" else 0
    got, dbg, _ = G.run_gpu(case, debug=True, flags=flags)
    _check(case, got, dbg, direction)


def test_pair_scan_general_A():
    g = torch.Generator().manual_seed(17)
    A_log = torch.log(torch.rand((S.BIG.d_inner, 16), generator=g) * 8 + 0.25)
    case = _case(232, A_log=A_log)
    got, dbg, _ = G.run_gpu(case, debug=True)
    _check(case, got, dbg, "r2l")


def test_pair_scan_forced_general_path():
    case = _case(233)
    got, dbg, _ = G.run_gpu(case, debug=True, flags=bd.R2L_FLAG_GENERAL_A)
    _check(case, got, dbg, "r2l")
