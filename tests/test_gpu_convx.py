"""conv + SiLU fused into x_proj (the kernel the layer uses once a batch has at
least one 128-row tile per SM) against the oracle of "Bifocal Diffusion Language
Models" (arXiv 2606.27732v1, §3.4 steps ❶–❹): u, [Δr | B | C], y, ĥ and h⁺,
on sequences whose lengths end tiles part-way, in both directions."""
import numpy as np
import pytest
import torch

import oracle as O
from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

from . import gpu_util as G

pytestmark = pytest.mark.gpu

L = 2400                                    # B·L = 19,200 rows: at least one 128-row tile per SM
LENS = [2400, 2399, 1, 17, 2000, 100, 0, 1537]
CHECK = (1, 2, 3, 7)                        # sequences compared against the oracle in full


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bd.load()


def _flip_rows(a, n):
    out = np.array(a, copy=True)
    out[:n] = a[:n][::-1]
    return out


@pytest.mark.parametrize("direction", ["r2l", "l2r"])
def test_fused_conv_x_proj(direction):
    case = S.make_case(1, B=8, L=L)
    case.lengths = torch.tensor(LENS, dtype=torch.int32)
    case.h = S.poison_padding(case.h, case.lengths)
    case.weights = [S.make_weights(case.dims, torch.bfloat16, seed=241, x_proj_std=0.8, D_value=0.0,
                                   ln="seeded")]
    flags = bd.R2L_FLAG_FORWARD_SCAN if direction == "l2r" else 0
    got, dbg, _ = G.run_gpu(case, debug=True, flags=flags)

    lengths = case.lengths.numpy()
    h64 = S.to_f64(case.h)
    w64 = S.weights_f64(case.weights[0])
    src = O.flip_valid(h64, lengths) if direction == "l2r" else h64
    _, inter = O.sidecar_forward(src, w64, case.s[0], lengths, "bf16", batch_indices=CHECK,
                                 return_intermediates=True)
    want = O.sidecar_forward(h64, w64, case.s[0], lengths, "bf16", batch_indices=CHECK, direction=direction)
    R = case.dims.dt_rank
    for b in CHECK:
        n = LENS[b]
        rows = slice(b * L, b * L + n)
        dbc = S.to_f64(dbg["dbc"][rows])
        pairs = [("u", S.to_f64(dbg["u"][rows]), inter[b]["u"]),
                 ("dr", dbc[:, :R], inter[b]["dr"]),
                 ("B", dbc[:, R:R + 16], inter[b]["B"]),
                 ("C", dbc[:, R + 16:R + 32], inter[b]["C"]),
                 ("y", S.to_f64(dbg["y"][rows]), inter[b]["y"]),
                 ("hhat", S.to_f64(dbg["hhat"][rows]), inter[b]["hhat"])]
        for name, g, w in pairs:
            if direction == "l2r":
                w = _flip_rows(w, n)
            e = G.err_norm(g, w)
            assert e <= G.TOL_BF16, f"{direction} {name} b={b} (len {n}): err {e:.3e}"
        e = G.err_bf16(S.to_f64(got[b, :n]), want[b, :n])
        assert e <= G.TOL_BF16, f"{direction} h+ b={b} (len {n}): err {e:.3e}"
    for b, n in enumerate(LENS):
        assert torch.equal(got[b, n:].view(torch.int16), case.h[b, n:].view(torch.int16)), \
            f"padding of sequence {b} was written"
