"""The separate conv + SiLU kernel (batches below one 128-row tile per SM, where
x_proj runs on its own, unsplit or split along K) against the oracle of
"Bifocal Diffusion Language Models" (arXiv 2606.27732v1, §3.4 steps ❶–❷), at
four batch sizes: 9600, 3200, 600 and 128 tokens (16 tokens per conv thread at
the first two, 8 at the others).  Lengths end part-way through a thread's tokens;
u, Δr, C, y, o and ĥ are compared, in both directions,
and padding rows of h must stay untouched.  At 600 and 128 tokens out_proj
also runs split along K, its partial sums added by the LayerNorm kernel."""
import numpy as np
import pytest
import torch

import oracle as O
from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

from . import gpu_util as G

pytestmark = pytest.mark.gpu

# (B, L, lengths, sequences checked in full), all below the 18,944 rows where the
# fused conv/x_proj kernel takes over; x_proj runs unsplit at 9600 rows (75
# tiles) and split along K at 3200, 600 and 128; out_proj runs split along K
# into the LayerNorm kernel at 600 rows (3 slices) and 128 (8 slices)
CASES = {
    "b8_l1200": (8, 1200, [1200, 1199, 1, 0, 1185, 1200, 17, 1200], (1, 6)),
    "b4_l800": (4, 800, [800, 793, 9, 800], (1, 2)),
    "b2_l300": (2, 300, [300, 299], (0, 1)),
    "b1_l128": (1, 128, [121], (0,)),
}


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
@pytest.mark.parametrize("shape", sorted(CASES))
def test_conv_small_batches(shape, direction):
    B, L, lens, check = CASES[shape]
    case = S.make_case(1, B=B, L=L)
    case.lengths = torch.tensor(lens, dtype=torch.int32)
    case.h = S.poison_padding(case.h, case.lengths)
    case.weights = [S.make_weights(case.dims, torch.bfloat16, seed=263, x_proj_std=0.8, D_value=0.0,
                                   ln="seeded")]
    flags = bd.R2L_FLAG_FORWARD_SCAN if direction == "l2r" else 0
    got, dbg, _ = G.run_gpu(case, debug=True, flags=flags)

    lengths = case.lengths.numpy()
    h64 = S.to_f64(case.h)
    w64 = S.weights_f64(case.weights[0])
    src = O.flip_valid(h64, lengths) if direction == "l2r" else h64
    _, inter = O.sidecar_forward(src, w64, case.s[0], lengths, "bf16", batch_indices=check,
                                 return_intermediates=True)
    R = case.dims.dt_rank
    for b in check:
        n = lens[b]
        rows = slice(b * L, b * L + n)
        dbc = S.to_f64(dbg["dbc"][rows])
        for name, g, w in [("u", S.to_f64(dbg["u"][rows]), inter[b]["u"]),
                           ("dr", dbc[:, :R], inter[b]["dr"]),
                           ("C", dbc[:, R + 16:R + 32], inter[b]["C"]),
                           ("y", S.to_f64(dbg["y"][rows]), inter[b]["y"]),
                           ("o", S.to_f64(dbg["o"][rows]), inter[b]["o"]),
                           ("hhat", S.to_f64(dbg["hhat"][rows]), inter[b]["hhat"])]:
            if direction == "l2r":
                w = _flip_rows(w, n)
            e = G.err_norm(g, w)
            assert e <= G.TOL_BF16, f"{shape} {direction} {name} b={b} (len {n}): err {e:.3e}"
    for b, n in enumerate(lens):
        assert torch.equal(got[b, n:].view(torch.int16), case.h[b, n:].view(torch.int16)), \
            f"padding of sequence {b} was written"
