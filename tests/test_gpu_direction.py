"""The left-to-right control (R2L_FLAG_FORWARD_SCAN, the "L2R Mamba" row of
Table 4 of "Bifocal Diffusion Language Models", arXiv 2606.27732v1) against the
oracle, and the flip equivalence of §3.4 steps ❶–❸ on the GPU: the reverse
layer equals flipping each sequence, running the forward layer and flipping
back — bit for bit when neither run splits sequences into chunks."""
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


def _flip(h, lengths):
    out = h.clone()
    for b, n in enumerate(lengths):
        out[b, :n] = h[b, :n].flip(0)
    return out


def test_forward_layer_against_oracle():
    case = S.make_case(1, B=2, L=640)
    case.lengths = torch.tensor([640, 333], dtype=torch.int32)
    case.h = S.poison_padding(case.h, case.lengths)
    case.weights = [S.make_weights(case.dims, torch.bfloat16, seed=211, x_proj_std=0.8, D_value=0.0,
                                   ln="seeded")]
    got, _, _ = G.run_gpu(case, flags=bd.R2L_FLAG_FORWARD_SCAN)
    want = O.sidecar_forward(S.to_f64(case.h), S.weights_f64(case.weights[0]), case.s[0],
                             case.lengths.numpy(), "bf16", direction="l2r")
    for b, n in enumerate(case.lengths.tolist()):
        e = G.err_bf16(S.to_f64(got[b, :n]), want[b, :n])
        assert e <= G.TOL_BF16, f"b={b}: {e:.3e}"
        assert torch.isnan(got[b, n:].float()).all()


def test_forward_layer_fp32():
    case = S.make_case(0)
    case.weights = [S.make_weights(case.dims, torch.float32, seed=212, x_proj_std=0.5, D_value=0.3,
                                   ln="seeded")]
    got, _, _ = G.run_gpu(case, flags=bd.R2L_FLAG_FORWARD_SCAN)
    want = O.sidecar_forward(S.to_f64(case.h), S.weights_f64(case.weights[0]), case.s[0], None, "f32",
                             direction="l2r")
    e = G.err_fp32(S.to_f64(got[0]), want[0])
    assert e <= G.TOL_FP32, f"{e:.3e}"


def test_flip_equivalence_bitwise():
    """flip(R2L(h)) == L2R(flip(h)) on the GPU, per sequence, bit for bit
    (batch 8 keeps every sequence in one chunk, so both runs do the same
    arithmetic on the same values in the same order)."""
    B, L = 8, 256
    lengths = [256, 200, 1, 255, 17, 128, 96, 250]
    case = S.make_case(1, B=B, L=L)
    case.lengths = torch.tensor(lengths, dtype=torch.int32)
    case.h = S.poison_padding(case.h, case.lengths)
    case.weights = [S.make_weights(case.dims, torch.bfloat16, seed=213, x_proj_std=0.8, ln="seeded")]
    r2l, _, _ = G.run_gpu(case)
    flipped = S.Case(case.name, case.dims, case.dtype, B, L, _flip(case.h, lengths), case.weights, case.s,
                     lengths=case.lengths)
    l2r, _, _ = G.run_gpu(flipped, flags=bd.R2L_FLAG_FORWARD_SCAN)
    back = _flip(l2r, lengths)
    for b, n in enumerate(lengths):
        assert torch.equal(back[b, :n].view(torch.int16), r2l[b, :n].view(torch.int16)), f"sequence {b}"
