"""The sidecar stack captured in a CUDA graph gives the same bits as direct
calls (the forward path enqueues work only: no allocation, no host sync), on
the denoise-step shape of cached parallel decoding ("Bifocal Diffusion
Language Models", arXiv 2606.27732v1, §3.5): 7 hooks over the G = 128
generation positions of each request."""
import pytest
import torch

from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

from . import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bd.load()


def test_stack_in_cuda_graph_matches_direct_calls():
    case = S.make_case(5, B=4, L=128)
    dims = bd.dims_of(case.dims, case.dtype)
    wdev = G.device_weights(case)
    ws = bd.alloc_workspace(dims, case.B, case.L)

    direct = case.h.cuda()
    bd.sidecar_stack(direct, wdev, dims, case.s, None, ws)
    torch.cuda.synchronize()

    h = case.h.cuda()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):          # first call outside capture
        warm = case.h.cuda()
        bd.sidecar_stack(warm, wdev, dims, case.s, None, ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bd.sidecar_stack(h, wdev, dims, case.s, None, ws)
    h.copy_(case.h.cuda())                 # capture does not run the work
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int16), direct.view(torch.int16))
    # a second replay applies the stack again (the hidden state is updated in place)
    again = direct.clone()
    bd.sidecar_stack(again, wdev, dims, case.s, None, ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int16), again.view(torch.int16))


def test_denoise_block_against_oracle():
    """The full denoise-step shape (B=8, G=128, 7 hooks): the final h⁺ against
    the oracle's stack on requests 0 and 7; and the last hook, run through the
    debug entry point on the GPU's hidden state after six hooks, against the
    oracle's hook on that input (h⁺, pre-gate ĥ and y, requests 0 and 7)."""
    case = S.make_case(5)
    before, got, dbg = G.run_gpu_stack_last_debug(case)
    want = G.run_oracle(case, [0, 7])
    for b in (0, 7):
        e = G.err_bf16(S.to_f64(got[b]), want[b])
        assert e <= G.TOL_BF16, f"b={b}: {e:.3e}"
    G.check_sampled_rows(case, got, dbg, full=(0, 7), hook=6, h_in=before)
