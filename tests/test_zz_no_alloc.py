"""r2l_reverse_scan_noalloc against r2l_reverse_scan.

The allocation-free entry point serves callers that may not allocate device
memory while they run (a runtime that reserves all device memory at start-up,
a plug-in whose host owns the allocator); its scratch is a fixed array inside
the library.  It must give the same results as the workspace entry point, on
consecutive calls that share that array.  This file is named so that pytest
collects it last."""
import numpy as np
import pytest
import torch

from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import synthetic as S

from . import gpu_util as G
from .test_gpu_scan import make_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bd.load()


def _dev(inp):
    return {k: v.to("cuda").contiguous() for k, v in inp.items()}


def _with_workspace(d, dims, B, L, lens, T):
    y = torch.full((B * L, d["u"].shape[1]), float("nan"), dtype=d["u"].dtype, device="cuda")
    bd.reverse_scan(d["u"], d["z"], d["dt_raw"], d["bc"], d["A_log"], d["D"], d["dt_b"], y, dims, B, L, lens, T)
    return y


def _no_alloc(d, dims, B, L, lens, T):
    y = torch.full((B * L, d["u"].shape[1]), float("nan"), dtype=d["u"].dtype, device="cuda")
    bd.reverse_scan_noalloc(d["u"], d["z"], d["dt_raw"], d["bc"], d["A_log"], d["D"], d["dt_b"], y, dims, B, L,
                            lens, T)
    return y


def _compare(a, b, B, L, lens):
    a, b = a.cpu(), b.cpu()
    for s in range(B):
        n = L if lens is None else int(lens[s])
        e = G.err_norm(S.to_f64(a[s * L: s * L + n]), S.to_f64(b[s * L: s * L + n]))
        assert e <= 5e-3, f"sequence {s}: {e:.3e}"
        assert torch.isnan(a[s * L + n: (s + 1) * L].float()).all()


def test_no_alloc_matches_workspace_entry_on_two_calls():
    # two different problems back to back through the shared static scratch;
    # both split sequences into several chunks, so the carry scratch is used
    cases = [(3, 300, 256, [300, 7, 161], 48, 61, True),
             (2, 517, 384, [400, 517], 64, 62, False)]
    for B, L, E, lens, T, seed, structured in cases:
        dims = bd.make_dims(64, E, dt_rank=8, dtype=torch.bfloat16)
        assert 0 < bd.reverse_scan_workspace_size(dims, B, L, T) <= bd.NOALLOC_SCRATCH_BYTES
        d = _dev(make_scan_inputs(B, L, E, seed=seed, structured_A=structured))
        lt = torch.tensor(lens, dtype=torch.int32, device="cuda")
        ref = _with_workspace(d, dims, B, L, lt, T)
        got = _no_alloc(d, dims, B, L, lt, T)
        torch.cuda.synchronize()
        _compare(got, ref, B, L, lens)


def test_no_alloc_rejects_requests_beyond_capacity():
    # 64 sequences x 4096 channels x 64 chunks of carries is far beyond 16 MiB
    B, L, E = 64, 1024, 4096
    dims = bd.make_dims(2048, E, dtype=torch.bfloat16)
    assert bd.reverse_scan_workspace_size(dims, B, L, 16) > bd.NOALLOC_SCRATCH_BYTES
    t = torch.empty((16,), dtype=torch.bfloat16, device="cuda")
    f = torch.empty((16,), dtype=torch.float32, device="cuda")
    st = bd.reverse_scan_noalloc(t, t.view(1, 16), t, f.view(1, 16), f, f, f, t, dims, B, L, None, 16, check=False)
    assert st == 4   # R2L_ERR_WORKSPACE, nothing enqueued
