"""The C ABI on the CPU: the library loads, exports every function the header
declares, and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest
import torch

from reverse_selective_ssm_b200 import binding as bd
from reverse_selective_ssm_b200 import build as bld

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    bld.build()
    return bd.load()


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"R2L_API\s+[\w\s\*]*?\b(r2l_\w+)\s*\(", src))
    return sorted(names)


def test_exports_every_declared_function(lib):
    names = header_functions()
    assert names, "no R2L_API declarations found"
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(bd.EXPORTS) <= set(names)


def test_abi_version_and_status_strings(lib):
    assert lib.r2l_abi_version() == 1
    for code, name in bd.STATUS.items():
        assert lib.r2l_status_string(code).decode().startswith(name)
    assert lib.r2l_status_string(99).decode() == "R2L_ERR_UNKNOWN"


def test_workspace_size(lib):
    d = bd.make_dims(2048, 4096)
    a = bd.workspace_size(d, 8, 4096)
    assert a > 8 * 4096 * 4096 * 2 * 4          # xz, u, y at least
    # dt_rank 128 runs dt_proj inside the scan: no [M, d_inner] dt_raw region
    assert a < 8 * 4096 * 4096 * 2 * 5
    # dt_rank 64 (dt_proj as its own GEMM) adds the dt_raw region back; its Δr|B|C rows are 384 B shorter
    assert bd.workspace_size(bd.make_dims(2048, 4096, dt_rank=64), 8, 4096) >= a + 8 * 4096 * (4096 * 2 - 384)
    assert bd.workspace_size(d, 8, 4096) == a     # deterministic
    assert bd.workspace_size(d, 16, 4096) > a
    assert bd.workspace_size(d, 0, 4096) == 0
    assert bd.workspace_size(d, 1, -1) == 0
    assert bd.workspace_size(bd.make_dims(0, 4096), 1, 1) == 0
    f = bd.make_dims(64, 128, dt_rank=4, dtype=torch.float32)
    assert bd.workspace_size(f, 1, 64) > 64 * 128 * 4 * 5


FAKE = 0x10000  # a 16-byte aligned non-null value; never dereferenced on the host


def _weights(ln=True):
    w = bd.Weights()
    for f, _ in bd.Weights._fields_:
        setattr(w, f, FAKE)
    if not ln:
        w.ln_w = None
        w.ln_b = None
    return w


def _call(lib, hidden=FAKE, w=None, dims=None, s=0.5, B=1, L=8, lengths=None, ws=FAKE, ws_bytes=None):
    dims = dims or bd.make_dims(64, 128, dt_rank=4, dtype=torch.float32)
    w = w or _weights()
    if ws_bytes is None:
        ws_bytes = bd.workspace_size(dims, max(B, 1), max(L, 1)) or 1
    return lib.r2l_sidecar_forward(hidden, ctypes.byref(w), ctypes.byref(dims), s, B, L, lengths, ws,
                                   ws_bytes, None)


def test_host_validation(lib):
    assert _call(lib, hidden=None) == 1
    assert _call(lib, B=0) == 1
    assert _call(lib, L=0) == 1
    d = bd.make_dims(64, 128, d_state=8, dt_rank=4, dtype=torch.float32)
    assert _call(lib, dims=d) == 2
    d = bd.make_dims(64, 128, d_conv=3, dt_rank=4, dtype=torch.float32)
    assert _call(lib, dims=d) == 2
    d = bd.make_dims(64, 128, dt_rank=4, dtype=torch.float32)
    d.dtype = 7
    assert _call(lib, dims=d) == 1
    assert _call(lib, hidden=FAKE + 4) == 3
    assert _call(lib, ws=FAKE + 8) == 3
    assert _call(lib, ws=None) == 4
    assert _call(lib, ws_bytes=16) == 4
    w = _weights()
    w.A_log = None
    assert _call(lib, w=w) == 1
    w = _weights()
    w.ln_b = None            # only one of the two LN pointers
    assert _call(lib, w=w) == 1
    w = _weights()
    w.x_proj_w = FAKE + 2
    assert _call(lib, w=w) == 3
    assert _call(lib, lengths=FAKE + 1) == 3


def test_zero_gate_enqueues_nothing(lib):
    """tanh(s) == 0 returns R2L_OK before any CUDA call (works with no GPU):
    the identity at initialisation of §3.4 step ❹."""
    assert _call(lib, s=0.0) == 0
    assert _call(lib, s=-0.0) == 0
    w = _weights()
    arr = (bd.Weights * 3)(w, w, w)
    s = (ctypes.c_float * 3)(0.0, 0.0, 0.0)
    dims = bd.make_dims(64, 128, dt_rank=4, dtype=torch.float32)
    n = bd.workspace_size(dims, 1, 8)
    assert lib.r2l_sidecar_stack(FAKE, arr, s, 3, ctypes.byref(dims), 1, 8, None, FAKE, n, None) == 0


def test_stack_and_debug_argument_checks(lib):
    dims = bd.make_dims(64, 128, dt_rank=4, dtype=torch.float32)
    n = bd.workspace_size(dims, 1, 8)
    w = _weights()
    s = (ctypes.c_float * 1)(0.5)
    assert lib.r2l_sidecar_stack(FAKE, None, s, 1, ctypes.byref(dims), 1, 8, None, FAKE, n, None) == 1
    assert lib.r2l_sidecar_stack(FAKE, ctypes.byref(w), s, 0, ctypes.byref(dims), 1, 8, None, FAKE, n, None) == 1
    assert lib.r2l_sidecar_forward_debug(FAKE, ctypes.byref(w), ctypes.byref(dims), 0.5, 1, 8, None, FAKE,
                                         n, None, None) == 1
    st = lib.r2l_get_device_status(None, None, None)
    assert st == 1


def _bwd(lib, dims=None, B=2, L=40, ldz=128, ldbc=32, lengths=None, ws=FAKE, ws_bytes=None, chunk=0, bad=None):
    dims = dims or bd.make_dims(64, 128, dtype=torch.float32)
    if ws_bytes is None:
        ws_bytes = bd.reverse_scan_backward_workspace_size(dims, B, L, chunk) or 1
    p = [FAKE] * 19
    if bad is not None:
        p[bad[0]] = bad[1]
    return lib.r2l_reverse_scan_backward(p[0], p[1], ldz, p[2], p[3], ldbc, p[4], p[5], p[6], p[7], p[8], p[9],
                                         128, p[10], p[11], 32, p[12], p[13], p[14], ctypes.byref(dims), B, L,
                                         lengths, chunk, ws, ws_bytes, None)


def test_scan_backward_argument_checks(lib):
    """r2l_reverse_scan_backward rejects bad arguments on the host (no GPU
    needed): null pointers, unsupported dtype / direction / widths,
    misalignment and a short workspace."""
    f32 = bd.make_dims(64, 128, dtype=torch.float32)
    n = bd.reverse_scan_backward_workspace_size(f32, 2, 40, 0)
    assert n >= 3 * (2 * 3 * 128 * 16 * 4)              # three [B][chunks][E][16] fp32 arrays (T = 16: 3 chunks)
    assert bd.reverse_scan_backward_workspace_size(f32, 2, 40, 8) > n   # shorter chunks, more carries
    assert bd.reverse_scan_backward_workspace_size(bd.make_dims(64, 128), 2, 40, 0) == n      # bf16 u, z: same scratch
    assert bd.reverse_scan_backward_workspace_size(bd.make_dims(64, 96, dtype=torch.float32), 2, 40, 0) == 0
    assert _bwd(lib, bad=(0, None)) == 1
    assert _bwd(lib, bad=(14, None)) == 1
    assert _bwd(lib, B=0) == 1
    assert _bwd(lib, chunk=-1) == 1
    assert _bwd(lib, dims=bd.make_dims(64, 96, dtype=torch.float32), ldz=96) == 2      # E % 64
    assert _bwd(lib, dims=bd.make_dims(64, 128, dtype=torch.float32, flags=bd.R2L_FLAG_FORWARD_SCAN)) == 2
    assert _bwd(lib, ldz=64) == 1
    assert _bwd(lib, ldbc=34) == 3
    assert _bwd(lib, ldz=130) == 3
    assert _bwd(lib, bad=(7, FAKE + 4)) == 3
    assert _bwd(lib, lengths=FAKE + 2) == 3
    assert _bwd(lib, ws=None) == 4
    assert _bwd(lib, ws_bytes=16) == 4
    assert _bwd(lib, ws=FAKE + 8) == 3
    big = bd.make_dims(64, 128, dtype=torch.float32)
    assert bd.reverse_scan_backward_workspace_size(big, 65535, 65535, 1) == 0     # beyond the launch grid
    assert _bwd(lib, B=65535, L=65535, chunk=1, ws_bytes=1 << 40) == 2


def _hook_bwd(lib, dims=None, B=2, L=40, ws=FAKE, ws_bytes=None, w=None, g=None, dh_out=FAKE, ds=FAKE + 16,
              lengths=None):
    dims = dims or bd.make_dims(64, 128, dt_rank=8)
    w = w or _weights()
    if g is None:
        g = bd.Grads()
        for f, _ in bd.Grads._fields_:
            setattr(g, f, FAKE)
    if ws_bytes is None:
        ws_bytes = bd.sidecar_backward_workspace_size(dims, B, L) or 1
    return lib.r2l_sidecar_backward(FAKE, ctypes.byref(w), ctypes.byref(dims), 0.5, B, L, lengths, dh_out, FAKE, ds,
                                    ctypes.byref(g), ws, ws_bytes, None)


def test_hook_backward_argument_checks(lib):
    """r2l_sidecar_backward rejects bad arguments on the host (no GPU needed)."""
    bf = bd.make_dims(64, 128, dt_rank=8)
    n = bd.sidecar_backward_workspace_size(bf, 2, 40)
    assert n > bd.workspace_size(bf, 2, 40)                  # the forward's regions and the gradient's
    assert bd.sidecar_backward_workspace_size(bf, 4, 40) > n
    assert bd.sidecar_backward_workspace_size(bd.make_dims(64, 128, dt_rank=8, dtype=torch.float32), 2, 40) == 0
    assert _hook_bwd(lib, dh_out=None) == 1
    assert _hook_bwd(lib, B=0) == 1
    assert _hook_bwd(lib, dims=bd.make_dims(64, 128, dt_rank=8, dtype=torch.float32)) == 2
    assert _hook_bwd(lib, dims=bd.make_dims(64, 128, dt_rank=8, flags=bd.R2L_FLAG_FORWARD_SCAN)) == 2
    assert _hook_bwd(lib, dims=bd.make_dims(64, 96, dt_rank=8)) == 2                     # d_inner % 64
    g = bd.Grads()
    for f, _ in bd.Grads._fields_:
        setattr(g, f, FAKE)
    g.A_log = None
    assert _hook_bwd(lib, g=g) == 1
    g.A_log = FAKE + 4
    assert _hook_bwd(lib, g=g) == 3
    g.A_log = FAKE
    g.ln_w = None                                                              # the hook has a LayerNorm
    assert _hook_bwd(lib, g=g) == 1
    assert _hook_bwd(lib, ds=FAKE + 2) == 3
    assert _hook_bwd(lib, ws=None) == 4
    assert _hook_bwd(lib, ws_bytes=16) == 4
    assert _hook_bwd(lib, ws=FAKE + 8) == 3


def _train_fwd(lib, dims=None, B=2, L=40, hidden=FAKE, out=FAKE + 1024, ws=FAKE, ws_bytes=None, lengths=None):
    dims = dims or bd.make_dims(64, 128, dt_rank=8)
    w = _weights()
    if ws_bytes is None:
        ws_bytes = bd.sidecar_backward_workspace_size(dims, B, L) or 1
    return lib.r2l_sidecar_forward_train(hidden, out, ctypes.byref(w), ctypes.byref(dims), 0.5, B, L, lengths, ws,
                                         ws_bytes, None)


def test_train_forward_argument_checks(lib):
    """r2l_sidecar_forward_train rejects bad arguments on the host: an output
    that aliases the input (the gradient reads the input again), shapes the
    gradient does not support, a workspace smaller than the gradient's."""
    assert _train_fwd(lib, out=None) == 1
    assert _train_fwd(lib, out=FAKE) == 1                                       # out == hidden
    assert _train_fwd(lib, hidden=None) == 1
    assert _train_fwd(lib, B=0) == 1
    assert _train_fwd(lib, dims=bd.make_dims(64, 128, dt_rank=8, dtype=torch.float32)) == 2
    assert _train_fwd(lib, dims=bd.make_dims(64, 128, dt_rank=8, flags=bd.R2L_FLAG_FORWARD_SCAN)) == 2
    assert _train_fwd(lib, out=FAKE + 1032) == 3
    assert _train_fwd(lib, lengths=FAKE + 2) == 3
    assert _train_fwd(lib, ws=None) == 4
    dims = bd.make_dims(64, 128, dt_rank=8)
    assert _train_fwd(lib, ws_bytes=bd.workspace_size(dims, 2, 40)) == 4        # the forward's alone is too small
