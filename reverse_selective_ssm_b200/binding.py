"""ctypes binding of libr2l (include/r2l.h): argument marshalling only.

Every step of the layer runs in the CUDA library; this module turns torch
tensors into the raw device pointers and sizes the C ABI takes, calls it, and
raises :class:`R2LError` on a non-zero status.  There is no fallback: if the
shared library is missing or cannot be loaded, :func:`load` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libr2l.so")

R2L_BF16, R2L_FP32 = 0, 1
R2L_FLAG_GENERAL_A = 0x1
R2L_FLAG_FORWARD_SCAN = 0x2
R2L_FLAG_SAVED_FORWARD = 0x4
R2L_DEVFLAG_LENGTH_CLAMPED = 0x1

STATUS = {0: "R2L_OK", 1: "R2L_ERR_INVALID_ARG", 2: "R2L_ERR_UNSUPPORTED", 3: "R2L_ERR_ALIGNMENT",
          4: "R2L_ERR_WORKSPACE", 5: "R2L_ERR_CUDA", 6: "R2L_ERR_DEVICE_CHECK"}

EXPORTS = ("r2l_abi_version", "r2l_status_string", "r2l_workspace_size", "r2l_sidecar_forward",
           "r2l_sidecar_forward_debug", "r2l_sidecar_forward_profiled", "r2l_sidecar_stack",
           "r2l_get_device_status", "r2l_reverse_scan_workspace_size", "r2l_reverse_scan",
           "r2l_reverse_scan_noalloc", "r2l_reverse_scan_backward_workspace_size",
           "r2l_reverse_scan_backward", "r2l_sidecar_backward_workspace_size", "r2l_sidecar_backward",
           "r2l_sidecar_forward_train")

NOALLOC_SCRATCH_BYTES = 16 << 20

STAGES = ("in_proj", "conv", "x_proj", "dt_proj", "scan", "out_proj", "ln_residual")


class R2LError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _LIB.r2l_status_string(status).decode() if _LIB is not None else STATUS.get(status, "?")
        super().__init__(f"{where}: {msg} (status {status})")


class Dims(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("d_inner", ctypes.c_int), ("d_state", ctypes.c_int),
                ("dt_rank", ctypes.c_int), ("d_conv", ctypes.c_int), ("dtype", ctypes.c_int),
                ("flags", ctypes.c_uint)]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "in_proj_w", "conv_w", "conv_b", "x_proj_w", "dt_proj_w", "dt_proj_b", "A_log", "D",
        "out_proj_w", "ln_w", "ln_b")]


class Grads(ctypes.Structure):
    """r2l_grads: fp32 device arrays shaped like the weights."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "in_proj_w", "conv_w", "conv_b", "x_proj_w", "dt_proj_w", "dt_proj_b", "A_log", "D",
        "out_proj_w", "ln_w", "ln_b")]


class DebugOut(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("x", "z", "u", "dbc", "y", "o", "hhat")]


_LIB: Optional[ctypes.CDLL] = None

# key of the synthetic weight dict -> field of the C struct
_WMAP = (("W_in", "in_proj_w"), ("conv_w", "conv_w"), ("conv_b", "conv_b"), ("W_x", "x_proj_w"),
         ("W_dt", "dt_proj_w"), ("b_dt", "dt_proj_b"), ("A_log", "A_log"), ("D", "D"),
         ("W_out", "out_proj_w"), ("ln_w", "ln_w"), ("ln_b", "ln_b"))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libr2l.so (raises if it is missing: there is no other implementation)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"libr2l.so not found at {path}; build it with "
                           "`python -m reverse_selective_ssm_b200.build`")
    lib = ctypes.CDLL(path)
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.r2l_abi_version.restype = ci
    lib.r2l_status_string.restype = ctypes.c_char_p
    lib.r2l_status_string.argtypes = [ci]
    lib.r2l_workspace_size.restype = ctypes.c_size_t
    lib.r2l_workspace_size.argtypes = [ctypes.POINTER(Dims), ci, ci]
    fwd = [vp, ctypes.POINTER(Weights), ctypes.POINTER(Dims), cf, ci, ci, vp, vp, ctypes.c_size_t, vp]
    lib.r2l_sidecar_forward.restype = ci
    lib.r2l_sidecar_forward.argtypes = fwd
    lib.r2l_sidecar_forward_debug.restype = ci
    lib.r2l_sidecar_forward_debug.argtypes = fwd + [ctypes.POINTER(DebugOut)]
    lib.r2l_sidecar_forward_profiled.restype = ci
    lib.r2l_sidecar_forward_profiled.argtypes = fwd + [ctypes.POINTER(vp), ci, ctypes.POINTER(ci)]
    lib.r2l_sidecar_stack.restype = ci
    lib.r2l_sidecar_stack.argtypes = [vp, ctypes.POINTER(Weights), ctypes.POINTER(cf), ci,
                                      ctypes.POINTER(Dims), ci, ci, vp, vp, ctypes.c_size_t, vp]
    lib.r2l_reverse_scan_workspace_size.restype = ctypes.c_size_t
    lib.r2l_reverse_scan_workspace_size.argtypes = [ctypes.POINTER(Dims), ci, ci, ci]
    lib.r2l_reverse_scan.restype = ci
    lib.r2l_reverse_scan.argtypes = [vp, vp, ci, vp, vp, ci, vp, vp, vp, vp, ctypes.POINTER(Dims), ci, ci, vp,
                                     ci, vp, ctypes.c_size_t, vp]
    lib.r2l_reverse_scan_noalloc.restype = ci
    lib.r2l_reverse_scan_noalloc.argtypes = [vp, vp, ci, vp, vp, ci, vp, vp, vp, vp, ctypes.POINTER(Dims), ci,
                                             ci, vp, ci, vp]
    lib.r2l_reverse_scan_backward_workspace_size.restype = ctypes.c_size_t
    lib.r2l_reverse_scan_backward_workspace_size.argtypes = [ctypes.POINTER(Dims), ci, ci, ci]
    lib.r2l_reverse_scan_backward.restype = ci
    lib.r2l_reverse_scan_backward.argtypes = [vp, vp, ci, vp, vp, ci, vp, vp, vp, vp, vp, vp, ci, vp, vp, ci,
                                              vp, vp, vp, ctypes.POINTER(Dims), ci, ci, vp, ci, vp,
                                              ctypes.c_size_t, vp]
    lib.r2l_sidecar_backward_workspace_size.restype = ctypes.c_size_t
    lib.r2l_sidecar_backward_workspace_size.argtypes = [ctypes.POINTER(Dims), ci, ci]
    lib.r2l_sidecar_backward.restype = ci
    lib.r2l_sidecar_backward.argtypes = [vp, ctypes.POINTER(Weights), ctypes.POINTER(Dims), cf, ci, ci, vp, vp, vp,
                                         vp, ctypes.POINTER(Grads), vp, ctypes.c_size_t, vp]
    lib.r2l_sidecar_forward_train.restype = ci
    lib.r2l_sidecar_forward_train.argtypes = [vp, vp, ctypes.POINTER(Weights), ctypes.POINTER(Dims), cf, ci, ci, vp,
                                              vp, ctypes.c_size_t, vp]
    lib.r2l_get_device_status.restype = ci
    lib.r2l_get_device_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    _LIB = lib
    return lib


def make_dims(d_model: int, d_inner: int, d_state: int = 16, dt_rank: int = 128, d_conv: int = 4,
              dtype: torch.dtype = torch.bfloat16, flags: int = 0) -> Dims:
    code = {torch.bfloat16: R2L_BF16, torch.float32: R2L_FP32}[dtype]
    return Dims(d_model, d_inner, d_state, dt_rank, d_conv, code, flags)


def dims_of(dims, dtype: torch.dtype, flags: int = 0) -> Dims:
    """From a :class:`synthetic.Dims`-like object."""
    return make_dims(dims.d_model, dims.d_inner, dims.d_state, dims.dt_rank, dims.d_conv, dtype, flags)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libr2l takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libr2l takes contiguous tensors")
    return t.data_ptr()


def weights_struct(w: Dict[str, Optional[torch.Tensor]]) -> Weights:
    """Weights struct from a dict of device tensors (keys as in synthetic.WEIGHT_KEYS)."""
    ws = Weights()
    for key, field in _WMAP:
        setattr(ws, field, _ptr(w.get(key)))
    return ws


def workspace_size(dims: Dims, B: int, L: int) -> int:
    return int(load().r2l_workspace_size(ctypes.byref(dims), B, L))


def alloc_workspace(dims: Dims, B: int, L: int, device="cuda") -> torch.Tensor:
    n = workspace_size(dims, B, L)
    if n == 0:
        raise ValueError("invalid dims for a workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def sidecar_forward(hidden: torch.Tensor, weights, dims: Dims, s: float, lengths=None,
                    workspace: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> int:
    """r2l_sidecar_forward on hidden [B, L, d] (in place)."""
    lib = load()
    B, L = hidden.shape[0], hidden.shape[1]
    if workspace is None:
        workspace = alloc_workspace(dims, B, L, hidden.device)
    w = weights if isinstance(weights, Weights) else weights_struct(weights)
    st = lib.r2l_sidecar_forward(_ptr(hidden), ctypes.byref(w), ctypes.byref(dims), float(s), B, L,
                                 _ptr(lengths), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if check and st != 0:
        raise R2LError(st, "r2l_sidecar_forward")
    return st


def sidecar_forward_debug(hidden: torch.Tensor, weights, dims: Dims, s: float, lengths=None,
                          workspace: Optional[torch.Tensor] = None, stream=None,
                          outputs: Optional[Dict[str, torch.Tensor]] = None, check: bool = True) -> int:
    lib = load()
    B, L = hidden.shape[0], hidden.shape[1]
    if workspace is None:
        workspace = alloc_workspace(dims, B, L, hidden.device)
    w = weights if isinstance(weights, Weights) else weights_struct(weights)
    dbg = DebugOut()
    for k, v in (outputs or {}).items():
        setattr(dbg, k, _ptr(v))
    st = lib.r2l_sidecar_forward_debug(_ptr(hidden), ctypes.byref(w), ctypes.byref(dims), float(s), B, L,
                                       _ptr(lengths), _ptr(workspace), workspace.numel(),
                                       _stream_ptr(stream), ctypes.byref(dbg))
    if check and st != 0:
        raise R2LError(st, "r2l_sidecar_forward_debug")
    return st


def sidecar_forward_profiled(hidden: torch.Tensor, weights, dims: Dims, s: float, events, lengths=None,
                             workspace: Optional[torch.Tensor] = None, stream=None,
                             check: bool = True) -> int:
    """r2l_sidecar_forward_profiled: records ``events`` (len(STAGES)+1 torch
    CUDA events with timing) at the stage boundaries; returns the number of
    kernels the call enqueued."""
    lib = load()
    B, L = hidden.shape[0], hidden.shape[1]
    if workspace is None:
        workspace = alloc_workspace(dims, B, L, hidden.device)
    w = weights if isinstance(weights, Weights) else weights_struct(weights)
    for e in events:            # torch creates the CUDA event lazily on first record
        if not e.cuda_event:
            e.record(stream if stream is not None else torch.cuda.current_stream())
    ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    n = ctypes.c_int(0)
    st = lib.r2l_sidecar_forward_profiled(_ptr(hidden), ctypes.byref(w), ctypes.byref(dims), float(s), B, L,
                                          _ptr(lengths), _ptr(workspace), workspace.numel(),
                                          _stream_ptr(stream), ev, len(events), ctypes.byref(n))
    if check and st != 0:
        raise R2LError(st, "r2l_sidecar_forward_profiled")
    return int(n.value)


def sidecar_stack(hidden: torch.Tensor, weights_list: Sequence, dims: Dims, s_list: Sequence[float],
                  lengths=None, workspace: Optional[torch.Tensor] = None, stream=None,
                  check: bool = True) -> int:
    lib = load()
    B, L = hidden.shape[0], hidden.shape[1]
    if workspace is None:
        workspace = alloc_workspace(dims, B, L, hidden.device)
    n = len(weights_list)
    arr = (Weights * n)(*[w if isinstance(w, Weights) else weights_struct(w) for w in weights_list])
    sarr = (ctypes.c_float * n)(*[float(x) for x in s_list])
    st = lib.r2l_sidecar_stack(_ptr(hidden), arr, sarr, n, ctypes.byref(dims), B, L, _ptr(lengths),
                               _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if check and st != 0:
        raise R2LError(st, "r2l_sidecar_stack")
    return st


def reverse_scan_workspace_size(dims: Dims, B: int, L: int, chunk_tokens: int = 0) -> int:
    return int(load().r2l_reverse_scan_workspace_size(ctypes.byref(dims), B, L, chunk_tokens))


def reverse_scan(u: torch.Tensor, z: torch.Tensor, dt_raw: torch.Tensor, bc: torch.Tensor,
                 A_log: torch.Tensor, D: torch.Tensor, dt_b: torch.Tensor, y: torch.Tensor, dims: Dims,
                 B: int, L: int, lengths=None, chunk_tokens: int = 0,
                 workspace: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> int:
    """r2l_reverse_scan.  u, dt_raw, y: [B·L, E]; z: [B·L, ldz] (first E columns);
    bc: [B·L, ldbc] fp32 with B in columns 0..15 and C in 16..31."""
    lib = load()
    if workspace is None:
        n = reverse_scan_workspace_size(dims, B, L, chunk_tokens)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=u.device)
    st = lib.r2l_reverse_scan(_ptr(u), _ptr(z), z.stride(0), _ptr(dt_raw), _ptr(bc), bc.stride(0), _ptr(A_log),
                              _ptr(D), _ptr(dt_b), _ptr(y), ctypes.byref(dims), B, L, _ptr(lengths),
                              chunk_tokens, _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if check and st != 0:
        raise R2LError(st, "r2l_reverse_scan")
    return st


def reverse_scan_noalloc(u: torch.Tensor, z: torch.Tensor, dt_raw: torch.Tensor, bc: torch.Tensor,
                         A_log: torch.Tensor, D: torch.Tensor, dt_b: torch.Tensor, y: torch.Tensor, dims: Dims,
                         B: int, L: int, lengths=None, chunk_tokens: int = 0, stream=None,
                         check: bool = True) -> int:
    """r2l_reverse_scan_noalloc: as :func:`reverse_scan`, with the library's
    static device scratch instead of a caller workspace (nothing is allocated)."""
    lib = load()
    st = lib.r2l_reverse_scan_noalloc(_ptr(u), _ptr(z), z.stride(0), _ptr(dt_raw), _ptr(bc), bc.stride(0),
                                      _ptr(A_log), _ptr(D), _ptr(dt_b), _ptr(y), ctypes.byref(dims), B, L,
                                      _ptr(lengths), chunk_tokens, _stream_ptr(stream))
    if check and st != 0:
        raise R2LError(st, "r2l_reverse_scan_noalloc")
    return st


def reverse_scan_backward_workspace_size(dims: Dims, B: int, L: int, chunk_tokens: int = 0) -> int:
    return int(load().r2l_reverse_scan_backward_workspace_size(ctypes.byref(dims), B, L, chunk_tokens))


def reverse_scan_backward(u: torch.Tensor, z: torch.Tensor, dt_raw: torch.Tensor, bc: torch.Tensor,
                          A_log: torch.Tensor, D: torch.Tensor, dt_b: torch.Tensor, dy: torch.Tensor,
                          du: torch.Tensor, dz: torch.Tensor, ddt_raw: torch.Tensor, dbc: torch.Tensor,
                          dA_log: torch.Tensor, dD: torch.Tensor, ddt_b: torch.Tensor, dims: Dims, B: int, L: int,
                          lengths=None, chunk_tokens: int = 0, workspace: Optional[torch.Tensor] = None,
                          stream=None, check: bool = True) -> int:
    """r2l_reverse_scan_backward (fp32).  u, dt_raw, dy, du, ddt_raw: [B·L, E];
    z, dz: [B·L, ld] (first E columns); bc, dbc: [B·L, ld] with B in columns
    0..15 and C in 16..31; dA_log [E, 16]; dD, ddt_b [E]."""
    lib = load()
    if workspace is None:
        n = reverse_scan_backward_workspace_size(dims, B, L, chunk_tokens)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=u.device)
    st = lib.r2l_reverse_scan_backward(_ptr(u), _ptr(z), z.stride(0), _ptr(dt_raw), _ptr(bc), bc.stride(0),
                                       _ptr(A_log), _ptr(D), _ptr(dt_b), _ptr(dy), _ptr(du), _ptr(dz), dz.stride(0),
                                       _ptr(ddt_raw), _ptr(dbc), dbc.stride(0), _ptr(dA_log), _ptr(dD),
                                       _ptr(ddt_b), ctypes.byref(dims), B, L, _ptr(lengths), chunk_tokens,
                                       _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if check and st != 0:
        raise R2LError(st, "r2l_reverse_scan_backward")
    return st


def get_device_status(workspace: torch.Tensor, stream=None):
    """(status, flags) after synchronising the stream."""
    lib = load()
    flags = ctypes.c_uint32(0)
    st = lib.r2l_get_device_status(_ptr(workspace), _stream_ptr(stream), ctypes.byref(flags))
    return st, int(flags.value)


def weights_to_device(w: Dict[str, Optional[torch.Tensor]], device="cuda"):
    return {k: (None if v is None else v.to(device).contiguous()) for k, v in w.items()}


# weight-dict key -> r2l_grads field, as for the weights
GRAD_KEYS = tuple(k for k, _ in _WMAP)


def sidecar_backward_workspace_size(dims: Dims, B: int, L: int) -> int:
    return int(load().r2l_sidecar_backward_workspace_size(ctypes.byref(dims), B, L))


def alloc_grads(weights: Dict[str, Optional[torch.Tensor]], device="cuda") -> Dict[str, Optional[torch.Tensor]]:
    """fp32 gradient buffers shaped like a hook's weights (None where the
    weight is None)."""
    return {k: None if v is None else torch.empty(v.shape, dtype=torch.float32, device=device)
            for k, v in weights.items()}


def sidecar_forward_train(hidden: torch.Tensor, weights, dims: Dims, s: float, lengths=None,
                          workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, stream=None,
                          check: bool = True):
    """r2l_sidecar_forward_train: returns (out = h⁺, workspace); hidden is not
    written.  Pass the same workspace to sidecar_backward with dims carrying
    R2L_FLAG_SAVED_FORWARD to skip the forward's recomputation."""
    lib = load()
    B, L = hidden.shape[0], hidden.shape[1]
    if workspace is None:
        workspace = torch.empty(max(sidecar_backward_workspace_size(dims, B, L), 16), dtype=torch.uint8,
                                device=hidden.device)
    if out is None:
        out = torch.empty_like(hidden)
    w = weights if isinstance(weights, Weights) else weights_struct(weights)
    st = lib.r2l_sidecar_forward_train(_ptr(hidden), _ptr(out), ctypes.byref(w), ctypes.byref(dims), float(s), B, L,
                                       _ptr(lengths), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if check and st != 0:
        raise R2LError(st, "r2l_sidecar_forward_train")
    return out, workspace


def sidecar_backward(hidden: torch.Tensor, weights, dims: Dims, s: float, dh_out: torch.Tensor,
                     grads: Dict[str, Optional[torch.Tensor]], lengths=None, workspace: Optional[torch.Tensor] = None,
                     stream=None, check: bool = True, dh: Optional[torch.Tensor] = None,
                     ds: Optional[torch.Tensor] = None):
    """r2l_sidecar_backward: returns (dh [B, L, d] fp32, ds (a 1-element fp32
    device tensor)); grads (from alloc_grads) receives every parameter's
    gradient.  dh and ds may be given (fp32 [B, L, d] and at least 4 floats,
    caller-owned); they are allocated here otherwise."""
    lib = load()
    B, L = hidden.shape[0], hidden.shape[1]
    if workspace is None:
        workspace = torch.empty(max(sidecar_backward_workspace_size(dims, B, L), 16), dtype=torch.uint8,
                                device=hidden.device)
    w = weights if isinstance(weights, Weights) else weights_struct(weights)
    g = Grads()
    for key, field in _WMAP:
        setattr(g, field, _ptr(grads.get(key)))
    if dh is None:
        dh = torch.empty(dh_out.shape, dtype=torch.float32, device=hidden.device)
    elif dh.dtype != torch.float32 or dh.shape != dh_out.shape:
        raise ValueError("dh must be fp32 and shaped like dh_out")
    if ds is None:
        ds = torch.zeros(4, dtype=torch.float32, device=hidden.device)
    elif ds.dtype != torch.float32 or ds.numel() < 4:
        raise ValueError("ds must be fp32 with at least 4 elements")
    st = lib.r2l_sidecar_backward(_ptr(hidden), ctypes.byref(w), ctypes.byref(dims), float(s), B, L, _ptr(lengths),
                                  _ptr(dh_out), _ptr(dh), _ptr(ds), ctypes.byref(g), _ptr(workspace),
                                  workspace.numel(), _stream_ptr(stream))
    if check and st != 0:
        raise R2LError(st, "r2l_sidecar_backward")
    return dh, ds[:1]
