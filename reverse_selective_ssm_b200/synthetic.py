"""Seeded synthetic inputs for the R2L sidecar.

This module only draws numbers: hidden states, weights, gates and lengths, on
the CPU with ``torch.Generator`` so every consumer (the CUDA library, the CPU
oracle, the benchmark) sees identical bits.  It holds none of the layer's
arithmetic.

Shapes follow the serving setup of "Bifocal Diffusion Language Models"
(arXiv 2606.27732v1): §4.1 (Qwen3-1.7B backbone, d_model = 2048, 28 decoder
layers, a hook after every 4th, d_state = 16, d_conv = 4, expand 2) and the
throughput sweep of §4.3 / Table 3 (batch 8, prompt length 4096).  The pages
train on a web corpus and publish no weights, so everything here is drawn:

  * hidden states ~ N(0, 1), stored in the activation dtype;
  * W_in, conv_w, conv_b, W_x, W_dt, W_out ~ N(0, 0.02);
  * A_log[c, m] = log(m + 1) (so A = -(1..d_state) per channel), D = 1;
  * a per-channel target step dt0 ~ logUniform[1e-3, 1e-1] and the dt_proj
    bias set to the inverse softplus of dt0 (a weight-initialisation recipe);
  * LayerNorm weight 1 and bias 0 unless asked for seeded values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

WEIGHT_KEYS = ("W_in", "conv_w", "conv_b", "W_x", "W_dt", "b_dt", "A_log", "D",
               "W_out", "ln_w", "ln_b")
GEMM_WEIGHTS = ("W_in", "W_x", "W_dt", "W_out")


@dataclass(frozen=True)
class Dims:
    d_model: int
    d_inner: int
    d_state: int = 16
    dt_rank: int = 128
    d_conv: int = 4


@dataclass
class Case:
    """One workload: hidden [B, L, d_model], per-hook weights and gates."""
    name: str
    dims: Dims
    dtype: torch.dtype
    B: int
    L: int
    h: torch.Tensor
    weights: List[Dict[str, Optional[torch.Tensor]]]
    s: List[float]
    lengths: Optional[torch.Tensor] = None     # int32 [B] or None (all L)
    meta: dict = field(default_factory=dict)

    @property
    def valid_tokens(self) -> int:
        if self.lengths is None:
            return self.B * self.L
        return int(self.lengths.clamp(0, self.L).sum())


def _normal(gen, shape, std, dtype):
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * std).to(dtype)


def make_weights(dims: Dims, dtype: torch.dtype, seed: int, *, std: float = 0.02,
                 x_proj_std: Optional[float] = None, D_value: float = 1.0,
                 ln: str = "unit", dt_min: float = 1e-3, dt_max: float = 1e-1,
                 A_log: Optional[torch.Tensor] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Draw one hook's weights.

    ``ln`` is "unit" (γ=1, β=0), "seeded" (γ ~ 1+N(0,0.1), β ~ N(0,0.1)) or
    "none" (no LayerNorm: both pointers null).  GEMM weights are stored in
    ``dtype``; the vectors (conv, dt bias, A_log, D, LN) in float32.
    """
    g = torch.Generator().manual_seed(seed)
    d, E, N, R, W = dims.d_model, dims.d_inner, dims.d_state, dims.dt_rank, dims.d_conv
    xs = std if x_proj_std is None else x_proj_std
    w: Dict[str, Optional[torch.Tensor]] = {}
    w["W_in"] = _normal(g, (2 * E, d), std, dtype)
    w["conv_w"] = _normal(g, (E, W), std, torch.float32)
    w["conv_b"] = _normal(g, (E,), std, torch.float32)
    w["W_x"] = _normal(g, (R + 2 * N, E), xs, dtype)
    w["W_dt"] = _normal(g, (E, R), std, dtype)
    u01 = torch.rand((E,), generator=g, dtype=torch.float64)
    dt0 = torch.exp(u01 * (math.log(dt_max) - math.log(dt_min)) + math.log(dt_min))
    w["b_dt"] = (dt0 + torch.log(-torch.expm1(-dt0))).to(torch.float32)
    if A_log is None:
        w["A_log"] = torch.log(torch.arange(1, N + 1, dtype=torch.float32)).repeat(E, 1).contiguous()
    else:
        w["A_log"] = A_log.to(torch.float32).contiguous()
    w["D"] = torch.full((E,), float(D_value), dtype=torch.float32)
    w["W_out"] = _normal(g, (d, E), std, dtype)
    if ln == "unit":
        w["ln_w"] = torch.ones(d, dtype=torch.float32)
        w["ln_b"] = torch.zeros(d, dtype=torch.float32)
    elif ln == "seeded":
        w["ln_w"] = 1.0 + _normal(g, (d,), 0.1, torch.float32)
        w["ln_b"] = _normal(g, (d,), 0.1, torch.float32)
    elif ln == "none":
        w["ln_w"] = None
        w["ln_b"] = None
    else:
        raise ValueError(ln)
    return w


def _sequence_generator(seed: int, index: int) -> torch.Generator:
    """The generator of global sequence ``index`` of a batch drawn with ``seed``."""
    return torch.Generator().manual_seed(seed * 1_000_003 + index)


def make_hidden(B: int, L: int, d: int, dtype: torch.dtype, seed: int, first: int = 0) -> torch.Tensor:
    """Hidden states [B, L, d] ~ N(0, 1).  Row b is global sequence first + b
    and depends on (seed, first + b) only, so a contiguous slice of a global
    batch (one rank's shard) is drawn with the same bits as the whole."""
    out = torch.empty((B, L, d), dtype=torch.float32)
    for b in range(B):
        out[b] = torch.randn((L, d), generator=_sequence_generator(seed, first + b), dtype=torch.float32)
    return out.to(dtype)


def make_lengths(B: int, lo: int, hi: int, seed: int, first: int = 0) -> torch.Tensor:
    """Valid lengths ~ U{lo..hi}, one draw per global sequence (as make_hidden)."""
    vals = [int(torch.randint(lo, hi + 1, (1,), generator=_sequence_generator(seed + 7919, first + b)))
            for b in range(B)]
    return torch.tensor(vals, dtype=torch.int32)


def shard_first(B: int, shard) -> int:
    """First global sequence of a rank's shard: rank r of n takes sequences
    [r·B, (r+1)·B) of a global batch of n·B (B sequences per rank)."""
    if shard is None:
        return 0
    rank, world = shard
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    return rank * B


def poison_padding(h: torch.Tensor, lengths: torch.Tensor) -> torch.Tensor:
    """Fill rows at or past each sequence's length with NaN sentinels."""
    h = h.clone()
    for b, n in enumerate(lengths.tolist()):
        if n < h.shape[1]:
            h[b, n:] = float("nan")
    return h


BIG = Dims(d_model=2048, d_inner=4096, d_state=16, dt_rank=128, d_conv=4)
TINY = Dims(d_model=64, d_inner=128, d_state=16, dt_rank=4, d_conv=4)

# The five workloads.  Config 2 is the serving shape the throughput numbers are
# quoted on (batch 8, prompt 4096).
CONFIG_NAMES = {
    0: "tiny-fp32 B=1 L=64 d=64 E=128 N=16 R=4",
    1: "single bf16 B=1 L=2048 d=2048 E=4096 N=16 R=128",
    2: "serving bf16 B=8 L=4096 d=2048 E=4096 N=16 R=128",
    3: "stack7 bf16 B=4 L=8192 d=2048 E=4096 N=16 R=128 x7 hooks",
    4: "ragged bf16 B=256 L=512 len~U[64,512] d=2048 E=4096 N=16 R=128",
    5: "denoise-step bf16 B=8 G=128 d=2048 E=4096 N=16 R=128 x7 hooks",
}


def _meta(first: int, B: int, shard) -> dict:
    world = 1 if shard is None else shard[1]
    return {"first_sequence": first, "global_batch": B * world}


def make_case(cfg: int, *, B: Optional[int] = None, L: Optional[int] = None,
              weights: bool = True, shard=None) -> Case:
    """Build one of the workloads (``B``/``L`` override for smaller runs).

    ``shard`` = (rank, world): the case holds rank's contiguous slice of a
    global batch of world·B sequences (B per rank); the weights are the same
    on every rank, and the slice's hidden states and lengths are bit for bit
    the rows of the global batch."""
    if cfg == 0:
        dims, dt = TINY, torch.float32
        Bv, Lv = (B or 1), (L or 64)
        first = shard_first(Bv, shard)
        h = make_hidden(Bv, Lv, dims.d_model, dt, seed=0, first=first)
        ws = [make_weights(dims, dt, seed=100)] if weights else []
        return Case(CONFIG_NAMES[0], dims, dt, Bv, Lv, h, ws, [0.5], meta=_meta(first, Bv, shard))
    if cfg == 1:
        dims, dt = BIG, torch.bfloat16
        Bv, Lv = (B or 1), (L or 2048)
        first = shard_first(Bv, shard)
        h = make_hidden(Bv, Lv, dims.d_model, dt, seed=1, first=first)
        ws = [make_weights(dims, dt, seed=101)] if weights else []
        return Case(CONFIG_NAMES[1], dims, dt, Bv, Lv, h, ws, [1.0], meta=_meta(first, Bv, shard))
    if cfg == 2:
        dims, dt = BIG, torch.bfloat16
        Bv, Lv = (B or 8), (L or 4096)
        first = shard_first(Bv, shard)
        h = make_hidden(Bv, Lv, dims.d_model, dt, seed=2, first=first)
        ws = [make_weights(dims, dt, seed=102)] if weights else []
        return Case(CONFIG_NAMES[2], dims, dt, Bv, Lv, h, ws, [0.3], meta=_meta(first, Bv, shard))
    if cfg == 3:
        dims, dt = BIG, torch.bfloat16
        Bv, Lv = (B or 4), (L or 8192)
        first = shard_first(Bv, shard)
        h = make_hidden(Bv, Lv, dims.d_model, dt, seed=3, first=first)
        g = torch.Generator().manual_seed(3)
        s = (torch.rand((7,), generator=g, dtype=torch.float64) * 2.0 - 1.0).tolist()
        ws = [make_weights(dims, dt, seed=300 + k) for k in range(7)] if weights else []
        return Case(CONFIG_NAMES[3], dims, dt, Bv, Lv, h, ws, s, meta=_meta(first, Bv, shard))
    if cfg == 4:
        dims, dt = BIG, torch.bfloat16
        Bv, Lv = (B or 256), (L or 512)
        first = shard_first(Bv, shard)
        lengths = make_lengths(Bv, min(64, Lv), Lv, seed=4, first=first)
        h = poison_padding(make_hidden(Bv, Lv, dims.d_model, dt, seed=4, first=first), lengths)
        ws = [make_weights(dims, dt, seed=104)] if weights else []
        return Case(CONFIG_NAMES[4], dims, dt, Bv, Lv, h, ws, [0.7], lengths=lengths,
                    meta=_meta(first, Bv, shard))
    if cfg == 5:
        # one denoising step of cached parallel decoding (§3.5, "Inference with
        # prefix KV cache"): the 7 hooks run over the generation block alone,
        # G = 128 positions of each of B = 8 requests (§4.1 throughput setup)
        dims, dt = BIG, torch.bfloat16
        Bv, Lv = (B or 8), (L or 128)
        first = shard_first(Bv, shard)
        h = make_hidden(Bv, Lv, dims.d_model, dt, seed=5, first=first)
        g = torch.Generator().manual_seed(5)
        s = (torch.rand((7,), generator=g, dtype=torch.float64) * 2.0 - 1.0).tolist()
        ws = [make_weights(dims, dt, seed=500 + k) for k in range(7)] if weights else []
        return Case(CONFIG_NAMES[5], dims, dt, Bv, Lv, h, ws, s, meta=_meta(first, Bv, shard))
    raise ValueError(f"unknown config {cfg}")


def to_f64(t):
    """Exact float64 numpy copy of a CPU tensor (None passes through)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def weights_f64(w: Dict[str, Optional[torch.Tensor]]) -> Dict[str, object]:
    return {k: to_f64(v) for k, v in w.items()}


def make_scan_bwd_case(B: int, L: int, E: int, seed: int, lengths: Optional[torch.Tensor] = None,
                       dt_min: float = 1e-3, dt_max: float = 1e-1) -> Dict[str, torch.Tensor]:
    """Inputs of the scan-gradient entry point, fp32 on the host: the scan's
    own inputs with the distributions they have inside the layer (u, z ~
    N(0, 1); B, C ~ N(0, 1); dt_raw ~ N(0, 0.1) around the per-channel bias
    of a logUniform[dt_min, dt_max] step; A_log = log(1..16); D = 1) and an
    upstream gradient dy ~ N(0, 1).  Rows at or past a sequence's length are
    NaN in every per-position input (they must not be read)."""
    g = torch.Generator().manual_seed(seed)
    M = B * L
    c = {
        "u": torch.randn((M, E), generator=g),
        "z": torch.randn((M, E), generator=g),
        "dt_raw": torch.randn((M, E), generator=g) * 0.1,
        "bc": torch.randn((M, 32), generator=g),
        "dy": torch.randn((M, E), generator=g),
    }
    u01 = torch.rand((E,), generator=g, dtype=torch.float64)
    dt0 = torch.exp(u01 * (math.log(dt_max) - math.log(dt_min)) + math.log(dt_min))
    c["dt_b"] = (dt0 + torch.log(-torch.expm1(-dt0))).to(torch.float32)
    c["A_log"] = torch.log(torch.arange(1, 17, dtype=torch.float32)).repeat(E, 1).contiguous()
    c["D"] = torch.ones(E)
    if lengths is not None:
        for b, n in enumerate(lengths.tolist()):
            if n < L:
                for k in ("u", "z", "dt_raw", "bc", "dy"):
                    c[k][b * L + n:(b + 1) * L] = float("nan")
    return c
