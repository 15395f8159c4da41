"""B200-native (sm_100a) R2L sidecar forward: a reverse Mamba-1 block with a
stream-local LayerNorm and a tanh(s)-gated residual, behind a C ABI (libr2l).

The CUDA library is loaded on first use by :mod:`reverse_selective_ssm_b200.binding`;
importing this package alone loads nothing.
"""
__all__ = ["binding", "synthetic"]
