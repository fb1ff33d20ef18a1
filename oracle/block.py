"""Oracle for the Mamba-2 block pieces around the SSD -- TEST INFRASTRUCTURE.

"SSM 家族全景图（下）：Mamba-2 与 Jamba", section 5 (Mamba-2 Block 的数据流):
the main path passes a one-dimensional causal convolution and then SiLU
before the SSD; the gate path passes SiLU; the two paths are multiplied
elementwise.  The pages give no kernel width; the convolution here is
depthwise (one filter per channel) with width K, bias optional, and causal:
output t sees inputs t-K+1 .. t, with zeros before the first token.  With
packed sequences a tap never reaches into an earlier sequence (the same cut
as the SSD's decay at a boundary).  Plain fp64 numpy, one tap at a time.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import as_f64


def silu(v: np.ndarray) -> np.ndarray:
    """SiLU(v) = v * sigmoid(v) = v / (1 + e^-v)."""
    return v / (1.0 + np.exp(-v))


def conv1d_silu(u, weight, bias=None, seq_idx=None) -> np.ndarray:
    """u (b, L, C), weight (C, K), bias (C) or None, seq_idx (b, L) or None ->
    SiLU(bias_c + sum_k weight[c, k] * u[b, t - (K-1) + k, c]), (b, L, C) fp64;
    a tap at s < 0, or (with seq_idx) at a token of another sequence, adds 0."""
    u = as_f64(u)
    w = as_f64(weight)
    b, L, C = u.shape
    K = w.shape[1]
    pre = np.zeros((b, L, C)) if bias is None else np.broadcast_to(as_f64(bias), (b, L, C)).copy()
    seq = None if seq_idx is None else np.asarray(seq_idx.cpu() if hasattr(seq_idx, "cpu") else seq_idx)
    for k in range(K):
        shift = K - 1 - k  # this tap reads token t - shift
        if shift >= L:
            continue
        src = np.zeros((b, L, C))
        src[:, shift:] = u[:, : L - shift]
        if seq is not None and shift > 0:
            same = np.zeros((b, L), dtype=bool)
            same[:, shift:] = seq[:, shift:] == seq[:, : L - shift]
            src *= same[:, :, None]
        pre += w[None, None, :, k] * src
    return silu(pre)


def gate(y, z) -> np.ndarray:
    """The gate path: y * SiLU(z), elementwise, fp64."""
    return as_f64(y) * silu(as_f64(z))
