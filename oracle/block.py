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


def _taps(u, K, seq_idx):
    """For each tap k of a width-K causal filter over u (b, L, C): (k, shift,
    src), where the tap reads token t - shift (shift = K-1-k) and src[t] is
    that input, 0 where t - shift < 0 or (with seq_idx) lies in another
    sequence."""
    b, L, C = u.shape
    seq = None if seq_idx is None else np.asarray(seq_idx.cpu() if hasattr(seq_idx, "cpu") else seq_idx)
    for k in range(K):
        shift = K - 1 - k
        if shift >= L:
            continue
        src = np.zeros((b, L, C))
        src[:, shift:] = u[:, : L - shift]
        if seq is not None and shift > 0:
            same = np.zeros((b, L), dtype=bool)
            same[:, shift:] = seq[:, shift:] == seq[:, : L - shift]
            src *= same[:, :, None]
        yield k, shift, src


def _pre(u, w, bias, seq_idx):
    """The pre-activation bias_c + sum_k weight[c, k] * u[b, t - (K-1) + k, c]."""
    b, L, C = u.shape
    pre = np.zeros((b, L, C)) if bias is None else np.broadcast_to(as_f64(bias), (b, L, C)).copy()
    for k, _, src in _taps(u, w.shape[1], seq_idx):
        pre += w[None, None, :, k] * src
    return pre


def conv1d_silu(u, weight, bias=None, seq_idx=None) -> np.ndarray:
    """u (b, L, C), weight (C, K), bias (C) or None, seq_idx (b, L) or None ->
    SiLU(bias_c + sum_k weight[c, k] * u[b, t - (K-1) + k, c]), (b, L, C) fp64;
    a tap at s < 0, or (with seq_idx) at a token of another sequence, adds 0."""
    return silu(_pre(as_f64(u), as_f64(weight), bias, seq_idx))


def silu_grad(v: np.ndarray) -> np.ndarray:
    """dSiLU/dv = s (1 + v (1 - s)) with s = 1 / (1 + e^-v)."""
    s = 1.0 / (1.0 + np.exp(-v))
    return s * (1.0 + v * (1.0 - s))


def conv1d_silu_bwd(u, weight, bias, dout, seq_idx=None, with_scale: bool = False) -> tuple:
    """Gradients of sum(dout * conv1d_silu(u, weight, bias, seq_idx)):
    (du (b, L, C), dweight (C, K), dbias (C)), fp64.  With g = dout * SiLU'(pre),
    each tap k that the forward takes (reading token t - shift for output t)
    sends w[c, k] g[t] back to du[t - shift] and adds g[t] u[t - shift] to
    dweight[c, k]; dbias = sum over rows and tokens of g.  With ``with_scale``
    two more arrays follow: the sums of the magnitudes of the terms of dweight
    and of dbias (the scale a rounding error in those sums is measured against)."""
    u, w = as_f64(u), as_f64(weight)
    b, L, C = u.shape
    g = as_f64(dout) * silu_grad(_pre(u, w, bias, seq_idx))
    du = np.zeros((b, L, C))
    dw = np.zeros(w.shape)
    dw_abs = np.zeros(w.shape)
    for k, shift, src in _taps(u, w.shape[1], seq_idx):
        valid = np.zeros((b, L, 1))  # the tap reads a real input (not the zero before a row or sequence)
        valid[:, shift:] = 1.0
        if seq_idx is not None and shift > 0:
            seq = np.asarray(seq_idx.cpu() if hasattr(seq_idx, "cpu") else seq_idx)
            valid[:, shift:, 0] = seq[:, shift:] == seq[:, : L - shift]
        du[:, : L - shift] += (w[None, None, :, k] * g * valid)[:, shift:]
        dw[:, k] = np.einsum("blc,blc->c", g, src)
        dw_abs[:, k] = np.einsum("blc,blc->c", np.abs(g), np.abs(src))
    if with_scale:
        return du, dw, g.sum(axis=(0, 1)), dw_abs, np.abs(g).sum(axis=(0, 1))
    return du, dw, g.sum(axis=(0, 1))


def gate(y, z) -> np.ndarray:
    """The gate path: y * SiLU(z), elementwise, fp64."""
    return as_f64(y) * silu(as_f64(z))
