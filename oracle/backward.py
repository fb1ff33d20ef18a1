"""Oracle for the SSD backward pass -- TEST INFRASTRUCTURE ONLY.

The pages give the forward recurrence ("22 · Mamba 2 — Transformers are
SSMs", section 3.1; the D feed-through from "从Transformer的二次复杂度困境到
Mamba的线性突围", continuous SSM equations) and say that the backward pass
recomputes the forward's states instead of storing them (the same page, the
hardware-aware algorithm: recomputation), but they give no gradient formulas.
These are the adjoint of the recurrence, derived here.  Per batch row b and
head h (group g), forward:

    a_t = exp(dt_t A_h)  (0 at the first token of a new packed sequence)
    h_t = a_t h_{t-1} + dt_t x_t B_t^T          h_{-1} = h0
    y_t = h_t C_t + D_h x_t                     final = h_{T-1}

Backward, with G_t = dLoss/dh_t (P x N) swept from the last token:

    G_t   = dy_t C_t^T + a_{t+1} G_{t+1}        (G_{T-1} also gets dfinal)
    dx_t  = dt_t G_t B_t + D_h dy_t
    dB_t += dt_t G_t^T x_t                      (summed over the group's heads)
    dC_t += h_t^T dy_t                          (summed over the group's heads)
    ddt_t = <G_t, x_t B_t^T> + A_h a_t <G_t, h_{t-1}>
    dA_h  = sum_t dt_t a_t <G_t, h_{t-1}>
    dD_h  = sum_t <dy_t, x_t>
    dh0   = a_0 G_0

where <., .> sums over all entries.  A reset token (a_t = 0) passes no
gradient to h_{t-1}, dt_t's decay term or A.  Plain fp64 numpy, token by token
(the states are recomputed first, as the pages describe), for small inputs.

With the Mamba-2 block's gate ("SSM 家族全景图（下）：Mamba-2 与 Jamba",
section 5) the output is out = y * SiLU(z), SiLU(v) = v / (1 + e^-v).  Given
dout, the gate's own gradient is dz = dout * y * SiLU'(z), with
SiLU'(v) = s (1 + v (1 - s)) and s = 1 / (1 + e^-v), and the SSD receives
dy = dout * SiLU(z) (``ssd_bwd_gated``).
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import as_f64, as_i32


def _upstream(a):
    """An upstream gradient at the precision given: fp64 arrays as they are
    (a gradient formed in fp64, such as the gate's dout * SiLU(z)), anything
    else widened through fp32 like the inputs."""
    if isinstance(a, np.ndarray) and a.dtype == np.float64:
        return np.ascontiguousarray(a)
    return as_f64(a)


def ssd_bwd(x, dt, A, B, C, D, initial_states, dy, dfinal=None, seq_idx=None) -> dict:
    """Gradients of sum(dy * y) + sum(dfinal * final) with respect to every
    input.  Shapes as the forward: x (b,L,H,P), dt (b,L,H), A (H), B and C
    (b,L,G,N), D (H) or None, initial_states (b,H,P,N) or None, dy like y,
    dfinal (b,H,P,N) or None, seq_idx (b,L) or None (then dfinal is not
    supported: the final states are per sequence).  Returns a dict of fp64
    arrays dx, ddt, dA, dB, dC, dD (or None), dh0 (or None)."""
    x, dt, A, B, C = as_f64(x), as_f64(dt), as_f64(A), as_f64(B), as_f64(C)
    Dv = None if D is None else as_f64(D)
    h0 = None if initial_states is None else as_f64(initial_states)
    dy = _upstream(dy)
    dfin = None if dfinal is None else _upstream(dfinal)
    seq = None if seq_idx is None else as_i32(seq_idx)
    if seq is not None and dfin is not None:
        raise ValueError("dfinal with packed sequences is not supported here")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = H // G
    grp = np.arange(H) // hpg
    Bh = B[:, :, grp]  # (b, L, H, N): each head's B and C
    Ch = C[:, :, grp]

    a = np.exp(dt * A[None, None, :])  # (b, L, H)
    if seq is not None:
        reset = np.zeros((b, L), dtype=bool)
        reset[:, 1:] = seq[:, 1:] != seq[:, :-1]
        a = np.where(reset[:, :, None], 0.0, a)

    # recompute the states: hs[:, t] = h_t, hprev[:, t] = h_{t-1}
    hs = np.zeros((b, L, H, P, N))
    h = np.zeros((b, H, P, N)) if h0 is None else h0.copy()
    hprev = np.zeros_like(hs)
    for t in range(L):
        hprev[:, t] = h
        h = a[:, t, :, None, None] * h + (dt[:, t, :, None, None] * x[:, t, :, :, None]) * Bh[:, t, :, None, :]
        hs[:, t] = h

    dx = np.zeros_like(x)
    ddt = np.zeros_like(dt)
    dA = np.zeros(H)
    dBh = np.zeros((b, L, H, N))
    dCh = np.zeros((b, L, H, N))
    Gt = np.zeros((b, H, P, N)) if dfin is None else dfin.copy()
    for t in range(L - 1, -1, -1):
        if t < L - 1:
            Gt = a[:, t + 1, :, None, None] * Gt
        Gt = Gt + dy[:, t, :, :, None] * Ch[:, t, :, None, :]
        dx[:, t] = dt[:, t, :, None] * np.einsum("bhpn,bhn->bhp", Gt, Bh[:, t])
        dBh[:, t] = dt[:, t, :, None] * np.einsum("bhpn,bhp->bhn", Gt, x[:, t])
        dCh[:, t] = np.einsum("bhpn,bhp->bhn", hs[:, t], dy[:, t])
        g_in = np.einsum("bhpn,bhp,bhn->bh", Gt, x[:, t], Bh[:, t])
        g_dec = np.einsum("bhpn,bhpn->bh", Gt, hprev[:, t])
        ddt[:, t] = g_in + A[None, :] * a[:, t] * g_dec
        dA += np.sum(dt[:, t] * a[:, t] * g_dec, axis=0)
    if Dv is not None:
        dx += Dv[None, None, :, None] * dy
    dD = None if Dv is None else np.einsum("blhp,blhp->h", dy, x)
    dh0 = None if h0 is None else a[:, 0, :, None, None] * Gt
    dB = np.zeros((b, L, G, N))
    dC = np.zeros((b, L, G, N))
    for h_ in range(H):
        dB[:, :, grp[h_]] += dBh[:, :, h_]
        dC[:, :, grp[h_]] += dCh[:, :, h_]
    return {"dx": dx, "ddt": ddt, "dA": dA, "dB": dB, "dC": dC, "dD": dD, "dh0": dh0}


def silu(v):
    """SiLU(v) = v / (1 + e^-v), elementwise, fp64."""
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def silu_grad(v):
    """dSiLU/dv = s (1 + v (1 - s)) with s = 1 / (1 + e^-v), elementwise, fp64."""
    v = np.asarray(v, dtype=np.float64)
    s = 1.0 / (1.0 + np.exp(-v))
    return s * (1.0 + v * (1.0 - s))


def ssd_bwd_gated(x, dt, A, B, C, D, initial_states, z, dout, dfinal=None, seq_idx=None, backward_fn=None) -> dict:
    """Gradients of sum(dout * y * SiLU(z)) + sum(dfinal * final): the ungated
    output y comes from the forward oracle (fp64), the SSD's gradients from
    ``backward_fn`` (default ``ssd_bwd``) on dy = dout * SiLU(z).  Returns the
    same dict plus dz."""
    from . import ssd_fwd
    seq = None if seq_idx is None else as_i32(seq_idx)
    num_seqs = None if seq is None else int(seq.max()) + 1
    y, _ = ssd_fwd(x, dt, A, B, C, D, initial_states, seq_idx=seq, num_seqs=num_seqs)
    zz, do = as_f64(z), as_f64(dout)
    g = (backward_fn or ssd_bwd)(x, dt, A, B, C, D, initial_states, do * silu(zz), dfinal, seq)
    g["dz"] = do * y * silu_grad(zz)
    return g
