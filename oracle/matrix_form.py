"""The SSD forward as one explicit matrix product -- TEST INFRASTRUCTURE ONLY.

This is the "matrix transform" statement of the method, used to pin the
sequential oracle on tiny inputs.  It builds, per (batch row, head), the lower
triangular semiseparable matrix

    M[j, i] = C_j . B_i * L[j, i] * dt_i      (j >= i),   0 above the diagonal
    L[j, i] = a_j * a_{j-1} * ... * a_{i+1}    (empty product = 1 on the diagonal)

and returns y = M x + z * (C h0^T) + D x, where z_j = a_j ... a_0 carries the
initial state (the state before token 0, so a_0 applies to it).

Sources:
  * "22 · Mamba 2 — Transformers are SSMs" (paper story), section 2.1: the
    unrolled form y_t = sum_s C_t^T (A_t ... A_{s+1}) B_s x_s and the matrix
    M_{j,i}; section 3.2: the dual form Y = (L o Q K^T) V with Q = C, K = B,
    V = Delta x and L_{j,i} = a_j ... a_{i+1}.
  * "SSM 家族全景图（下）：Mamba-2 与 Jamba", section 二.1: the same M as a lower
    triangular semiseparable matrix.
  * "Transformers与SSMs的隐藏联系", section 4.2: a_t = 0 where a new packed
    sequence starts.

O(T^2) memory and O(T^3)-ish work in plain numpy: tiny T only.
"""
from __future__ import annotations

import numpy as np

from . import as_f64, as_i32


def decay_factors(dt_h: np.ndarray, A_h: float, seq_row=None) -> np.ndarray:
    """a_t = exp(dt_t * A_h), forced to 0 where seq_row changes (length T)."""
    a = np.exp(dt_h * A_h)
    if seq_row is not None:
        for t in range(1, len(a)):
            if seq_row[t] != seq_row[t - 1]:
                a[t] = 0.0
    return a


def decay_matrix(a: np.ndarray) -> np.ndarray:
    """L[j, i] = prod_{k=i+1..j} a_k for j >= i, else 0."""
    T = len(a)
    Lm = np.zeros((T, T))
    for j in range(T):
        Lm[j, j] = 1.0
        for i in range(j - 1, -1, -1):
            Lm[j, i] = Lm[j, i + 1] * a[i + 1]
    return Lm


def semiseparable_matrix(dt_h, A_h, B_g, C_g, seq_row=None) -> np.ndarray:
    """M (T x T) for one head: (L o C B^T) scaled by dt on the input side."""
    a = decay_factors(dt_h, A_h, seq_row)
    Lm = decay_matrix(a)
    CB = C_g @ B_g.T
    return Lm * CB * dt_h[None, :]


def ssd_matrix_form(x, dt, A, B, C, D=None, initial_states=None, seq_idx=None, num_seqs=None):
    """y (b,L,H,P) and final states via explicit M; tiny inputs only.

    Final states use the same unrolled sum evaluated at each sequence's last
    token: h_e = sum_{s<=e} L[e,s] dt_s x_s B_s^T + z_e h0.
    """
    x, dt, A, B, C = (as_f64(v) for v in (x, dt, A, B, C))
    D, h0, si = as_f64(D), as_f64(initial_states), as_i32(seq_idx)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros_like(x)
    if si is not None:
        ns = int(si.max()) + 1 if num_seqs is None else num_seqs
        final = np.zeros((ns, H, P, N))
    else:
        final = np.zeros((b, H, P, N))
    for bi in range(b):
        row = None if si is None else si[bi]
        for h in range(H):
            g = h // (H // G)
            a = decay_factors(dt[bi, :, h], A[h], row)
            Lm = decay_matrix(a)
            M = Lm * (C[bi, :, g] @ B[bi, :, g].T) * dt[bi, :, h][None, :]
            yh = M @ x[bi, :, h]
            z = np.cumprod(a)  # z_j = a_0 ... a_j
            if h0 is not None:
                yh = yh + z[:, None] * (C[bi, :, g] @ h0[bi, h].T)
            if D is not None:
                yh = yh + D[h] * x[bi, :, h]
            y[bi, :, h] = yh
            # states at the ends: weights L[e, s] dt_s on x_s B_s^T
            ends = [L - 1] if row is None else [t for t in range(L) if t == L - 1 or row[t + 1] != row[t]]
            for e in ends:
                w = Lm[e] * dt[bi, :, h]
                st = (x[bi, :, h] * w[:, None]).T @ B[bi, :, g]
                if h0 is not None:
                    st = st + z[e] * h0[bi, h]
                if row is None:
                    final[bi, h] = st
                else:
                    final[row[e], h] = st
    return y, final
