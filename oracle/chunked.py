"""The four chunked SSD steps, written out literally in fp64 -- TEST INFRASTRUCTURE ONLY.

This checks the block decomposition itself (independently of any GPU code)
against the sequential oracle: chunking is an exact re-association, so for
every chunk size Q the result must equal the recurrence up to rounding.

The steps, per (batch row, head), with tokens split into chunks of Q (the last
chunk may be short):

  a0  cs_t = sum_{k = chunk start .. t} dt_k A            (log of the decay, in-chunk)
  a1  Y_diag[t] = sum_{s <= t in the chunk, no boundary in (s, t]}
                     (C_t . B_s) exp(cs_t - cs_s) dt_s x_s
  a2  S_c = sum_{s in the chunk, no boundary in (s, e]} exp(cs_e - cs_s) dt_s x_s B_s^T
                                                             (e = last token of the chunk)
  a3  H_{c+1} = [no boundary in [t0, e]] exp(cs_e) H_c + S_c,   H_0 = h0
  a4  y_t = Y_diag[t] + [no boundary in [t0, t]] exp(cs_t) C_t H_c^T + D x_t

"boundary at k" means seq_idx[k] != seq_idx[k-1]; the initial state belongs
to the first sequence.  Packed final states come from the same sums evaluated
at each sequence's last token instead of the chunk's.

Sources:
  * "SSM 家族全景图（下）：Mamba-2 与 Jamba", section 三.4: the four steps --
    intra-chunk outputs, per-chunk final states, the state scan across
    chunks (sequence shortened to 1/Q), and the output correction from each
    chunk's true initial state.
  * "22 · Mamba 2 — Transformers are SSMs", section 4.1: M = M_intra + M_inter,
    chunk sizes 64-256; section 3.2: the decay mask L as a product of a's,
    i.e. a difference of cumulative sums in log space.
  * "Transformers与SSMs的隐藏联系", section 3.2 (chunks of length Q) and the
    chunk count ceil(T/Q) in its pseudo-code (a short last chunk); section
    4.2: a_t = 0 at packed-sequence boundaries.
"""
from __future__ import annotations

import numpy as np

from . import as_f64, as_i32


def ssd_chunked(x, dt, A, B, C, D=None, initial_states=None, seq_idx=None, num_seqs=None,
                chunk_size: int = 64, return_intermediates: bool = False):
    x, dt, A, B, C = (as_f64(v) for v in (x, dt, A, B, C))
    D, h0, si = as_f64(D), as_f64(initial_states), as_i32(seq_idx)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    Q = int(chunk_size)
    nc = -(-L // Q)
    y = np.zeros_like(x)
    if si is not None:
        ns = int(si.max()) + 1 if num_seqs is None else num_seqs
        final = np.zeros((ns, H, P, N))
    else:
        final = np.zeros((b, H, P, N))
    inter = {"cs": np.zeros((b, H, nc, Q)), "chunk_states": np.zeros((b, nc, H, P, N)),
             "prev_states": np.zeros((b, nc, H, P, N))}
    for bi in range(b):
        row = si[bi] if si is not None else np.zeros(L, dtype=np.int32)
        # boundary[k]: a new sequence starts at token k (never at k = 0)
        boundary = np.zeros(L, dtype=bool)
        boundary[1:] = row[1:] != row[:-1]
        for h in range(H):
            g = h // (H // G)
            Hc = h0[bi, h].copy() if h0 is not None else np.zeros((P, N))
            for c in range(nc):
                t0, t1 = c * Q, min(L, (c + 1) * Q)
                n = t1 - t0
                tok = np.arange(t0, t1)
                # a0: in-chunk cumulative sum of dt*A
                cs = np.cumsum(dt[bi, t0:t1, h] * A[h])
                inter["cs"][bi, h, c, :n] = cs
                # boundary prefix counts inside the chunk, for "no boundary in (s, t]"
                nb = np.cumsum(boundary[t0:t1].astype(np.int64))  # boundaries in [t0, t]
                Xc, Bc, Cc, dtc = x[bi, t0:t1, h], B[bi, t0:t1, g], C[bi, t0:t1, g], dt[bi, t0:t1, h]
                # a1: masked decay-weighted C B^T applied to dt*x
                same = nb[:, None] == nb[None, :]  # no boundary in (s, t]  (s <= t)
                causal = tok[:, None] >= tok[None, :]
                seg = np.where(causal & same, np.exp(np.where(causal, cs[:, None] - cs[None, :], 0.0)), 0.0)
                W = (Cc @ Bc.T) * seg * dtc[None, :]
                y_diag = W @ Xc
                # a4 (uses H_c, the state entering the chunk)
                carry = (nb == 0).astype(np.float64)  # no boundary in [t0, t]
                y_off = (carry * np.exp(cs))[:, None] * (Cc @ Hc.T)
                yc = y_diag + y_off
                if D is not None:
                    yc = yc + D[h] * Xc
                y[bi, t0:t1, h] = yc
                inter["prev_states"][bi, c, h] = Hc
                # a2: state contributed by this chunk, evaluated at its last token
                e = n - 1
                w = np.where(nb == nb[e], np.exp(cs[e] - cs), 0.0) * dtc
                Sc = (Xc * w[:, None]).T @ Bc
                inter["chunk_states"][bi, c, h] = Sc
                # a5: packed final states at sequence ends inside this chunk
                if si is not None:
                    for k in range(n):
                        t = t0 + k
                        if t == L - 1 or row[t + 1] != row[t]:
                            wk = np.where((nb == nb[k]) & (np.arange(n) <= k), np.exp(cs[k] - cs), 0.0) * dtc
                            st = (Xc * wk[:, None]).T @ Bc
                            if nb[k] == 0:
                                st = st + np.exp(cs[k]) * Hc
                            final[row[t], h] = st
                # a3: pass the state to the next chunk
                keep = 1.0 if nb[e] == 0 else 0.0
                Hc = keep * np.exp(cs[e]) * Hc + Sc
            if si is None:
                final[bi, h] = Hc
    if return_intermediates:
        return y, final, inter
    return y, final
