"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, independent of the oracle's own code.

Each ``pin_*`` function takes an oracle callable with the signature of
``oracle.ssd_fwd`` and raises AssertionError when the callable disagrees.
They are shared by the pin tests (run against the real oracle) and the
mutation tests (run against copies of the oracle with planted mistakes, each
of which some pin must reject).

Sources, by page title and section:
  * "22 · Mamba 2 — Transformers are SSMs": section 2.1 (matrix form y = M x),
    2.2 (N-semiseparable: off-diagonal blocks of rank <= N), 3.1 (scalar A
    recurrence), 3.2 (dual form), 4.1 (block decomposition).
  * "从Transformer的二次复杂度困境到Mamba的线性突围": "Mamba-2与状态空间对偶性"
    (all a_t = 1 gives causal linear attention); continuous SSM (D skip).
  * "Transformers与SSMs的隐藏联系" section 4.2 (A_t = 0 at packed boundaries).
  * "SSM 家族全景图（下）：Mamba-2 与 Jamba" section 三.4 (four chunked steps).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import ssd_inputs as si

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "worked_examples.json")
KEYS = ("x", "dt", "A", "B", "C", "D", "initial_states")


def rel(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def small_inputs(b=2, L=40, H=4, P=3, N=5, G=2, seed=7, h0_std=0.3, with_D=True):
    shape = si.SSDShape("pin", b, L, H, P, N, G, 16, "f32", h0_std=h0_std, seed=seed, has_D=with_D)
    d = si.make_inputs(shape)
    return {k: d[k] for k in KEYS}


def pin_golden(fwd):
    """Hand-worked examples (tests/golden/worked_examples.json)."""
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        T, P, N = len(c["dt"]), c["P"], c["N"]
        x = torch.tensor(c["x"], dtype=torch.float32).view(1, T, 1, P)
        B = torch.tensor(c["B"], dtype=torch.float32).view(1, T, 1, N)
        C = torch.tensor(c["C"], dtype=torch.float32).view(1, T, 1, N)
        dt = torch.tensor(c["dt"], dtype=torch.float32).view(1, T, 1)
        A = torch.tensor([c["A"]], dtype=torch.float32)
        D = torch.tensor([c["D"]], dtype=torch.float32)
        h0 = None if c["h0"] is None else torch.tensor(c["h0"], dtype=torch.float32).view(1, 1, P, N)
        sq = None if c["seq_idx"] is None else torch.tensor(c["seq_idx"], dtype=torch.int32).view(1, T)
        y, f = fwd(x, dt, A, B, C, D, h0, seq_idx=sq)
        want_y = np.array(c["y"], dtype=np.float64).reshape(1, T, 1, P)
        want_f = np.array(c["final"], dtype=np.float64)
        want_f = want_f.reshape(want_f.shape[0], 1, P, N)
        # the fixture's A is a double; the oracle sees it rounded to fp32, so
        # the decay differs from 1/2 by ~1e-8 relative
        assert np.allclose(y, want_y, rtol=0, atol=1e-6), (c["name"], y.ravel(), want_y.ravel())
        assert np.allclose(f, want_f, rtol=0, atol=1e-6), (c["name"], f.ravel(), want_f.ravel())


def pin_matrix_form(fwd):
    """y = M x with M written out (section 2.1 / 3.2 of the paper story), tiny T,
    with and without packing, initial state and D, G > 1."""
    from oracle.matrix_form import ssd_matrix_form
    for L in (1, 2, 7, 64):
        d = small_inputs(L=L, seed=11 + L)
        y, f = fwd(*[d[k] for k in KEYS])
        y2, f2 = ssd_matrix_form(*[d[k] for k in KEYS])
        assert rel(y, y2) < 1e-12 and rel(f, f2) < 1e-12, ("matrix form", L, rel(y, y2), rel(f, f2))
    d = small_inputs(b=2, L=50, seed=3)
    sq, ns = si.seq_idx_from_lengths([[1, 16, 9, 24], [17, 33]])
    y, f = fwd(*[d[k] for k in KEYS], seq_idx=sq, num_seqs=ns)
    y2, f2 = ssd_matrix_form(*[d[k] for k in KEYS], seq_idx=sq, num_seqs=ns)
    assert rel(y, y2) < 1e-12 and rel(f, f2) < 1e-12, ("matrix form packed", rel(y, y2), rel(f, f2))
    d = small_inputs(b=1, L=256, H=2, P=2, N=3, G=1, seed=5)
    y, f = fwd(*[d[k] for k in KEYS])
    y2, f2 = ssd_matrix_form(*[d[k] for k in KEYS])
    assert rel(y, y2) < 1e-12 and rel(f, f2) < 1e-12, ("matrix form T=256", rel(y, y2))


def pin_geometric_closed_form(fwd):
    """P = N = 1, B = C = x = 1, constant dt and A: h_t = a^{t+1} h0 + dt (1 - a^{t+1}) / (1 - a),
    y_t = h_t + D."""
    T, dtv, Av, h0v, Dv = 200, 0.05, -3.0, 0.7, 0.25
    a = math.exp(dtv * np.float32(Av))
    one = torch.ones(1, T, 1, 1)
    y, f = fwd(one, torch.full((1, T, 1), dtv), torch.tensor([Av]), one, one,
               torch.tensor([Dv]), torch.full((1, 1, 1, 1), h0v))
    dt32 = float(np.float32(dtv))
    a = math.exp(dt32 * float(np.float32(Av)))
    t = np.arange(T)
    h = a ** (t + 1) * np.float32(h0v) + dt32 * (1 - a ** (t + 1)) / (1 - a)
    want = h + float(np.float32(Dv))
    assert np.allclose(y.ravel(), want, rtol=1e-12, atol=1e-13), ("geometric", np.abs(y.ravel() - want).max())
    assert abs(f.ravel()[0] - h[-1]) < 1e-12


def pin_unit_decay_is_linear_attention(fwd):
    """A = 0 => a = 1 => y = tril(C B^T) (dt * x) + D x (causal linear attention)."""
    d = small_inputs(b=1, L=33, H=2, P=3, N=4, G=1, seed=21, h0_std=0.0)
    d["A"] = torch.zeros_like(d["A"])
    y, _ = fwd(*[d[k] for k in KEYS])
    x, dt, B, C, D = (np.asarray(d[k].double()) for k in ("x", "dt", "B", "C", "D"))
    for h in range(2):
        K = np.tril(C[0, :, 0] @ B[0, :, 0].T)
        want = K @ (dt[0, :, h, None] * x[0, :, h]) + D[h] * x[0, :, h]
        assert rel(y[0, :, h], want) < 1e-12, ("linear attention", h)


def pin_zero_decay_every_token_alone(fwd):
    """Every token its own packed sequence => a_t = 0 for t > 0:
    y_t = (C_t . B_t) dt_t x_t + D x_t, final state of sequence t = dt_t x_t B_t^T."""
    d = small_inputs(b=1, L=20, H=2, P=3, N=4, G=1, seed=8, h0_std=0.0)
    sq = torch.arange(20, dtype=torch.int32).view(1, 20)
    y, f = fwd(*[d[k] for k in KEYS], seq_idx=sq, num_seqs=20)
    x, dt, B, C, D = (np.asarray(d[k].double()) for k in ("x", "dt", "B", "C", "D"))
    for h in range(2):
        cb = np.sum(C[0, :, 0] * B[0, :, 0], axis=1)
        want = (cb * dt[0, :, h])[:, None] * x[0, :, h] + D[h] * x[0, :, h]
        assert rel(y[0, :, h], want) < 1e-12
        for t in range(20):
            st = dt[0, t, h] * np.outer(x[0, t, h], B[0, t, 0])
            assert rel(f[t, h], st) < 1e-12


def pin_rank_bound(fwd):
    """The map x -> y is N-semiseparable: every block M[j0:j1, i0:i1] strictly
    below the diagonal (i1 <= j0) has rank <= N; generic inputs reach N."""
    T, N = 24, 3
    d = small_inputs(b=1, L=T, H=1, P=1, N=N, G=1, seed=4, h0_std=0.0, with_D=False)
    M = np.zeros((T, T))
    for i in range(T):
        x = torch.zeros(1, T, 1, 1)
        x[0, i, 0, 0] = 1.0
        y, _ = fwd(x, d["dt"], d["A"], d["B"], d["C"], None, None)
        M[:, i] = y[0, :, 0, 0]
    assert np.allclose(np.triu(M, 1), 0.0), "not causal"
    for j0 in range(1, T):
        blk = M[j0:, :j0]
        s = np.linalg.svd(blk, compute_uv=False)
        tol = 1e-9 * max(s[0], 1e-300)
        r = int(np.sum(s > tol))
        assert r <= N, ("rank", j0, r)
        if min(blk.shape) >= N and j0 >= N and T - j0 >= N:
            assert r == N, ("rank below N", j0, r)


def pin_chunk_size_invariance(fwd):
    """The literal four chunked steps equal the oracle for every chunk size,
    including Q = 1 (pure recurrence) and Q = T (pure quadratic form)."""
    from oracle.chunked import ssd_chunked
    d = small_inputs(b=2, L=67, H=4, P=3, N=5, G=2, seed=13)
    y, f = fwd(*[d[k] for k in KEYS])
    for Q in (1, 3, 16, 64, 67):
        y2, f2 = ssd_chunked(*[d[k] for k in KEYS], chunk_size=Q)
        assert rel(y2, y) < 1e-12 and rel(f2, f) < 1e-12, ("chunked", Q, rel(y2, y), rel(f2, f))
    sq, ns = si.seq_idx_from_lengths([[5, 16, 16, 30], [64, 3]])
    y, f = fwd(*[d[k] for k in KEYS], seq_idx=sq, num_seqs=ns)
    for Q in (1, 4, 16, 32, 67):
        y2, f2 = ssd_chunked(*[d[k] for k in KEYS], seq_idx=sq, num_seqs=ns, chunk_size=Q)
        assert rel(y2, y) < 1e-12 and rel(f2, f) < 1e-12, ("chunked packed", Q, rel(y2, y), rel(f2, f))


def pin_packing_equivalence(fwd):
    """A packed row equals independent runs of its sequences (zero initial
    state each) concatenated; per-sequence final states equal each run's."""
    d = small_inputs(b=1, L=45, H=4, P=3, N=5, G=2, seed=17, h0_std=0.0)
    lens = [7, 1, 16, 21]
    sq, ns = si.seq_idx_from_lengths([lens])
    y, f = fwd(*[d[k] for k in KEYS], seq_idx=sq, num_seqs=ns)
    t0 = 0
    for s, n in enumerate(lens):
        part = {k: (v[:, t0:t0 + n] if k in ("x", "dt", "B", "C") else v) for k, v in d.items()}
        yp, fp = fwd(*[part[k] for k in KEYS])
        assert rel(y[:, t0:t0 + n], yp) < 1e-12, ("packed y", s)
        assert rel(f[s], fp[0]) < 1e-12, ("packed final", s)
        t0 += n


def pin_state_carry_and_linearity(fwd):
    """run(0:L) == run(0:k) then run(k:L) started from the first part's final
    state; and y(x, h0) = y(x, 0) + y(0, h0)."""
    d = small_inputs(b=2, L=41, seed=23)
    y, f = fwd(*[d[k] for k in KEYS])
    k = 19
    a = {kk: (v[:, :k] if kk in ("x", "dt", "B", "C") else v) for kk, v in d.items()}
    b_ = {kk: (v[:, k:] if kk in ("x", "dt", "B", "C") else v) for kk, v in d.items()}
    ya, fa = fwd(*[a[kk] for kk in KEYS])
    b_["initial_states"] = torch.from_numpy(fa).float()
    yb, fb = fwd(*[b_[kk] for kk in KEYS])
    # the carried state is rounded to fp32 on the way back in
    assert rel(np.concatenate([ya, yb], axis=1), y) < 1e-6
    assert rel(fb, f) < 1e-6
    z = dict(d)
    z["initial_states"] = None
    y_x, _ = fwd(*[z[kk] for kk in KEYS])
    z = dict(d)
    z["x"] = torch.zeros_like(d["x"])
    y_h, _ = fwd(*[z[kk] for kk in KEYS])
    assert rel(y_x + y_h, y) < 1e-12, "linearity"


def pin_initial_state_decay(fwd):
    """x = 0: y_t = (a_0 ... a_t) C_t h0^T (the state before token 0 decays by a_0)."""
    d = small_inputs(b=1, L=30, H=2, P=3, N=4, G=1, seed=29, with_D=False)
    d["x"] = torch.zeros_like(d["x"])
    y, f = fwd(*[d[k] for k in KEYS])
    dt, A, C, h0 = (np.asarray(d[k].double()) for k in ("dt", "A", "C", "initial_states"))
    for h in range(2):
        z = np.exp(np.cumsum(dt[0, :, h] * A[h]))
        want = z[:, None] * (C[0, :, 0] @ h0[0, h].T)
        assert rel(y[0, :, h], want) < 1e-12
        assert rel(f[0, h], z[-1] * h0[0, h]) < 1e-12


def pin_skip_only(fwd):
    """B = 0 and h0 = 0: the state stays zero and y = D x exactly."""
    d = small_inputs(b=1, L=12, seed=31, h0_std=0.0)
    d["B"] = torch.zeros_like(d["B"])
    y, f = fwd(*[d[k] for k in KEYS])
    x, D = np.asarray(d["x"].double()), np.asarray(d["D"].double())
    assert np.array_equal(y, x * D[None, None, :, None])
    assert not f.any()


def pin_grouping(fwd):
    """G groups == G = H with each head given its group's B/C, group of head h
    = h // (H/G) (contiguous heads share B/C); permuting heads inside a group
    permutes the outputs."""
    d = small_inputs(b=1, L=25, H=6, P=2, N=3, G=2, seed=37)
    y, f = fwd(*[d[k] for k in KEYS])
    e = dict(d)
    idx = torch.tensor([h // 3 for h in range(6)])
    e["B"] = d["B"][:, :, idx].contiguous()
    e["C"] = d["C"][:, :, idx].contiguous()
    y2, f2 = fwd(*[e[k] for k in KEYS])
    assert rel(y2, y) < 1e-14 and rel(f2, f) < 1e-14, "group expansion"
    perm = torch.tensor([2, 0, 1, 5, 3, 4])
    p = dict(d)
    for k in ("x", "dt"):
        p[k] = d[k][:, :, perm].contiguous()
    p["A"], p["D"] = d["A"][perm].contiguous(), d["D"][perm].contiguous()
    p["initial_states"] = d["initial_states"][:, perm].contiguous()
    y3, f3 = fwd(*[p[k] for k in KEYS])
    assert rel(y3, y[:, :, perm.numpy()]) < 1e-14 and rel(f3, f[:, perm.numpy()]) < 1e-14


ALL_PINS = [pin_golden, pin_matrix_form, pin_geometric_closed_form, pin_unit_decay_is_linear_attention,
            pin_zero_decay_every_token_alone, pin_rank_bound, pin_chunk_size_invariance,
            pin_packing_equivalence, pin_state_carry_and_linearity, pin_initial_state_decay,
            pin_skip_only, pin_grouping]
