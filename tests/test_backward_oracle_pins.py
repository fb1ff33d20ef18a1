"""Pins for the backward oracle (``oracle/backward.py``).

The pages give no gradient formulas; the oracle's are derived from the
recurrence.  They are checked here against (1) PyTorch autograd of a plain
fp64 recurrence written in this file (autograd differentiates it, nothing is
retyped from the oracle), and (2) central finite differences of the C forward
oracle (``oracle.ssd_fwd``), which its own pins tie to the pages."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward
import ssd_inputs as si


def _autograd(d, dy, dfinal, z=None):
    """fp64 recurrence in PyTorch; returns the gradient of sum(dy*y) + sum(dfinal*final),
    or, with a gate z, of sum(dy * y * z * sigmoid(z)) + sum(dfinal*final) (plus dz)."""
    t64 = {k: (v.double().clone().requires_grad_(True) if isinstance(v, torch.Tensor) and k != "seq_idx" else v)
           for k, v in d.items()}
    zt = None if z is None else torch.from_numpy(np.asarray(z, dtype=np.float64)).requires_grad_(True)
    x, dt, A, B, C, D, h0 = (t64[k] for k in ("x", "dt", "A", "B", "C", "D", "initial_states"))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    grp = torch.arange(H) // (H // G)
    seq = d.get("seq_idx")
    h = torch.zeros(b, H, P, N, dtype=torch.float64) if h0 is None else h0
    ys = []
    for t in range(L):
        a = torch.exp(dt[:, t] * A[None, :])  # (b, H)
        if seq is not None and t > 0:
            a = torch.where((seq[:, t] != seq[:, t - 1])[:, None], torch.zeros_like(a), a)
        Bt, Ct = B[:, t][:, grp], C[:, t][:, grp]  # (b, H, N)
        h = a[:, :, None, None] * h + (dt[:, t, :, None, None] * x[:, t, :, :, None]) * Bt[:, :, None, :]
        y = torch.einsum("bhpn,bhn->bhp", h, Ct)
        if D is not None:
            y = y + D[None, :, None] * x[:, t]
        ys.append(y)
    yy = torch.stack(ys, 1)
    if zt is not None:
        yy = yy * zt * torch.sigmoid(zt)
    loss = (yy * torch.from_numpy(dy)).sum()
    if dfinal is not None:
        loss = loss + (h * torch.from_numpy(dfinal)).sum()
    loss.backward()
    g = lambda k: None if t64[k] is None else t64[k].grad.numpy()
    out = {"dx": g("x"), "ddt": g("dt"), "dA": g("A"), "dB": g("B"), "dC": g("C"), "dD": g("D"),
           "dh0": g("initial_states")}
    if zt is not None:
        out["dz"] = zt.grad.numpy()
    return out


CASES = [
    # b, L, H, P, N, G, h0, D, dfinal, packed
    (2, 20, 4, 3, 5, 2, 0.5, True, True, None),
    (1, 17, 2, 4, 3, 1, 0.0, False, False, None),
    (2, 24, 4, 2, 3, 4, 0.3, True, False, [[5, 1, 18], [24]]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}L{c[1]}H{c[2]}G{c[5]}{'_packed' if c[9] else ''}")
def test_backward_matches_autograd(case):
    b, L, H, P, N, G, h0s, withD, withF, packed = case
    d = si.make_inputs(si.SSDShape("bwd", b, L, H, P, N, G, 64, "f32", h0_std=h0s, seed=L * 7 + H))
    if not withD:
        d["D"] = None
    if packed is not None:
        d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths(packed)
    rng = np.random.default_rng(L)
    f32 = lambda a: a.astype(np.float32).astype(np.float64)  # the oracle widens its inputs through fp32
    dy = f32(rng.standard_normal((b, L, H, P)))
    dfinal = f32(rng.standard_normal((b, H, P, N))) if withF else None
    got = backward.ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"], dy, dfinal,
                           d.get("seq_idx"))
    want = _autograd(d, dy, dfinal)
    for k, w in want.items():
        if w is None:
            assert got[k] is None, k
            continue
        assert np.allclose(got[k], w, rtol=1e-10, atol=1e-10 * max(1.0, np.abs(w).max())), k


def test_backward_matches_finite_differences_of_the_forward_oracle():
    b, L, H, P, N, G = 1, 12, 2, 3, 4, 1
    d = si.make_inputs(si.SSDShape("bwd_fd", b, L, H, P, N, G, 64, "f32", h0_std=0.5, seed=3))
    rng = np.random.default_rng(4)
    dy = rng.standard_normal((b, L, H, P)).astype(np.float32).astype(np.float64)
    dfinal = rng.standard_normal((b, H, P, N)).astype(np.float32).astype(np.float64)
    got = backward.ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"], dy, dfinal)

    def loss(dd):
        y, f = oracle.ssd_fwd(dd["x"], dd["dt"], dd["A"], dd["B"], dd["C"], dd["D"], dd["initial_states"])
        return float((y * dy).sum() + (f * dfinal).sum())

    probes = [("A", (1,)), ("D", (0,)), ("dt", (0, 5, 1)), ("x", (0, 3, 0, 2)), ("B", (0, 7, 0, 1)),
              ("C", (0, 9, 0, 3)), ("initial_states", (0, 1, 2, 3))]
    names = {"A": "dA", "D": "dD", "dt": "ddt", "x": "dx", "B": "dB", "C": "dC", "initial_states": "dh0"}
    for key, idx in probes:
        v = float(d[key][idx])
        eps = 2.0 ** (np.floor(np.log2(max(abs(v), 1e-2))) - 10)  # a power of two: v +- eps stays exact in fp32
        plus = {k: (t.clone() if isinstance(t, torch.Tensor) else t) for k, t in d.items()}
        minus = {k: (t.clone() if isinstance(t, torch.Tensor) else t) for k, t in d.items()}
        plus[key][idx] = v + eps
        minus[key][idx] = v - eps
        fd = (loss(plus) - loss(minus)) / (2 * eps)
        an = float(got[names[key]][idx])
        assert abs(fd - an) <= 1e-4 * max(1.0, abs(an)), (key, fd, an)


@pytest.mark.parametrize("case", CASES + [(2, 200, 4, 8, 16, 2, 0.4, True, True, None),
                                          (1, 300, 2, 8, 8, 1, 0.2, True, False, [[70, 1, 100, 129]])],
                         ids=lambda c: f"b{c[0]}L{c[1]}H{c[2]}G{c[5]}{'_packed' if c[9] else ''}")
def test_c_backward_matches_the_numpy_backward(case):
    """The C backward (checkpointed recompute) agrees with the numpy one,
    which autograd and finite differences pin; L up to 300 spans several
    64-token checkpoints."""
    b, L, H, P, N, G, h0s, withD, withF, packed = case
    d = si.make_inputs(si.SSDShape("bwd_c", b, L, H, P, N, G, 64, "f32", h0_std=h0s, seed=L + H))
    if not withD:
        d["D"] = None
    if packed is not None:
        d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths(packed)
    rng = np.random.default_rng(L + 1)
    f32 = lambda a: a.astype(np.float32).astype(np.float64)
    dy = f32(rng.standard_normal((b, L, H, P)))
    dfinal = f32(rng.standard_normal((b, H, P, N))) if withF else None
    args = (d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"])
    want = backward.ssd_bwd(*args, dy, dfinal, d.get("seq_idx"))
    got = oracle.ssd_bwd(*args, dy=dy, dfinal=dfinal, seq_idx=d.get("seq_idx"))
    for k, w in want.items():
        if w is None:
            assert got[k] is None, k
            continue
        assert np.allclose(got[k], w, rtol=1e-11, atol=1e-11 * max(1.0, np.abs(w).max())), k


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}L{c[1]}H{c[2]}G{c[5]}{'_packed' if c[9] else ''}")
def test_gated_backward_matches_autograd(case):
    """The gate out = y * SiLU(z): dz and the SSD's gradients through it,
    against autograd of y * z * sigmoid(z) written out here."""
    b, L, H, P, N, G, h0s, withD, withF, packed = case
    d = si.make_inputs(si.SSDShape("bwd_gate", b, L, H, P, N, G, 64, "f32", h0_std=h0s, seed=L * 5 + H))
    if not withD:
        d["D"] = None
    if packed is not None:
        d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths(packed)
        withF = False
    rng = np.random.default_rng(L + 7)
    f32 = lambda a: a.astype(np.float32).astype(np.float64)
    dout = f32(rng.standard_normal((b, L, H, P)))
    z = f32(2.0 * rng.standard_normal((b, L, H, P)))  # both signs, well into the curved part of SiLU
    dfinal = f32(rng.standard_normal((b, H, P, N))) if withF else None
    got = backward.ssd_bwd_gated(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"], z, dout,
                                 dfinal, d.get("seq_idx"))
    want = _autograd(d, dout, dfinal, z=z)
    for k, w in want.items():
        if w is None:
            assert got[k] is None, k
            continue
        assert np.allclose(got[k], w, rtol=1e-9, atol=1e-9 * max(1.0, np.abs(w).max())), k


def test_silu_grad_is_the_derivative():
    v = np.linspace(-8.0, 8.0, 161)
    h = 1e-6
    fd = (backward.silu(v + h) - backward.silu(v - h)) / (2 * h)
    assert np.allclose(backward.silu_grad(v), fd, rtol=1e-7, atol=1e-9)
    assert backward.silu_grad(0.0) == 0.5  # s(0) = 1/2, and the v (1 - s) term vanishes


def test_one_token_closed_form():
    """L = 1, P = N = 1: y = (a h0 + dt x B) C + D x with a = exp(dt A), so by
    hand dx = (dt B C + D) dy, dB = dt x C dy, dC = h dy, dD = x dy,
    ddt = (x B + A a h0) C dy, dA = dt a h0 C dy, dh0 = a C dy (a final-state
    gradient adds dfinal times the same derivatives of h)."""
    x, dt, A, B, C, D, h0, dy, df = 0.75, 0.125, -2.0, -1.5, 0.5, 0.25, 0.625, 1.25, -0.375
    t = lambda v, shape: torch.full(shape, v, dtype=torch.float32)
    got = backward.ssd_bwd(t(x, (1, 1, 1, 1)), t(dt, (1, 1, 1)), t(A, (1,)), t(B, (1, 1, 1, 1)), t(C, (1, 1, 1, 1)),
                           t(D, (1,)), t(h0, (1, 1, 1, 1)), np.full((1, 1, 1, 1), dy), np.full((1, 1, 1, 1), df))
    a = np.exp(dt * A)
    h = a * h0 + dt * x * B
    g = C * dy + df  # dLoss/dh
    want = {"dx": dt * B * g + D * dy, "dB": dt * x * g, "dC": h * dy, "dD": x * dy,
            "ddt": x * B * g + A * a * h0 * g, "dA": dt * a * h0 * g, "dh0": a * g}
    for k, w in want.items():
        assert np.allclose(np.asarray(got[k]).ravel()[0], w, rtol=1e-14, atol=0), (k, got[k], w)
