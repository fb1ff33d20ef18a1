"""Sequence parallelism on one GPU: the two state kernels against their
definitions, and a sequence split into ranges (ranks simulated in one
process, the gather done by stacking) against the oracle over the whole."""
import numpy as np
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
from mamba_ssd_chunked_03_b200 import seqpar
import oracle
import ssd_inputs as si
from gpu_util import rel_l2, state_err

pytestmark = pytest.mark.gpu


def test_total_decay_kernel():
    g = torch.Generator().manual_seed(3)
    dt = torch.rand(3, 1000, 5, generator=g) * 0.01
    A = -torch.rand(5, generator=g) * 2
    got = ssd.total_decay(dt.cuda(), A.cuda()).cpu().double().numpy()
    want = np.exp(A.double().numpy()[None, :] * dt.double().numpy().sum(axis=1))
    assert np.abs(got - want).max() <= 1e-6 * np.abs(want).max()


@pytest.mark.parametrize("rank", [0, 1, 3])
@pytest.mark.parametrize("with_h0", [True, False])
def test_state_fold_kernel(rank, with_h0):
    g = torch.Generator().manual_seed(rank + 10 * with_h0)
    R, b, H, P, N = 4, 2, 3, 16, 24
    S = torch.randn(R, b, H, P, N, generator=g)
    Dk = torch.rand(R, b, H, generator=g)
    h0 = torch.randn(b, H, P, N, generator=g) if with_h0 else None
    got = ssd.state_fold(S.cuda(), Dk.cuda(), None if h0 is None else h0.cuda(), rank, (b, H, P, N))
    want = np.zeros((b, H, P, N)) if h0 is None else h0.double().numpy()
    for k in range(rank):
        want = Dk[k].double().numpy()[:, :, None, None] * want + S[k].double().numpy()
    assert np.abs(got.cpu().double().numpy() - want).max() <= 1e-5 * max(1.0, np.abs(want).max())


@pytest.mark.parametrize("cuts", [[0, 333, 700], [0, 250, 500, 700], [0, 64, 65, 700]])
def test_simulated_split_matches_the_whole_sequence(cuts):
    shape = si.SSDShape("split_seq", 2, 700, 4, 64, 128, 2, 64, "bf16", h0_std=0.3, seed=21)
    d = si.make_inputs(shape)
    yw, fw = oracle.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"])
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    parts = [{k: (g[k][:, lo:hi].contiguous() if k in ("x", "dt", "B", "C") else g[k]) for k in g}
             for lo, hi in zip(cuts[:-1], cuts[1:])]
    summaries = [seqpar.local_summary(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], 64) for p in parts]
    S = torch.stack([s for s, _ in summaries])
    Dk = torch.stack([dk for _, dk in summaries])
    ys, f = [], None
    for r, p in enumerate(parts):
        h_in = seqpar.carry_in(S, Dk, g["initial_states"], r, tuple(S.shape[1:]))
        y, f = ssd.fwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], chunk_size=64, initial_states=h_in)
        ys.append(y.float().cpu())
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1).double().numpy()
    assert rel_l2(y, yw) <= 1e-2, rel_l2(y, yw)
    assert state_err(f.cpu().double().numpy(), fw) <= 1e-2
