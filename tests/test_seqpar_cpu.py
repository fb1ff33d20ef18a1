"""Sequence parallelism on the CPU: the composition rule the split relies on,
pinned on the oracle, and the exchange logic of ``seqpar.fwd_seqpar`` and
``seqpar.bwd_seqpar`` on two and three gloo ranks (with the per-rank
operations done by the oracle, since these ranks have no GPU).

The rule: over a contiguous token range the recurrence is affine in the
state, h_out = D h_in + S, with S the range's end state from a zero state and
D = exp(A sum dt); a sequence split into ranges and carried through them
equals the sequence run whole."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from oracle import backward, block
import ssd_inputs as si

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _split(d, lo, hi):
    return {k: (v[:, lo:hi].contiguous() if k in ("x", "dt", "B", "C") else v) for k, v in d.items()}


def _whole(d):
    return oracle.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"])


class OracleOps:
    """The per-rank operations of seqpar, on the oracle (fp64)."""

    @staticmethod
    def local_forward(x, dt, A, B, C, D, chunk_size, initial_states, z=None):
        y, f = oracle.ssd_fwd(x, dt, A, B, C, D, initial_states)
        if z is not None:
            y = block.gate(y, z)
        return torch.from_numpy(y), torch.from_numpy(f).float()

    @staticmethod
    def total_decay(dt, A):
        s = dt.double().sum(dim=1)  # (b, H)
        return torch.exp(A.double()[None, :] * s).float()

    @staticmethod
    def state_fold(states, decays, initial_states, rank, shape):
        h = torch.zeros(shape, dtype=torch.float64) if initial_states is None else initial_states.double().clone()
        for k in range(rank):
            h = decays[k].double()[:, :, None, None] * h + states[k].double()
        return h.float()

    @staticmethod
    def local_backward(x, dt, A, B, C, D, dy, initial_states, dfinal_states, z=None):
        b, _, H, P = x.shape
        h0 = initial_states if initial_states is not None else torch.zeros(b, H, P, B.shape[3])
        if z is None:
            g = oracle.ssd_bwd(x, dt, A, B, C, D, h0, dy, dfinal_states, None)
        else:
            g = backward.ssd_bwd_gated(x, dt, A, B, C, D, h0, z, dy, dfinal_states, None,
                                       backward_fn=oracle.ssd_bwd)
        out = {k: (None if v is None else torch.from_numpy(np.asarray(v)).float()) for k, v in g.items()
               if k != "dh0"}
        out["dinitial_states"] = torch.from_numpy(g["dh0"]).float()
        return out


@pytest.mark.parametrize("cuts", [[0, 90, 91, 200], [0, 64, 128, 200], [0, 200]])
def test_split_sequence_composes_to_the_whole(cuts):
    shape = si.SSDShape("sp", 2, 200, 3, 8, 8, 1, 64, "f32", h0_std=0.5, seed=5)
    d = si.make_inputs(shape)
    yw, fw = _whole(d)
    h = d["initial_states"].double().numpy()
    ys = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        p = _split(d, lo, hi)
        # the range's summary: end state from zero, total decay
        _, S = oracle.ssd_fwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], None)
        Dk = np.exp(p["A"].double().numpy()[None, :] * p["dt"].double().numpy().sum(axis=1))
        y, f = oracle.ssd_fwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], torch.from_numpy(h).float())
        ys.append(y)
        h_next = Dk[:, :, None, None] * h + S
        # the carried state is the range's true end state
        assert np.abs(h_next - f).max() <= 1e-5 * max(1.0, np.abs(f).max())
        h = h_next
    y = np.concatenate(ys, axis=1)
    assert np.abs(y - yw).max() <= 1e-5 * max(1.0, np.abs(yw).max())
    assert np.abs(h - fw).max() <= 1e-5 * max(1.0, np.abs(fw).max())


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gate(seed=22):
    return 2.0 * torch.randn(2, 200, 3, 8, generator=torch.Generator().manual_seed(seed))


def _rank_main(rank, world, port, cuts, out, gated=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mamba_ssd_chunked_03_b200 import seqpar
        shape = si.SSDShape("sp", 2, 200, 3, 8, 8, 1, 64, "f32", h0_std=0.5, seed=5)
        d = si.make_inputs(shape)
        p = _split(d, cuts[rank], cuts[rank + 1])
        z = _gate()[:, cuts[rank]:cuts[rank + 1]].contiguous() if gated else None
        y, f = seqpar.fwd_seqpar(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], 64, d["initial_states"],
                                 ops=OracleOps, z=z)
        out[rank] = (np.asarray(y), np.asarray(f))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts,gated", [([0, 117, 200], False), ([0, 64, 65, 200], False), ([0, 90, 200], True)],
                         ids=["2_ranks", "3_ranks", "2_ranks_gated"])
def test_fwd_seqpar_gloo_ranks(cuts, gated):
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, cuts, out, gated)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        shape = si.SSDShape("sp", 2, 200, 3, 8, 8, 1, 64, "f32", h0_std=0.5, seed=5)
        yw, fw = _whole(si.make_inputs(shape))
        if gated:
            yw = block.gate(yw, _gate())
        y = np.concatenate([out[r][0] for r in range(world)], axis=1)
        assert np.abs(y - yw).max() <= 1e-5 * max(1.0, np.abs(yw).max())
        assert np.abs(out[world - 1][1] - fw).max() <= 1e-5 * max(1.0, np.abs(fw).max())


def _bwd_data(gated=False):
    shape = si.SSDShape("sp", 2, 200, 3, 8, 8, 1, 64, "f32", h0_std=0.5, seed=5)
    d = si.make_inputs(shape)
    g = torch.Generator().manual_seed(21)
    dy = torch.randn(2, 200, 3, 8, generator=g)
    dfinal = torch.randn(2, 3, 8, 8, generator=g)
    d["z"] = 2.0 * torch.randn(2, 200, 3, 8, generator=g) if gated else None
    return d, dy, dfinal


def _bwd_rank_main(rank, world, port, cuts, out, gated=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mamba_ssd_chunked_03_b200 import seqpar
        d, dy, dfinal = _bwd_data(gated)
        lo, hi = cuts[rank], cuts[rank + 1]
        p = _split(d, lo, hi)
        z = None if d["z"] is None else d["z"][:, lo:hi].contiguous()
        g = seqpar.bwd_seqpar(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], dy[:, lo:hi].contiguous(), 64,
                              d["initial_states"], dfinal, ops=OracleOps, z=z)
        out[rank] = {k: (None if v is None else v.numpy()) for k, v in g.items()}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts,gated", [([0, 117, 200], False), ([0, 64, 65, 200], False), ([0, 90, 200], True)],
                         ids=["2_ranks", "3_ranks", "2_ranks_gated"])
def test_bwd_seqpar_gloo_ranks(cuts, gated):
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_bwd_rank_main, args=(r, world, port, cuts, out, gated)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        d, dy, dfinal = _bwd_data(gated)
        args = (d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"])
        ref = (oracle.ssd_bwd(*args, dy, dfinal, None) if not gated else
               backward.ssd_bwd_gated(*args, d["z"], dy, dfinal, None, backward_fn=oracle.ssd_bwd))
        tol = lambda w: 1e-5 * max(1.0, np.abs(w).max())
        for k in ("dx", "ddt", "dB", "dC") + (("dz",) if gated else ()):
            got = np.concatenate([out[r][k] for r in range(world)], axis=1)
            assert np.abs(got - ref[k]).max() <= tol(ref[k]), k
        for r in range(world):  # the shared parameters: every rank holds the sum
            assert np.abs(out[r]["dA"] - ref["dA"]).max() <= tol(ref["dA"])
            assert np.abs(out[r]["dD"] - ref["dD"]).max() <= tol(ref["dD"])
        assert np.abs(out[0]["dinitial_states"] - ref["dh0"]).max() <= tol(ref["dh0"])
        assert all(out[r]["dinitial_states"] is None for r in range(1, world))
