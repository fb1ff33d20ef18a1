"""Parity of the CUDA backward (``ssd_bwd``) with the fp64 backward oracle.

The cases of the host emulation (``test_bwd_emu_cpu.py``) run here compiled
by nvcc on the GPU, plus sizes only a GPU finishes quickly: a mid-size bf16
problem and a packed one compared in full, and the benchmark's c1 layout
(b 8, L 2048, H 80, P 64, N 128, bf16) at full size compared on one batch
row: every gradient of a row except dA and dD depends on that row's inputs
only, and dA, dD (sums over rows) are compared at the smaller sizes.  bf16
calls at headdim 64, dstate 128 without a gate run the tensor-core kernels
(k_bwd_state_walk_tc, k_bwd_chunk_tc); the others the CUDA-core ones, so
both are held to the same tolerances here."""
import numpy as np
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
import oracle
from bwd_cases import (CASES, CONV_CASES, KEYS, RANDOM_SEEDS, case_inputs, compare, conv_case_inputs, conv_compare,
                       dfinal_like, dy_like, inputs, oracle_bwd, random_case)
from oracle import block

pytestmark = pytest.mark.gpu


def _gpu_bwd(d, dy, dfinal, chunk=0):
    c = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    g = ssd.bwd(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], dy.cuda(), initial_states=c["initial_states"],
                seq_idx=c.get("seq_idx"), dfinal_states=None if dfinal is None else dfinal.cuda(), chunk_size=chunk,
                want_dD=True, want_dinitial_states=True, z=c.get("z"))
    torch.cuda.synchronize()
    out = {k: (None if v is None else v.cpu().numpy()) for k, v in g.items()}
    out["dh0"] = out.pop("dinitial_states")
    return out


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(case):
    d, dy, dfinal, chunk = case_inputs(case)
    out = _gpu_bwd(d, dy, dfinal, chunk)
    compare(out, oracle_bwd(d, dy, dfinal))
    if d["initial_states"] is None:
        b, H, P, N = d["x"].shape[0], d["x"].shape[2], d["x"].shape[3], d["B"].shape[3]
        ref0 = oracle_bwd(dict(d, initial_states=torch.zeros(b, H, P, N)), dy, dfinal)
        compare(out, ref0, keys=("dh0",))


def test_backward_is_deterministic():
    d, dy, dfinal, _ = case_inputs(CASES[1])
    first = _gpu_bwd(d, dy, dfinal)
    second = _gpu_bwd(d, dy, dfinal)
    for k in KEYS:
        assert np.array_equal(first[k], second[k]), k


@pytest.mark.parametrize("packed", [False, True], ids=["dense", "packed"])
def test_backward_mid_size(packed):
    b, L, H, P, N, G = (2, 1024, 8, 64, 128, 1) if not packed else (2, 1024, 4, 64, 128, 2)
    d = inputs(b, L, H, P, N, G, "bf16", h0=0.0 if packed else 0.2, packed=(32, 400) if packed else None, seed=77)
    dy = dy_like(b, L, H, P, torch.bfloat16, 78)
    dfinal = None if packed else dfinal_like(b, H, P, N, 79)
    compare(_gpu_bwd(d, dy, dfinal), oracle_bwd(d, dy, dfinal))


def test_backward_c1_layout_one_row():
    b, L, H, P, N, G = 8, 2048, 80, 64, 128, 1
    d = inputs(b, L, H, P, N, G, "bf16", h0=0.1, seed=1001)
    dy = dy_like(b, L, H, P, torch.bfloat16, 5)
    dfinal = dfinal_like(b, H, P, N, 6)
    out = _gpu_bwd(d, dy, dfinal)
    row = {k: (v[:1] if isinstance(v, torch.Tensor) and k not in ("A", "D") else v) for k, v in d.items()}
    ref = oracle_bwd(row, dy[:1], dfinal[:1])
    got = {k: out[k][:1] for k in ("dx", "ddt", "dB", "dC", "dh0")}
    compare(got, ref, keys=("dx", "ddt", "dB", "dC", "dh0"))


def test_autograd_function_routes_through_the_library():
    d, dy, dfinal, _ = case_inputs(CASES[1])
    c = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    leaves = {k: c[k].clone().requires_grad_(True) for k in ("x", "dt", "A", "B", "C", "D", "initial_states")}
    y, fin = ssd.ssd_chunked(leaves["x"], leaves["dt"], leaves["A"], leaves["B"], leaves["C"], leaves["D"],
                             chunk_size=64, initial_states=leaves["initial_states"])
    loss = (y.double() * dy.cuda().double()).sum() + (fin.double() * dfinal.cuda().double()).sum()
    loss.backward()
    ref = oracle_bwd(d, dy, dfinal)
    got = {"dx": leaves["x"].grad, "ddt": leaves["dt"].grad, "dA": leaves["A"].grad, "dB": leaves["B"].grad,
           "dC": leaves["C"].grad, "dD": leaves["D"].grad, "dh0": leaves["initial_states"].grad}
    compare({k: v.float().cpu().numpy() for k, v in got.items()}, ref)


@pytest.mark.parametrize("cuts", [[0, 333, 700], [0, 64, 65, 700]], ids=["2_ranks", "3_ranks"])
def test_simulated_seqpar_backward_matches_the_whole_sequence(cuts):
    """The exchange of ``seqpar.bwd_seqpar`` with the library's kernels, ranks
    simulated in one process (gathers done by stacking).  The states crossing
    ranks come from the fp32 forward, so the bound is ten times the
    single-call one."""
    from mamba_ssd_chunked_03_b200 import seqpar
    import ssd_inputs as si
    b, L, H, P, N = 2, 700, 4, 64, 128
    d = si.make_inputs(si.SSDShape("split_bwd", b, L, H, P, N, 2, 64, "f32", h0_std=0.3, seed=23))
    dy = dy_like(b, L, H, P, torch.float32, 31)
    dfinal = dfinal_like(b, H, P, N, 31)
    ref = oracle_bwd(d, dy, dfinal)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    ops = seqpar.LibraryOps
    spans = list(zip(cuts[:-1], cuts[1:]))
    parts = [{k: (g[k][:, lo:hi].contiguous() if k in ("x", "dt", "B", "C") else g[k]) for k in g} for lo, hi in spans]
    dys = [dy[:, lo:hi].contiguous().cuda() for lo, hi in spans]
    summ = [seqpar.local_summary(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], 64) for p in parts]
    S, Dk = torch.stack([s for s, _ in summ]), torch.stack([k for _, k in summ])
    shape = (b, H, P, N)
    h_in = [seqpar.carry_in(S, Dk, g["initial_states"], r, shape) for r in range(len(parts))]
    T = [ops.adjoint_summary(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], dys[r]) for r, p in enumerate(parts)]
    R = len(parts)
    out = []
    for r, p in enumerate(parts):
        after = list(range(R - 1, r, -1))
        lam = ops.state_fold(torch.stack([T[k] for k in after]) if after else None,
                             torch.stack([Dk[k] for k in after]) if after else None, dfinal.cuda(), len(after), shape)
        out.append(ops.local_backward(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], dys[r], h_in[r], lam))
    torch.cuda.synchronize()
    got = {k: torch.cat([o[k] for o in out], dim=1).cpu().numpy() for k in ("dx", "ddt", "dB", "dC")}
    got["dA"] = sum(o["dA"] for o in out).cpu().numpy()
    got["dD"] = sum(o["dD"] for o in out).cpu().numpy()
    got["dh0"] = out[0]["dinitial_states"].cpu().numpy()
    compare(got, ref, keys=("dx", "ddt", "dA", "dB", "dC", "dD", "dh0"), rel_l2=1e-4)


def test_autograd_function_through_the_gate():
    """ssd_chunked with a gate z: y * SiLU(z) forward, dz and the SSD's
    gradients backward."""
    d, dy, _, _ = case_inputs(next(c for c in CASES if c[0] == "gated_f32_ragged_Q16"))
    c = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    leaves = {k: c[k].clone().requires_grad_(True) for k in ("x", "dt", "A", "B", "C", "D", "initial_states", "z")}
    y, _ = ssd.ssd_chunked(leaves["x"], leaves["dt"], leaves["A"], leaves["B"], leaves["C"], leaves["D"],
                           chunk_size=64, initial_states=leaves["initial_states"], z=leaves["z"])
    (y.double() * dy.cuda().double()).sum().backward()
    ref = oracle_bwd(d, dy, None)
    names = {"dx": "x", "ddt": "dt", "dA": "A", "dB": "B", "dC": "C", "dD": "D", "dh0": "initial_states", "dz": "z"}
    compare({k: leaves[v].grad.float().cpu().numpy() for k, v in names.items()}, ref)


@pytest.mark.parametrize("case", CONV_CASES, ids=lambda c: c[0])
def test_conv_backward_matches_oracle(case):
    u, w, bias, dout, seq = conv_case_inputs(case)
    cu = lambda t: None if t is None else t.cuda()
    du, dw, db = ssd.conv1d_silu_bwd(cu(u), cu(w), cu(bias), cu(dout), cu(seq))
    torch.cuda.synchronize()
    conv_compare(du.cpu().numpy(), dw.cpu().numpy(), None if db is None else db.cpu().numpy(),
                 block.conv1d_silu_bwd(u, w, bias, dout, seq, with_scale=True))


def test_conv_autograd_function_routes_through_the_library():
    """fp32 u, so that the gradient handed back in u's dtype is the library's
    fp32 du unrounded (packed rows, as the forward kernel takes channels % 4)."""
    u, w, bias, dout, _ = conv_case_inputs(CONV_CASES[0])
    import ssd_inputs as si
    seq = si.seq_idx_from_lengths([[20, 1, 49], [35, 35]])[0]
    leaves = [t.cuda().requires_grad_(True) for t in (u, w, bias)]
    out = ssd.causal_conv1d_silu(leaves[0], leaves[1], leaves[2], seq.cuda())
    (out.double() * dout.cuda().double()).sum().backward()
    conv_compare(leaves[0].grad.cpu().numpy(), leaves[1].grad.cpu().numpy(), leaves[2].grad.cpu().numpy(),
                 block.conv1d_silu_bwd(u, w, bias, dout, seq, with_scale=True))


@pytest.mark.parametrize("seed", RANDOM_SEEDS)
def test_backward_on_random_shapes(seed):
    """The seeded random problems of the host emulation's sweep, on the GPU."""
    d, dy, dfinal, chunk, _ = random_case(seed)
    compare(_gpu_bwd(d, dy, dfinal, chunk), oracle_bwd(d, dy, dfinal))


def test_backward_with_ids_out_of_order():
    from bwd_cases import out_of_order_case
    d, dy, dfinal, chunk = out_of_order_case()
    compare(_gpu_bwd(d, dy, dfinal, chunk), oracle_bwd(d, dy, dfinal))


TC_EDGE = [
    # b, L, H, P, N, G, dtype, h0, dfinal, has_D, per-row lengths (packed) or None
    (1, 200, 4, 64, 128, 2, "bf16", 0.3, True, False, None),      # ragged last chunk (8 tokens), no D
    (2, 65, 2, 64, 128, 1, "bf16", 0.0, True, True, None),        # one full chunk and one token
    (1, 300, 4, 64, 128, 2, "bf16", 0.0, False, True, [[1, 63, 1, 100, 135]]),  # one-token sequences, a
                                                                   # boundary on a chunk edge
]


@pytest.mark.parametrize("case", TC_EDGE, ids=lambda c: f"L{c[1]}_H{c[2]}_G{c[5]}_{'packed' if c[10] else 'dense'}")
def test_tensor_core_backward_edge_cases(case):
    b, L, H, P, N, G, dtype, h0, with_df, has_D, lengths = case
    d = inputs(b, L, H, P, N, G, dtype, h0, None, seed=L + H, has_D=has_D, lengths=lengths)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    dy = dy_like(b, L, H, P, torch.bfloat16, L + 1)
    assert ssd.bwd_path(g["x"], dy.cuda(), g["B"], g["C"]) == "tcgen05"
    dfinal = dfinal_like(b, H, P, N, L + 2) if with_df else None
    compare(_gpu_bwd(d, dy, dfinal), oracle_bwd(d, dy, dfinal))


def test_tensor_core_dinitial_only_matches_a_full_call():
    b, L, H, P, N, G = 2, 300, 4, 64, 128, 2
    d = inputs(b, L, H, P, N, G, "bf16", 0.2, None, seed=91)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    dy = dy_like(b, L, H, P, torch.bfloat16, 92).cuda()
    full = ssd.bwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], dy, initial_states=g["initial_states"],
                   want_dinitial_states=True)
    only = ssd.bwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], dy, initial_states=g["initial_states"],
                   want_dinitial_states=True, dinitial_only=True)
    torch.cuda.synchronize()
    assert torch.equal(full["dinitial_states"], only["dinitial_states"])
