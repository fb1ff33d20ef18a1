"""ssd_fwd_noalloc, the entry point for callers that cannot allocate device
memory when they call (for instance a plugin inside a host runtime that owns
all device memory, or a latency-critical loop that must not call cudaMalloc).

It takes the same arguments as ssd_fwd but brings its own scratch: a fixed
32 MiB device array inside the library, and it takes ssd_fwd's kernel path
when that path's workspace fits the array.  These tests call it through the C
ABI and compare it with ssd_fwd on several calls in a row (the array keeps
the previous call's contents, so a stale value would show up in a later
call), compare a tensor-core call with the oracle, and check that a problem
too large for the array is refused without touching the outputs.  This file
is collected last so that a failure here cannot hide other tests in a run
that stops at the first failure.
"""
import ctypes

import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
import ssd_inputs as si
from gpu_util import TOL, rel_l2, run_oracle, state_err, to_dev

pytestmark = pytest.mark.gpu


def _entry():
    f = ssd.lib.ssd_fwd_noalloc
    f.argtypes = [ctypes.POINTER(ssd.Args), ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _outputs(g, num_seqs):
    b, L, H, P = g["x"].shape
    N = g["B"].shape[3]
    rows = num_seqs if g.get("seq_idx") is not None else b
    y = torch.full_like(g["x"], float("nan"))
    f = torch.full((rows, H, P, N), float("nan"), device=g["x"].device, dtype=torch.float32)
    return y, f


def _noalloc(g, Q, num_seqs=None):
    y, f = _outputs(g, num_seqs)
    a = ssd.make_args(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], Q, g["initial_states"],
                      g.get("seq_idx"), num_seqs, y, f)
    st = _entry()(ctypes.byref(a), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ssd.SSD_OK, ssd.lib.ssd_status_string(st)
    torch.cuda.synchronize()
    return y, f


def _reference(g, Q, num_seqs=None):
    y, f = ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=Q,
                   initial_states=g["initial_states"], seq_idx=g.get("seq_idx"), num_seqs=num_seqs)
    torch.cuda.synchronize()
    return y, f


def _case_packed():
    s = si.SSDShape("na_packed", 1, 300, 4, 64, 64, 2, 64, "bf16", seed=21)
    d = si.make_inputs(s)
    d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths([[70, 1, 64, 165]])
    return d, s


def _case_f32():
    s = si.SSDShape("na_f32", 2, 257, 4, 32, 128, 1, 128, "f32", h0_std=0.3, seed=22)
    return si.make_inputs(s), s


def _case_bf16():
    s = si.SSDShape("na_bf16", 2, 500, 8, 64, 128, 4, 64, "bf16", h0_std=0.1, seed=23)
    return si.make_inputs(s), s


def test_calls_in_a_row_match_ssd_fwd():
    cases = [_case_packed(), _case_f32(), _case_bf16(), _case_packed()]
    for d, s in cases:
        g = to_dev(d)
        ns = d.get("num_seqs")
        y, f = _noalloc(g, s.chunk_size, ns)
        yr, fr = _reference(g, s.chunk_size, ns)
        y64, yr64 = y.double().cpu().numpy(), yr.double().cpu().numpy()
        f64, fr64 = f.double().cpu().numpy(), fr.double().cpu().numpy()
        assert rel_l2(y64, yr64) <= TOL[s.dtype], (s.name, rel_l2(y64, yr64))
        assert state_err(f64, fr64) <= TOL[s.dtype], (s.name, state_err(f64, fr64))


def test_problem_larger_than_the_scratch_is_refused():
    s = si.SSDShape("na_big", 2, 2048, 32, 64, 128, 1, 64, "bf16", seed=24)  # ~68 MB of workspace
    g = to_dev(si.make_inputs(s))
    y, f = _outputs(g, None)
    a = ssd.make_args(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], s.chunk_size, None, None, None, y, f,
                      generic=True)
    assert ssd.lib.ssd_fwd_workspace_size(ctypes.byref(a)) > 32 << 20
    st = _entry()(ctypes.byref(a), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert st == ssd.SSD_ERR_WORKSPACE
    assert bool(torch.isnan(y).all()) and bool(torch.isnan(f).all())


def test_tensor_core_path_matches_the_oracle():
    # two-head tensor-core kernel (N 128, heads per group even), ragged tail, h0
    s = si.SSDShape("na_tc", 2, 300, 8, 64, 128, 2, 64, "bf16", h0_std=0.2, seed=25)
    d = si.make_inputs(s)
    g = to_dev(d)
    a = ssd.make_args(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], s.chunk_size)
    assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) == b"tcgen05"
    yr, fr = run_oracle(d)
    for _ in range(2):  # two calls in a row on the shared array
        y, f = _noalloc(g, s.chunk_size)
        y64, f64 = y.double().cpu().numpy(), f.double().cpu().numpy()
        assert rel_l2(y64, yr) <= TOL["bf16"], rel_l2(y64, yr)
        assert state_err(f64, fr) <= TOL["bf16"], state_err(f64, fr)
