"""Failure detection on the GPU without a fault: the two-head kernel's state
hand-over between CTAs is a bounded wait.  SSD_FLAG_TEST_STALL points that
wait at a flag nothing sets, so it runs out after its 1 s limit; the kernel
then drains its copies, stores and MMAs, frees its tensor memory and exits.
The tests check that the call returns, that the timeout is reported (by
``device_status`` and by ``fwd(check_status=True)``), and that the context and
the same workspace then serve a normal call that matches the oracle."""
import time

import numpy as np
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
import ssd_inputs as si
from gpu_util import TOL, rel_l2, run_oracle, state_err, to_dev

pytestmark = pytest.mark.gpu

# 160 head pairs of 4 chunks over at most 148 persistent CTAs: pairs are
# split between CTAs, so states are handed over
SHAPE = si.SSDShape("stall", 4, 200, 80, 64, 128, 1, 64, "bf16", h0_std=0.1, seed=77)


def _call(g, ws, **kw):
    return ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=SHAPE.chunk_size,
                   initial_states=g["initial_states"], workspace=ws, **kw)


def _workspace(g):
    need = ssd.workspace_size(g["x"], g["B"], SHAPE.chunk_size)
    return torch.empty(need, dtype=torch.uint8, device="cuda")


def test_stalled_handover_times_out_and_the_next_call_is_correct():
    d = si.make_inputs(SHAPE)
    g = to_dev(d)
    assert ssd.main_kernel(g["x"], g["dt"], g["B"], SHAPE.chunk_size) == "k_ssd_fwd_pair"
    ws = _workspace(g)
    t0 = time.monotonic()
    _call(g, ws, flags=ssd.SSD_FLAG_TEST_STALL)  # asynchronous: returns SSD_OK
    st = ssd.device_status(g["x"], g["B"], SHAPE.chunk_size, ws)
    waited = time.monotonic() - t0
    assert st == ssd.SSD_ERR_TIMEOUT, st
    assert waited < 30.0, waited  # one bounded wait (1 s) per CTA, in parallel
    torch.cuda.synchronize()      # no fault: the context is still usable
    # the same stream and workspace, a normal call
    y, f = _call(g, ws)
    assert ssd.device_status(g["x"], g["B"], SHAPE.chunk_size, ws) == ssd.SSD_OK
    yr, fr = run_oracle(d)
    y = y.float().cpu().numpy().astype(np.float64)
    f = f.cpu().numpy().astype(np.float64)
    assert rel_l2(y, yr) <= TOL["bf16"], rel_l2(y, yr)
    assert state_err(f, fr) <= TOL["bf16"], state_err(f, fr)


def test_check_status_raises_on_a_timeout_and_passes_otherwise():
    g = to_dev(si.make_inputs(SHAPE))
    ws = _workspace(g)
    with pytest.raises(ssd.SSDError) as e:
        _call(g, ws, flags=ssd.SSD_FLAG_TEST_STALL, check_status=True)
    assert e.value.status == ssd.SSD_ERR_TIMEOUT
    y, _ = _call(g, ws, check_status=True)
    assert torch.isfinite(y.float()).all()
