"""The recurrent (decode) step ``ssd_step`` against the oracle.

One step is the oracle's forward over a single token with the state as the
initial state: y is that token's output and the state becomes the final
state.  Also, T steps in a row must reproduce the chunked forward over the
same T tokens (outputs token by token and the final state)."""
import numpy as np
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
import oracle
import ssd_inputs as si
from gpu_util import TOL, rel_l2, state_err

pytestmark = pytest.mark.gpu

STEP_CASES = [
    # b, H, P, N, G, dtype
    (3, 4, 64, 128, 2, "bf16"),
    (2, 6, 32, 64, 3, "f32"),
    (1, 8, 64, 256, 1, "bf16"),
    (2, 4, 16, 16, 2, "f32"),
    (5, 80, 64, 128, 1, "bf16"),   # the c1 head layout
]


def _step_inputs(b, H, P, N, G, dtype, seed, with_d=True):
    shape = si.SSDShape("step", b, 1, H, P, N, G, 64, dtype, h0_std=0.5, seed=seed)
    d = si.make_inputs(shape)
    if not with_d:
        d["D"] = None
    return d


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: "b{}_H{}_P{}_N{}_G{}_{}".format(*c))
@pytest.mark.parametrize("with_d", [True, False])
def test_step_matches_the_oracle(case, with_d):
    b, H, P, N, G, dtype = case
    d = _step_inputs(b, H, P, N, G, dtype, seed=b * 100 + N + with_d, with_d=with_d)
    yr, fr = oracle.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"])
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    state = g["initial_states"].clone()
    y = ssd.step(g["x"][:, 0], g["dt"][:, 0], g["A"], g["B"][:, 0], g["C"][:, 0], g["D"], state)
    torch.cuda.synchronize()
    y = y.float().cpu().numpy().astype(np.float64)
    f = state.cpu().numpy().astype(np.float64)
    assert rel_l2(y, yr[:, 0]) <= TOL[dtype], rel_l2(y, yr[:, 0])
    assert state_err(f, fr) <= TOL[dtype], state_err(f, fr)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_steps_reproduce_the_chunked_forward(dtype):
    b, T, H, P, N, G = 2, 150, 4, 64, 128, 2
    shape = si.SSDShape("steps", b, T, H, P, N, G, 64, dtype, h0_std=0.3, seed=7)
    d = si.make_inputs(shape)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    y_fwd, f_fwd = ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=64,
                           initial_states=g["initial_states"])
    state = g["initial_states"].clone()
    ys = [ssd.step(g["x"][:, t].contiguous(), g["dt"][:, t].contiguous(), g["A"], g["B"][:, t].contiguous(),
                   g["C"][:, t].contiguous(), g["D"], state) for t in range(T)]
    torch.cuda.synchronize()
    y_steps = torch.stack(ys, dim=1).float().cpu().numpy().astype(np.float64)
    ref = y_fwd.float().cpu().numpy().astype(np.float64)
    tol = 2 * TOL[dtype]  # two roundings of y in bf16, one per side
    assert rel_l2(y_steps, ref) <= tol, rel_l2(y_steps, ref)
    assert state_err(state.cpu().numpy().astype(np.float64), f_fwd.cpu().numpy().astype(np.float64)) <= tol
