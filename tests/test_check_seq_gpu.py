"""SSD_FLAG_CHECK_SEQ on the GPU: ``fwd(check_seq=True)`` copies seq_idx to
the host and checks the packing precondition ("Transformers与SSMs的隐藏联系",
section 4.2: ids per sequence, non-decreasing along a row, no sequence in two
rows, ids in [0, num_seqs)) before anything is launched.  Valid ids run and
match the oracle; each violation raises SSDError(SSD_ERR_INVALID_ARG) and
leaves the outputs untouched."""
import numpy as np
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
import ssd_inputs as si
from gpu_util import TOL, rel_l2, run_oracle, state_err, to_dev

pytestmark = pytest.mark.gpu


def _packed(rows, dtype="bf16", Q=64, seed=5):
    b = len(rows)
    L = max(len(r) for r in rows)
    s = si.SSDShape("chk", b, L, 4, 64, 128, 2, Q, dtype, seed=seed)
    d = si.make_inputs(s)
    d["seq_idx"] = torch.tensor(rows, dtype=torch.int32)
    d["num_seqs"] = max(0, int(d["seq_idx"].max())) + 1
    d["initial_states"] = None
    return d


def _run(d, num_seqs):
    g = to_dev(d)
    y = torch.full_like(g["x"], 7.0)
    f = torch.full((num_seqs, g["x"].shape[2], 64, 128), 7.0, device="cuda")
    ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=64, seq_idx=g["seq_idx"],
            num_seqs=num_seqs, y=y, final_states=f, check_seq=True)
    torch.cuda.synchronize()
    return y, f


def _ids(lengths, first=0):
    return sum(([first + i] * n for i, n in enumerate(lengths)), [])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_valid_ids_run_and_match_the_oracle(dtype):
    rows = [_ids([37, 64, 27]), _ids([100, 28], first=3)]
    d = _packed(rows, dtype)
    y, f = _run(d, 5)
    yr, fr = run_oracle(d)
    y = y.float().cpu().numpy().astype(np.float64)
    f = f.cpu().numpy().astype(np.float64)
    assert rel_l2(y, yr) <= TOL[dtype], rel_l2(y, yr)
    assert state_err(f, fr) <= TOL[dtype], state_err(f, fr)


BAD = {
    "decreasing_along_a_row": ([_ids([40, 40, 48], first=0)[::-1]], 3),
    "id_out_of_range": ([_ids([64, 64])], 1),
    "negative_id": ([[-1] * 8 + [0] * 120], 1),
    "id_in_two_rows": ([_ids([64, 64]), _ids([128], first=1)], 2),
}


@pytest.mark.parametrize("name", sorted(BAD))
def test_violations_raise_before_any_launch(name):
    rows, num_seqs = BAD[name]
    d = _packed(rows)
    with pytest.raises(ssd.SSDError) as e:
        _run(d, num_seqs)
    assert e.value.status == ssd.SSD_ERR_INVALID_ARG
    # nothing ran: the preset outputs are untouched
    g = to_dev(d)
    y = torch.full_like(g["x"], 7.0)
    with pytest.raises(ssd.SSDError):
        ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=64, seq_idx=g["seq_idx"],
                num_seqs=num_seqs, y=y, check_seq=True)
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
