"""``ssd_fwd_host`` (the forward from and to host memory, the batch in row
pieces on two streams so that one piece's copies in overlap the previous
piece's compute and copies out) against ``ssd_fwd`` on device buffers, which
``test_parity_gpu.py`` holds to the oracle.

A piece is a forward over fewer rows, or over a token range of every row
(negative piece sizes, and the library's choice under eight rows), whose
state goes on to the next piece.  Either can change how the tensor-core path
splits the state passing among CTAs.  There the chunk states are formed from
bf16 operands, so a different split rounds the states, and through them y,
differently; a gated y on the two-head kernel is rounded to bf16 twice
(before and after the gate pass).  The comparison is therefore not bitwise:
1e-5 (relative L2) on the fp32 path, 2e-3 on the bf16 one, both well inside
the oracle tolerances (1e-5 and 1e-2).  Token pieces that do not start on a
64-token boundary move the bf16 path's chunk tiling, and are held to the
oracle's bf16 tolerance.  Only the current stream is synchronised before the
host outputs are read: the call must order its second stream's part before
it."""
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
import ssd_inputs as si

pytestmark = pytest.mark.gpu

CASES = [
    # name, shape, piece sizes: rows, or (< 0) tokens of every row; 0: the
    # library's choice (here 64-token pieces, as the batch is under 8 rows);
    # the last piece ragged for 2, 3, -64 and -100
    ("bf16_tc", si.SSDShape("host_bf16", 5, 300, 8, 64, 128, 2, 64, "bf16", h0_std=0.2, seed=5),
     [0, 1, 2, 3, 5, -64, -100]),
    ("bf16_pair_c1_heads", si.SSDShape("host_pair", 3, 256, 80, 64, 128, 1, 64, "bf16", seed=8), [0, 1]),
    ("bf16_long_split", si.SSDShape("host_long", 1, 1000, 8, 64, 128, 1, 64, "bf16", h0_std=0.2, seed=12),
     [0, -128, -100]),
    ("f32_generic", si.SSDShape("host_f32", 3, 200, 4, 16, 16, 1, 64, "f32", h0_std=0.1, seed=6), [1, 2, -64, -50]),
    ("packed_one_piece", si.SSDShape("host_packed", 2, 600, 4, 64, 128, 1, 64, "bf16", packed=(50, 300), seed=7),
     [1]),
]


def _rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / max(b.norm(), 1e-30))


@pytest.mark.parametrize("name,shape,rows_list", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("gated", [False, True], ids=["plain", "gated"])
def test_host_entry_matches_the_device_call(name, shape, rows_list, gated):
    d = si.make_inputs(shape)
    seq, ns = d.get("seq_idx"), d.get("num_seqs")
    z = None
    if gated:
        g = torch.Generator().manual_seed(shape.seed + 1)
        z = torch.randn(d["x"].shape, generator=g).to(d["x"].dtype)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    y_ref, f_ref = ssd.fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], shape.chunk_size,
                           dev["initial_states"], dev.get("seq_idx"), ns, z=None if z is None else z.cuda())
    torch.cuda.synchronize()
    y_ref, f_ref = y_ref.cpu(), f_ref.cpu()
    host = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    zh = None if z is None else z.pin_memory()
    for rows in rows_list:
        tol = 1e-5 if shape.dtype == "f32" else (1e-2 if rows < 0 and -rows % 64 else 2e-3)
        y, f = ssd.fwd_host(host["x"], host["dt"], host["A"], host["B"], host["C"], host["D"], shape.chunk_size,
                            host["initial_states"], host.get("seq_idx"), ns, z=zh, rows_per_piece=rows)
        torch.cuda.current_stream().synchronize()
        assert y.device.type == "cpu" and f.device.type == "cpu"
        assert _rel(y, y_ref) <= tol, (rows, _rel(y, y_ref))
        assert _rel(f, f_ref) <= tol, (rows, _rel(f, f_ref))


def test_host_entry_reuses_caller_buffers_and_workspace():
    """Preallocated pinned outputs and a device workspace of the size the
    library asks for are used as given, call after call."""
    shape = si.SSDShape("host_reuse", 4, 256, 8, 64, 128, 1, 64, "bf16", seed=9)
    d = si.make_inputs(shape)
    host = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    need = ssd.fwd_host_workspace_size(d["x"], d["B"], shape.chunk_size, rows_per_piece=1)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    y = torch.empty(d["x"].shape, dtype=d["x"].dtype, pin_memory=True)
    f = torch.empty(4, 8, 64, 128, dtype=torch.float32, pin_memory=True)
    outs = []
    for _ in range(3):
        y2, f2 = ssd.fwd_host(host["x"], host["dt"], host["A"], host["B"], host["C"], host["D"], 64,
                              y=y, final_states=f, rows_per_piece=1, workspace=ws)
        torch.cuda.current_stream().synchronize()
        assert y2.data_ptr() == y.data_ptr() and f2.data_ptr() == f.data_ptr()
        outs.append((y.clone(), f.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[1][0], outs[2][0])
    assert torch.equal(outs[0][1], outs[2][1])


def test_host_entry_with_pageable_memory():
    """Host tensors that are not page-locked: the copies are then staged by the
    driver and do not overlap, but the results are those of pinned buffers."""
    shape = si.SSDShape("host_pageable", 3, 200, 8, 64, 128, 1, 64, "bf16", h0_std=0.1, seed=11)
    d = si.make_inputs(shape)
    pinned = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    y_p, f_p = ssd.fwd_host(pinned["x"], pinned["dt"], pinned["A"], pinned["B"], pinned["C"], pinned["D"], 64,
                            pinned["initial_states"], rows_per_piece=1)
    torch.cuda.current_stream().synchronize()
    y_out = torch.empty(d["x"].shape, dtype=d["x"].dtype)  # pageable outputs too
    f_out = torch.empty(3, 8, 64, 128, dtype=torch.float32)
    y, f = ssd.fwd_host(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 64, d["initial_states"],
                        y=y_out, final_states=f_out, rows_per_piece=1)
    torch.cuda.current_stream().synchronize()
    assert not y.is_pinned()
    assert torch.equal(y, y_p) and torch.equal(f, f_p)


def _packed_row_case(lens, ids, num_seqs, seed):
    L = sum(lens)
    shape = si.SSDShape("host_seqp", 1, L, 8, 64, 128, 1, 64, "bf16", h0_std=0.2, seed=seed)
    d = si.make_inputs(shape)
    d["seq_idx"] = torch.cat([torch.full((n,), i, dtype=torch.int32) for n, i in zip(lens, ids)]).view(1, L)
    d["num_seqs"] = num_seqs
    return shape, d


def _host_vs_device(d, num_seqs, z):
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    y_ref, f_ref = ssd.fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], 64, dev["initial_states"],
                           dev["seq_idx"], num_seqs, z=None if z is None else z.cuda())
    torch.cuda.synchronize()
    host = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    final = torch.full((num_seqs, 8, 64, 128), float("nan")).pin_memory()
    y, f = ssd.fwd_host(host["x"], host["dt"], host["A"], host["B"], host["C"], host["D"], 64,
                        host["initial_states"], host["seq_idx"], num_seqs, final_states=final,
                        z=None if z is None else z.pin_memory())
    torch.cuda.current_stream().synchronize()
    return y, f, y_ref.cpu(), f_ref.cpu()


@pytest.mark.parametrize("gated", [False, True], ids=["plain", "gated"])
def test_host_packed_row_in_sequence_pieces(gated):
    """One row of packed sequences is cut at sequence starts (here into 7
    pieces): every id comes back from exactly one piece, ids that never occur
    (0, 3, 7 and 11, at the ends and between pieces) as zeros over a host
    buffer that starts as NaN, and h0 enters the row's first sequence only."""
    lens = [300, 410, 90, 700, 260, 500, 333, 407]
    shape, d = _packed_row_case(lens, [1, 2, 4, 5, 6, 8, 9, 10], 12, seed=21)
    z = torch.randn(d["x"].shape, generator=torch.Generator().manual_seed(22)).to(d["x"].dtype) if gated else None
    y, f, y_ref, f_ref = _host_vs_device(d, 12, z)
    assert not torch.isnan(f).any()
    assert not f[[0, 3, 7, 11]].any()
    assert _rel(y, y_ref) <= 2e-3, _rel(y, y_ref)
    assert _rel(f, f_ref) <= 2e-3, _rel(f, f_ref)


def test_host_packed_row_out_of_order_runs_whole():
    """Ids that do not increase along the row cannot be cut into independent
    pieces; the call then runs as one piece, on the exact kernel."""
    shape, d = _packed_row_case([100, 150, 130], [2, 0, 1], 3, seed=23)
    y, f, y_ref, f_ref = _host_vs_device(d, 3, None)
    assert torch.equal(y, y_ref) and torch.equal(f, f_ref)
