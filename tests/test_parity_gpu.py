"""GPU parity: the CUDA path against the fp64 CPU oracle on the same seeded
inputs.  Tolerances (stated by the task's target and written here): relative
L2 over y <= 1e-5 on the fp32 path and <= 1e-2 on the bf16-input /
fp32-accumulate path; final states max|diff| <= tol * max(1, max|ref|).

Every case is compared element by element over the whole output.  The small
cases span several chunks, ragged tails, groups, packed boundaries inside
chunks and on chunk edges; the full-size workloads run in the launch
configuration the benchmark times, with the oracle on every unit.
"""
import numpy as np
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
import ssd_inputs as si
from gpu_util import TOL, rel_l2, run_gpu, run_oracle, state_err, to_dev

pytestmark = pytest.mark.gpu

SMALL = [
    # b, L, H, P, N, G, Q, h0_std
    (2, 300, 4, 64, 128, 2, 64, 0.5),
    (1, 513, 2, 64, 256, 1, 256, 0.0),
    (2, 200, 6, 32, 64, 3, 128, 0.2),
    (1, 64, 2, 16, 16, 1, 16, 0.0),
    (1, 1, 2, 64, 128, 1, 64, 0.3),
    (3, 130, 4, 128, 32, 4, 32, 0.0),
    (1, 1000, 8, 64, 128, 2, 64, 0.1),
    (1, 777, 4, 64, 64, 1, 128, 0.0),
    (1, 100, 2, 256, 256, 1, 256, 0.1),
    (2, 255, 4, 64, 128, 1, 256, 0.0),
    # more head pairs than SMs: the two-head kernel splits pairs between CTAs
    # and hands the state over (4 chunks per row; ragged 13-chunk rows)
    (4, 200, 80, 64, 128, 1, 64, 0.1),
    (2, 777, 160, 64, 128, 2, 64, 0.0),
    # N = 64 on the two-head kernel (state zero-padded to 128 rows), with hand-over
    (4, 200, 80, 64, 64, 1, 64, 0.1),
]


def _id(c):
    return "b{}_L{}_H{}_P{}_N{}_G{}_Q{}_h{}".format(*c)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", SMALL, ids=_id)
def test_small_shapes(case, dtype):
    b, L, H, P, N, G, Q, h0 = case
    shape = si.SSDShape("small", b, L, H, P, N, G, Q, dtype, h0_std=h0, seed=hash(case) % 10000)
    d = si.make_inputs(shape)
    y, f = run_gpu(d, Q)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= TOL[dtype], rel_l2(y, yr)
    assert state_err(f, fr) <= TOL[dtype], state_err(f, fr)


def test_config_c0_fp32_full():
    s = si.CONFIGS["c0"]
    d = si.make_inputs(s)
    y, f = run_gpu(d, s.chunk_size)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-5, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-5, state_err(f, fr)


PACKED = [
    # per-row lengths, Q, h0_std
    ([[5, 16, 16, 27, 64, 1, 1, 30]], 16, 0.0),        # boundaries on chunk edges and mid-chunk
    ([[100, 37, 1, 118], [256]], 64, 0.3),              # two rows, ids numbered across rows
    ([[1] * 40 + [88]], 32, 0.0),                       # single-token sequences
    ([[300, 212]], 256, 0.2),                           # one boundary, long chunks
    ([[64, 64, 64, 64]], 64, 0.0),                      # every boundary on a chunk edge
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", PACKED, ids=lambda c: f"Q{c[1]}_rows{len(c[0])}_n{sum(map(len, c[0]))}")
def test_packed(case, dtype):
    rows, Q, h0 = case
    L = sum(rows[0])
    assert all(sum(r) == L for r in rows)
    shape = si.SSDShape("packed", len(rows), L, 4, 64, 64, 2, Q, dtype, h0_std=h0, seed=L + Q)
    d = si.make_inputs(shape)
    d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths(rows)
    y, f = run_gpu(d, Q)
    yr, fr = run_oracle(d)
    assert f.shape == fr.shape == (d["num_seqs"], 4, 64, 64)
    assert rel_l2(y, yr) <= TOL[dtype], rel_l2(y, yr)
    assert state_err(f, fr) <= TOL[dtype], state_err(f, fr)


PACKED_TC = [
    # per-row lengths, N, Q, h0_std: bf16 with Q >= 64 runs on the exact tensor-core kernel
    ([[5, 16, 16, 27, 64, 1, 1, 30]], 128, 64, 0.3),   # ends mid-chunk, on chunk edges, 1-token sequences
    ([[100, 37, 1, 118], [256]], 256, 64, 0.2),         # two rows, ids numbered across rows
    ([[300, 212]], 128, 256, 0.0),                      # one boundary, 256-token chunks
    ([[64, 64, 1, 63, 64, 60]], 64, 128, 0.1),          # N = 64 (zero-padded), ends before chunk edges
]


@pytest.mark.parametrize("case", PACKED_TC, ids=lambda c: f"N{c[1]}_Q{c[2]}_rows{len(c[0])}_n{sum(map(len, c[0]))}")
def test_packed_on_the_tensor_core_path(case):
    rows, N, Q, h0 = case
    L = sum(rows[0])
    shape = si.SSDShape("packed_tc", len(rows), L, 4, 64, N, 2, Q, "bf16", h0_std=h0, seed=L + N)
    d = si.make_inputs(shape)
    d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths(rows)
    g = to_dev(d)
    assert ssd.kernel_path(g["x"], g["B"], Q, seq_idx=g["seq_idx"], num_seqs=d["num_seqs"]) == "tcgen05"
    y, f = run_gpu(d, Q)
    yr, fr = run_oracle(d)
    assert f.shape == fr.shape == (d["num_seqs"], 4, 64, N)
    assert rel_l2(y, yr) <= 1e-2, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)


def test_packed_absent_ids_get_zero_states_on_the_tensor_core_path():
    shape = si.SSDShape("packed", 1, 160, 2, 64, 128, 1, 64, "bf16", seed=19)
    d = si.make_inputs(shape)
    sq = torch.tensor([[0] * 70 + [2] * 90], dtype=torch.int32)  # ids 1 and 3 never occur
    d["seq_idx"], d["num_seqs"] = sq, 4
    y, f = run_gpu(d, 64)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2
    assert not f[1].any() and not f[3].any()
    assert state_err(f, fr) <= 1e-2


def test_packed_absent_ids_get_zero_states():
    shape = si.SSDShape("packed", 1, 96, 2, 64, 64, 1, 32, "bf16", seed=9)
    d = si.make_inputs(shape)
    sq = torch.tensor([[0] * 40 + [2] * 56], dtype=torch.int32)  # id 1 and 3 never occur
    d["seq_idx"], d["num_seqs"] = sq, 4
    y, f = run_gpu(d, 32)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2
    assert not f[1].any() and not f[3].any()
    assert state_err(f, fr) <= 1e-2


@pytest.mark.parametrize("order", ["increasing", "out_of_order"])
def test_packed_absent_ids_are_zeroed_in_a_dirty_buffer(order):
    """Ids that never occur get zero final states written, whatever the caller's
    buffer held (here NaN).  Increasing ids take the per-run kernels; ids out of
    order leave the run list unusable and every unit to the exact kernel."""
    shape = si.SSDShape("packed_dirty", 1, 200, 4, 64, 128, 1, 64, "bf16", h0_std=0.2, seed=41)
    d = si.make_inputs(shape)
    ids = [0] * 80 + [3] * 120 if order == "increasing" else [3] * 80 + [0] * 120
    d["seq_idx"], d["num_seqs"] = torch.tensor([ids], dtype=torch.int32), 5
    g = to_dev(d)
    final = torch.full((5, 4, 64, 128), float("nan"), device="cuda")
    y, f = ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=64,
                   initial_states=g["initial_states"], seq_idx=g["seq_idx"], num_seqs=5, final_states=final)
    torch.cuda.synchronize()
    assert f.data_ptr() == final.data_ptr()
    yr, fr = run_oracle(d)
    f = f.cpu().numpy().astype(np.float64)
    assert rel_l2(y.float().cpu().numpy().astype(np.float64), yr) <= 1e-2
    assert not np.isnan(f).any()
    assert not f[[1, 2, 4]].any()
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)


def test_determinism():
    s = si.SSDShape("det", 2, 700, 8, 64, 128, 2, 64, "bf16", h0_std=0.1, seed=77)
    d = si.make_inputs(s)
    y1, f1 = run_gpu(d, 64)
    y2, f2 = run_gpu(d, 64)
    assert np.array_equal(y1, y2) and np.array_equal(f1, f2)


def test_chunk_size_invariance_on_gpu():
    """The same inputs through every supported chunk size agree with each
    other and with the oracle (chunking is an exact re-association)."""
    s = si.SSDShape("q", 1, 600, 4, 64, 64, 2, 64, "f32", h0_std=0.2, seed=5)
    d = si.make_inputs(s)
    yr, fr = run_oracle(d)
    for Q in (16, 32, 64, 128, 256):
        y, f = run_gpu(d, Q)
        assert rel_l2(y, yr) <= 1e-5, (Q, rel_l2(y, yr))
        assert state_err(f, fr) <= 1e-5, (Q, state_err(f, fr))


@pytest.mark.parametrize("case", [
    # b, L, H, P, N, G, Q, h0_std: N = 128 shapes the two-head kernel does not take
    (1, 300, 6, 64, 128, 3, 64, 0.2),    # H not a multiple of 4
    (2, 200, 3, 64, 128, 1, 64, 0.0),    # an odd number of heads per group
    (1, 300, 3, 64, 64, 1, 64, 0.2),     # N = 64, zero-padded to 128 rows
], ids=_id)
def test_single_head_kernel_takes_the_other_n128_shapes(case):
    b, L, H, P, N, G, Q, h0 = case
    shape = si.SSDShape("sh", b, L, H, P, N, G, Q, "bf16", h0_std=h0, seed=H * 10 + G)
    d = si.make_inputs(shape)
    g = to_dev(d)
    assert ssd.main_kernel(g["x"], g["dt"], g["B"], Q) == "k_ssd_fwd_fast"
    y, f = run_gpu(d, Q)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)


@pytest.mark.parametrize("case", [
    # b, L, H, P, N, G, Q, h0_std: fewer head pairs than SMs and at least two
    # chunk steps per SM, so the two-head kernel runs split (a state-only pass
    # first; each CTA folds the local states of the CTAs before it)
    (1, 8192, 8, 64, 128, 1, 64, 0.3),     # 4 pairs of 128 chunks: each pair over ~37 CTAs
    (1, 12000, 4, 64, 128, 2, 128, 0.0),   # two groups, a ragged tail, Q = 128
    (2, 4800, 4, 64, 64, 1, 256, 0.2),     # two rows, N = 64 zero-padded
], ids=_id)
def test_split_two_head_kernel(case):
    b, L, H, P, N, G, Q, h0 = case
    shape = si.SSDShape("split", b, L, H, P, N, G, Q, "bf16", h0_std=h0, seed=L + H)
    d = si.make_inputs(shape)
    g = to_dev(d)
    assert ssd.main_kernel(g["x"], g["dt"], g["B"], Q) == "k_ssd_fwd_pair"
    assert ssd.launch_count(g["x"], g["B"], Q) == 4  # C B^T, state-only pass, fused, exact
    y, f = run_gpu(d, Q)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)


def test_unaligned_dt_takes_the_single_head_kernel():
    """The two-head kernel reads dt by TMA (16-byte aligned base); a dt view
    that starts 4 bytes into its storage goes to the single-head kernel."""
    s = si.SSDShape("ua", 2, 300, 8, 64, 128, 1, 64, "bf16", h0_std=0.1, seed=12)
    d = si.make_inputs(s)
    g = to_dev(d)
    store = torch.empty(g["dt"].numel() + 1, device="cuda", dtype=torch.float32)
    dt = store[1:].view_as(g["dt"])
    dt.copy_(g["dt"])
    assert dt.data_ptr() % 16 != 0
    assert ssd.main_kernel(g["x"], dt, g["B"], 64) == "k_ssd_fwd_fast"
    assert ssd.main_kernel(g["x"], g["dt"], g["B"], 64) == "k_ssd_fwd_pair"
    y, f = ssd.fwd(g["x"], dt, g["A"], g["B"], g["C"], g["D"], chunk_size=64, initial_states=g["initial_states"])
    torch.cuda.synchronize()
    yr, fr = run_oracle(d)
    assert rel_l2(y.float().cpu().numpy(), yr) <= 1e-2
    assert state_err(f.cpu().numpy(), fr) <= 1e-2


def test_device_status_reports_no_timeout_after_a_normal_call():
    s = si.SSDShape("st", 2, 300, 8, 64, 128, 1, 64, "bf16", h0_std=0.1, seed=8)
    g = to_dev(si.make_inputs(s))
    assert ssd.main_kernel(g["x"], g["dt"], g["B"], 64) == "k_ssd_fwd_pair"
    need = ssd.workspace_size(g["x"], g["B"], 64)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")  # the call must clear its error word
    ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=64,
            initial_states=g["initial_states"], workspace=ws)
    assert ssd.device_status(g["x"], g["B"], 64, ws) == ssd.SSD_OK


def test_generic_flag_matches_default_path():
    s = si.SSDShape("g", 2, 333, 4, 64, 128, 1, 64, "bf16", h0_std=0.1, seed=6)
    d = si.make_inputs(s)
    y1, f1 = run_gpu(d, 64)
    y2, f2 = run_gpu(d, 64, generic=True)
    assert rel_l2(y1, y2) <= 1e-2 and state_err(f1, f2) <= 1e-2


@pytest.mark.parametrize("N", [128, 256])
def test_strong_decay_heads_take_the_exact_kernel(N):
    """Heads whose in-chunk decay is too steep for the factorised fast kernel
    (dt*A ~ -30 per token) are handled by the exact kernel in the same call;
    the other heads by the fast kernel.  Both must match the oracle."""
    s = si.SSDShape("steep", 2, 300, 4, 64, N, 2, 64, "bf16", h0_std=0.2, seed=31)
    d = si.make_inputs(s)
    d["dt"][:, :, 0] = 2.0
    d["A"][0] = -16.0
    d["dt"][0, 100:140, 3] = 1.5   # one steep stretch in one row of head 3
    d["A"][3] = -12.0
    y, f = run_gpu(d, 64)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)


@pytest.mark.parametrize("N", [128, 256])
def test_packed_strong_decay_runs_take_the_exact_kernel(N):
    """Packed sequences run per (sequence, head) on the fast kernel; a head
    with a steep stretch inside one sequence sends its (row, head) to the exact
    kernel, which redoes the whole row for that head.  Two sequences share the
    steep head's row, so the exact kernel rewrites outputs the fast kernel also
    wrote; both rows and every sequence's final state must match the oracle."""
    s = si.SSDShape("steep_packed", 2, 320, 4, 64, N, 2, 64, "bf16", h0_std=0.2, seed=33)
    d = si.make_inputs(s)
    d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths([[130, 190], [64, 100, 156]])
    d["dt"][0, 140:180, 3] = 1.5   # inside the second sequence of row 0
    d["A"][3] = -12.0
    g = to_dev(d)
    assert ssd.main_kernel(g["x"], g["dt"], g["B"], 64, seq_idx=g["seq_idx"], num_seqs=d["num_seqs"]) == "k_ssd_fwd_fast"
    y, f = run_gpu(d, 64)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)


def test_packed_ids_out_of_order_take_the_exact_kernel():
    """Sequence ids that do not increase along the tokens cannot be listed as
    independent runs; every unit then goes to the exact kernel."""
    s = si.SSDShape("packed_order", 1, 240, 4, 64, 128, 1, 64, "bf16", h0_std=0.3, seed=35)
    d = si.make_inputs(s)
    d["seq_idx"] = torch.tensor([[2] * 50 + [0] * 100 + [1] * 90], dtype=torch.int32)
    d["num_seqs"] = 3
    y, f = run_gpu(d, 64)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)


def test_zero_step_tokens():
    """dt = 0 tokens (a_t = 1, no input) still get their D x term."""
    s = si.SSDShape("dt0", 1, 200, 4, 64, 128, 1, 64, "bf16", h0_std=0.1, seed=41)
    d = si.make_inputs(s)
    d["dt"][0, 10:20, 1] = 0.0
    d["dt"][0, 150, 2] = 0.0
    y, f = run_gpu(d, 64)
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)


def test_rejected_call_raises_and_leaves_outputs():
    s = si.SSDShape("r", 1, 64, 2, 64, 64, 1, 64, "bf16", seed=1)
    g = to_dev(si.make_inputs(s))
    y = torch.full_like(g["x"], 7.0)
    with pytest.raises(ssd.SSDError):
        ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=48, y=y)
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())


# ---- full-size workloads, every unit -----------------------------------------

FULL = ["c1", "c3", "c4"] + [f"c2_N{n}_Q{q}" for n in (64, 128, 256) for q in (64, 128, 256)]


@pytest.mark.parametrize("name", FULL)
def test_full_size(name):
    """The whole y and every final state of each benchmark workload, in the
    launch configuration the benchmark times, against the oracle run on every
    (batch, head) unit.  Besides the stated bound over the whole tensor, each
    unit's own slice of y is held to it, so that one wrong hand-over or split
    point between CTAs cannot hide in the average."""
    s = si.CONFIGS[name]
    d = si.make_inputs(s)
    y, f = run_gpu(d, s.chunk_size)
    assert np.isfinite(y).all() and np.isfinite(f).all()
    yr, fr = run_oracle(d)
    assert rel_l2(y, yr) <= 1e-2, rel_l2(y, yr)
    assert state_err(f, fr) <= 1e-2, state_err(f, fr)
    err = y - yr
    num = np.sqrt((err * err).sum(axis=(1, 3)))    # (b, H): per unit
    den = np.sqrt((yr * yr).sum(axis=(1, 3)))
    worst = float((num / np.maximum(den, 1e-300)).max())
    assert worst <= 1e-2, worst
