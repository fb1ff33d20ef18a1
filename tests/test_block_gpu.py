"""The Mamba-2 block pieces on the GPU against the oracle: the causal
depthwise conv1d + SiLU (``ssd_conv1d_silu``)."""
import numpy as np
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd
import ssd_inputs as si
from gpu_util import TOL, rel_l2
from oracle import block

pytestmark = pytest.mark.gpu


def _conv_inputs(b, L, C, K, dtype, seed, with_bias=True):
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(b, L, C, generator=g).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    w = torch.randn(C, K, generator=g) * 0.5
    bias = torch.randn(C, generator=g) * 0.1 if with_bias else None
    return u, w, bias


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_conv1d_silu(K, dtype):
    u, w, bias = _conv_inputs(2, 77, 5376 if dtype == "bf16" else 100, K, dtype, seed=K)
    got = ssd.conv1d_silu(u.cuda(), w.cuda(), bias.cuda())
    torch.cuda.synchronize()
    want = block.conv1d_silu(u, w, bias)
    assert rel_l2(got.float().cpu().double().numpy(), want) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_conv1d_silu_packed_and_without_bias(dtype):
    u, w, _ = _conv_inputs(2, 100, 64, 4, dtype, seed=9, with_bias=False)
    seq, _ = si.seq_idx_from_lengths([[3, 1, 40, 56], [33, 67]])
    got = ssd.conv1d_silu(u.cuda(), w.cuda(), None, seq.cuda())
    torch.cuda.synchronize()
    want = block.conv1d_silu(u, w, None, seq)
    assert rel_l2(got.float().cpu().double().numpy(), want) <= TOL[dtype]


def test_conv1d_silu_strip_edges():
    """Lengths around the 32-token strips and a single token."""
    for L in (1, 31, 32, 33, 65):
        u, w, bias = _conv_inputs(1, L, 16, 4, "f32", seed=L)
        got = ssd.conv1d_silu(u.cuda(), w.cuda(), bias.cuda())
        torch.cuda.synchronize()
        assert rel_l2(got.cpu().double().numpy(), block.conv1d_silu(u, w, bias)) <= 1e-5, L


GATE_CASES = [
    # name, b, L, H, N, G, dtype, generic, packed, steep
    ("two_head_shape_gate_pass", 2, 300, 8, 128, 1, "bf16", False, None, False),
    ("single_head_N256", 1, 200, 4, 256, 2, "bf16", False, None, False),
    ("packed_per_sequence", 1, 260, 4, 128, 2, "bf16", False, [[100, 60, 100]], False),
    ("exact_kernel", 2, 300, 4, 128, 2, "bf16", False, None, True),
    ("generic_fp32", 2, 150, 4, 64, 2, "f32", False, None, False),
    ("generic_forced_bf16", 1, 150, 4, 128, 1, "bf16", True, None, False),
]


@pytest.mark.parametrize("case", GATE_CASES, ids=lambda c: c[0])
def test_gate_is_applied_where_y_is_formed(case):
    name, b, L, H, N, G, dtype, generic, packed, steep = case
    import oracle
    shape = si.SSDShape("gate", b, L, H, 64, N, G, 64, dtype, h0_std=0.2, seed=L + H)
    d = si.make_inputs(shape)
    if packed is not None:
        d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths(packed)
    if steep:
        d["dt"][0, 100:140, 1] = 1.5
        d["A"][1] = -12.0
    gen = torch.Generator().manual_seed(77)
    z = torch.randn(b, L, H, 64, generator=gen).to(d["x"].dtype)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    if name == "two_head_shape_gate_pass":  # the two-head kernel, then the gate pass over y
        assert ssd.main_kernel(g["x"], g["dt"], g["B"], 64) == "k_ssd_fwd_pair"
        assert ssd.main_kernel(g["x"], g["dt"], g["B"], 64, z=g["x"]) == "k_ssd_fwd_pair"
        assert ssd.launch_count(g["x"], g["B"], 64, z=g["x"]) == ssd.launch_count(g["x"], g["B"], 64) + 1
    y, f = ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=64,
                   initial_states=g["initial_states"], seq_idx=g.get("seq_idx"), num_seqs=d.get("num_seqs"),
                   generic=generic, z=z.cuda())
    torch.cuda.synchronize()
    yr, fr = oracle.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"],
                            seq_idx=d.get("seq_idx"), num_seqs=d.get("num_seqs"))
    want = block.gate(yr, z)
    got = y.float().cpu().double().numpy()
    assert rel_l2(got, want) <= TOL[dtype], rel_l2(got, want)
    from gpu_util import state_err
    assert state_err(f.cpu().double().numpy(), fr) <= TOL[dtype]
