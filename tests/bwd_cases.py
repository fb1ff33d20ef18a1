"""Cases, inputs and the comparison rule shared by the backward tests (the
host emulation in ``test_bwd_emu_cpu.py`` and the GPU parity tests in
``test_bwd_gpu.py``)."""
import numpy as np
import torch

import oracle
from oracle import backward
import ssd_inputs as si

# The kernels compute in fp32 and the oracle in fp64 on the same (fp32- or
# bf16-valued) inputs, so the gap is fp32 rounding in sums of at most
# Q + P + N terms per stage, a few of them chained (measured below 1e-6
# relative at these sizes); both bounds leave a wide margin over that.
REL_L2 = 1e-5
MAX_ABS = 1e-4
KEYS = ("dx", "ddt", "dA", "dB", "dC", "dD", "dh0", "dz")

CASES = [
    # id, (b, L, H, P, N, G), dtype, h0 std, dfinal, packed (lo, hi) or per-row lengths, D, chunk
    ("f32_ragged_Q16", (1, 50, 2, 8, 16, 1), "f32", 0.5, True, None, True, 16),
    ("f32_groups_auto", (2, 150, 4, 24, 40, 2), "f32", 0.3, True, None, True, 0),
    ("bf16_packed", (2, 150, 4, 16, 32, 2), "bf16", 0.0, False, (5, 40), False, 0),
    # sequences starting exactly at a chunk start, one-token sequences, a row starting with two of them
    ("f32_packed_edges", (2, 64, 2, 8, 8, 1), "f32", 0.4, False, [[16, 1, 15, 32], [1, 1, 30, 2, 30]], True, 16),
    ("f32_chunk1", (1, 7, 2, 4, 4, 2), "f32", 0.5, True, None, True, 1),
    ("f32_one_token", (2, 1, 2, 4, 8, 1), "f32", 0.5, True, None, True, 0),
    # dstate 256 at headdim 64: a 64-token chunk does not fit one CTA's shared memory, 32 does
    ("bf16_N256_chunk32", (1, 70, 2, 64, 256, 1), "bf16", 0.2, True, None, True, 0),
    ("f32_hpg4", (1, 40, 8, 8, 16, 2), "f32", 0.0, True, None, True, 8),
]
# the same with the block's gate (out = y SiLU(z)): dy is then the gradient of the gated output
GATED = {"f32_ragged_Q16", "bf16_packed", "f32_packed_edges", "bf16_N256_chunk32"}
CASES += [("gated_" + c[0],) + c[1:] for c in CASES if c[0] in GATED]


def dy_like(b, L, H, P, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(b, L, H, P, generator=g).to(dtype)


def dfinal_like(b, H, P, N, seed):
    g = torch.Generator().manual_seed(seed + 1)
    return torch.randn(b, H, P, N, generator=g)


def inputs(b, L, H, P, N, G, dtype="f32", h0=0.0, packed=None, seed=1, has_D=True, lengths=None):
    d = si.make_inputs(si.SSDShape("bwd", b, L, H, P, N, G, 64, dtype, h0_std=h0, packed=packed,
                                   seed=seed, has_D=has_D))
    if lengths is not None:
        d["seq_idx"], d["num_seqs"] = si.seq_idx_from_lengths(lengths)
    return d


def gate_like(b, L, H, P, dtype, seed):
    """z ~ N(0, 2^2): both signs, well into the curved part of SiLU."""
    g = torch.Generator().manual_seed(seed + 2)
    return (2.0 * torch.randn(b, L, H, P, generator=g)).to(dtype)


def case_inputs(case):
    """(inputs, dy, dfinal, chunk) of one CASES entry; a gated case carries
    its gate in inputs["z"]."""
    name, (b, L, H, P, N, G), dtype, h0, with_df, packed, with_D, chunk = case
    d = inputs(b, L, H, P, N, G, dtype, h0, packed if isinstance(packed, tuple) else None, seed=L * 3 + H,
               has_D=with_D, lengths=packed if isinstance(packed, list) else None)
    d["z"] = gate_like(b, L, H, P, d["x"].dtype, L + N) if name.startswith("gated_") else None
    dy = dy_like(b, L, H, P, d["x"].dtype, L + P)
    dfinal = dfinal_like(b, H, P, N, L) if with_df else None
    return d, dy, dfinal, chunk


def oracle_bwd(d, dy, dfinal):
    args = (d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["initial_states"])
    if d.get("z") is not None:
        return backward.ssd_bwd_gated(*args, d["z"], dy, dfinal, d["seq_idx"], backward_fn=oracle.ssd_bwd)
    return oracle.ssd_bwd(*args, dy, dfinal, d["seq_idx"])


def compare(out, ref, keys=KEYS, rel_l2=REL_L2):
    """Every gradient the oracle gives: finite, within ``rel_l2`` in relative
    L2 and within MAX_ABS * max(1, max |ref|) element by element.  dA and dD
    are signed sums over every token, where cancellation can leave the sum
    far smaller than its terms: their error is bounded by ``rel_l2`` times
    the sum of the terms' magnitudes (the oracle's dA_abs and dD_abs)."""
    for k in keys:
        if ref.get(k) is None:
            continue
        got = np.asarray(out[k], dtype=np.float64)
        want = ref[k]
        assert got.shape == want.shape, f"{k}: shape {got.shape} != {want.shape}"
        assert np.isfinite(got).all(), f"{k}: non-finite values"
        if k in ("dA", "dD") and ref.get(k + "_abs") is not None:
            err = np.abs(got - want)
            assert (err <= rel_l2 * ref[k + "_abs"] + 1e-30).all(), f"{k}: {err} against {ref[k + '_abs']}"
            continue
        rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
        mad = np.abs(got - want).max()
        assert rel <= rel_l2, f"{k}: rel L2 {rel:.3g}"
        assert mad <= MAX_ABS * max(1.0, np.abs(want).max()), f"{k}: max abs {mad:.3g}"


# conv1d + SiLU backward: id, (b, L, C, K), dtype, per-row packed lengths or None, bias
CONV_CASES = [
    ("f32_K4_strips", (2, 70, 300, 4), "f32", None, True),
    ("bf16_K3_packed", (2, 64, 260, 3), "bf16", [[7, 1, 40, 16], [1, 63]], False),
    ("f32_K1", (1, 33, 5, 1), "f32", None, True),
    ("f32_one_token", (1, 1, 8, 4), "f32", None, True),
    ("f32_K2_packed_on_a_strip_edge", (1, 64, 8, 2), "f32", [[32, 32]], True),
    ("bf16_K4_c1_channels", (1, 100, 5376, 4), "bf16", None, True),
    # 64-token bf16 strips with a ragged last one; a partial second channel block
    ("bf16_K4_strips", (2, 150, 264, 4), "bf16", None, True),
    # sequence starts on either side of the 64-token strip edges (rows staged by 16-byte copies)
    ("bf16_K4_packed_strips", (1, 200, 16, 4), "bf16", [[63, 2, 65, 70]], False),
]


def conv_case_inputs(case):
    """(u, weight, bias, dout, seq_idx) of one CONV_CASES entry."""
    name, (b, L, C, K), dtype, packed, with_bias = case
    g = torch.Generator().manual_seed(L * 7 + C + K)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    u = torch.randn(b, L, C, generator=g).to(dt)
    w = torch.randn(C, K, generator=g) * 0.5
    bias = torch.randn(C, generator=g) * 0.1 if with_bias else None
    dout = torch.randn(b, L, C, generator=g).to(dt)
    seq = si.seq_idx_from_lengths(packed)[0] if packed else None
    return u, w, bias, dout, seq


def conv_compare(du, dw, db, ref):
    """du, dw, dbias against the fp64 oracle's (du, dw, dbias[, dw_abs,
    dbias_abs]): du by the SSD backward's bounds (fp32 sums of at most K
    terms); dw and dbias, signed sums over every token, element by element
    within REL_L2 times the sums of their terms' magnitudes when the oracle
    gives them (``with_scale``), else by the same relative bounds."""
    scales = {"dw": ref[3], "dbias": ref[4]} if len(ref) > 3 else {}
    for name, got, want in (("du", du, ref[0]), ("dw", dw, ref[1]), ("dbias", db, ref[2])):
        if got is None:
            continue
        got = np.asarray(got, dtype=np.float64)
        assert got.shape == want.shape, name
        assert np.isfinite(got).all(), name
        if name in scales:
            err = np.abs(got - want)
            assert (err <= REL_L2 * scales[name] + 1e-30).all(), f"{name}: {err.max():.3g}"
            continue
        rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
        assert rel <= REL_L2, f"{name}: rel L2 {rel:.3g}"
        assert np.abs(got - want).max() <= MAX_ABS * max(1.0, np.abs(want).max()), name


def random_case(seed: int):
    """One seeded random backward problem: (inputs with "z", dy, dfinal, chunk,
    description).  Odd headdim and dstate (partial tiles, odd padded strides),
    random chunk lengths, packed rows with one- and two-token sequences, and
    the gate, D, h0 and dfinal each on or off."""
    import random
    rng = random.Random(seed)
    G = rng.choice([1, 1, 2, 3])
    H = G * rng.choice([1, 2, 3])
    b, L = rng.randint(1, 3), rng.randint(1, 200)
    P, N = rng.randint(1, 70), rng.randint(1, 70)
    chunk = rng.choice([0, 0, rng.randint(1, 64)])
    dtype = rng.choice(["f32", "bf16"])
    packed = rng.random() < 0.4
    lengths = None
    if packed:
        lengths = []
        for _ in range(b):
            row, left = [], L
            while left > 0:
                k = min(left, rng.choice([1, 2, rng.randint(1, 80)]))
                row.append(k)
                left -= k
            lengths.append(row)
    h0 = rng.choice([0.0, 0.4])
    with_D, gate = rng.random() < 0.7, rng.random() < 0.4
    d = inputs(b, L, H, P, N, G, dtype, h0, None, seed=seed + 100, has_D=with_D, lengths=lengths)
    d["z"] = gate_like(b, L, H, P, d["x"].dtype, seed) if gate else None
    dy = dy_like(b, L, H, P, d["x"].dtype, seed)
    dfinal = None if packed or rng.random() < 0.3 else dfinal_like(b, H, P, N, seed)
    desc = (f"b{b}L{L}H{H}G{G}P{P}N{N}Q{chunk}_{dtype}{'_packed' if packed else ''}{'_gate' if gate else ''}"
            f"{'_D' if with_D else ''}{'_h0' if h0 else ''}{'_dfinal' if dfinal is not None else ''}")
    return d, dy, dfinal, chunk, desc


RANDOM_SEEDS = list(range(1000, 1012))


def out_of_order_case():
    """A packed batch whose ids do not increase along the tokens (a change of
    id starts a sequence, whatever its value), with a gate: (inputs, dy,
    dfinal, chunk)."""
    b, L, H, P, N, G = 2, 90, 4, 16, 24, 2
    d = inputs(b, L, H, P, N, G, "f32", 0.3, None, seed=5)
    seq = torch.tensor([[7] * 20 + [3] * 1 + [5] * 40 + [0] * 29,
                        [2] * 45 + [9] * 45], dtype=torch.int32)
    d["seq_idx"], d["num_seqs"] = seq, 10
    d["z"] = gate_like(b, L, H, P, torch.float32, 5)
    return d, dy_like(b, L, H, P, torch.float32, 5), None, 16
