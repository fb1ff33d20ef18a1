"""The backward kernels (``csrc/ssd_bwd.cuh``) run on the CPU through the
test-only emulation in ``tests/emu`` and compared with the fp64 backward
oracle, before any GPU runs them.

The emulator compiles the kernels' own source with g++ under
AddressSanitizer + UBSan (exact-size buffers: any access past an input,
output, workspace or shared-memory buffer aborts) or ThreadSanitizer (real
threads: a shared-memory race aborts), and fills outputs, workspace and
shared memory with NaN first, so a value read before it was written shows up.
Each block's threads also run in reverse order once, which exposes a missing
barrier in the other direction.  Planted mistakes in a copy of the kernels
must be caught.  The GPU parity tests (``test_bwd_gpu.py``) run the same
kernels compiled by nvcc."""
import os
import re
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import emu_bwd
from bwd_cases import (CASES, KEYS, RANDOM_SEEDS, case_inputs, compare, dfinal_like, dy_like, gate_like, inputs,
                       oracle_bwd, random_case)

pytestmark = pytest.mark.skipif(not emu_bwd.available(), reason="g++ not available")


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_emulated_backward_matches_oracle(case):
    name, (b, L, H, P, N, G), _, _, _, _, with_D, chunk = case
    d, dy, dfinal = case_inputs(case)[:3]
    out = emu_bwd.run(d, dy, dfinal, chunk_size=chunk, z=d["z"])
    assert out["status"] == 0
    assert out["launches"] == 6
    if name == "bf16_N256_chunk32":
        assert out["chunk"] == 32  # 64 would not fit the shared memory of one CTA
    elif chunk:
        assert out["chunk"] == chunk
    ref = oracle_bwd(d, dy, dfinal)
    compare(out, ref)
    if d["initial_states"] is None:
        # the gradient at a zero initial state: the oracle's, with a zero h0 passed
        d0 = dict(d, initial_states=torch.zeros(b, H, P, N))
        assert np.allclose(out["dh0"], oracle_bwd(d0, dy, dfinal)["dh0"], rtol=1e-4, atol=1e-5)
    if not with_D:
        # dD is the gradient at D = 0: sum over rows and tokens of dy . x (dy reaching y, after the gate)
        dyy = dy.double().numpy()
        if d["z"] is not None:
            zz = d["z"].double().numpy()
            dyy = dyy * zz / (1.0 + np.exp(-zz))
        want = np.einsum("blhp,blhp->h", dyy, d["x"].double().numpy())
        assert np.allclose(out["dD"], want, rtol=1e-5, atol=1e-5)


def test_reverse_thread_order_gives_the_same_bits():
    d = inputs(2, 150, 4, 24, 40, 2, "f32", 0.3, seed=11)
    dy = dy_like(2, 150, 4, 24, torch.float32, 5)
    dfinal = dfinal_like(2, 4, 24, 40, 5)
    fwd_order = emu_bwd.run(d, dy, dfinal)
    rev_order = emu_bwd.run(d, dy, dfinal, reverse=True)
    for k in KEYS:
        assert np.array_equal(fwd_order[k], rev_order[k]), k


def test_threads_under_thread_sanitizer():
    d = inputs(1, 40, 2, 8, 16, 1, "f32", 0.3, seed=3)
    dy = dy_like(1, 40, 2, 8, torch.float32, 3)
    out = emu_bwd.run(d, dy, dfinal_like(1, 2, 8, 16, 3), chunk_size=16, kind="tsan")
    assert out["status"] == 0
    assert "ThreadSanitizer" not in out["stderr"]
    compare(out, oracle_bwd(d, dy, dfinal_like(1, 2, 8, 16, 3)))


@pytest.mark.parametrize("kw,status", [
    (dict(headdim=257), 2),
    (dict(dstate=300), 2),
    (dict(chunk_size=65), 2),
    (dict(chunk_size=-1), 1),
    (dict(ngroups=3), 1),
    (dict(seqlen=0), 1),
])
def test_emulated_plan_rejects(kw, status):
    shp = dict(batch=1, seqlen=8, nheads=2, headdim=4, dstate=4, ngroups=1)
    shp.update(kw)
    x = torch.zeros(shp["batch"], max(shp["seqlen"], 1), shp["nheads"], shp["headdim"])
    d = {"x": x, "dt": torch.zeros(x.shape[:3]), "A": torch.zeros(shp["nheads"]),
         "B": torch.zeros(x.shape[0], x.shape[1], shp["ngroups"], shp["dstate"]),
         "C": torch.zeros(x.shape[0], x.shape[1], shp["ngroups"], shp["dstate"]), "D": None}
    # the driver reads sizes from args.txt: write the requested ones
    out = _run_with_sizes(d, shp, kw.get("chunk_size", 0))
    assert out == status


def _run_with_sizes(d, shp, chunk):
    exe = emu_bwd.build("asan")
    with tempfile.TemporaryDirectory() as tmp:
        for k in ("x", "dt", "A", "B", "C"):
            d[k].numpy().tofile(os.path.join(tmp, k + ".bin"))
        d["x"].numpy().tofile(os.path.join(tmp, "dy.bin"))
        kv = dict(shp, chunk_size=chunk, dtype=0, has_D=0, has_h0=0, has_seq=0, has_dfinal=0, want_dD=0,
                  want_dh0=0, reverse=0)
        with open(os.path.join(tmp, "args.txt"), "w") as f:
            f.write("".join(f"{k} {v}\n" for k, v in kv.items()))
        r = subprocess.run([exe, tmp], capture_output=True, text=True, timeout=120,
                           env=dict(os.environ, ASAN_OPTIONS="detect_leaks=0"))
        return int(r.stdout.split()[1])


def test_packed_with_dfinal_is_unsupported():
    d = inputs(1, 32, 2, 4, 4, 1, "f32", packed=(4, 12), seed=2)
    dy = dy_like(1, 32, 2, 4, torch.float32, 2)
    assert emu_bwd.run(d, dy, dfinal_like(1, 2, 4, 4, 2))["status"] == 2


# Planted mistakes in a copy of the kernels: each must make the emulated run
# fail (sanitizer abort, non-finite output or a parity miss).
MUTANTS = [
    # a missing barrier between the Q x Q matrices and their use by other threads
    ("drop_barrier", r"(        if \(s == t\) dg\[t\] = xy\[i\]\[j\];\n      }\n  }\n)  __syncthreads\(\);", r"\1"),
    # the in-chunk sum of dx runs one token past the chunk
    ("dx_past_chunk", r"(tile_mac<false>\(acc, tl, Km, 1, sQ, nullptr, dys, sP, 1, tl\.r\[0\], )Qc\);", r"\1Qc + 1);"),
    # the adjoint carried across chunks skips the chunk decay
    ("no_decay_backward", r"lam\[k\] = fmaf\(dl, lam\[k\], vt\[j\]\[k\]\);", "lam[k] = lam[k] + vt[j][k];"),
    # the pair sum of dl loses dt
    ("pairs_no_dt", r"blk = fmaf\(Mm\[u \* sQ \+ s2\], w\[s2\], blk\);", "blk += Mm[u * sQ + s2];"),
    # the h_in terms are taken for every token, also after a sequence boundary
    ("hin_always", r"ein\[t\] = seg\[t\] == -1 \? expf\(cs\[t\]\) : 0\.f;", "ein[t] = expf(cs[t]);"),
    # tiles numbered with the wrong divisor: parts of a non-square product are never written
    ("tile_index", r"const int tr = tile / TC;", "const int tr = tile / (TC + 1);"),
    # the gate's slope taken as the logistic's (run with a gate)
    ("gate_slope", r"return s \* fmaf\(v, 1\.f - s, 1\.f\);", "return s * (1.f - s);"),
    # no barrier between rewriting dy through the gate and reading it (run with a gate)
    ("gate_barrier", r"(          dys\[t \* sP \+ p\] = dout \* gate_silu\(zz\);\n        }\n    }\n)    __syncthreads\(\);",
     r"\1"),
]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_emulator_catches_planted_mistakes(mutant, monkeypatch):
    name, pat, rep = mutant
    src = open(emu_bwd.KERNELS).read()
    bad, n = re.subn(pat, rep, src)
    assert n == 1, f"mutant {name} did not apply"
    with tempfile.TemporaryDirectory() as tmp:
        os.makedirs(os.path.join(tmp, "k"))
        with open(os.path.join(tmp, "k", "ssd_bwd.cuh"), "w") as f:
            f.write(bad)
        monkeypatch.setattr(emu_bwd, "KERNELS", os.path.join(tmp, "k", "ssd_bwd.cuh"))
        monkeypatch.setattr(emu_bwd, "OUT", os.path.join(tmp, "out"))
        d = inputs(2, 80, 2, 8, 16, 1, "f32", 0.5, packed=None, seed=9,
                    lengths=[[20, 1, 30, 29], [40, 40]] if name == "hin_always" else None)
        d["z"] = gate_like(2, 80, 2, 8, torch.float32, 9) if name.startswith("gate") else None
        dy = dy_like(2, 80, 2, 8, torch.float32, 9)
        dfinal = None if name == "hin_always" else dfinal_like(2, 2, 8, 16, 9)
        ref = oracle_bwd(d, dy, dfinal)
        caught = False
        for reverse in (False, True):
            try:
                out = emu_bwd.run(d, dy, dfinal, chunk_size=16, reverse=reverse, z=d["z"])
                compare(out, ref)
            except (AssertionError, RuntimeError):
                caught = True
        assert caught, f"mutant {name} survived"


@pytest.mark.parametrize("seed", RANDOM_SEEDS)
def test_emulated_backward_on_random_shapes(seed):
    d, dy, dfinal, chunk, _ = random_case(seed)
    out = emu_bwd.run(d, dy, dfinal, chunk_size=chunk, z=d["z"], reverse=seed % 2 == 1)
    assert out["status"] == 0
    compare(out, oracle_bwd(d, dy, dfinal))


@pytest.mark.parametrize("packed", [False, True], ids=["dense", "packed"])
def test_emulated_backward_on_the_gpu_tests_mid_sizes(packed):
    """The mid-size problems of the GPU tests, under the sanitizers too."""
    b, L, H, P, N, G = (2, 1024, 8, 64, 128, 1) if not packed else (2, 1024, 4, 64, 128, 2)
    d = inputs(b, L, H, P, N, G, "bf16", h0=0.0 if packed else 0.2, packed=(32, 400) if packed else None, seed=77)
    d["z"] = None
    dy = dy_like(b, L, H, P, torch.bfloat16, 78)
    dfinal = None if packed else dfinal_like(b, H, P, N, 79)
    compare(emu_bwd.run(d, dy, dfinal, timeout=1200), oracle_bwd(d, dy, dfinal))


def test_dinitial_only_gives_the_same_bits_and_writes_nothing_else():
    d, dy, dfinal, chunk = case_inputs(CASES[1])
    full = emu_bwd.run(d, dy, None, chunk_size=chunk, z=d["z"])
    only = emu_bwd.run(d, dy, None, chunk_size=chunk, z=d["z"], flags=1)
    assert only["status"] == 0 and only["launches"] == 2
    assert np.array_equal(only["dh0"], full["dh0"])
    assert all(only[k] is None for k in ("dx", "ddt", "dA", "dB", "dC", "dD", "dz"))


def test_emulated_backward_with_ids_out_of_order():
    from bwd_cases import out_of_order_case
    d, dy, dfinal, chunk = out_of_order_case()
    out = emu_bwd.run(d, dy, dfinal, chunk_size=chunk, z=d["z"])
    compare(out, oracle_bwd(d, dy, dfinal))
