"""The tcgen05 building blocks of the fused kernel, one at a time: shared
memory layouts (K-major and MN-major, 128-byte swizzle), matrix and
instruction descriptors, MMA shapes (M = 64 and M = 128) and TMEM load
shapes.  Each mode computes D = A B^T on one CTA; D must match a float64
matmul of the same bf16 values to fp32-accumulation accuracy."""
import ctypes
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "cuda", "libtcprobe.so")

SHAPES = {0: (64, 64, 128), 1: (64, 64, 64), 2: (64, 64, 128), 3: (128, 64, 64),
          4: (128, 64, 64), 5: (128, 64, 128), 6: (128, 64, 64)}


@pytest.mark.parametrize("mode", list(SHAPES))
def test_mma_mode(mode):
    lib = ctypes.CDLL(LIB)
    lib.tc_probe_mma.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_void_p]
    M, N, K = SHAPES[mode]
    g = torch.Generator().manual_seed(100 + mode)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    Ad, Bd = A.cuda(), B.cuda()
    D = torch.full((M, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.tc_probe_mma(mode, Ad.data_ptr(), Bd.data_ptr(), D.data_ptr(), err.data_ptr(),
                          torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0 and int(err.item()) == 0
    want = A.double().numpy() @ B.double().numpy().T
    got = D.double().cpu().numpy()
    assert np.isfinite(got).all(), "unwritten outputs"
    rel = np.abs(got - want).max() / np.abs(want).max()
    assert rel < 1e-5, (mode, rel)


def _expected_layout():
    """The lane / column maps the kernels assume (the mma.sync m16n8 fragment)."""
    exp = np.zeros(4384, dtype=np.int64)
    for t in range(128):  # 16x256b.x4 load after filling (lane << 16) | column
        q, i = divmod(t, 32)
        for j in range(4):
            for e in range(4):
                lane = 32 * q + i // 4 + 8 * (e >> 1)
                col = 8 * j + 2 * (i % 4) + (e & 1)
                exp[t * 16 + 4 * j + e] = (lane << 16) | col
    for lane in range(128):  # 16x128b.x4 store of (thread << 8) | register
        q, l = divmod(lane, 32)
        for c in range(16):
            if l >= 16:
                exp[2048 + lane * 16 + c] = 0xFFFFFFFF
                continue
            e, r = divmod(l, 8)
            i = 4 * r + c % 4
            exp[2048 + lane * 16 + c] = ((32 * q + i) << 8) | (2 * (c // 4) + e)
    for i in range(32):  # 8 x 8 transpose: element ids row * 8 + column
        lo = 2 * (i % 4) * 8 + i // 4
        hi = (2 * (i % 4) + 1) * 8 + i // 4
        exp[4096 + i] = lo | (hi << 16)
    for i in range(32):  # ldmatrix.x4.trans: column i/4 of matrix k, rows 2(i%4), 2(i%4)+1
        for k in range(4):
            lo = 64 * k + 8 * (2 * (i % 4)) + i // 4
            exp[4128 + 4 * i + k] = lo | ((lo + 8) << 16)
    for e in range(128):  # stmatrix.x4.trans: shared row r of matrix k holds column r of the fragment
        vals = []
        for h in range(2):
            k, rc = divmod(2 * e + h, 64)
            r, c = divmod(rc, 8)
            vals.append(64 * k + 8 * c + r)
        exp[4256 + e] = vals[0] | (vals[1] << 16)
    return exp


def test_fragment_layouts():
    lib = ctypes.CDLL(LIB)
    lib.tc_probe_layout.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    out = torch.zeros(4384, dtype=torch.int32, device="cuda")
    assert lib.tc_probe_layout(out.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.int64) & 0xFFFFFFFF
    exp = _expected_layout()
    bad = np.nonzero(got != exp)[0]
    if len(bad):
        dump = os.environ.get("SSD_PROBE_DUMP")
        if dump:
            np.save(dump, got)
        names = ["16x256b load", "16x128b store", "8x8 transpose", "ldmatrix.trans", "stmatrix.trans"]
        part = lambda k: 0 if k < 2048 else 1 if k < 4096 else 2 if k < 4128 else 3 if k < 4256 else 4
        first = {n: [(int(k), hex(int(got[k])), hex(int(exp[k]))) for k in bad if part(k) == ni][:4]
                 for ni, n in enumerate(names)}
        raise AssertionError(f"{len(bad)} mismatches: {first}")

