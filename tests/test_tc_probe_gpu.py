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

SHAPES = {0: (64, 64, 128), 1: (64, 64, 64), 2: (64, 64, 128), 3: (128, 64, 64)}


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
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
