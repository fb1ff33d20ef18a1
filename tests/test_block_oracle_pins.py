"""Pins for the block-piece oracle (causal depthwise conv1d + SiLU, and the
SiLU gate) against library routines and closed forms, independent of the
oracle's own code."""
import numpy as np
import pytest
import scipy.special
import torch

from oracle import block


def _rand(shape, seed):
    # fp32-representable values: the oracle widens its inputs through fp32
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32).astype(np.float64)


def test_silu_is_x_times_the_logistic():
    v = np.linspace(-30, 30, 1001)
    assert np.allclose(block.silu(v), v * scipy.special.expit(v), rtol=1e-13, atol=1e-300)
    assert block.silu(np.array([0.0]))[0] == 0.0


@pytest.mark.parametrize("K", [1, 2, 4])
def test_each_channel_is_a_numpy_convolution(K):
    b, L, C = 2, 37, 5
    u, w, bias = _rand((b, L, C), 1), _rand((C, K), 2), _rand((C,), 3)
    got = block.conv1d_silu(u, w, bias)
    for bb in range(b):
        for c in range(C):
            pre = np.convolve(u[bb, :, c], w[c, ::-1])[:L] + bias[c]
            assert np.allclose(got[bb, :, c], pre * scipy.special.expit(pre), rtol=1e-12, atol=1e-12)


def test_an_impulse_gives_back_the_filter():
    K, L = 4, 10
    u = np.zeros((1, L, 1))
    u[0, 3, 0] = 1.0
    w = np.array([[0.5, -1.0, 2.0, 0.25]])
    got = block.conv1d_silu(u, w)
    pre = np.zeros(L)
    pre[3:3 + K] = w[0, ::-1]  # output 3 + j sees the impulse through tap K-1-j
    assert np.allclose(got[0, :, 0], block.silu(pre), rtol=1e-14, atol=1e-15)


def test_the_first_token_sees_only_itself():
    u, w, bias = _rand((3, 6, 4), 4), _rand((4, 4), 5), _rand((4,), 6)
    got = block.conv1d_silu(u, w, bias)
    pre0 = bias + w[:, 3] * u[:, 0]
    assert np.allclose(got[:, 0], block.silu(pre0), rtol=1e-13)


def test_packed_sequences_equal_their_parts_run_alone():
    b, L, C, K = 2, 30, 3, 4
    u, w, bias = _rand((b, L, C), 7), _rand((C, K), 8), _rand((C,), 9)
    lens = [[7, 1, 22], [30]]
    seq = np.zeros((b, L), dtype=np.int32)
    sid = 0
    for r, row in enumerate(lens):
        t = 0
        for n in row:
            seq[r, t:t + n] = sid
            sid += 1
            t += n
    got = block.conv1d_silu(u, w, bias, torch.from_numpy(seq))
    for r, row in enumerate(lens):
        t = 0
        for n in row:
            alone = block.conv1d_silu(u[r:r + 1, t:t + n], w, bias)
            assert np.allclose(got[r:r + 1, t:t + n], alone, rtol=1e-13)
            t += n


def test_gate():
    y, z = _rand((4, 9), 10), _rand((4, 9), 11)
    assert np.allclose(block.gate(y, z), y * z * scipy.special.expit(z), rtol=1e-13)
