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


def _torch_conv_silu(u, w, bias, lens=None):
    """An fp64 depthwise causal conv1d + SiLU written with torch's conv1d
    (groups = channels, left padding K - 1); with per-row sequence lengths,
    each sequence is convolved alone and the pieces concatenated."""
    b, L, C = u.shape
    K = w.shape[1]
    rows = []
    for r in range(b):
        pieces = []
        for lo, hi in (_bounds(lens[r]) if lens else [(0, L)]):
            x = u[r:r + 1, lo:hi].transpose(1, 2)  # (1, C, n)
            x = torch.nn.functional.pad(x, (K - 1, 0))
            pieces.append(torch.nn.functional.conv1d(x, w[:, None, :], bias, groups=C).transpose(1, 2))
        rows.append(torch.cat(pieces, dim=1))
    pre = torch.cat(rows, dim=0)
    return pre * torch.sigmoid(pre)


def _bounds(lengths):
    out, t = [], 0
    for n in lengths:
        out.append((t, t + n))
        t += n
    return out


@pytest.mark.parametrize("K,with_bias,lens", [(1, True, None), (2, False, None), (4, True, None),
                                               (4, True, [[7, 1, 22], [30]]), (3, False, [[1, 1, 28], [15, 15]])])
def test_conv_backward_matches_autograd(K, with_bias, lens):
    b, L, C = 2, 30, 3
    u, w = _rand((b, L, C), 20 + K), _rand((C, K), 21)
    bias = _rand((C,), 22) if with_bias else None
    dout = _rand((b, L, C), 23)
    seq = None
    if lens:
        seq = np.concatenate([np.full(n, i, dtype=np.int32) for i, n in
                              enumerate([n for row in lens for n in row])]).reshape(b, L)
    du, dw, db = block.conv1d_silu_bwd(u, w, bias, dout, None if seq is None else torch.from_numpy(seq))
    ut, wt = torch.tensor(u, requires_grad=True), torch.tensor(w, requires_grad=True)
    bt = torch.tensor(bias, requires_grad=True) if with_bias else None
    (_torch_conv_silu(ut, wt, bt, lens) * torch.from_numpy(dout)).sum().backward()
    assert np.allclose(du, ut.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dw, wt.grad.numpy(), rtol=1e-12, atol=1e-12)
    if with_bias:
        assert np.allclose(db, bt.grad.numpy(), rtol=1e-12, atol=1e-12)
    # the forward written here agrees with the oracle's forward
    assert np.allclose(_torch_conv_silu(torch.tensor(u), torch.tensor(w), None if bias is None else torch.tensor(bias),
                                        lens).numpy(),
                       block.conv1d_silu(u, w, bias, None if seq is None else torch.from_numpy(seq)), rtol=1e-12)
