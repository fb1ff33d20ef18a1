"""The Python binding rejects bad arguments before anything reaches the
library: CPU tensors, wrong shapes or dtypes.  No kernel runs here."""
import pytest
import torch

import mamba_ssd_chunked_03_b200 as ssd


def _fwd_args(**kw):
    b, L, H, P, N, G = 1, 8, 2, 4, 8, 1
    d = dict(x=torch.zeros(b, L, H, P), dt=torch.zeros(b, L, H), A=torch.zeros(H), B=torch.zeros(b, L, G, N),
             C=torch.zeros(b, L, G, N), D=None)
    d.update(kw)
    return d


def test_fwd_rejects_cpu_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        ssd.fwd(**_fwd_args())


@pytest.mark.parametrize("kw,exc", [
    ({"x": torch.zeros(1, 8, 2, 4, dtype=torch.float16)}, TypeError),       # dtype
    ({"B": torch.zeros(1, 8, 1, 9)}, ValueError),                           # B / C shape mismatch
    ({"dt": torch.zeros(1, 8, 3)}, ValueError),                             # dt shape
    ({"A": torch.zeros(2, dtype=torch.float64)}, TypeError),                # A dtype
    ({"D": torch.zeros(3)}, ValueError),                                    # D shape
])
def test_fwd_rejects_bad_shapes_and_dtypes(kw, exc):
    with pytest.raises(exc):
        ssd.fwd(**_fwd_args(**kw))


def test_step_rejects_bad_arguments():
    b, H, P, N, G = 2, 4, 8, 8, 2
    x, dt, A = torch.zeros(b, H, P), torch.zeros(b, H), torch.zeros(H)
    B, C, st = torch.zeros(b, G, N), torch.zeros(b, G, N), torch.zeros(b, H, P, N)
    with pytest.raises(ValueError):
        ssd.step(x, dt, A, B, C, None, st)  # CPU tensors
    with pytest.raises(ValueError):
        ssd.step(x, dt, A, B, C, None, torch.zeros(b, H, P, N + 1))  # state shape
    with pytest.raises(TypeError):
        ssd.step(x.double(), dt, A, B.double(), C.double(), None, st)  # dtype


def test_conv_rejects_bad_arguments():
    u, w = torch.zeros(1, 8, 16), torch.zeros(16, 4)
    with pytest.raises(ValueError):
        ssd.conv1d_silu(u, w)  # CPU tensors
    with pytest.raises(ValueError):
        ssd.conv1d_silu(u, torch.zeros(15, 4))  # weight rows != channels
    with pytest.raises(TypeError):
        ssd.conv1d_silu(u, w.double())


def test_total_decay_and_fold_reject_cpu_tensors():
    with pytest.raises(ValueError):
        ssd.total_decay(torch.zeros(1, 4, 2), torch.zeros(2))
    with pytest.raises(ValueError):
        ssd.state_fold(torch.zeros(2, 1, 2, 4, 4), torch.zeros(2, 1, 2), None, 1, (1, 2, 4, 4))


def test_bwd_rejects_bad_arguments():
    d = _fwd_args()
    dy = torch.zeros_like(d["x"])
    with pytest.raises(ValueError, match="CUDA"):
        ssd.bwd(**d, dy=dy)  # CPU tensors
    with pytest.raises(TypeError):
        ssd.bwd(**_fwd_args(x=torch.zeros(1, 8, 2, 4, dtype=torch.float16)), dy=dy)


def test_autograd_wrapper_rejects_cpu_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        ssd.ssd_chunked(**_fwd_args())
