"""The conv1d + SiLU backward kernels (``csrc/ssd_conv_bwd.cuh``) on the CPU
through the test-only emulation in ``tests/emu`` (AddressSanitizer + UBSan,
exact-size buffers, NaN-filled outputs and workspace), against the fp64
oracle, before any GPU runs them.  ``test_bwd_gpu.py`` runs the same
cases on the GPU."""
import pytest

import emu_bwd
from bwd_cases import CONV_CASES, conv_case_inputs, conv_compare
from oracle import block

pytestmark = pytest.mark.skipif(not emu_bwd.available(), reason="g++ not available")


@pytest.mark.parametrize("case", CONV_CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("reverse", [False, True], ids=["fwd_order", "rev_order"])
def test_emulated_conv_backward_matches_oracle(case, reverse):
    u, w, bias, dout, seq = conv_case_inputs(case)
    out = emu_bwd.run_conv(u, w, bias, dout, seq, reverse=reverse)
    assert out["status"] == 0 and out["launches"] == 2
    conv_compare(out["du"], out["dw"], out["dbias"], block.conv1d_silu_bwd(u, w, bias, dout, seq, with_scale=True))


def test_emulated_conv_backward_without_dbias():
    u, w, bias, dout, seq = conv_case_inputs(CONV_CASES[0])
    out = emu_bwd.run_conv(u, w, bias, dout, seq, want_dbias=False)
    assert out["status"] == 0 and out["dbias"] is None
    ref = block.conv1d_silu_bwd(u, w, bias, dout, seq)
    conv_compare(out["du"], out["dw"], None, ref)


def test_emulated_conv_backward_rejects_width_5():
    u, w, bias, dout, seq = conv_case_inputs(CONV_CASES[2])
    import torch
    assert emu_bwd.run_conv(u, torch.zeros(u.shape[2], 5), bias, dout, seq)["status"] == 2
