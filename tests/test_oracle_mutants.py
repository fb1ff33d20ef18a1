"""Planted mistakes in a copy of the CPU oracle must each fail some pin.

Each mutant is the oracle's C source with one plausible slip (a dropped term,
a wrong sign or index, a swapped operand), compiled to a temporary library.
If every pin still passed on a mutant, the pins would not be tying the oracle
to the pages.  CPU only; the real oracle is never modified.
"""
import ctypes
import functools
import os
import subprocess
import tempfile

import pytest

import oracle
import oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")

MUTANTS = {
    "decay_sign_flipped": ("double a = exp(dtv * a_log);", "double a = exp(-dtv * a_log);"),
    "dt_dropped_from_input": ("const double u = dtv * (double)xt[p];", "const double u = (double)xt[p];"),
    "skip_term_dropped": ("yt[p] = acc + d_skip * (double)xt[p];", "yt[p] = acc;"),
    "readout_before_update": (
        "        Sp[n] = a * Sp[n] + u * (double)Bt[n];\n        acc += Sp[n] * (double)Ct[n];",
        "        acc += Sp[n] * (double)Ct[n];\n        Sp[n] = a * Sp[n] + u * (double)Bt[n];"),
    "B_and_C_swapped": (
        "        Sp[n] = a * Sp[n] + u * (double)Bt[n];\n        acc += Sp[n] * (double)Ct[n];",
        "        Sp[n] = a * Sp[n] + u * (double)Ct[n];\n        acc += Sp[n] * (double)Bt[n];"),
    "group_index_interleaved": ("const int64_t g = h / (H / G);", "const int64_t g = h % G;"),
    "reset_one_token_late": ("if (seq_idx && t > 0 && seq_idx[tok] != seq_idx[tok - 1]) a = 0.0;",
                             "if (seq_idx && t > 1 && seq_idx[tok - 1] != seq_idx[tok - 2]) a = 0.0;"),
    "reset_ignored": ("if (seq_idx && t > 0 && seq_idx[tok] != seq_idx[tok - 1]) a = 0.0;",
                      "if (seq_idx && t > 0 && seq_idx[tok] != seq_idx[tok - 1]) a = a;"),
    "initial_state_not_decayed": ("double a = exp(dtv * a_log);",
                                  "double a = (t == 0) ? 1.0 : exp(dtv * a_log);"),
    "decay_applied_after_input": ("        Sp[n] = a * Sp[n] + u * (double)Bt[n];",
                                  "        Sp[n] = a * (Sp[n] + u * (double)Bt[n]);"),
}


@functools.lru_cache(maxsize=None)
def _mutant_lib(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    d = tempfile.mkdtemp(prefix="oracle_mutant_")
    path = os.path.join(d, f"{name}.c")
    with open(path, "w") as fh:
        fh.write(src.replace(old, new))
    so = os.path.join(d, f"lib{name}.so")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", so, path, "-lm"],
                   check=True)
    return oracle.load_library(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    lib = _mutant_lib(name)
    fwd = functools.partial(oracle.ssd_fwd, lib=lib)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(fwd)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the planted mistake {name}"


# ----------------------------------------------------------------------------- block pieces
# Planted mistakes in a copy of oracle/block.py (conv1d + SiLU, gate): each must
# fail some pin of tests/test_block_oracle_pins.py.
BLOCK_MUTANTS = {
    "tap_direction_reversed": ("pre += w[None, None, :, k] * src",
                               "pre += w[None, None, :, w.shape[1] - 1 - k] * src"),
    "taps_shifted_by_one": ("shift = K - 1 - k", "shift = K - k"),
    "bias_dropped": ("pre = np.zeros((b, L, C)) if bias is None", "pre = np.zeros((b, L, C)) if True"),
    "packing_cut_ignored": ("            src *= same[:, :, None]\n", ""),
    "silu_sign_flipped": ("return v / (1.0 + np.exp(-v))", "return v / (1.0 + np.exp(v))"),
    "conv_grad_lands_on_the_output_token": ("du[:, : L - shift] += (w[None, None, :, k] * g * valid)[:, shift:]",
                                            "du += w[None, None, :, k] * g * valid"),
    "conv_grad_without_the_silu_slope": ("g = as_f64(dout) * silu_grad(_pre(u, w, bias, seq_idx))",
                                         "g = as_f64(dout) + 0.0 * _pre(u, w, bias, seq_idx)"),
    "conv_grad_ignores_the_packing_cut": ("            valid[:, shift:, 0] = seq[:, shift:] == seq[:, : L - shift]\n", ""),
}


@pytest.mark.parametrize("name", sorted(BLOCK_MUTANTS))
def test_block_mutant_fails_a_pin(name, monkeypatch, tmp_path):
    import importlib.util
    import sys

    import oracle.block
    import test_block_oracle_pins as bpins
    src = open(oracle.block.__file__).read()
    old, new = BLOCK_MUTANTS[name]
    assert src.count(old) == 1, name
    path = tmp_path / "block_mutant.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("oracle.block_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    spec.loader.exec_module(mod)
    monkeypatch.setattr(bpins, "block", mod)
    pins_run = [lambda: bpins.test_silu_is_x_times_the_logistic(),
                *[functools.partial(bpins.test_each_channel_is_a_numpy_convolution, K) for K in (1, 2, 4)],
                bpins.test_an_impulse_gives_back_the_filter, bpins.test_the_first_token_sees_only_itself,
                bpins.test_packed_sequences_equal_their_parts_run_alone, bpins.test_gate,
                *[functools.partial(bpins.test_conv_backward_matches_autograd, *c) for c in
                  [(4, True, None), (4, True, [[7, 1, 22], [30]])]]]
    failed = 0
    for pin in pins_run:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught {name}"


# ----------------------------------------------------------------------------- backward
# Planted mistakes in a copy of oracle/backward.py: each must fail some pin of
# tests/test_backward_oracle_pins.py.
BACKWARD_MUTANTS = {
    "carry_dropped": ("Gt = a[:, t + 1, :, None, None] * Gt", "Gt = 0.0 * Gt"),
    "dh0_not_decayed": ("dh0 = None if h0 is None else a[:, 0, :, None, None] * Gt",
                        "dh0 = None if h0 is None else Gt"),
    "ddt_decay_term_dropped": ("ddt[:, t] = g_in + A[None, :] * a[:, t] * g_dec", "ddt[:, t] = g_in"),
    "dA_without_dt": ("dA += np.sum(dt[:, t] * a[:, t] * g_dec, axis=0)", "dA += np.sum(a[:, t] * g_dec, axis=0)"),
    "dB_not_summed_over_group": ("dB[:, :, grp[h_]] += dBh[:, :, h_]", "dB[:, :, grp[h_]] = dBh[:, :, h_]"),
    "reset_ignored": ("a = np.where(reset[:, :, None], 0.0, a)", "a = a"),
    "skip_term_dropped_from_dx": ("dx += Dv[None, None, :, None] * dy", "dx += 0.0 * dy"),
    "gate_grad_is_the_logistic_slope": ("return s * (1.0 + v * (1.0 - s))", "return s * (1.0 - s)"),
    "gate_not_applied_to_dy": ("do * silu(zz), dfinal, seq)", "do, dfinal, seq)"),
}


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTANTS))
def test_backward_mutant_fails_a_pin(name, monkeypatch, tmp_path):
    import importlib.util

    import oracle.backward
    import test_backward_oracle_pins as bw
    src = open(oracle.backward.__file__).read()
    old, new = BACKWARD_MUTANTS[name]
    assert src.count(old) == 1, name
    path = tmp_path / "backward_mutant.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("oracle.backward_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    spec.loader.exec_module(mod)
    monkeypatch.setattr(bw, "backward", mod)
    failed = 0
    for case in bw.CASES:
        try:
            bw.test_backward_matches_autograd(case)
        except AssertionError:
            failed += 1
    try:
        bw.test_backward_matches_finite_differences_of_the_forward_oracle()
    except AssertionError:
        failed += 1
    for case in bw.CASES:
        try:
            bw.test_gated_backward_matches_autograd(case)
        except AssertionError:
            failed += 1
    try:
        bw.test_one_token_closed_form()
    except AssertionError:
        failed += 1
    assert failed > 0, f"no pin caught {name}"
