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
