"""The CPU oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
import oracle_pins as pins
import ssd_inputs as si


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.ssd_fwd)


def test_unit_sampling_matches_full_run():
    """Computing a subset of (b, h) units gives the same numbers as the full run."""
    d = pins.small_inputs(b=3, L=30, H=4, seed=41)
    y, f = oracle.ssd_fwd(*[d[k] for k in pins.KEYS])
    units = [1, 6, 11]
    ys, fs = oracle.ssd_fwd(*[d[k] for k in pins.KEYS], units=units)
    for u in units:
        b, h = divmod(u, 4)
        assert np.array_equal(ys[b, :, h], y[b, :, h])
        assert np.array_equal(fs[b, h], f[b, h])
    other = [u for u in range(12) if u not in units]
    for u in other:
        b, h = divmod(u, 4)
        assert not ys[b, :, h].any()


def test_thread_count_does_not_change_results():
    d = pins.small_inputs(b=2, L=50, H=4, seed=43)
    y1, f1 = oracle.ssd_fwd(*[d[k] for k in pins.KEYS], nthreads=1)
    y4, f4 = oracle.ssd_fwd(*[d[k] for k in pins.KEYS], nthreads=4)
    assert np.array_equal(y1, y4) and np.array_equal(f1, f4)


def test_bf16_inputs_are_widened_exactly():
    """bf16 tensors reach the oracle as their exact values."""
    shape = si.SSDShape("b", 1, 20, 2, 4, 8, 1, 16, "bf16", seed=3)
    d = si.make_inputs(shape)
    y, _ = oracle.ssd_fwd(*[d[k] for k in pins.KEYS])
    e = {k: (v.float() if v is not None else None) for k, v in d.items() if k in pins.KEYS}
    y2, _ = oracle.ssd_fwd(*[e[k] for k in pins.KEYS])
    assert np.array_equal(y, y2)


def test_bad_arguments_rejected():
    lib = oracle._get_lib()
    rc = lib.oracle_ssd_fwd(1, 4, 3, 2, 2, 2, *([None] * 8), 0, None, None, None, 0, 0)
    assert rc == -1
