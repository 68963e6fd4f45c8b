"""The CPU oracle against its pins (see oracle_pins.py), plus the directional claims the pages
make about windows and compensators."""
import numpy as np
import pytest

import oracle
from oracle_pins import PINS, rand_inputs, rel


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin, orc):
    pin(orc.load())


def _quality(W, r, fmt="int8", seed=77, T=192, D=32, nh=8, gate="scalar"):
    q, k, v, g, beta = rand_inputs(seed, T, nh, D, gate, outlier=True)
    S0 = np.random.default_rng(seed).standard_normal((nh, D, D))
    exact, _ = oracle.plain_run(q, k, v, g, beta, S0=S0)
    res = oracle.o2_run(q, k, v, g, beta, W=W, r=r, fmt=fmt, S0=S0)
    return rel(res.o, exact)


def test_direction_window_beats_every_step(orc):
    """"LeapQuant ..." Abstract: quantizing once per window limits the accumulation of
    rounding error that per-step write-back suffers ("Low-Bit GDN ..." Abstract)."""
    for fmt in ("int8", "int4_g32"):
        e1 = _quality(1, 0, fmt)
        e32 = _quality(32, 0, fmt)
        assert e32 < e1, (fmt, e32, e1)


def test_direction_compensators_help_on_outliers(orc):
    """"LeapQuant ..." Abstract: keeping the largest outliers as compensator pairs lowers the
    error each quantization adds."""
    for fmt in ("int8", "int4_g32"):
        e0 = _quality(16, 0, fmt, gate="diag")
        e4 = _quality(16, 4, fmt, gate="diag")
        assert e4 <= e0, (fmt, e4, e0)


def test_zero_steps_and_empty_batch(orc):
    z = np.zeros((0, 0, 16))
    res = oracle.o2_run(z, z, z, np.zeros((0, 0)), np.zeros((0, 0)), W=4)
    assert res.o.shape == (0, 0, 16) and res.codes.shape == (0, 16, 16)
    o, S = oracle.plain_run(np.zeros((0, 2, 4)), np.zeros((0, 2, 4)), np.zeros((0, 2, 4)),
                            np.zeros((0, 2)), np.zeros((0, 2)))
    assert o.shape == (0, 2, 4) and not S.any()
