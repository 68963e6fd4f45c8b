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


def test_smoothing_exponent_near_ties_are_reported(orc):
    """A residual column max-abs within 1e-6 of a power of 4 sits where the smoothing exponent
    steps; the oracle reports the head as a near tie (another correct implementation may put
    the column on the other side), and does not for column maxima away from one."""
    lib = orc.load()
    rng = np.random.default_rng(29)
    S = rng.uniform(-1, 1, size=(16, 16))
    S *= (2.0 + rng.uniform(size=16))[None, :] / np.abs(S).max(axis=0)  # column maxima in [2, 3)
    assert oracle.window_end(S, "int8", smooth=True, lib=lib).near_tie == 0
    S[3, 5] = 4.0 * (1 - 3e-7)  # just below 4 = 2^2
    assert oracle.window_end(S, "int8", smooth=True, lib=lib).near_tie == 1
    assert oracle.window_end(S, "int8", smooth=False, lib=lib).near_tie == 0
