"""Host checks of the parity harness's acceptance logic (no GPU): a loose scale row is accepted
only when it is the oracle's own alternative result -- one write-vector entry of that row,
lying on a rounding midpoint, rounded to its other neighbour -- and rejected otherwise."""
import numpy as np

import oracle
from gdn_harness import U_MIDPOINT_NOISE, _midpoint_distance, _o2, explain_loose_row
from oracle_pins import rand_inputs
from workloads import Workload


def test_midpoint_distance():
    q = 2.0 ** -7  # bf16 quantum in [1, 2)
    u = np.array([1.0, 1.0 + q / 2, 1.0 + q / 2 + q / 64, -(1.0 + q / 2), 0.0])
    d = _midpoint_distance(u, "bf16")
    assert np.allclose(d, [0.5, 0.0, 1 / 64, 0.0, 1.0])
    assert _midpoint_distance(np.array([1.0 + 2.0 ** -24]), "f32")[0] == 0.0


def _setup(seed):
    wl = Workload("harness", B=1, H=3, D=16, T=24, W=8, act="bf16", buf="bf16", warmup=0)
    q, k, v, g, beta = rand_inputs(seed, wl.T, wl.heads, wl.D)
    S0 = np.random.default_rng(seed).standard_normal((wl.heads, wl.D, wl.D)).astype(np.float32)
    res = _o2(wl, q, k, v, g, beta, S0, None, want_u_raw=True)
    res.rerun = (q, k, v, g, beta, S0, None)
    return wl, res


def test_loose_row_explained_only_by_a_midpoint_flip():
    for seed in range(40):
        wl, res = _setup(seed)
        # the entry of the last window closest to a midpoint, over all heads and rows
        last = res.u_raw[wl.T - wl.W:]
        d = _midpoint_distance(last, wl.buf)
        t, a, v = np.unravel_index(np.argmin(d), d.shape)
        if d[t, a, v] > U_MIDPOINT_NOISE:
            continue
        t += wl.T - wl.W
        q, k, vv, g, beta, S0, _ = res.rerun
        one = slice(a, a + 1)
        flip = np.zeros((wl.T, 1, wl.D), np.uint8)
        flip[t, 0, v] = 1
        alt = _o2(wl, q[:, one], k[:, one], vv[:, one], g[:, one], beta[:, one], S0[one], None,
                  u_flip=flip)
        if np.array_equal(alt.scales[0, v], res.scales[a, v]):
            continue  # this flip does not reach the scale: try another case
        assert explain_loose_row(wl, res, int(a), int(v), alt.scales[0, v])
        assert not explain_loose_row(wl, res, int(a), int(v), res.scales[a, v] * (1 + 3e-3))
        return
    raise AssertionError("no case with a write-vector entry on a midpoint")
