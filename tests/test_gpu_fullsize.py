"""CUDA path vs the CPU oracle at the workloads' full sizes, in the launch configuration the
benchmark times (every head of the batch, one launch per decode step through
gdn_decode_window_steps), compared on sampled heads that the oracle recomputes from their own
inputs: every head of the first and the last sequence plus random others; the serving and KDA
workloads also with residual smoothing. Also the largest window and compensator count the build
accepts.

Each run also reports the quality figure: the GPU output against the unquantized fp64
recurrence from the same initial state (not a parity bar; the windowed low-bit state is an
approximation of it)."""
import numpy as np
import pytest

import bit_recurrent_state_gdn_b200 as gdn
import oracle
from gdn_harness import (
    _heads_np, compare, gpu_run, oracle_initial_state, oracle_run, rel_l2, sample_heads,
)
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu

# heads sampled per workload: sized so the oracle's share stays at a few seconds
SAMPLE = {"gdn-mid": 48, "kda": 40, "gdn-long-int4": 16, "gdn-serving": 80}


def _quality(wl, run, heads, S0):
    o_gpu = _heads_np(run.o, heads)
    q, k, v, g, beta = (_heads_np(run.inputs[n], heads) for n in ("q", "k", "v", "g", "beta"))
    o_ref, _ = oracle.plain_run(q, k, v, g, beta, S0=S0, state_round="none")
    return rel_l2(o_gpu, o_ref)


@pytest.mark.parametrize("name", list(SAMPLE) + ["gdn-serving+smooth", "kda+smooth"])
def test_full_size_sampled_heads(name):
    base, _, extra = name.partition("+")
    wl = WORKLOADS[base].with_(smooth=extra == "smooth")
    run = gpu_run(wl)
    assert int(run.state.status[0].item()) == 0
    heads = sample_heads(wl, SAMPLE[base], seed=wl.seed)
    S0 = oracle_initial_state(wl, heads)
    res = oracle_run(wl, heads, run.inputs, S0)
    p = compare(wl, run, heads, res)
    quality = _quality(wl, run, heads, S0)
    print(f"\n{name}: heads={len(heads)} o_rel={p.o_rel:.2e} (unrounded {p.o_rel_unrounded:.2e}) "
          f"flips={p.flip_frac:.2e} scale_rel={p.scale_rel:.1e} (rows above 1e-4: {p.scale_loose_rows} of {p.scale_rows}) comp_rel={p.comp_rel:.1e} "
          f"tie_heads={p.tie_heads} quality_vs_fp64_recurrence={quality:.3e}")
    p.check()
    assert np.isfinite(quality)


def _largest_window(D, r, gate):
    """Largest W the build accepts for this head size / rank / gate (the step kernel's shared
    memory grows with W)."""
    lo, hi = 1, 4096
    while lo < hi:
        mid = (lo + hi + 1) // 2
        try:
            gdn.gdn_state_sizes(gdn.make_config(1, 1, D, mid, r, gate, "int8", "bf16", "bf16"))
            lo = mid
        except gdn.GdnError:
            hi = mid - 1
    return lo


@pytest.mark.parametrize("gate", ["scalar", "diag"])
def test_largest_window_and_compensator_count(gate):
    r = 16  # the largest compensator count per head
    W = _largest_window(128, r, gate)
    assert W >= 64
    wl = WORKLOADS["kda"].with_(name=f"max-{gate}", B=2, H=3, T=W + W // 3, W=W, r=r,
                                gate=gate, warmup=48)
    run = gpu_run(wl)
    heads = np.arange(wl.heads)
    res = oracle_run(wl, heads, run.inputs, oracle_initial_state(wl, heads))
    compare(wl, run, heads, res).check()
