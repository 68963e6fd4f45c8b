"""Residual smoothing ("LeapQuant: Efficient Linear Attention with Accurate Recurrent State
Quantization", Abstract: the residual is smoothed before quantization; reading: per-key-column
power-of-two factors) on the GPU against the oracle's buffered form with the same smoothing:
outputs, codes, scales, compensators and the smoothing exponents, through every kernel that
quantizes or reads a frozen state (initial quantize, tensor-core and FMA steps and window ends,
materialisation, forced flushes). All calls go through the C ABI."""
import numpy as np
import pytest
import torch

import bit_recurrent_state_gdn_b200 as gdn
import oracle
from gdn_harness import (
    GpuRun, cfg_of, compare, gpu_run, gpu_warmup, oracle_initial_state, oracle_run, rel_l2,
    _heads_np,
)
from workloads import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu

MID, KDA, LONG4 = WORKLOADS["gdn-mid"], WORKLOADS["kda"], WORKLOADS["gdn-long-int4"]

CASES = {
    "tiny-d16-f32": WORKLOADS["gdn-tiny"].with_(name="sm-tiny", H=3, outliers=True, warmup=16,
                                                smooth=True),
    "kda-d16-r2": WORKLOADS["gdn-tiny"].with_(name="sm-kda-d16", H=3, gate="diag", r=2,
                                              outliers=True, warmup=16, smooth=True),
    "gdn-int8": MID.with_(name="sm-gdn-int8", B=2, H=4, T=150, warmup=48, smooth=True),
    "kda-int8-r4": KDA.with_(name="sm-kda-int8", B=2, H=4, T=150, warmup=48, smooth=True),
    "gdn-int4": LONG4.with_(name="sm-gdn-int4", B=2, H=4, T=300, warmup=48, smooth=True),
    "kda-int4-r2": LONG4.with_(name="sm-kda-int4", B=1, H=4, T=100, W=32, r=2, gate="diag",
                               warmup=48, smooth=True),
    "gdn-int8-f32": MID.with_(name="sm-gdn-f32", B=1, H=4, T=100, W=32, act="f32", buf="f32",
                              warmup=32, smooth=True),
    "kda-int8-w160": KDA.with_(name="sm-kda-w160", B=1, H=2, T=170, W=160, r=2, warmup=32,
                               smooth=True),
}


def _parity(wl, T=None):
    run = gpu_run(wl, T=T)
    heads = np.arange(wl.heads)
    res = oracle_run(wl, heads, run.inputs, oracle_initial_state(wl, heads))
    return run, res, compare(wl, run, heads, res)


@pytest.mark.parametrize("name", list(CASES))
def test_smoothed_window_decode_parity(name):
    wl = CASES[name]
    run, res, p = _parity(wl)
    print(name, p)
    p.check()
    assert np.any(res.sexp != 0), "the case never smooths"
    assert int(run.state.status[0].item()) == 0


@pytest.mark.parametrize("name", ["gdn-int8", "gdn-int4", "kda-int8-r4"])
def test_smoothed_initial_quantize(name):
    wl = CASES[name]
    _, res, p = _parity(wl, T=0)
    p.check()
    assert np.any(res.sexp != 0)


@pytest.mark.parametrize("name", ["gdn-int8", "gdn-int4", "kda-int8-r4"])
def test_smoothed_materialize_mid_window(name):
    wl = CASES[name].with_(T=90)
    run, res, p = _parity(wl)
    p.check()
    S = torch.empty((wl.heads, wl.D, wl.D), device="cuda")
    gdn.gdn_state_materialize(cfg_of(wl), run.state, S)
    torch.cuda.synchronize()
    assert rel_l2(S.double().cpu().numpy(), res.S) < 1e-4


@pytest.mark.parametrize("name", ["gdn-int8", "kda-int8-r4"])
def test_smoothed_forced_flush(name):
    wl = CASES[name].with_(B=3, H=2, T=130)
    cfg = cfg_of(wl)
    inputs = decode_inputs(wl, "cuda")
    S0 = gpu_warmup(wl)
    st = gdn.GdnState.allocate(cfg)
    gdn.gdn_state_quantize(cfg, S0, st)
    o = torch.empty_like(inputs["q"])
    flush_mask = np.zeros((wl.T, wl.heads), np.uint8)
    plan = {10: [1, 0, 0], 37: [0, 1, 1], 71: [1, 1, 0]}
    for t in range(wl.T):
        gdn.gdn_decode_window_step(cfg, st, *(inputs[n][t] for n in ("q", "k", "v", "g", "beta")),
                                   o[t])
        if t in plan:
            gdn.gdn_window_flush(cfg, st, torch.tensor(plan[t], dtype=torch.int32, device="cuda"))
            flush_mask[t] = np.repeat(plan[t], wl.H)
    torch.cuda.synchronize()
    heads = np.arange(wl.heads)
    res = oracle_run(wl, heads, inputs, oracle_initial_state(wl, heads), flush_mask)
    compare(wl, GpuRun(o, st, S0, inputs), heads, res).check()


def test_smoothing_lowers_the_error_against_the_unquantized_recurrence():
    """What the page claims for the step: with the outlier key channels of the recipe and no
    compensators, the smoothed state's outputs are closer to the unquantized fp64 recurrence."""
    wl = MID.with_(name="sm-quality", B=2, H=8, T=128, warmup=64)
    errs = {}
    for smooth in (False, True):
        w = wl.with_(smooth=smooth)
        run = gpu_run(w)
        heads = np.arange(w.heads)
        q, k, v, g, beta = (_heads_np(run.inputs[n], heads) for n in ("q", "k", "v", "g", "beta"))
        o_ref, _ = oracle.plain_run(q, k, v, g, beta, S0=oracle_initial_state(w, heads))
        errs[smooth] = rel_l2(_heads_np(run.o, heads), o_ref)
    print("quality vs fp64 recurrence", errs)
    assert errs[True] < errs[False], errs
