"""CUDA path vs the CPU oracle, element by element, on seeded inputs small enough for the oracle
to finish in seconds (several tiles of every kernel, a ragged final window), plus the edge cases
of the method. All calls go through the C ABI."""
import numpy as np
import pytest
import torch

import bit_recurrent_state_gdn_b200 as gdn
import oracle
from gdn_harness import (
    cfg_of, compare, gpu_codes, gpu_run, gpu_warmup, oracle_initial_state, oracle_run, rel_l2,
    round_act, _heads_np,
)
from workloads import WORKLOADS, decode_inputs, torch_dtype

pytestmark = pytest.mark.gpu

MID, KDA, LONG4 = WORKLOADS["gdn-mid"], WORKLOADS["kda"], WORKLOADS["gdn-long-int4"]

# T not a multiple of W: the run ends inside a window
SMALL = {
    "gdn-tiny": WORKLOADS["gdn-tiny"],
    "gdn-int8": MID.with_(name="gdn-int8-small", B=2, H=4, T=150, warmup=48),
    "kda-int8-r4": KDA.with_(name="kda-small", B=2, H=4, T=150, warmup=48),
    "gdn-int4": LONG4.with_(name="gdn-int4-small", B=2, H=4, T=300, warmup=48),
    "kda-int4-r2": LONG4.with_(name="kda-int4-small", B=1, H=4, T=100, W=32, r=2, gate="diag",
                               warmup=48),
    "gdn-int8-f32": MID.with_(name="gdn-f32", B=1, H=4, T=100, W=32, act="f32", buf="f32",
                              warmup=32),
    "gdn-int8-bf16-f32buf": MID.with_(name="gdn-f32buf", B=1, H=4, T=100, W=32, buf="f32",
                                      warmup=32),
    "kda-d16-f32-r2": WORKLOADS["gdn-tiny"].with_(name="kda-d16", H=3, gate="diag", r=2,
                                                  outliers=True, warmup=16),
    "gdn-d16-bf16-r3": WORKLOADS["gdn-tiny"].with_(name="gdn-d16-bf16", H=3, r=3, act="bf16",
                                                   buf="bf16", T=70, warmup=16),
    # diagonal gate with a window past the tensor-core flush's limit (FMA path)
    "kda-int8-w160": KDA.with_(name="kda-w160", B=1, H=2, T=170, W=160, r=2, warmup=32),
    "gdn-int8-w16": MID.with_(name="gdn-w16", B=2, H=3, T=50, W=16, warmup=32),
    "gdn-int8-w20": MID.with_(name="gdn-w20", B=2, H=3, T=50, W=20, r=1, warmup=32),
    # tensor-core flush with three 16-pair blocks (window 40 / 48: 48 padded pairs)
    "gdn-int8-w40-r3": MID.with_(name="gdn-w40", B=2, H=3, T=90, W=40, r=3, warmup=32),
    "gdn-int4-w48": MID.with_(name="gdn-w48-int4", B=2, H=3, T=100, W=48, fmt="int4_g32",
                              warmup=32),
}


def _parity(wl, T=None, flush_mask=None, inputs=None):
    run = gpu_run(wl, T=T, inputs=inputs)
    heads = np.arange(wl.heads)
    S0 = oracle_initial_state(wl, heads)
    res = oracle_run(wl, heads, run.inputs, S0, flush_mask)
    return run, res, compare(wl, run, heads, res)


@pytest.mark.parametrize("name", list(SMALL))
def test_window_decode_parity(name):
    wl = SMALL[name]
    _, _, p = _parity(wl)
    p.check()


def test_warmup_state_matches_oracle():
    """fp32-state baseline kernel over the warm-up tokens vs the oracle's plain recurrence."""
    for wl in (SMALL["gdn-int8"], SMALL["kda-int8-r4"]):
        S_gpu = gpu_warmup(wl).reshape(wl.heads, wl.D, wl.D).double().cpu().numpy()
        S_orc = oracle_initial_state(wl, np.arange(wl.heads))
        assert rel_l2(S_gpu, S_orc) < 1e-5


@pytest.mark.parametrize("fmt,tol", [("fp32", 1e-5), ("bf16", 2e-3)])
@pytest.mark.parametrize("gate", ["scalar", "diag"])
def test_baseline_step_parity(fmt, tol, gate):
    wl = MID.with_(B=2, H=3, T=40, gate=gate, warmup=0)
    cfg = gdn.make_config(wl.B, wl.H, wl.D, gate=gate, fmt=fmt, act="bf16")
    inp = decode_inputs(wl, "cuda")
    rng = np.random.default_rng(1)
    S0 = rng.standard_normal((wl.heads, wl.D, wl.D)).astype(np.float32) * 0.3
    sdt = torch.float32 if fmt == "fp32" else torch.bfloat16
    S = torch.from_numpy(S0).to(sdt).cuda().contiguous()
    S0_used = S.double().cpu().numpy()
    o = torch.empty_like(inp["q"])
    for t in range(wl.T):
        gdn.gdn_baseline_step(cfg, S, inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                              inp["beta"][t], o[t])
    torch.cuda.synchronize()
    heads = np.arange(wl.heads)
    q, k, v, g, beta = (_heads_np(inp[n], heads) for n in ("q", "k", "v", "g", "beta"))
    o_ref, S_ref = oracle.plain_run(q, k, v, g, beta, S0=S0_used,
                                    state_round="f32" if fmt == "fp32" else "bf16")
    assert rel_l2(_heads_np(o, heads), round_act(o_ref, "bf16")) < max(tol, 2e-3)
    assert rel_l2(S.double().cpu().numpy().reshape(S_ref.shape), S_ref) < tol


def test_window_one_is_quantize_every_step():
    wl = SMALL["gdn-int8"].with_(W=1, T=20)
    _, _, p = _parity(wl)
    p.check()


def test_window_longer_than_run_never_flushes():
    wl = SMALL["gdn-int8"].with_(W=200, T=150)
    run, res, p = _parity(wl)
    p.check()
    assert (run.state.pos.cpu().numpy() == 150).all()
    S = torch.empty((wl.heads, wl.D, wl.D), device="cuda")
    gdn.gdn_state_materialize(cfg_of(wl), run.state, S)
    assert rel_l2(S.double().cpu().numpy(), res.S) < 1e-4


@pytest.mark.parametrize("name", ["gdn-int8", "kda-int8-r4", "gdn-int4"])
def test_materialize_mid_window(name):
    wl = SMALL[name].with_(T=90)
    run, res, p = _parity(wl)
    p.check()
    S = torch.empty((wl.heads, wl.D, wl.D), device="cuda")
    gdn.gdn_state_materialize(cfg_of(wl), run.state, S)
    torch.cuda.synchronize()
    assert rel_l2(S.double().cpu().numpy(), res.S) < 1e-4


@pytest.mark.parametrize("name", ["gdn-int8", "kda-int8-r4"])
def test_forced_flush_ragged_windows(name):
    """Forced flushes of chosen sequences desynchronise the windows of a batch."""
    wl = SMALL[name].with_(B=3, H=2, T=130)
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
            m = torch.tensor(plan[t], dtype=torch.int32, device="cuda")
            gdn.gdn_window_flush(cfg, st, m)
            flush_mask[t] = np.repeat(plan[t], wl.H)
    torch.cuda.synchronize()
    from gdn_harness import GpuRun
    run = GpuRun(o, st, S0, inputs)
    heads = np.arange(wl.heads)
    res = oracle_run(wl, heads, inputs, oracle_initial_state(wl, heads), flush_mask)
    compare(wl, run, heads, res).check()
    assert len(set(st.pos.cpu().numpy().tolist())) > 1


def test_flush_of_empty_window_is_noop():
    wl = SMALL["gdn-int8"].with_(T=64)   # ends exactly on a window boundary: pos == 0
    run = gpu_run(wl)
    before = run.state.clone()
    gdn.gdn_window_flush(cfg_of(wl), run.state)
    torch.cuda.synchronize()
    for n, t in before.tensors().items():
        assert torch.equal(t, getattr(run.state, n)), n


def test_checkpoint_resume_is_bit_identical():
    wl = SMALL["kda-int8-r4"]
    cfg = cfg_of(wl)
    inputs = decode_inputs(wl, "cuda")
    S0 = gpu_warmup(wl)
    a = gdn.GdnState.allocate(cfg)
    gdn.gdn_state_quantize(cfg, S0, a)
    o1 = torch.empty_like(inputs["q"])
    args = lambda lo, hi: [inputs[n][lo:hi].contiguous() for n in ("q", "k", "v", "g", "beta")]
    gdn.gdn_decode_window_steps(cfg, a, *args(0, 77), o1[:77])
    torch.cuda.synchronize()
    host = {n: t.cpu() for n, t in a.tensors().items()}        # checkpoint mid-window
    gdn.gdn_decode_window_steps(cfg, a, *args(77, wl.T), o1[77:])
    b = gdn.GdnState.allocate(cfg)
    for n, t in b.tensors().items():
        t.copy_(host[n])
    o2 = torch.empty_like(o1[77:])
    gdn.gdn_decode_window_steps(cfg, b, *args(77, wl.T), o2)
    torch.cuda.synchronize()
    assert torch.equal(o1[77:], o2)
    for n in ("codes", "scales", "comp_idx", "comp_u", "pos"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n


def test_scalar_gate_through_diagonal_kernel_matches_gdn():
    wl = SMALL["gdn-int8"].with_(T=100)
    inputs = decode_inputs(wl, "cuda")
    S0 = gpu_warmup(wl)
    r_gdn = gpu_run(wl, inputs=inputs, S0=S0)
    wl_d = wl.with_(gate="diag")
    inputs_d = dict(inputs)
    inputs_d["g"] = inputs["g"][..., None].expand(*inputs["g"].shape, wl.D).contiguous()
    r_kda = gpu_run(wl_d, inputs=inputs_d, S0=S0)
    assert rel_l2(r_kda.o.double().cpu().numpy(), r_gdn.o.double().cpu().numpy()) < 1e-3
    heads = np.arange(wl.heads)
    d = np.abs(gpu_codes(wl, r_gdn.state, heads).astype(int) -
               gpu_codes(wl, r_kda.state, heads).astype(int))
    assert d.max() <= 1 and (d > 0).mean() < 1e-3


def test_empty_batch_and_zero_steps():
    wl = SMALL["gdn-int8"].with_(B=0)
    cfg = cfg_of(wl)
    st = gdn.GdnState.allocate(cfg)
    e = torch.empty(0, device="cuda")
    gdn.gdn_state_quantize(cfg, torch.empty(0, device="cuda"), st)
    z = torch.empty((0,), dtype=torch.bfloat16, device="cuda")
    gdn.gdn_decode_window_step(cfg, st, z, z, z, e, e, z)
    wl1 = SMALL["gdn-int8"]
    cfg1 = cfg_of(wl1)
    st1 = gdn.GdnState.allocate(cfg1)
    zq = torch.empty((0, wl1.B, wl1.H, wl1.D), dtype=torch.bfloat16, device="cuda")
    gdn.gdn_decode_window_steps(cfg1, st1, zq, zq, zq, torch.empty((0, wl1.B, wl1.H), device="cuda"),
                                torch.empty((0, wl1.B, wl1.H), device="cuda"), zq)
    torch.cuda.synchronize()


def test_bad_pos_is_reported_and_skipped():
    wl = SMALL["gdn-int8"].with_(T=5)
    run = gpu_run(wl)
    cfg = cfg_of(wl)
    st = run.state
    assert int(st.status[0]) == 0
    before = st.clone()
    st.pos[3] = wl.W   # invalid: the kernel must skip head 3 and report
    inp = decode_inputs(wl, "cuda", T=1)
    o = torch.zeros_like(inp["q"][0])
    gdn.gdn_decode_window_step(cfg, st, *(inp[n][0] for n in ("q", "k", "v", "g", "beta")), o)
    torch.cuda.synchronize()
    assert int(st.status[0]) & 0x2
    assert torch.equal(st.codes.view(wl.heads, -1)[3], before.codes.view(wl.heads, -1)[3])
    assert int(st.pos[0]) == int(before.pos[0]) + 1


def test_host_buffer_pipeline_matches_device_path():
    wl = SMALL["kda-int8-r4"]
    cfg = cfg_of(wl)
    inputs = decode_inputs(wl, "cuda")
    S0 = gpu_warmup(wl)
    ref = gpu_run(wl, inputs=inputs, S0=S0)
    st = gdn.GdnState.allocate(cfg)
    gdn.gdn_state_quantize(cfg, S0, st)
    host = {n: t.cpu().pin_memory() for n, t in inputs.items()}
    o_host = torch.empty(inputs["q"].shape, dtype=inputs["q"].dtype).pin_memory()
    staging = torch.empty(gdn.gdn_host_staging_bytes(cfg), dtype=torch.uint8, device="cuda")
    gdn.gdn_decode_window_steps_host(cfg, st, host["q"], host["k"], host["v"], host["g"],
                                     host["beta"], o_host, staging)
    torch.cuda.synchronize()
    assert torch.equal(o_host, ref.o.cpu())
    for n in ("codes", "scales", "comp_idx", "comp_u", "pos"):
        assert torch.equal(getattr(st, n), getattr(ref.state, n)), n


def test_status_word_stays_clear():
    run = gpu_run(SMALL["kda-int8-r4"])
    assert int(run.state.status[0]) == 0
