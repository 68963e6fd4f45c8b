"""Chunkwise prefill (include/gdnq_prefill.h) against the oracle's plain fp64 recurrence on the
same seeded inputs: every output and the final state, for one chunk, several chunks with a
ragged tail, a single token, an empty prompt, a zero and a warmed-up initial state, prompts
split over calls, and a 128-head batch on sampled heads, with the scalar (GDN) gate and with
the per-key-channel (KDA) gate (plus strong per-channel decays at the kernel's documented
bound). All calls go through the C ABI."""
import numpy as np
import pytest
import torch

import bit_recurrent_state_gdn_b200 as gdn
import oracle
from gdn_harness import (
    O_TOL, _heads_np, gpu_warmup, oracle_initial_state, rel_l2, round_act, sample_heads,
)
from workloads import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu

MID = WORKLOADS["gdn-mid"]
KDA = WORKLOADS["kda"].with_(r=0)
# Final state: the prefill's fp32 state feeds gdn_state_quantize, so its bar is set by what the
# kernels achieve (a few 1e-6 rel-L2), not by the outputs' bf16 bar: rel-L2 over the compared
# heads, and entry by entry the largest error of a state row relative to that row's largest
# entry (an error big enough to move an int8 code, 1/254 of the row's absmax, fails it).
S_TOL = 5e-5
S_ELEM_TOL = 5e-4

CASES = {
    "one-chunk": MID.with_(name="pf-64", B=1, H=3, T=64, warmup=32),
    "ragged": MID.with_(name="pf-200", B=2, H=2, T=200, warmup=32),
    "zero-state": MID.with_(name="pf-zero", B=1, H=2, T=150, warmup=0),
    "single-token": MID.with_(name="pf-1", B=1, H=2, T=1, warmup=32),
    "long": MID.with_(name="pf-1000", B=1, H=2, T=1000, warmup=48),
    # per-key-channel gate (16-token chunks): one chunk, ragged tail, zero state, one token, long
    "kda-one-chunk": KDA.with_(name="kpf-16", B=1, H=3, T=16, warmup=32),
    "kda-ragged": KDA.with_(name="kpf-200", B=2, H=2, T=200, warmup=32),
    "kda-zero-state": KDA.with_(name="kpf-zero", B=1, H=2, T=37, warmup=0),
    "kda-single-token": KDA.with_(name="kpf-1", B=1, H=2, T=1, warmup=32),
    "kda-long": KDA.with_(name="kpf-1000", B=1, H=2, T=1000, warmup=48),
}


def head_major(x):
    """[L][B][H](...) -> [B][H][L](...) contiguous."""
    return x.permute(1, 2, 0, *range(3, x.dim())).contiguous()


def pf_run(wl, inp, S0, cuts=None):
    cfg = gdn.make_config(wl.B, wl.H, wl.D, gate=wl.gate, act="bf16")
    S = S0.clone()
    L = inp["q"].shape[0]
    o = torch.empty((wl.B, wl.H, L, wl.D), dtype=torch.bfloat16, device="cuda")
    cuts = cuts or [0, L]
    hm = {n: head_major(inp[n]) for n in ("q", "k", "v", "g", "beta")}
    for lo, hi in zip(cuts, cuts[1:]):
        part = {n: t[:, :, lo:hi].contiguous() for n, t in hm.items()}
        op = torch.empty_like(part["q"])
        gdn.gdn_prefill(cfg, part["q"], part["k"], part["v"], part["g"], part["beta"], op, S)
        o[:, :, lo:hi] = op
    torch.cuda.synchronize()
    return o, S


def compare(wl, inp, o, S, heads):
    q, k, v, g, beta = (_heads_np(inp[n], heads) for n in ("q", "k", "v", "g", "beta"))
    S0 = oracle_initial_state(wl, heads)
    o_ref, S_ref = oracle.plain_run(q, k, v, g, beta, S0=S0)
    L = q.shape[0]
    h = torch.as_tensor(heads, device="cuda")
    o_gpu = o.view(-1, L, wl.D)[h].permute(1, 0, 2).double().cpu().numpy()
    S_gpu = S.view(-1, wl.D, wl.D)[h].double().cpu().numpy()
    row_max = np.maximum(np.abs(S_ref).max(axis=-1, keepdims=True), 1e-30)
    s_elem = float((np.abs(S_gpu - S_ref) / row_max).max()) if S_ref.size else 0.0
    return ((rel_l2(o_gpu, round_act(o_ref, "bf16")) if L else 0.0), rel_l2(S_gpu, S_ref),
            s_elem)


def check(m):
    o_rel, s_rel, s_elem = m
    assert o_rel <= O_TOL and s_rel <= S_TOL and s_elem <= S_ELEM_TOL, m


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_parity(name):
    wl = CASES[name]
    inp = decode_inputs(wl, "cuda")
    o, S = pf_run(wl, inp, gpu_warmup(wl))
    m = compare(wl, inp, o, S, np.arange(wl.heads))
    print(name, m)
    check(m)


@pytest.mark.parametrize("name", ["ragged", "kda-ragged"])
def test_prefill_split_over_calls_carries_the_state(name):
    wl = CASES[name]
    inp = decode_inputs(wl, "cuda")
    S0 = gpu_warmup(wl)
    o, S = pf_run(wl, inp, S0, cuts=[0, 5, 70, 131, 200])  # chunk boundaries inside the calls
    m = compare(wl, inp, o, S, np.arange(wl.heads))
    print(name, m)
    check(m)


def test_kda_prefill_strong_decays():
    """Per-channel log-gates three times the recipe's, floored at -10 per token: 8-token sums
    reach -80, the bound up to which the chunk's decay factors e^{+-(G_t - G_r)} stay finite."""
    wl = KDA.with_(name="kpf-strong", B=1, H=4, T=160, warmup=32)
    inp = decode_inputs(wl, "cuda")
    inp["g"] = (3.0 * inp["g"]).clamp_min(-10.0)
    inp["g"][5:13, :, :, :7] = -10.0  # a run of 8 tokens at the floor on a few channels
    o, S = pf_run(wl, inp, gpu_warmup(wl))
    m = compare(wl, inp, o, S, np.arange(wl.heads))
    print("strong", m)
    assert np.all(np.isfinite(m))
    check(m)


@pytest.mark.parametrize("base", ["gdn", "kda"])
def test_prefill_batch_sampled_heads(base):
    wl = (MID if base == "gdn" else KDA).with_(name="pf-batch", B=4, H=32, T=512, warmup=32)
    inp = decode_inputs(wl, "cuda")
    o, S = pf_run(wl, inp, gpu_warmup(wl))
    heads = sample_heads(wl, 24, seed=3)
    m = compare(wl, inp, o, S, heads)
    print("batch", m)
    check(m)


@pytest.mark.parametrize("name", ["one-chunk", "kda-one-chunk"])
def test_empty_prompt_leaves_the_state(name):
    wl = CASES[name]
    cfg = gdn.make_config(wl.B, wl.H, wl.D, gate=wl.gate)
    S0 = gpu_warmup(wl)
    S = S0.clone()
    z = torch.empty((wl.B, wl.H, 0, wl.D), dtype=torch.bfloat16, device="cuda")
    zf = torch.empty((wl.B, wl.H, 0), dtype=torch.float32, device="cuda")
    zg = torch.empty((wl.B, wl.H, 0, wl.D) if wl.gate == "diag" else (wl.B, wl.H, 0),
                     dtype=torch.float32, device="cuda")
    gdn.gdn_prefill(cfg, z, z, z, zg, zf, z, S)
    torch.cuda.synchronize()
    assert torch.equal(S, S0)


@pytest.mark.parametrize("base", ["gdn", "kda"])
def test_prefill_then_window_decode(base):
    """The state a prefill leaves, quantized, starts the windowed decode: the decode's outputs
    match the oracle running the same prompt and decode tokens through the plain recurrence
    then the windowed form."""
    wb = MID if base == "gdn" else KDA
    wl = wb.with_(name="pf-decode", B=1, H=4, T=64, W=64, warmup=0)
    prompt = wb.with_(name="pf-prompt", B=1, H=4, T=300, warmup=0, seed=4242)
    pin = decode_inputs(prompt, "cuda")
    _, S = pf_run(prompt, pin, torch.zeros((1, 4, 128, 128), device="cuda"))
    cfg = gdn.make_config(wl.B, wl.H, wl.D, wl.W, 0, wl.gate, "int8", "bf16", "bf16")
    st = gdn.GdnState.allocate(cfg)
    gdn.gdn_state_quantize(cfg, S, st)
    inp = decode_inputs(wl, "cuda")
    o = torch.empty_like(inp["q"])
    gdn.gdn_decode_window_steps(cfg, st, inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], o)
    torch.cuda.synchronize()
    heads = np.arange(4)
    pq, pk, pv, pg, pb = (_heads_np(pin[n], heads) for n in ("q", "k", "v", "g", "beta"))
    _, S_ref = oracle.plain_run(pq, pk, pv, pg, pb, state_round="f32", want_o=False)
    q, k, v, g, beta = (_heads_np(inp[n], heads) for n in ("q", "k", "v", "g", "beta"))
    res = oracle.o2_run(q, k, v, g, beta, W=wl.W, fmt="int8", S0=S_ref, round_storage=True)
    o_rel = rel_l2(_heads_np(o, heads), round_act(res.o, "bf16"))
    assert o_rel <= O_TOL, o_rel


@pytest.mark.parametrize("name", ["gdn-prefill", "kda-prefill"])
def test_prefill_full_size_sampled_heads(name):
    """The prompt workloads the benchmark times (8 x 32 heads, 4096-token prompts, one launch),
    checked on sampled heads against the plain fp64 recurrence."""
    wl = WORKLOADS[name]
    inp = decode_inputs(wl, "cuda")
    o, S = pf_run(wl, inp, torch.zeros((wl.B, wl.H, wl.D, wl.D), device="cuda"))
    assert bool(torch.isfinite(S).all())
    heads = sample_heads(wl, 4, seed=wl.seed)
    m = compare(wl, inp, o, S, heads)
    print(name, m)
    check(m)
