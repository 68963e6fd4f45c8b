"""Pure-write sliding window (include/gdnq_pw.h) against the oracle's pw_run with GPU storage
roundings, element by element: outputs, the history's codes and scales, the FP8 pairs in every
ring slot, the window count and the materialised logical state. Windows of 0 (every-step
quantization), 1, 3, 8 (the pages' PW-S8) and 16 pairs; int8 and int4 histories; scalar and
per-channel gates; bf16 and fp32 activations; runs long enough for the ring to wrap several
times, split over two calls; batches that put several heads on one CTA; the full serving batch
on sampled heads. All calls go through the C ABI."""
import numpy as np
import pytest
import torch

import bit_recurrent_state_gdn_b200 as gdn
import oracle
from gdn_harness import (
    FLIP_FRAC, O_TOL, SCALE_TOL, SCALE_TOL_ROUNDING, _heads_np, gpu_codes, gpu_scales,
    gpu_warmup, oracle_initial_state, rel_l2, round_act, sample_heads,
)
from workloads import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu

MID, KDA, SERVE = WORKLOADS["gdn-mid"], WORKLOADS["kda"], WORKLOADS["gdn-serving"]

# (workload, pairs per head); T > Wp in all but one case, so pairs leave the window and merge
CASES = {
    "s8-int4": (MID.with_(name="pw-s8-int4", B=2, H=4, T=40, fmt="int4_g32", warmup=48), 8),
    "s8-int8-kda": (KDA.with_(name="pw-s8-kda", B=2, H=4, T=40, r=0, warmup=48), 8),
    "s0-int8": (MID.with_(name="pw-s0", B=2, H=3, T=20, warmup=32), 0),
    "s1-int4": (MID.with_(name="pw-s1", B=1, H=4, T=20, fmt="int4_g32", warmup=32), 1),
    "s3-int4-kda-f32": (KDA.with_(name="pw-s3-f32", B=1, H=4, T=30, r=0, fmt="int4_g32",
                                  act="f32", buf="f32", warmup=32), 3),
    "s16-int8": (MID.with_(name="pw-s16", B=1, H=3, T=45, warmup=32), 16),
    "s8-short-run": (MID.with_(name="pw-short", B=1, H=3, T=5, fmt="int4_g32", warmup=32), 8),
    # 640 heads: several heads per CTA and every stage of the ring (oracle on sampled heads)
    "s8-int4-many": (MID.with_(name="pw-many", B=40, H=16, T=24, fmt="int4_g32", warmup=32), 8),
}


def pw_cfg(wl, Wp):
    return gdn.make_pw_config(wl.B, wl.H, wl.D, Wp, wl.gate, wl.fmt, wl.act)


def pw_gpu_run(wl, Wp, T=None, split=True, draw="cuda"):
    """``draw``: the device the seeded inputs are drawn on (then copied to the GPU)."""
    T = wl.T if T is None else T
    cfg = pw_cfg(wl, Wp)
    inp = {n: x.to("cuda") for n, x in decode_inputs(wl, draw, T).items()}
    S0 = gpu_warmup(wl, draw=draw)
    st = gdn.PwState.allocate(cfg)
    gdn.gdn_pw_quantize(cfg, S0, st)
    o = torch.empty_like(inp["q"])
    cuts = [0, T // 2, T] if split and T > 1 else [0, T]
    for lo, hi in zip(cuts, cuts[1:]):
        part = [inp[n][lo:hi] for n in ("q", "k", "v", "g", "beta")]
        gdn.gdn_pw_decode_steps(cfg, st, *part, o[lo:hi])
    S = torch.empty_like(S0)
    gdn.gdn_pw_materialize(cfg, st, S)
    torch.cuda.synchronize()
    return cfg, st, inp, o, S


def expected_count(T, Wp):
    if Wp == 0:
        return 0
    return T if T < Wp else Wp + T % Wp


def gpu_pairs(st, heads, Wp, D):
    """Dequantised pairs [n][2][Wp][D] of the chosen heads (x block, y block)."""
    Wr = (Wp + 3) // 4 * 4
    h = torch.as_tensor(heads, device=st.pairs.device)
    codes = st.pairs.view(-1, 2, Wp, D)[h].view(torch.float8_e4m3fn).double()
    sc = st.pscales.view(-1, 2, Wr)[h][:, :, :Wp].double()
    return (codes * sc[..., None]).cpu().numpy()


def compare(wl, Wp, st, inp, o, S, heads, draw="cuda"):
    S0 = oracle_initial_state(wl, heads, draw)
    q, k, v, g, beta = (_heads_np(inp[n], heads) for n in ("q", "k", "v", "g", "beta"))
    T = q.shape[0]
    res = oracle.pw_run(q, k, v, g, beta, Wp=Wp, fmt=wl.fmt, S0=S0, prec32=True)
    out = {}
    out["o_rel"] = rel_l2(_heads_np(o, heads), round_act(res.o, wl.act))
    codes = gpu_codes(wl, st, heads)
    diff = np.abs(codes.astype(int) - res.codes.astype(int))
    out["flip_frac"] = float((diff > 0).mean())
    out["max_code_diff"] = int(diff.max())
    sc = gpu_scales(wl, st, heads)
    ref = res.scales.reshape(sc.shape)
    row_max = np.maximum(np.abs(ref).max(axis=-1, keepdims=True), 1e-30)
    srel = (np.abs(sc - ref) / row_max).max(axis=-1)          # [n][D] per row
    same = diff.reshape(len(heads), wl.D, -1).max(axis=-1) == 0
    out["scale_rel_max"] = float(srel[same].max()) if same.any() else 0.0
    loose = same & (srel > SCALE_TOL)
    out["scale_loose_rows"] = int(loose.sum())
    out["scale_unexplained"] = (explain_loose_rows(wl, Wp, heads, loose, draw) if loose.any()
                                else 0)
    out["rows"] = int(same.sum())
    if Wp > 0:
        live = min(T, Wp)  # slots 0 .. live-1 hold pairs
        gp = gpu_pairs(st, heads, Wp, wl.D)
        out["px_rel"] = rel_l2(gp[:, 0, :live], res.px[:, :live])
        out["py_rel"] = rel_l2(gp[:, 1, :live], res.py[:, :live])
    h = torch.as_tensor(heads, device=st.count.device)
    out["count_ok"] = bool((st.count[h].cpu().numpy() == expected_count(T, Wp)).all())
    Sg = S.view(-1, wl.D, wl.D)[h].double().cpu().numpy()
    out["S_rel"] = rel_l2(Sg, res.S)
    return out


def explain_loose_rows(wl, Wp, heads, loose, draw="cuda"):
    """How many loose scale rows are NOT preceded by a code flip in the same row: the run is
    repeated one step per call (runs are bit-identical however they are split) and the codes of
    the loose rows' heads after every earlier step are compared with the oracle's after the same
    number of steps."""
    T = wl.T
    hl = np.unique(np.nonzero(loose)[0])
    cfg = pw_cfg(wl, Wp)
    inp = {n: x.to("cuda") for n, x in decode_inputs(wl, draw, T).items()}
    st = gdn.PwState.allocate(cfg)
    gdn.gdn_pw_quantize(cfg, gpu_warmup(wl, draw=draw), st)
    o = torch.empty_like(inp["q"])
    S0 = oracle_initial_state(wl, heads[hl], draw)
    q, k, v, g, beta = (_heads_np(inp[n], heads[hl]) for n in ("q", "k", "v", "g", "beta"))
    flipped = np.zeros((len(hl), wl.D), bool)
    for t in range(T - 1):
        gdn.gdn_pw_decode_steps(cfg, st, *(inp[n][t:t + 1] for n in ("q", "k", "v", "g", "beta")),
                                o[t:t + 1])
        torch.cuda.synchronize()
        gc = gpu_codes(wl, st, heads[hl])
        res = oracle.pw_run(q[:t + 1], k[:t + 1], v[:t + 1], g[:t + 1], beta[:t + 1], Wp=Wp,
                            fmt=wl.fmt, S0=S0, prec32=True)
        flipped |= (gc != res.codes).any(axis=-1)
    return int((loose[hl] & ~flipped).sum())


# Bars. Outputs and the logical state: rel-L2 O_TOL (as the window form). History codes: equal
# but for one-LSB flips on at most FLIP_FRAC of the entries: both sides requantise every step
# from their own fp32 / fp64 arithmetic, so a value within rounding noise of a code boundary may
# land on either side, once per step. Scales: where a row's codes agree, within SCALE_TOL of the
# row's largest scale; a row beyond it is accepted only when a code of that row flipped at an
# earlier step (the flipped value is carried into the row's later values), on at most FLIP_FRAC
# of the rows and never beyond one bf16 ulp. FP8 pairs: an e4m3 rounding that lands the other
# way moves one element by one e4m3 step (2^-3 relative at most); rel-L2 over the stored pairs
# 1e-2.
PAIR_TOL = 1e-2


def check(m):
    assert m["o_rel"] <= O_TOL, m
    assert m["S_rel"] <= O_TOL, m
    assert m["max_code_diff"] <= 1, m
    assert m["flip_frac"] <= FLIP_FRAC, m
    assert m["scale_rel_max"] <= SCALE_TOL_ROUNDING, m
    assert m["scale_loose_rows"] <= max(1, int(FLIP_FRAC * m["rows"])), m
    assert m["scale_unexplained"] == 0, m
    assert m.get("px_rel", 0.0) <= PAIR_TOL and m.get("py_rel", 0.0) <= PAIR_TOL, m
    assert m["count_ok"], m


@pytest.mark.parametrize("name", list(CASES))
def test_pw_decode_parity(name):
    wl, Wp = CASES[name]
    cfg, st, inp, o, S = pw_gpu_run(wl, Wp)
    heads = sample_heads(wl, 48) if wl.heads > 64 else np.arange(wl.heads)
    m = compare(wl, Wp, st, inp, o, S, heads)
    print(name, m)
    check(m)
    assert int(st.status[0].item()) == 0


def test_pw_full_serving_batch_sampled_heads():
    """B = 1024, H = 32, PW-S8 over an int4 history, long enough for the window to wrap."""
    wl = SERVE.with_(name="pw-serving", fmt="int4_g32", T=12)
    cfg, st, inp, o, S = pw_gpu_run(wl, 8)
    heads = sample_heads(wl, 48, seed=5)
    m = compare(wl, 8, st, inp, o, S, heads)
    print("serving", m)
    check(m)
    assert int(st.status[0].item()) == 0


def test_pw_runs_are_bit_identical():
    wl, Wp = CASES["s8-int4-many"]
    a = pw_gpu_run(wl, Wp, T=12)
    b = pw_gpu_run(wl, Wp, T=12, split=False)
    assert torch.equal(a[3], b[3])
    for n in ("codes", "scales", "pairs", "pscales", "count"):
        assert torch.equal(getattr(a[1], n), getattr(b[1], n)), n


def test_pw_bad_count_is_reported_and_skipped():
    wl, Wp = CASES["s8-int4"]
    cfg = pw_cfg(wl, Wp)
    inp = decode_inputs(wl, "cuda", 1)
    st = gdn.PwState.allocate(cfg)
    gdn.gdn_pw_quantize(cfg, gpu_warmup(wl), st)
    st.count[3] = 2 * Wp  # out of range
    before = st.clone()
    o = torch.zeros_like(inp["q"])
    gdn.gdn_pw_decode_steps(cfg, st, inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], o)
    torch.cuda.synchronize()
    assert int(st.status[0].item()) & 0x2  # GDN_DEVICE_BAD_POS
    per = st.codes.numel() // wl.heads
    assert torch.equal(st.codes.view(wl.heads, per)[3], before.codes.view(wl.heads, per)[3])
    assert int(st.count[3].item()) == 2 * Wp
    assert not o.view(wl.heads, -1)[3].any()
    assert int(st.count[2].item()) == 1


def test_pw_quantize_matches_window_quantize():
    """The history quantizer is the window state's (same codes, scales, layout)."""
    wl = CASES["s8-int4"][0]
    S0 = gpu_warmup(wl)
    st = gdn.PwState.allocate(pw_cfg(wl, 8))
    gdn.gdn_pw_quantize(pw_cfg(wl, 8), S0, st)
    wcfg = gdn.make_config(wl.B, wl.H, wl.D, 8, 0, wl.gate, wl.fmt, wl.act, wl.act)
    ws = gdn.GdnState.allocate(wcfg)
    gdn.gdn_state_quantize(wcfg, S0, ws)
    torch.cuda.synchronize()
    assert torch.equal(st.codes, ws.codes) and torch.equal(st.scales, ws.scales)
    assert not st.count.any()
