"""Mixed per-head bit widths in one launch (GDN_FMT_MIXED), two ways:
  - against the oracle: the heads of each format, read out of the mixed state, against the
    oracle's buffered-window form run in that head's format (outputs, codes, scales,
    compensators, pos), with the acceptance bars of the uniform formats;
  - against the uniform launches: every head must come out exactly as it does in a launch whose
    whole state has that head's format -- outputs, codes, scales, compensators and pos
    bit-identical through decode steps with window flushes, a forced ragged flush and
    materialisation."""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import bit_recurrent_state_gdn_b200 as gdn
from gdn_harness import (GpuRun, compare, gpu_warmup, oracle_initial_state, oracle_run,
                         sample_heads)
from workloads import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu

MID, KDA = WORKLOADS["gdn-mid"], WORKLOADS["kda"]
CASES = {
    "gdn-r2": MID.with_(name="mixed-gdn", B=40, H=16, T=150, r=2, warmup=48),  # 3 heads a CTA
    "kda-r4": KDA.with_(name="mixed-kda", B=2, H=8, T=140, W=64, r=4, warmup=48),
    "gdn-w20": MID.with_(name="mixed-w20", B=2, H=6, T=50, W=20, warmup=32),
}


def _pattern(n, seed):
    rng = np.random.default_rng(seed)
    f = rng.choice(["int8", "int4_g32"], size=n)
    f[0], f[-1] = "int8", "int4_g32"  # both formats always present
    return list(f)


def _cfg(wl, fmt):
    return gdn.make_config(wl.B, wl.H, wl.D, wl.W, wl.r, wl.gate, fmt, wl.act, wl.buf)


def _run(wl, fmt, S0, inp, head_fmt=None, flush_mask=None):
    cfg = _cfg(wl, fmt)
    st = gdn.GdnState.allocate(cfg, head_fmt=head_fmt)
    gdn.gdn_state_quantize(cfg, S0, st)
    o = torch.empty_like(inp["q"])
    gdn.gdn_decode_window_steps(cfg, st, inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], o)
    S = torch.empty_like(S0)
    gdn.gdn_state_materialize(cfg, st, S)
    if flush_mask is not None:
        gdn.gdn_window_flush(cfg, st, flush_mask)
    torch.cuda.synchronize()
    assert int(st.status[0].item()) == 0
    return cfg, st, o, S


def _head_views(wl, st, fmt, n):
    """Per-head codes / scales of a state laid out for `fmt` ("mixed" slots are the larger)."""
    D = wl.D
    code_slot = D * D // 2 if fmt == "int4_g32" else D * D
    scale_slot = D * (D // 32) if fmt in ("int4_g32", "mixed") else D
    return st.codes.view(n, code_slot), st.scales.view(n, scale_slot)


def _format_view(wl, mst, mo, fmt, heads):
    """The heads ``heads`` of a mixed state and its outputs, laid out as a uniform state of
    ``fmt`` holding only those heads (the harness reads it like any other run)."""
    n, D, T = wl.heads, wl.D, mo.shape[0]
    idx = torch.as_tensor(heads, device="cuda")
    cb = D * D // 2 if fmt == "int4_g32" else D * D
    sb = D * (D // 32) if fmt == "int4_g32" else D
    rp = (wl.r + 3) // 4 * 4
    st = SimpleNamespace(
        codes=mst.codes.view(n, D * D)[idx, :cb].contiguous().view(-1),
        scales=mst.scales.view(n, D * (D // 32))[idx, :sb].contiguous().view(-1),
        comp_idx=mst.comp_idx.view(n, max(rp, 1))[idx].contiguous().view(-1) if wl.r else
        mst.comp_idx,
        comp_u=mst.comp_u.view(n, -1)[idx].contiguous().view(-1) if wl.r else mst.comp_u,
        pos=mst.pos[idx].contiguous())
    o = mo.view(T, n, D)[:, idx].contiguous().view(T, 1, len(heads), D)
    return GpuRun(o, st, None, None)


@pytest.mark.parametrize("name", list(CASES))
def test_mixed_launch_against_the_oracle(name):
    wl = CASES[name]
    fmts = np.array(_pattern(wl.heads, wl.seed))
    inp = decode_inputs(wl, "cuda")
    _, mst, mo, _ = _run(wl, "mixed", gpu_warmup(wl), inp, head_fmt=list(fmts))
    pick = set(sample_heads(wl, 64, seed=7).tolist()) if wl.heads > 64 else None
    for f in ("int8", "int4_g32"):
        heads = np.array([h for h in np.flatnonzero(fmts == f) if pick is None or h in pick])
        wf = wl.with_(fmt=f)
        res = oracle_run(wf, heads, inp, oracle_initial_state(wf, heads))
        p = compare(wf, _format_view(wl, mst, mo, f, heads), np.arange(len(heads)), res)
        print(name, f, len(heads), p)
        p.check()


@pytest.mark.parametrize("name", list(CASES))
def test_mixed_launch_equals_uniform_launches(name):
    wl = CASES[name]
    n, D = wl.heads, wl.D
    fmts = _pattern(n, wl.seed)
    inp = decode_inputs(wl, "cuda")
    S0 = gpu_warmup(wl)
    mask = (torch.arange(wl.B, device="cuda") % 2).to(torch.int32)  # flush every other sequence
    runs = {f: _run(wl, f, S0, inp, flush_mask=mask) for f in ("int8", "int4_g32")}
    _, mst, mo, mS = _run(wl, "mixed", S0, inp, head_fmt=fmts, flush_mask=mask)
    mcodes, mscales = _head_views(wl, mst, "mixed", n)
    rp = (wl.r + 3) // 4 * 4
    for f, (_, st, o, S) in runs.items():
        heads = [h for h in range(n) if fmts[h] == f]
        idx = torch.tensor(heads, device="cuda")
        codes, scales = _head_views(wl, st, f, n)
        assert torch.equal(mo.view(wl.T, n, D)[:, idx], o.view(wl.T, n, D)[:, idx]), f
        assert torch.equal(mS.view(n, D, D)[idx], S.view(n, D, D)[idx]), f
        cb, sb = codes.shape[1], scales.shape[1]
        assert torch.equal(mcodes[idx, :cb], codes[idx]), f
        assert torch.equal(mscales[idx, :sb], scales[idx]), f
        assert torch.equal(mst.pos[idx], st.pos[idx]), f
        if wl.r > 0:
            assert torch.equal(mst.comp_idx.view(n, rp)[idx], st.comp_idx.view(n, rp)[idx]), f
            assert torch.equal(mst.comp_u.view(n, -1)[idx], st.comp_u.view(n, -1)[idx]), f


def test_mixed_state_needs_head_formats():
    cfg = _cfg(CASES["gdn-r2"], "mixed")
    with pytest.raises(ValueError):
        gdn.GdnState.allocate(cfg)
    st = gdn.GdnState.allocate(cfg, head_fmt=["int8"] * (cfg.B * cfg.H))
    st.head_fmt = torch.empty(0, dtype=torch.int8, device="cuda")  # a null pointer
    S0 = torch.zeros((cfg.B, cfg.H, cfg.d_k, cfg.d_k), device="cuda")
    with pytest.raises(gdn.GdnError, match="head_fmt"):
        gdn.gdn_state_quantize(cfg, S0, st)
