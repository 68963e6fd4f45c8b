"""gdn_decode_window_steps_host_fixed (the host-buffer decode that stages through the library's
fixed device array and allocates nothing) against gdn_decode_window_steps_host (caller-provided
staging), on two calls in a row from the same state: outputs and state must be bit-identical,
the second call crossing a window flush. Kept in a file of its own, collected last, so that it
also runs after everything else the suite has done on the device."""
import pytest
import torch

import bit_recurrent_state_gdn_b200 as gdn
from gdn_harness import cfg_of, gpu_warmup
from workloads import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu

WL = WORKLOADS["gdn-mid"].with_(name="gdn-no-alloc", B=8, H=16, T=80, warmup=32)


def _host(x):
    return x.cpu().pin_memory()


def _state_tensors(st):
    return {n: t.clone() for n, t in st.tensors().items()}


def test_fixed_staging_matches_caller_staging_on_two_calls():
    cfg = cfg_of(WL)
    inp = decode_inputs(WL, "cuda")
    S0 = gpu_warmup(WL)
    ref, fix = gdn.GdnState.allocate(cfg), gdn.GdnState.allocate(cfg)
    gdn.gdn_state_quantize(cfg, S0, ref)
    gdn.gdn_state_quantize(cfg, S0, fix)
    staging = torch.empty(gdn.gdn_host_staging_bytes(cfg), dtype=torch.uint8, device="cuda")
    half = WL.T // 2
    for lo, hi in ((0, half), (half, WL.T)):  # two calls in a row
        h = {n: _host(t[lo:hi]) for n, t in inp.items()}
        o_ref = torch.empty_like(h["q"]).pin_memory()
        o_fix = torch.empty_like(h["q"]).pin_memory()
        gdn.gdn_decode_window_steps_host(cfg, ref, h["q"], h["k"], h["v"], h["g"], h["beta"],
                                         o_ref, staging)
        gdn.gdn_decode_window_steps_host_fixed(cfg, fix, h["q"], h["k"], h["v"], h["g"],
                                               h["beta"], o_fix)
        torch.cuda.synchronize()
        assert torch.equal(o_ref, o_fix), (lo, hi)
        a, b = _state_tensors(ref), _state_tensors(fix)
        for n in ("codes", "scales", "pos"):
            assert torch.equal(a[n], b[n]), (n, lo, hi)
    assert int(fix.status[0].item()) == 0
    assert int(fix.pos[0].item()) == WL.T % WL.W


def test_fixed_staging_rejects_a_batch_it_cannot_hold():
    # one staging slot is about 1 KiB per (sequence, head) here: 32768 heads need ~33 MiB
    big = WORKLOADS["gdn-serving"]
    cfg = cfg_of(big)
    st = gdn.GdnState.allocate(cfg)
    q = torch.zeros((1, big.B, big.H, big.D), dtype=torch.bfloat16).pin_memory()
    g = torch.zeros((1, big.B, big.H), dtype=torch.float32).pin_memory()
    with pytest.raises(gdn.GdnError, match="fixed staging"):
        gdn.gdn_decode_window_steps_host_fixed(cfg, st, q, q, q, g, g, torch.empty_like(q))
