"""One sequence's non-finite input stays in that sequence's heads. A persistent window-step CTA
works through several heads in turn on shared-memory stages, and with ragged windows (sequences
at different window positions) a stage may still hold rows of write vectors that an earlier
head left there; the buffer product reads such rows against zero coefficients, so they must
never carry another head's Inf or NaN. Here every head of the even sequences gets an Inf in its
value vector from some step on, the odd sequences' windows are restarted by a forced flush so
that they run at other positions, and every odd sequence must come out bit-identical to a run
without the bad inputs: outputs, codes, scales, buffered pairs and positions."""
import pytest
import torch

import bit_recurrent_state_gdn_b200 as gdn
from gdn_harness import cfg_of, gpu_warmup
from workloads import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu

# 1536 heads of 4: six heads a CTA on 2 x 148 CTAs, so every CTA walks heads of both parities
# through reused stages
WL = WORKLOADS["gdn-mid"].with_(name="isolation", B=384, H=4, T=48, warmup=16)
FIELDS = ("codes", "scales", "buf_k", "buf_u", "buf_L", "pos")


def _run(wl, inputs, S0):
    cfg = cfg_of(wl)
    st = gdn.GdnState.allocate(cfg)
    gdn.gdn_state_quantize(cfg, S0, st)
    o = torch.empty_like(inputs["q"])
    odd = (torch.arange(wl.B, device="cuda") % 2).to(torch.int32)
    for t in range(wl.T):
        gdn.gdn_decode_window_step(cfg, st, *(inputs[n][t] for n in ("q", "k", "v", "g", "beta")),
                                   o[t])
        if t == 9:
            gdn.gdn_window_flush(cfg, st, odd)  # the odd sequences restart their windows
    torch.cuda.synchronize()
    assert int(st.status[0].item()) == 0
    return o, st


@pytest.mark.parametrize("gate", ["scalar", "diag"])
def test_nonfinite_inputs_stay_in_their_sequence(gate):
    wl = WL.with_(gate=gate)
    inputs = decode_inputs(wl, "cuda")
    S0 = gpu_warmup(wl)
    even = torch.arange(wl.B, device="cuda") % 2 == 0
    bad = {n: t.clone() for n, t in inputs.items()}
    v = bad["v"]
    v[20:, even, :, 5] = float("inf")
    o_ref, st_ref = _run(wl, inputs, S0)
    o_bad, st_bad = _run(wl, bad, S0)
    odd = ~even
    assert not bool(torch.isfinite(o_bad[30:, even]).all())  # the bad input did enter
    assert torch.equal(o_bad[:, odd], o_ref[:, odd])
    for f in FIELDS:
        a, b = getattr(st_bad, f).view(wl.B, -1), getattr(st_ref, f).view(wl.B, -1)
        assert torch.equal(a[odd], b[odd]), f
    # positions really are ragged: even sequences run 10 steps ahead in their windows
    pos = st_ref.pos.view(wl.B, wl.H)
    assert bool((pos[even] - pos[odd] == 10).all())
