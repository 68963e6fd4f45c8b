"""The seeded input generators: shapes, dtypes, determinism and the stated distributions."""
import torch

from workloads import WORKLOADS, decode_inputs, outlier_scales, step_inputs
from workloads.generate import n_outlier_channels


def small(name, **kw):
    return WORKLOADS[name].with_(**{"B": 3, "H": 4, **kw})


def test_shapes_and_dtypes():
    for name in WORKLOADS:
        wl = small(name)
        s = step_inputs(wl, "decode", 0)
        D = wl.D
        act = torch.float32 if wl.act == "f32" else torch.bfloat16
        for x in (s.q, s.k, s.v):
            assert x.shape == (3, 4, D) and x.dtype == act
        assert s.beta.shape == (3, 4) and s.beta.dtype == torch.float32
        gshape = (3, 4) if wl.gate == "scalar" else (3, 4, D)
        assert s.g.shape == gshape and s.g.dtype == torch.float32


def test_deterministic_and_step_dependent():
    wl = small("gdn-mid")
    a, b = step_inputs(wl, "decode", 5), step_inputs(wl, "decode", 5)
    c = step_inputs(wl, "decode", 6)
    w = step_inputs(wl, "warmup", 5)
    assert torch.equal(a.q, b.q) and torch.equal(a.g, b.g)
    assert not torch.equal(a.q, c.q) and not torch.equal(a.q, w.q)


def test_distributions():
    wl = small("gdn-mid", H=16)
    s = step_inputs(wl, "decode", 1)
    nk = s.k.float().norm(dim=-1)
    assert torch.allclose(nk, torch.ones_like(nk), atol=1e-2)
    assert torch.all(s.g < 0) and torch.all((s.beta > 0) & (s.beta < 1))
    ks, vs = outlier_scales(wl)
    n = n_outlier_channels(wl.D)
    assert n == 3
    assert torch.all((ks == 20).sum(-1) == n) and torch.all((vs == 20).sum(-1) == n)
    tiny = WORKLOADS["gdn-tiny"]
    ks, vs = outlier_scales(tiny)
    assert torch.all(ks == 1) and torch.all(vs == 1)


def test_decode_inputs_stack_the_steps():
    wl = small("kda", T=5)
    d = decode_inputs(wl)
    assert d["q"].shape == (5, 3, 4, 128) and d["g"].shape == (5, 3, 4, 128)
    s3 = step_inputs(wl, "decode", 3)
    assert torch.equal(d["v"][3], s3.v) and torch.equal(d["beta"][3], s3.beta)
