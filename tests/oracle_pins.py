"""Pins for the CPU oracle: checks against what the pages and the mathematics fix, never against
the oracle's own formulas retyped.

Each ``pin_*`` takes a loaded oracle library and raises AssertionError when the oracle is wrong.
``test_oracle_pins.py`` runs them on the real oracle; ``test_oracle_mutants.py`` runs them on
deliberately broken copies and requires every break to be caught.

Kinds of pin used here:
  - hand-worked fixtures under tests/golden (values fixed by arithmetic done by hand);
  - closed forms: one write from a zero state, pure decay, exact retrieval with orthonormal keys,
    the delta-rule write identity at the written key;
  - agreement of independent formulations (literal matrix form, distributive plain form,
    buffered windows) where the mathematics says they are equal;
  - library routines for special cases: numpy rint / argsort, torch's bf16 and float8_e4m3fn
    conversions.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from golden_io import read


def _softplus(x):
    return np.log1p(np.exp(-np.abs(x))) + np.maximum(x, 0)


def rand_inputs(seed, T, nh, D, gate="scalar", unit=True, outlier=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, nh, D))
    k = rng.standard_normal((T, nh, D))
    v = rng.standard_normal((T, nh, D))
    if outlier:
        k[..., 1] *= 20.0
        v[..., 2] *= 20.0
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, nh))))
    gshape = (T, nh) if gate == "scalar" else (T, nh, D)
    g = -_softplus(rng.standard_normal(gshape))
    return q, k, v, g, beta


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def close(a, b, tol, what):
    e = rel(a, b)
    assert e <= tol, f"{what}: rel err {e:.3e} > {tol:.1e}"


# ---------------------------------------------------------------------------------------------
# Hand-worked fixtures
# ---------------------------------------------------------------------------------------------
def pin_golden_delta_rule_kda(lib):
    gd = read("delta_rule_kda_2x2.txt")
    D, T = 2, 2
    S0 = gd["S0"].reshape(1, D, D)
    q, k, v = (gd[n].reshape(T, 1, D) for n in ("q", "k", "v"))
    g = np.log(gd["a"]).reshape(T, 1, D)
    beta = gd["beta"].reshape(T, 1)
    for t, Sname in ((1, "S1"), (2, "S2")):
        o, S = oracle.plain_run(q[:t], k[:t], v[:t], g[:t], beta[:t], S0=S0, lib=lib)
        assert np.allclose(S[0].ravel(), gd[Sname], atol=1e-12), ("plain", Sname, S[0])
        assert np.allclose(o.ravel(), gd["o"][: t * D], atol=1e-12), ("plain o", o)
        o1, S1, _ = oracle.o1_run(q[:t], k[:t], v[:t], g[:t], beta[:t], W=1, fmt="none",
                                  S0=S0, lib=lib)
        assert np.allclose(S1[0].ravel(), gd[Sname], atol=1e-12), ("O1", Sname, S1[0])
        assert np.allclose(o1.ravel(), gd["o"][: t * D], atol=1e-12), ("O1 o", o1)
        res = oracle.o2_run(q[:t], k[:t], v[:t], g[:t], beta[:t], W=4, fmt="none", S0=S0, lib=lib)
        assert np.allclose(res.S[0].ravel(), gd[Sname], atol=1e-12), ("O2", Sname, res.S[0])
        assert np.allclose(res.o.ravel(), gd["o"][: t * D], atol=1e-12), ("O2 o", res.o)


def pin_golden_window_int8(lib):
    gd = read("window_int8_2x2.txt")
    D, T, W = 2, 3, 2
    S0 = gd["S0"].reshape(1, D, D)
    q, k, v = (gd[n].reshape(T, 1, D) for n in ("q", "k", "v"))
    g = np.log(gd["a"]).reshape(T, 1)
    beta = gd["beta"].reshape(T, 1)
    res = oracle.o2_run(q, k, v, g, beta, W=W, fmt="int8", S0=S0, lib=lib)
    assert np.allclose(res.o.ravel(), gd["o"], atol=1e-12), ("O2 o", res.o.ravel())
    assert np.allclose(res.S[0].ravel(), gd["S3"], atol=1e-12), ("O2 S3", res.S[0])
    r2 = oracle.o2_run(q[:2], k[:2], v[:2], g[:2], beta[:2], W=W, fmt="int8", S0=S0, lib=lib)
    assert np.array_equal(r2.codes[0].ravel(), gd["codes_after_window1"].astype(np.int8)), r2.codes
    assert np.allclose(r2.scales[0].ravel(), gd["scales_after_window1"], rtol=1e-15, atol=0)
    assert r2.pos[0] == 0
    o1, S1, _ = oracle.o1_run(q, k, v, g, beta, W=W, fmt="int8", S0=S0, lib=lib)
    assert np.allclose(o1.ravel(), gd["o"], atol=1e-12), ("O1 o", o1.ravel())
    assert np.allclose(S1[0].ravel(), gd["S3"], atol=1e-12), ("O1 S3", S1[0])


def pin_golden_compensator(lib):
    gd = read("compensator_2x2.txt")
    D = 2
    S0 = gd["S0"].reshape(1, D, D)
    q, k, v = (gd[n].reshape(1, 1, D) for n in ("q", "k", "v"))
    g = np.log(gd["a"]).reshape(1, 1, D)
    beta = gd["beta"].reshape(1, 1)
    r0 = oracle.o2_run(q[:0], k[:0], v[:0], g[:0], beta[:0], W=4, r=1, fmt="int8", S0=S0, lib=lib)
    assert list(r0.cidx[0]) == [int(gd["comp_idx"][0])], r0.cidx
    assert np.allclose(r0.cu[0].ravel(), gd["comp_u"], atol=0), r0.cu
    assert np.array_equal(r0.codes[0].ravel(), gd["codes0"].astype(np.int8)), r0.codes
    assert np.allclose(r0.scales[0].ravel(), gd["scales0"], rtol=1e-15, atol=0), r0.scales
    assert np.allclose(r0.S[0], S0[0], atol=1e-12), r0.S
    r1 = oracle.o2_run(q, k, v, g, beta, W=4, r=1, fmt="int8", S0=S0, lib=lib)
    assert np.allclose(r1.o.ravel(), gd["o"], atol=1e-12), r1.o
    o1, _, _ = oracle.o1_run(q, k, v, g, beta, W=4, r=1, fmt="int8", S0=S0, lib=lib)
    assert np.allclose(o1.ravel(), gd["o"], atol=1e-12), o1


def pin_golden_quantizer_int8(lib):
    gd = read("quantizer_int8_rows.txt")
    c, s = oracle.quantize(gd["S"].reshape(4, 4), "int8", lib=lib)
    assert np.array_equal(c.ravel(), gd["codes"].astype(np.int8)), c
    assert np.allclose(s.ravel(), gd["scales"], rtol=1e-15, atol=0), s
    c32, s32 = oracle.quantize(gd["S"].reshape(4, 4), "int8", prec32=True, lib=lib)
    assert np.array_equal(c32.ravel(), gd["codes"].astype(np.int8)), c32


def pin_golden_int4(lib):
    gd = read("int4_g32_row.txt")
    D = 32
    S = np.zeros((D, D))
    S[0, : len(gd["row0"])] = gd["row0"]
    c, s = oracle.quantize(S, "int4_g32", lib=lib)
    want = np.zeros(D, np.int8)
    want[: len(gd["codes0"])] = gd["codes0"]
    assert np.array_equal(c[0], want), c[0]
    assert s[0, 0] == gd["scale0"][0] and s[1, 0] == 0.0 and not c[1:].any()
    packed = oracle.pack_int4(c, lib=lib)
    wb = np.zeros(D // 2, np.uint8)
    wb[: len(gd["bytes0"])] = gd["bytes0"]
    assert np.array_equal(packed[0], wb), packed[0]
    assert np.array_equal(oracle.unpack_int4(packed, lib=lib), c)


# ---------------------------------------------------------------------------------------------
# Quantizer, rounding and compensator choice against library routines and bounds
# ---------------------------------------------------------------------------------------------
def pin_quantizer_properties(lib):
    rng = np.random.default_rng(7)
    D = 64   # two int4 groups per row, so a wrong group index shows
    for fmt, qmax in (("int8", 127), ("int4_g32", 7)):
        S = rng.standard_normal((D, D)) * rng.uniform(0.01, 50, size=(D, 1))
        S[:, 40:] *= 7.0
        S[5] = 0.0
        S[9, :32] = 0.0
        S = S.astype(np.float32).astype(np.float64)
        for prec32 in (False, True):
            c, s = oracle.quantize(S, fmt, prec32=prec32, lib=lib)
            ng = s.shape[1]
            gsz = D // ng
            assert gsz == (32 if fmt == "int4_g32" else D)
            deq = oracle.dequantize(c, s, fmt, lib=lib)
            srep = np.repeat(s, gsz, axis=1)
            assert np.all(np.abs(S - deq) <= srep / 2 * (1 + 1e-6) + 1e-300), (fmt, prec32)
            assert np.all(np.abs(c.astype(int)) <= qmax)
            cg = np.abs(c.astype(int)).reshape(D, ng, gsz).max(axis=-1)
            nz = np.abs(S).reshape(D, ng, gsz).max(axis=-1) > 0
            assert np.all(cg[nz] == qmax), (fmt, "some nonzero group lacks a full-range code")
            assert np.all(s[~nz] == 0) and np.all(cg[~nz] == 0)
            # the same decisions through numpy (fp64) / numpy float32 arithmetic (prec32)
            Sg = S.reshape(D, ng, gsz)
            if prec32:
                m = np.abs(Sg).max(axis=-1).astype(np.float32)
                sref = (m / np.float32(qmax)).astype(np.float32)
                with np.errstate(divide="ignore", invalid="ignore"):
                    t = (Sg.astype(np.float32) / sref[..., None]).astype(np.float32)
            else:
                sref = np.abs(Sg).max(axis=-1) / qmax
                with np.errstate(divide="ignore", invalid="ignore"):
                    t = Sg / sref[..., None]
            cref = np.where(sref[..., None] == 0, 0, np.clip(np.rint(t), -qmax, qmax))
            assert np.array_equal(c.reshape(D, ng, gsz), cref.astype(np.int8)), (fmt, prec32)
            assert np.array_equal(s, sref.astype(np.float64)), (fmt, prec32)
    packed = oracle.pack_int4(rng.integers(-7, 8, size=(D, D)).astype(np.int8), lib=lib)
    assert np.array_equal(oracle.pack_int4(oracle.unpack_int4(packed, lib=lib), lib=lib), packed)


def pin_bf16_rounding(lib):
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(2000) * 10.0 ** rng.uniform(-30, 30, 2000),
        rng.standard_normal(200) * 1e-39,                     # bf16 subnormals
        np.array([1 + 2.0**-8, 1 + 3 * 2.0**-8, -(1 + 2.0**-8), 2.0**-133, 1.5 * 2.0**-133]),
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([lib.orc_round_bf16(float(v)) for v in x])
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:10]
    assert lib.orc_round_bf16(1 + 2.0**-8) == 1.0
    assert lib.orc_round_bf16(1 + 3 * 2.0**-8) == 1 + 2.0**-6


def pin_select_columns_vs_sort(lib):
    rng = np.random.default_rng(5)
    for trial in range(20):
        D, r = 16, int(rng.integers(1, 6))
        S = rng.standard_normal((D, D)) * (1 + 10 * (rng.random(D) < 0.2))
        if trial % 4 == 0:   # exact ties of column max-abs: lower index first
            S[:, 3] = S[:, 9] = 0.0
            S[0, 3] = 50.0
            S[1, 9] = -50.0
        idx, _ = oracle.select_columns(S, r, lib=lib)
        ref = np.argsort(-np.abs(S).max(axis=0), kind="stable")[:r]
        assert list(idx) == list(ref), (idx, ref)


# ---------------------------------------------------------------------------------------------
# Closed forms of the recurrence
# ---------------------------------------------------------------------------------------------
def _all_forms(q, k, v, g, beta, S0=None, W=3):
    """State and outputs from the plain, literal and buffered (unquantized) forms."""
    out = {}
    o, S = oracle.plain_run(q, k, v, g, beta, S0=S0, lib=_all_forms.lib)
    out["plain"] = (o, S)
    o1, S1, _ = oracle.o1_run(q, k, v, g, beta, W=W, fmt="none", S0=S0, lib=_all_forms.lib)
    out["O1"] = (o1, S1)
    for w in (W, 10 ** 6):
        r = oracle.o2_run(q, k, v, g, beta, W=w, fmt="none", S0=S0, lib=_all_forms.lib)
        out[f"O2 W={w}"] = (r.o, r.S)
    return out


def pin_single_step_from_zero(lib):
    _all_forms.lib = lib
    for gate in ("scalar", "diag"):
        q, k, v, g, beta = rand_inputs(3, 1, 3, 8, gate)
        want_S = beta[0][:, None, None] * v[0][:, :, None] * k[0][:, None, :]
        want_o = beta[0][:, None] * v[0] * np.sum(k[0] * q[0], axis=-1)[:, None]
        for name, (o, S) in _all_forms(q, k, v, g, beta).items():
            close(S, want_S, 1e-13, f"{name} S1 = beta v k^T ({gate})")
            close(o[0], want_o, 1e-13, f"{name} o1 = beta v (k.q) ({gate})")
        for fmt in ("int8",):
            r = oracle.o2_run(q, k, v, g, beta, W=4, fmt=fmt, lib=lib)
            close(r.S, want_S, 1e-13, f"O2 {fmt} from zero")
            close(r.o[0], want_o, 1e-13, f"O2 {fmt} o1 from zero")


def pin_delta_write_at_key(lib):
    """With |k_t| = 1: S_t k_t = (1 - beta_t) S_{t-1} Diag(a_t) k_t + beta_t v_t, any state."""
    _all_forms.lib = lib
    T, nh, D = 5, 2, 6
    q, k, v, g, beta = rand_inputs(4, T, nh, D, "diag")
    S0 = np.random.default_rng(9).standard_normal((nh, D, D))
    prev = {name: S0 for name in ("plain", "O1", "O2 W=3", f"O2 W={10**6}")}
    for t in range(1, T + 1):
        forms = _all_forms(q[:t], k[:t], v[:t], g[:t], beta[:t], S0=S0)
        for name, (_, S) in forms.items():
            Sp = prev[name] * np.exp(g[t - 1])[:, None, :]
            lhs = np.einsum("hij,hj->hi", S, k[t - 1])
            rhs = (1 - beta[t - 1])[:, None] * np.einsum("hij,hj->hi", Sp, k[t - 1]) \
                + beta[t - 1][:, None] * v[t - 1]
            close(lhs, rhs, 1e-12, f"{name}: write identity at step {t}")
            prev[name] = S


def pin_exact_retrieval(lib):
    """a = 1, beta = 1, orthonormal keys: after writing (k_i, v_i), S k_i = v_i for all i."""
    _all_forms.lib = lib
    D, nh = 8, 2
    rng = np.random.default_rng(12)
    K = np.stack([np.linalg.qr(rng.standard_normal((D, D)))[0].T for _ in range(nh)], axis=1)
    v = rng.standard_normal((D, nh, D))
    q = rng.standard_normal((D, nh, D))
    g = np.zeros((D, nh))
    beta = np.ones((D, nh))
    S0 = rng.standard_normal((nh, D, D))
    for name, (_, S) in _all_forms(q, K, v, g, beta, S0=S0).items():
        got = np.einsum("hij,thj->thi", S, K)
        close(got, v, 1e-12, f"{name}: exact retrieval")


def pin_pure_decay(lib):
    """beta = 0: S_t = S_0 Diag(e^{L_t}), so o_t = S_0 (e^{L_t} * q_t); the gate scales key
    columns, not value rows."""
    _all_forms.lib = lib
    T, nh, D = 6, 2, 5
    q, k, v, g, beta = rand_inputs(6, T, nh, D, "diag")
    beta[:] = 0.0
    S0 = np.random.default_rng(2).standard_normal((nh, D, D))
    L = np.cumsum(g, axis=0)
    want = np.einsum("hij,thj->thi", S0, np.exp(L) * q)
    for name, (o, _) in _all_forms(q, k, v, g, beta, S0=S0).items():
        close(o, want, 1e-12, f"{name}: pure decay")
    # scalar gate, int8 state: codes survive every flush; scales pick up e^{L_W} per window
    q, k, v, g, beta = rand_inputs(8, 12, nh, 16, "scalar")
    beta[:] = 0.0
    S0 = np.random.default_rng(3).standard_normal((nh, 16, 16))
    for r in (0, 2):
        r0 = oracle.o2_run(q[:0], k[:0], v[:0], g[:0], beta[:0], W=4, r=r, S0=S0, lib=lib)
        r12 = oracle.o2_run(q, k, v, g, beta, W=4, r=r, S0=S0, lib=lib)
        assert r12.pos.tolist() == [0] * nh
        assert np.array_equal(r12.codes, r0.codes), f"codes changed under pure decay (r={r})"
        decay = np.exp(g.sum(axis=0))[:, None, None]
        close(r12.scales, r0.scales * decay, 1e-12, f"scales under pure decay (r={r})")
        if r:
            assert np.array_equal(r12.cidx, r0.cidx)
            close(r12.cu, r0.cu * decay, 1e-12, "compensators under pure decay")


def pin_kda_uniform_gate_is_gdn(lib):
    T, nh, D = 20, 3, 16
    q, k, v, g, beta = rand_inputs(21, T, nh, D, "scalar")
    gd = np.repeat(g[..., None], D, axis=-1)
    a = oracle.o2_run(q, k, v, g, beta, W=6, r=2, S0=None, lib=lib)
    b = oracle.o2_run(q, k, v, gd, beta, W=6, r=2, S0=None, lib=lib)
    assert np.array_equal(a.o, b.o) and np.array_equal(a.codes, b.codes)
    pa, _ = oracle.plain_run(q, k, v, g, beta, lib=lib)
    pb, _ = oracle.plain_run(q, k, v, gd, beta, lib=lib)
    assert np.array_equal(pa, pb)


# ---------------------------------------------------------------------------------------------
# Agreement of the formulations
# ---------------------------------------------------------------------------------------------
def pin_windowed_unquantized_is_plain(lib):
    """Buffered windows with the identity quantizer are the plain recurrence, wherever the
    windows end (natural or forced flushes), with or without compensator pairs."""
    T, nh, D = 19, 2, 8
    for gate in ("scalar", "diag"):
        q, k, v, g, beta = rand_inputs(31, T, nh, D, gate)
        S0 = np.random.default_rng(4).standard_normal((nh, D, D))
        po, pS = oracle.plain_run(q, k, v, g, beta, S0=S0, lib=lib)
        mask = np.random.default_rng(8).random((T, nh)) < 0.2
        for W in (1, 2, 3, 8):
            for r in (0, 2):
                for fm in (None, mask):
                    res = oracle.o2_run(q, k, v, g, beta, W=W, r=r, fmt="none", S0=S0,
                                        flush_mask=fm, lib=lib)
                    close(res.o, po, 1e-12, f"O2 none W={W} r={r} {gate}")
                    close(res.S, pS, 1e-12, f"O2 none state W={W} r={r} {gate}")
        o1, S1, _ = oracle.o1_run(q, k, v, g, beta, W=3, fmt="none", S0=S0, lib=lib)
        close(o1, po, 1e-12, f"O1 none {gate}")
        close(S1, pS, 1e-12, f"O1 none state {gate}")


def pin_literal_equals_buffered_quantized(lib):
    """O1 (dense, requantised every W steps) equals O2 (frozen low-bit state + buffer) for
    int8 and int4, with and without compensators; W = 1 is quantize-every-step."""
    for fmt, D in (("int8", 8), ("int4_g32", 32)):
        T, nh = 11, 2
        for gate in ("scalar", "diag"):
            q, k, v, g, beta = rand_inputs(41 + D, T, nh, D, gate)
            S0 = np.random.default_rng(D).standard_normal((nh, D, D))
            for W in (1, 2, 3, 8):
                for r in (0, 2):
                    o1, S1, _ = oracle.o1_run(q, k, v, g, beta, W=W, r=r, fmt=fmt, S0=S0, lib=lib)
                    res = oracle.o2_run(q, k, v, g, beta, W=W, r=r, fmt=fmt, S0=S0, lib=lib)
                    close(res.o, o1, 1e-10, f"O1 vs O2 {fmt} {gate} W={W} r={r}")
                    close(res.S, S1, 1e-10, f"O1 vs O2 state {fmt} {gate} W={W} r={r}")


def pin_compensator_decomposition(lib):
    """Right after quantization: state = dequant(codes) + compensator columns, exactly; the
    taken columns are zero in the codes; the rest is within half a step of the input."""
    D, nh, r = 16, 3, 3
    rng = np.random.default_rng(13)
    S0 = rng.standard_normal((nh, D, D))
    S0[:, :, 4] *= 30.0
    S0[:, :, 11] *= 12.0
    res = oracle.o2_run(np.zeros((0, nh, D)), np.zeros((0, nh, D)), np.zeros((0, nh, D)),
                        np.zeros((0, nh)), np.zeros((0, nh)), W=4, r=r, S0=S0, lib=lib)
    for h in range(nh):
        ref = np.argsort(-np.abs(S0[h]).max(axis=0), kind="stable")[:r]
        assert list(res.cidx[h]) == list(ref)
        deq = oracle.dequantize(res.codes[h], res.scales[h], "int8", lib=lib)
        assert not res.codes[h][:, res.cidx[h]].any()
        rebuilt = deq.copy()
        rebuilt[:, res.cidx[h]] += res.cu[h].T
        assert np.array_equal(rebuilt, res.S[h])
        assert np.array_equal(res.cu[h].T, S0[h][:, res.cidx[h]])
        keep = np.setdiff1d(np.arange(D), res.cidx[h])
        assert np.all(np.abs(S0[h][:, keep] - deq[:, keep]) <= res.scales[h] / 2 * (1 + 1e-12))


def pin_storage_roundings(lib):
    """round_storage keeps exactly what a GPU stores: bf16 write vectors, fp32 log-gates,
    fp32 scales and compensators."""
    T, nh, D = 10, 2, 16
    q, k, v, g, beta = rand_inputs(51, T, nh, D, "diag")
    S0 = np.random.default_rng(1).standard_normal((nh, D, D)).astype(np.float32)
    res = oracle.o2_run(q, k, v, g, beta, W=16, r=2, S0=S0, round_storage=True,
                        buf_round="bf16", lib=lib)
    P = int(res.pos[0])
    bu = res.bu[:, :P]
    assert np.array_equal(bu, torch.from_numpy(bu).to(torch.bfloat16).double().numpy())
    bL = res.bL[:, :P]
    assert np.array_equal(bL, bL.astype(np.float32).astype(np.float64))
    assert np.array_equal(res.scales, res.scales.astype(np.float32).astype(np.float64))
    assert np.array_equal(res.cu, res.cu.astype(np.float32).astype(np.float64))
    exact = oracle.o2_run(q, k, v, g, beta, W=16, r=2, S0=S0, lib=lib)
    close(res.o, exact.o, 2e-2, "storage roundings stay small")


def _bracket_bf16(x):
    """(toward zero, away from zero) bf16 neighbours of fp32 values, from their bit patterns."""
    b = np.asarray(x, np.float32).view(np.uint32)
    t = (b & np.uint32(0xFFFF0000))
    up = t + np.uint32(0x10000)
    return t.view(np.float32).astype(np.float64), up.view(np.float32).astype(np.float64)


def pin_round_other(lib):
    """The alternative rounding of a value is the other storage neighbour: together with the
    rounding it brackets the value (bf16 from fp32 bit patterns, single from numpy's nextafter);
    representable values have no other side."""
    rng = np.random.default_rng(17)
    x = (rng.standard_normal(3000) * 10.0 ** rng.uniform(-20, 20, 3000)).astype(np.float32)
    x = x[(x.view(np.uint32) & np.uint32(0xFFFF)) != 0]          # not bf16-representable
    t, up = _bracket_bf16(x)
    r = np.array([lib.orc_round_bf16(float(v)) for v in x])
    o = np.array([lib.orc_round_other(oracle.ROUND_BF16, float(v)) for v in x])
    assert np.array_equal(np.minimum(np.abs(r), np.abs(o)), np.abs(t))
    assert np.array_equal(np.maximum(np.abs(r), np.abs(o)), np.abs(up))
    assert np.all(np.sign(o) == np.sign(x))
    assert lib.orc_round_other(oracle.ROUND_BF16, 1 + 2.0**-8 + 2.0**-12) == 1.0
    assert lib.orc_round_other(oracle.ROUND_BF16, 1.5) == 1.5
    y = rng.standard_normal(2000) * 10.0 ** rng.uniform(-20, 20, 2000)
    y = y[y.astype(np.float32).astype(np.float64) != y]
    lo = np.nextafter(y.astype(np.float32), np.float32(0)).astype(np.float64)
    lo = np.where(np.abs(lo) > np.abs(y), np.nextafter(lo.astype(np.float32), np.float32(0)), lo)
    lo = np.where(np.abs(y.astype(np.float32).astype(np.float64)) < np.abs(y),
                  y.astype(np.float32).astype(np.float64), lo)
    hi = np.nextafter(lo.astype(np.float32), np.sign(y).astype(np.float32) * np.inf).astype(
        np.float64)
    o32 = np.array([lib.orc_round_other(oracle.ROUND_F32, float(v)) for v in y])
    r32 = y.astype(np.float32).astype(np.float64)
    assert np.array_equal(np.minimum(np.abs(r32), np.abs(o32)), np.abs(lo))
    assert np.array_equal(np.maximum(np.abs(r32), np.abs(o32)), np.abs(hi))


def pin_write_vectors_before_rounding(lib):
    """The exported write vectors are u_t = beta_t (v_t - S_{t-1} Diag(a_t) k_t) before their
    storage rounding, with S_{t-1} the logical state materialised after the previous step; the
    stored ones are their bf16 roundings, and a flipped entry is stored as its other neighbour
    while every earlier step stays as it was."""
    T, nh, D, W = 7, 3, 16, 16
    for gate in ("scalar", "diag"):
        q, k, v, g, beta = rand_inputs(61, T, nh, D, gate)
        S0 = np.random.default_rng(2).standard_normal((nh, D, D)).astype(np.float32)
        kw = dict(W=W, r=1, S0=S0, round_storage=True, buf_round="bf16", lib=lib)
        res = oracle.o2_run(q, k, v, g, beta, want_u_raw=True, **kw)
        prev = oracle.o2_run(q[:-1], k[:-1], v[:-1], g[:-1], beta[:-1], **kw)
        # the cumulative log-gates are stored in fp32 (round_storage), so the last step's
        # decay is e^{L_T - L_{T-1}} of the rounded sums
        gg = g[..., None] * np.ones((T, nh, D)) if gate == "scalar" else g
        Lc = np.zeros((T + 1, nh, D))
        for t in range(T):
            Lc[t + 1] = (Lc[t] + gg[t]).astype(np.float32)
        a = np.exp(Lc[T] - Lc[T - 1])
        w = np.einsum("hij,hj->hi", prev.S, a * k[-1])
        u = beta[-1][:, None] * (v[-1] - w)
        close(res.u_raw[-1], u, 1e-12, "write vector from the materialised state")
        ur = res.u_raw.transpose(1, 0, 2)                         # [nh][T][D]
        assert np.mean(ur == torch.from_numpy(ur).to(torch.bfloat16).double().numpy()) < 0.05
        assert np.array_equal(res.bu[:, :T], torch.from_numpy(ur).to(torch.bfloat16).double()
                              .numpy())
        flip = np.zeros((T, nh, D), np.uint8)
        flip[4, 1, 5] = 1
        alt = oracle.o2_run(q, k, v, g, beta, want_u_raw=True, u_flip=flip, **kw)
        assert np.array_equal(alt.u_raw[:5], res.u_raw[:5])
        assert alt.bu[1, 4, 5] == lib.orc_round_other(oracle.ROUND_BF16, res.u_raw[4, 1, 5])
        assert alt.bu[1, 4, 5] != res.bu[1, 4, 5]
        assert np.array_equal(alt.bu[[0, 2]], res.bu[[0, 2]])


# ---------------------------------------------------------------------------------------------
# Power compensators (reading: tokens spanning the dominant key subspace, subspace iteration)
# ---------------------------------------------------------------------------------------------
def _tokens(we):
    return we.cu.T @ we.ck  # sum_c cu_c ck_c^T


def pin_power_exact_low_rank(lib):
    """A state of rank r is carried entirely by r power tokens: residual 0, tokens = S."""
    rng = np.random.default_rng(71)
    for D, r in ((16, 2), (32, 4)):
        A, B = rng.standard_normal((D, r)), rng.standard_normal((D, r))
        S = A @ B.T
        we = oracle.window_end(S, "none", r=r, comp_rule="power", lib=lib)
        close(_tokens(we), S, 1e-10, "rank-r state rebuilt by its tokens")
        assert np.abs(we.residual).max() <= 1e-10 * np.abs(S).max()


def pin_power_planted_outlier(lib):
    """A dominant rank-one outlier planted on noise is the first token: its key is the
    outlier's key direction (up to sign), its value S times that key."""
    rng = np.random.default_rng(72)
    D = 32
    u, v = rng.standard_normal(D), rng.standard_normal(D)
    u, v = u / np.linalg.norm(u), v / np.linalg.norm(v)
    S = 0.02 * rng.standard_normal((D, D)) + 30.0 * np.outer(u, v)
    we = oracle.window_end(S, "none", r=1, comp_rule="power", lib=lib)
    v1 = np.linalg.svd(S)[2][0]  # LAPACK's top right singular vector
    assert abs(float(we.ck[0] @ v1)) >= 1 - 1e-12, we.ck[0] @ v1
    assert abs(float(we.ck[0] @ v)) >= 1 - 1e-4, we.ck[0] @ v
    close(we.cu[0], S @ we.ck[0], 1e-12, "token value = S key")


def pin_power_energy_matches_svd(lib):
    """With a clear spectral gap the tokens carry the top-r singular energy that LAPACK's SVD
    gives; the keys are orthonormal, the residual is orthogonal to them, and residual + tokens
    is the state exactly."""
    rng = np.random.default_rng(73)
    D, r = 32, 4
    U, _ = np.linalg.qr(rng.standard_normal((D, D)))
    V, _ = np.linalg.qr(rng.standard_normal((D, D)))
    sig = np.concatenate([[100.0, 50.0, 25.0, 12.0], np.linspace(1.0, 0.1, D - 4)])
    S = (U * sig) @ V.T
    we = oracle.window_end(S, "none", r=r, comp_rule="power", lib=lib)
    sv = np.linalg.svd(S, compute_uv=False)
    e_tok = float(np.sum(_tokens(we) ** 2))
    assert abs(e_tok - float(np.sum(sv[:r] ** 2))) <= 1e-9 * e_tok, (e_tok, sv[:r])
    assert np.allclose(we.ck @ we.ck.T, np.eye(r), atol=1e-12)
    assert np.abs(we.residual @ we.ck.T).max() <= 1e-10 * np.abs(S).max()
    close(we.residual + _tokens(we), S, 1e-13, "residual + tokens")
    # a random state (no gap): still orthonormal keys and an exact decomposition
    S2 = rng.standard_normal((D, D))
    we2 = oracle.window_end(S2, "none", r=r, comp_rule="power", lib=lib)
    assert np.allclose(we2.ck @ we2.ck.T, np.eye(r), atol=1e-12)
    close(we2.residual + _tokens(we2), S2, 1e-13, "residual + tokens, no gap")


def pin_power_start_and_ties(lib):
    """On a diagonal state the dominant key subspace is spanned by the coordinate vectors of
    the largest entries, which is where the iteration starts (largest column norms) and stays:
    the keys are exactly those e_j, ties going to the lower column."""
    D = 8
    d = np.array([0.5, -3.0, 1.0, 2.0, 0.25, -2.0, 0.1, 0.7])
    we = oracle.window_end(np.diag(d), "none", r=2, comp_rule="power", lib=lib)
    assert np.array_equal(we.ck, np.eye(D)[[1, 3]]), we.ck
    assert np.array_equal(we.cu, np.diag(d)[:, [1, 3]].T)
    tie = np.diag([1.0, 2.0, 2.0, 0.5])
    we = oracle.window_end(tie, "none", r=1, comp_rule="power", lib=lib)
    assert np.array_equal(we.ck, np.eye(4)[[1]]), we.ck


def pin_power_windows_agree(lib):
    """With power tokens: the literal form (O1) equals the buffered form (O2) with
    quantization on, and without quantization the buffered form is the plain recurrence."""
    T, nh, D = 12, 3, 16
    for gate in ("scalar", "diag"):
        q, k, v, g, beta = rand_inputs(81, T, nh, D, gate, outlier=True)
        S0 = np.random.default_rng(3).standard_normal((nh, D, D))
        for W, r in ((3, 2), (5, 1)):
            o1, S1, _ = oracle.o1_run(q, k, v, g, beta, W=W, r=r, fmt="int8", S0=S0,
                                      comp_rule="power", lib=lib)
            o2 = oracle.o2_run(q, k, v, g, beta, W=W, r=r, fmt="int8", S0=S0,
                               comp_rule="power", lib=lib)
            close(o2.o, o1, 1e-10, f"O1 = O2 with power tokens ({gate}, W={W})")
        plain, _ = oracle.plain_run(q, k, v, g, beta, S0=S0, lib=lib)
        ex = oracle.o2_run(q, k, v, g, beta, W=4, r=2, fmt="none", S0=S0, comp_rule="power",
                           lib=lib)
        close(ex.o, plain, 1e-10, f"unquantized windows with power tokens = plain ({gate})")


# ---------------------------------------------------------------------------------------------
# Residual smoothing (reading: per-column power-of-two factors m_j = 2^floor(E_j / 2))
# ---------------------------------------------------------------------------------------------
def pin_golden_smoothing(lib):
    gd = read("smoothing_4x4.txt")
    S = gd["S"].reshape(4, 4)
    we = oracle.window_end(S, "int8", r=0, smooth=True, lib=lib)
    assert list(we.sexp) == [int(x) for x in gd["sexp"]], we.sexp
    assert np.array_equal(we.codes.ravel(), gd["codes"].astype(np.int8)), we.codes
    assert np.allclose(we.scales.ravel() * 127, gd["absmax"], rtol=1e-15, atol=0), we.scales
    we1 = oracle.window_end(S, "int8", r=1, smooth=True, lib=lib)
    assert list(we1.cidx) == [0] and np.array_equal(we1.cu[0], gd["comp_u_r1"])
    assert list(we1.sexp) == [int(x) for x in gd["sexp_r1"]], we1.sexp
    assert np.array_equal(we1.codes.ravel(), gd["codes_r1"].astype(np.int8)), we1.codes
    assert np.allclose(we1.scales.ravel() * 127, gd["absmax_r1"], rtol=1e-15, atol=0)
    # the same as the initial quantization of the buffered form: the state it keeps is
    # dequant(codes, scales) Diag(2^e) plus the compensator column
    e0 = np.zeros((0, 1, 4))
    res = oracle.o2_run(e0, e0, e0, np.zeros((0, 1)), np.zeros((0, 1)), W=4, r=1, fmt="int8",
                        S0=S.reshape(1, 4, 4), smooth=True, lib=lib)
    assert np.array_equal(res.codes[0], we1.codes) and list(res.sexp[0]) == list(we1.sexp)
    kept = gd["codes_r1"].reshape(4, 4) * (gd["absmax_r1"].reshape(4, 1) / 127.0)
    kept = kept * 2.0 ** gd["sexp_r1"].reshape(1, 4)
    kept[:, 0] += gd["comp_u_r1"]
    assert np.allclose(res.S[0], kept, rtol=1e-15, atol=1e-300), res.S[0]


def pin_smooth_exponent(lib):
    """Hand values of e = floor(floor(log2 m) / 2) clamped to [-63, 63], and m_j = 2^e against
    the square root it stands for: 2^e <= sqrt(colmax) < 2^(e+1)."""
    cases = [(0.0, 0), (1.0, 0), (2.0, 0), (3.99, 0), (4.0, 1), (15.9, 1), (16.0, 2),
             (0.5, -1), (0.3, -1), (0.25, -1), (0.2, -2), (2.0 ** 200, 63), (2.0 ** -200, -63),
             (2.0 ** -127, -63), (2.0 ** -126, -63), (2.0 ** -125, -63), (2.0 ** -124, -62)]
    for m, e in cases:
        got = oracle.smooth_exponent(m, lib=lib)
        assert got == e, (m, got, e)
    rng = np.random.default_rng(3)
    for m in 10.0 ** rng.uniform(-30, 30, size=400):
        e = oracle.smooth_exponent(m, lib=lib)
        assert 2.0 ** e <= np.sqrt(m) < 2.0 ** (e + 1), (m, e)


def pin_smoothing_properties(lib):
    """On states with outlier key columns: the exponents follow the residual's column max-abs
    (compensator columns excluded), the kept state is within half a quantization step (times
    the column's factor) of the input, a uniform band of column maxima gives the unsmoothed
    codes, and smoothing lowers the reconstruction error (what the page claims for it)."""
    rng = np.random.default_rng(17)
    D = 64
    for fmt in ("int8", "int4_g32"):
        for r in (0, 3):
            S = rng.standard_normal((D, D)) * rng.uniform(0.05, 3.0, size=(D, 1))
            S[:, [3, 20, 41]] *= 20.0
            S[:, 50:] *= 0.05
            S = S.astype(np.float32).astype(np.float64)
            plain = oracle.window_end(S, fmt, r=r, smooth=False, lib=lib)
            sm = oracle.window_end(S, fmt, r=r, smooth=True, lib=lib)
            assert list(plain.cidx) == list(sm.cidx)
            R = S.copy()
            R[:, sm.cidx] = 0.0
            cm = np.abs(R).max(axis=0)
            m = 2.0 ** sm.sexp.astype(np.float64)
            nz = cm > 0
            assert np.all((m[nz] <= np.sqrt(cm[nz])) & (np.sqrt(cm[nz]) < 2 * m[nz]))
            assert np.all(sm.sexp[~nz] == 0)
            deq = oracle.dequantize(sm.codes, sm.scales, fmt, lib=lib) * m
            step = np.repeat(sm.scales, D // sm.scales.shape[1], axis=1) * m
            assert np.all(np.abs(R - deq) <= step / 2 * (1 + 1e-12))
            kept = deq.copy()
            kept[:, sm.cidx] += sm.cu.T
            kept_p = oracle.dequantize(plain.codes, plain.scales, fmt, lib=lib)
            kept_p[:, plain.cidx] += plain.cu.T
            assert rel(kept, S) < rel(kept_p, S), (fmt, r, rel(kept, S), rel(kept_p, S))
    # column maxima all in [4, 16): every e is 1, codes as without smoothing, scales halved
    S = rng.uniform(-1, 1, size=(D, D))
    S *= (4.0 + 11.9 * rng.uniform(size=D))[None, :] / np.abs(S).max(axis=0)
    for fmt in ("int8", "int4_g32"):
        plain = oracle.window_end(S, fmt, smooth=False, lib=lib)
        sm = oracle.window_end(S, fmt, smooth=True, lib=lib)
        assert np.all(sm.sexp == 1)
        assert np.array_equal(sm.codes, plain.codes)
        assert np.array_equal(sm.scales * 2.0, plain.scales)


def pin_smoothing_unquantized_is_exact(lib):
    """Without quantization the smoothing is undone exactly: the buffered form with and without
    it gives bit-identical outputs and states."""
    T, nh, D = 9, 2, 16
    for gate in ("scalar", "diag"):
        q, k, v, g, beta = rand_inputs(61, T, nh, D, gate, outlier=True)
        S0 = np.random.default_rng(5).standard_normal((nh, D, D)) * 3.0
        a = oracle.o2_run(q, k, v, g, beta, W=4, r=2, fmt="none", S0=S0, smooth=True, lib=lib)
        b = oracle.o2_run(q, k, v, g, beta, W=4, r=2, fmt="none", S0=S0, smooth=False, lib=lib)
        assert np.array_equal(a.o, b.o) and np.array_equal(a.S, b.S), gate
        assert np.any(a.sexp != 0)


def pin_smoothed_literal_equals_buffered(lib):
    """O1 (dense, requantised every W steps) equals O2 (frozen low-bit state + buffer) with
    residual smoothing too, for int8 and int4, with and without compensators."""
    for fmt, D in (("int8", 8), ("int4_g32", 32)):
        T, nh = 11, 2
        for gate in ("scalar", "diag"):
            q, k, v, g, beta = rand_inputs(71 + D, T, nh, D, gate, outlier=True)
            S0 = np.random.default_rng(D + 1).standard_normal((nh, D, D))
            S0[:, :, 1] *= 25.0
            for W in (1, 3, 8):
                for r in (0, 2):
                    o1, S1, _ = oracle.o1_run(q, k, v, g, beta, W=W, r=r, fmt=fmt, S0=S0,
                                              smooth=True, lib=lib)
                    res = oracle.o2_run(q, k, v, g, beta, W=W, r=r, fmt=fmt, S0=S0, smooth=True,
                                        lib=lib)
                    close(res.o, o1, 1e-10, f"smoothed O1 vs O2 {fmt} {gate} W={W} r={r}")
                    close(res.S, S1, 1e-10, f"smoothed O1 vs O2 state {fmt} {gate} W={W} r={r}")


# ---------------------------------------------------------------------------------------------
# PW: the pure-write sliding window
# ---------------------------------------------------------------------------------------------
def pin_golden_pure_write_window(lib):
    gd = read("pure_write_window_2x2.txt")
    D, T, Wp = 2, 3, 2
    q, k, v = (gd[n].reshape(T, 1, D) for n in ("q", "k", "v"))
    g = np.log(gd["a"]).reshape(T, 1)
    beta = gd["beta"].reshape(T, 1)
    S0 = gd["S0"].reshape(1, D, D)
    res = oracle.pw_run(q, k, v, g, beta, Wp=Wp, S0=S0, lib=lib)
    assert np.allclose(res.o.ravel(), gd["o"], atol=1e-12), ("PW o", res.o.ravel())
    assert np.allclose(res.S.ravel(), gd["S3"], atol=1e-12), ("PW S3", res.S.ravel())
    r2 = oracle.pw_run(q[:2], k[:2], v[:2], g[:2], beta[:2], Wp=Wp, S0=S0, lib=lib)
    H2 = (r2.codes[0] * r2.scales[0]).ravel()       # int8: one scale per row
    assert np.allclose(H2, gd["H2"], atol=1e-12), ("PW H2", H2)


def pin_e4m3_rounding(lib):
    """e4m3 against torch's float8_e4m3fn conversion (round to nearest even) on normals,
    subnormals, exact ties and the largest finite value; the FP8 vector round trip against
    s * e4m3(x / s) with s = absmax / 448 done through torch."""
    rng = np.random.default_rng(12)
    x = np.concatenate([
        rng.uniform(-447.0, 447.0, 3000),
        np.clip(rng.standard_normal(2000) * 2.0 ** rng.uniform(-12, 8, 2000), -460.0, 460.0),
        np.array([2.0**-9, 2.0**-10, 3 * 2.0**-10, 5 * 2.0**-10, 1 + 2.0**-4, 1 + 3 * 2.0**-4,
                  -(1 + 2.0**-4), 2.0**-6 * (1 + 2.0**-4), 17.0 * 2.0**-10, 448.0, -448.0,
                  464.0 - 2.0**-6, 0.0]),
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([lib.orc_round_e4m3(float(t)) for t in x])
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:10]
    # past 464 torch's conversion gives NaN; the saturating reading (a GPU's satfinite
    # conversion) keeps the largest finite value
    assert lib.orc_round_e4m3(500.0) == 448.0 and lib.orc_round_e4m3(-1e6) == -448.0
    for n in (5, 128):
        vec = rng.standard_normal(n) * 10.0 ** rng.uniform(-3, 3)
        out, s = oracle.fp8_vector(vec, lib=lib)
        ref_s = np.abs(vec).max() / 448.0
        t = torch.from_numpy(vec / ref_s).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        assert s == ref_s and np.allclose(out, ref_s * t, rtol=1e-15, atol=0), (n, out)
        j = int(np.argmax(np.abs(vec)))
        assert abs(out[j] - vec[j]) <= 1e-14 * abs(vec[j])   # the absmax entry is kept
    out, s = oracle.fp8_vector(np.zeros(4), lib=lib)
    assert s == 0.0 and not out.any()


def pin_pw_exact_is_plain(lib):
    """With an exact history and exact pairs the window only moves terms between two stores:
    outputs and final state are the plain recurrence's, for every window length and gate."""
    for gate, seed in (("scalar", 51), ("diag", 52)):
        q, k, v, g, beta = rand_inputs(seed, 9, 2, 6, gate)
        S0 = np.random.default_rng(seed).standard_normal((2, 6, 6))
        o_ref, S_ref = oracle.plain_run(q, k, v, g, beta, S0=S0, lib=lib)
        for Wp in (0, 1, 3, 12):
            res = oracle.pw_run(q, k, v, g, beta, Wp=Wp, S0=S0, quant=False, fp8=False, lib=lib)
            close(res.o, o_ref, 1e-12, f"PW exact o ({gate}, Wp={Wp})")
            close(res.S, S_ref, 1e-12, f"PW exact S ({gate}, Wp={Wp})")


def pin_pw_no_window_is_every_step_quantization(lib):
    """Wp = 0: each write joins the history at once, which is then requantised: the literal
    matrix form requantised after every step (window length 1)."""
    for fmt, D in (("int8", 8), ("int4_g32", 32)):
        for gate in ("scalar", "diag"):
            q, k, v, g, beta = rand_inputs(61, 7, 2, D, gate)
            S0 = np.random.default_rng(62).standard_normal((2, D, D))
            o1, S1, _ = oracle.o1_run(q, k, v, g, beta, W=1, fmt=fmt, S0=S0, lib=lib)
            res = oracle.pw_run(q, k, v, g, beta, Wp=0, fmt=fmt, S0=S0, lib=lib)
            close(res.o, o1, 1e-12, f"PW Wp=0 o ({fmt}, {gate})")
            close(res.S, S1, 1e-12, f"PW Wp=0 S ({fmt}, {gate})")


def pin_pw_superposition(lib):
    """When no pair leaves the window (Wp >= T) the writes never meet the quantizer: the state
    is the history's own quantised evolution (the every-step-quantised recurrence with v = 0)
    plus every write carried exactly (the plain recurrence from a zero state). The recurrence
    is linear in S, so the outputs add up the same way."""
    for gate in ("scalar", "diag"):
        q, k, v, g, beta = rand_inputs(71, 6, 2, 8, gate)
        S0 = np.random.default_rng(72).standard_normal((2, 8, 8))
        oh, Sh, _ = oracle.o1_run(q, k, np.zeros_like(v), g, beta, W=1, fmt="int8", S0=S0,
                                  lib=lib)
        ow, Sw = oracle.plain_run(q, k, v, g, beta, lib=lib)
        res = oracle.pw_run(q, k, v, g, beta, Wp=6, fmt="int8", S0=S0, fp8=False, lib=lib)
        close(res.o, oh + ow, 1e-12, f"PW superposition o ({gate})")
        close(res.S, Sh + Sw, 1e-12, f"PW superposition S ({gate})")


def pin_pw_window_timing(lib):
    """A write below half a quantization step of its row is visible in the outputs exactly
    while it is in the window (steps tau .. tau + Wp - 1), and on the step it joins the history
    (that step's output precedes the requantisation, which then rounds it away)."""
    D, T, tau, eps = 2, 12, 2, 1e-3
    S0 = np.array([[[1.0, 0.0], [1.0, 0.0]]])     # column 1 empty
    q = np.tile(np.array([0.0, 1.0]), (T, 1, 1))   # read column 1
    k = np.tile(np.array([0.0, 1.0]), (T, 1, 1))
    v = np.zeros((T, 1, D))
    v[tau, 0] = [eps, 0.0]
    g = np.zeros((T, 1))                            # a = 1
    beta = np.zeros((T, 1))
    beta[tau] = 1.0                                 # the one write; otherwise no transition
    for Wp in (0, 1, 3):
        res = oracle.pw_run(q, k, v, g, beta, Wp=Wp, S0=S0, lib=lib)
        want = np.zeros((T, 1, D))
        want[tau: tau + Wp + 1, 0, 0] = eps
        assert np.allclose(res.o, want, rtol=1e-12, atol=1e-18), (Wp, res.o[:, 0, 0])


PINS = [
    pin_golden_delta_rule_kda,
    pin_golden_window_int8,
    pin_golden_compensator,
    pin_golden_quantizer_int8,
    pin_golden_int4,
    pin_quantizer_properties,
    pin_bf16_rounding,
    pin_select_columns_vs_sort,
    pin_single_step_from_zero,
    pin_delta_write_at_key,
    pin_exact_retrieval,
    pin_pure_decay,
    pin_kda_uniform_gate_is_gdn,
    pin_windowed_unquantized_is_plain,
    pin_literal_equals_buffered_quantized,
    pin_compensator_decomposition,
    pin_storage_roundings,
    pin_round_other,
    pin_write_vectors_before_rounding,
    pin_power_exact_low_rank,
    pin_power_planted_outlier,
    pin_power_energy_matches_svd,
    pin_power_start_and_ties,
    pin_power_windows_agree,
    pin_golden_smoothing,
    pin_smooth_exponent,
    pin_smoothing_properties,
    pin_smoothing_unquantized_is_exact,
    pin_smoothed_literal_equals_buffered,
    pin_golden_pure_write_window,
    pin_e4m3_rounding,
    pin_pw_exact_is_plain,
    pin_pw_no_window_is_every_step_quantization,
    pin_pw_superposition,
    pin_pw_window_timing,
]
