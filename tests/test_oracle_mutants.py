"""Mutation check of the oracle's pins: each case plants one plausible mistake (a dropped term, a
wrong sign, index or operand) in a temporary copy of the oracle's C source, builds it, and
requires at least one pin to fail on it. The real oracle is never modified."""
import os

import pytest

import oracle
from oracle import build as orc_build
from oracle_pins import PINS

MUTANTS = [
    ("plain: delta term sign",
     "S[(size_t)i * D + j] += -bt * w[i] * kt[j] + bt * vt[i] * kt[j];",
     "S[(size_t)i * D + j] += bt * w[i] * kt[j] + bt * vt[i] * kt[j];"),
    ("plain: write outer product transposed",
     "S[(size_t)i * D + j] += -bt * w[i] * kt[j] + bt * vt[i] * kt[j];",
     "S[(size_t)i * D + j] += -bt * w[i] * kt[j] + bt * vt[j] * kt[i];"),
    ("plain: gate applied to value rows",
     "for (int j = 0; j < D; ++j) S[(size_t)i * D + j] *= a[j];",
     "for (int j = 0; j < D; ++j) S[(size_t)i * D + j] *= a[i];"),
    ("plain: output from the key instead of the query",
     "for (int j = 0; j < D; ++j) acc += S[(size_t)i * D + j] * qt[j];\n                    ot[i] = acc;\n                }\n            }\n            if (state_round",
     "for (int j = 0; j < D; ++j) acc += S[(size_t)i * D + j] * kt[j];\n                    ot[i] = acc;\n                }\n            }\n            if (state_round"),
    ("O1: beta dropped from the transition",
     "((j == l ? 1.0 : 0.0) - bt * kt[j] * kt[l])",
     "((j == l ? 1.0 : 0.0) - kt[j] * kt[l])"),
    ("O1: gate on the wrong side of the projection",
     "exp(gate_log(gt, Dg, j)) * ((j == l",
     "exp(gate_log(gt, Dg, l)) * ((j == l"),
    ("O1: window end one step early",
     "if ((t + 1) % W == 0) ties += dense_window_end(D, fmt, r, smooth, rule, S);",
     "if (t % W == 0) ties += dense_window_end(D, fmt, r, smooth, rule, S);"),
    ("O2: beta dropped from the write vector",
     "double u = bt * (vt[i] - w[i]);",
     "double u = (vt[i] - w[i]);"),
    ("O2: buffer decay factor with the wrong sign",
     "double f = exp(Lt[j] - s->bL[(size_t)p * D + j]);",
     "double f = exp(s->bL[(size_t)p * D + j] - Lt[j]);"),
    ("O2: output from w instead of r",
     "if (ot) ot[i] = rr[i] + u * kq;",
     "if (ot) ot[i] = w[i] + u * kq;"),
    ("O2: current write dropped from the output",
     "if (ot) ot[i] = rr[i] + u * kq;",
     "if (ot) ot[i] = rr[i];"),
    ("O2: compensators dropped from the step",
     "w[i] += s->cu[(size_t)cc * D + i] * ax;",
     "w[i] += 0.0 * ax;"),
    ("O2: key used for the query projection",
     "y[j] = exp(Lt[j]) * qt[j];",
     "y[j] = exp(Lt[j]) * kt[j];"),
    ("O2: log-gate not accumulated",
     "Lt[j] = Lt[j] + gate_log(gt, c->Dg, j);",
     "Lt[j] = gate_log(gt, c->Dg, j);"),
    ("O2: compensator not decayed at materialisation",
     "S[(size_t)i * D + j] += s->cu[(size_t)cc * D + i] * s->ck[(size_t)cc * D + j] * exp(L[j]);",
     "S[(size_t)i * D + j] += s->cu[(size_t)cc * D + i] * s->ck[(size_t)cc * D + j];"),
    ("O2: frozen state not decayed at materialisation",
     "S[(size_t)i * D + j] = s->F[(size_t)i * D + j] * exp(L[j]);",
     "S[(size_t)i * D + j] = s->F[(size_t)i * D + j];"),
    ("smoothing: factor not undone on the frozen state",
     "    if (c->smooth) unsmooth(D, s->sexp, s->F);",
     "    if (0) unsmooth(D, s->sexp, s->F);"),
    ("smoothing: exponent not halved",
     "int e = E >= 0 ? E / 2 : -((1 - E) / 2);  /* floor(E / 2) */",
     "int e = E;"),
    ("smoothing: exponent rounded toward zero",
     "int e = E >= 0 ? E / 2 : -((1 - E) / 2);  /* floor(E / 2) */",
     "int e = E / 2;"),
    ("smoothing: factors from row maxima",
     "for (int i = 0; i < D; ++i) m = fmax(m, fabs(S[(size_t)i * D + j]));\n            sexp[j]",
     "for (int i = 0; i < D; ++i) m = fmax(m, fabs(S[(size_t)j * D + i]));\n            sexp[j]"),
    ("smoothing: residual scaled up instead of down",
     "S[(size_t)i * D + j] = ldexp(S[(size_t)i * D + j], -sexp[j]);",
     "S[(size_t)i * D + j] = ldexp(S[(size_t)i * D + j], sexp[j]);"),
    ("quantizer: int8 range 128",
     "return fmt == ORC_FMT_INT4 ? 7 : 127;",
     "return fmt == ORC_FMT_INT4 ? 7 : 128;"),
    ("quantizer: ties away from zero",
     "double r = rint(t);",
     "double r = round(t);"),
    ("quantizer: truncation",
     "double r = rint(t);",
     "double r = trunc(t);"),
    ("quantizer: group of the wrong column",
     "S[(size_t)i * D + j] = scales[(size_t)i * ng + j / gs] * (double)codes[(size_t)i * D + j];",
     "S[(size_t)i * D + j] = scales[(size_t)i * ng + (D - 1 - j) / gs] * (double)codes[(size_t)i * D + j];"),
    ("int4: nibbles swapped",
     "packed[(size_t)i * (D / 2) + m] = (uint8_t)(lo | (hi << 4));",
     "packed[(size_t)i * (D / 2) + m] = (uint8_t)(hi | (lo << 4));"),
    ("compensators: ties to the higher index",
     "if (!taken[j] && (best < 0 || colmax[j] > colmax[best])) best = j;",
     "if (!taken[j] && (best < 0 || colmax[j] >= colmax[best])) best = j;"),
    ("compensators: chosen by column sum instead of max-abs",
     "for (int i = 0; i < D; ++i) colmax[j] = fmax(colmax[j], fabs(S[(size_t)i * D + j]));",
     "for (int i = 0; i < D; ++i) colmax[j] += S[(size_t)i * D + j];"),
    ("bf16: one mantissa bit too many",
     "int qexp = e - 8;",
     "int qexp = e - 9;"),
    ("PW: pair leaves the window one step late",
     "if (Wp > 0 && t >= Wp)",
     "if (Wp > 0 && t > Wp)"),
    ("PW: carried keys not erased by later writes",
     "yn[j] = a[j] * y[j] - bt * ky * kt[j];",
     "yn[j] = a[j] * y[j];"),
    ("PW: carried keys not gated",
     "yn[j] = a[j] * y[j] - bt * ky * kt[j];",
     "yn[j] = y[j] - bt * ky * kt[j];"),
    ("PW: new write missing from the output",
     "for (int i = 0; i < D; ++i) ot[i] += x[i] * kq;",
     "for (int i = 0; i < D; ++i) ot[i] += 0.0 * x[i] * kq;"),
    ("PW: carried pairs read with the key instead of the query",
     "for (int j = 0; j < D; ++j) yq += pyn[(size_t)sl * D + j] * qt[j];",
     "for (int j = 0; j < D; ++j) yq += pyn[(size_t)sl * D + j] * kt[j];"),
    ("PW: history requantised only when a pair joins it",
     "            if (quant) {\n                if (prec32)",
     "            if (quant && (Wp == 0 || t >= Wp)) {\n                if (prec32)"),
    ("PW: write vector without beta",
     "x[i] = bt * vt[i];",
     "x[i] = vt[i];"),
    ("e4m3: one mantissa bit too many",
     "int qexp = e - 4;",
     "int qexp = e - 5;"),
    ("e4m3: subnormal spacing too fine",
     "if (qexp < -9) qexp = -9;",
     "if (qexp < -10) qexp = -10;"),
    ("power tokens: keys not normalised",
     "xc[j] = n > 0.0 ? xc[j] / n : 0.0;",
     "xc[j] = xc[j];"),
    ("power tokens: S instead of S^T in the iteration",
     "acc += S[(size_t)i * D + j] * Y[(size_t)c * D + i];",
     "acc += S[(size_t)j * D + i] * Y[(size_t)c * D + i];"),
    ("power tokens: Gram-Schmidt projection added",
     "xc[j] -= dot * xp[j];",
     "xc[j] += dot * xp[j];"),
    ("power tokens: values from S^T",
     "acc += S[(size_t)i * D + j] * kc[j];",
     "acc += S[(size_t)j * D + i] * kc[j];"),
    ("power tokens: residual keeps the tokens",
     "S[(size_t)i * D + j] -= cu[(size_t)c * D + i] * ck[(size_t)c * D + j];",
     "S[(size_t)i * D + j] -= 0.0 * cu[(size_t)c * D + i] * ck[(size_t)c * D + j];"),
    ("power tokens: start from the smallest columns",
     "if (!taken[j] && (best < 0 || nrm[j] > nrm[best])) best = j;",
     "if (!taken[j] && (best < 0 || nrm[j] < nrm[best])) best = j;"),
    ("O2: token coefficient from the ungated key",
     "ax += s->ck[(size_t)cc * D + j] * x[j];",
     "ax += s->ck[(size_t)cc * D + j] * kt[j];"),
    ("alternative rounding: the rounding itself",
     "return round_to(mode, x) == lo ? hi : lo;",
     "return round_to(mode, x);"),
    ("alternative rounding: one quantum too far",
     "const double lo = floor(x / quantum) * quantum, hi = lo + quantum;",
     "const double lo = floor(x / quantum) * quantum - quantum, hi = lo + 3 * quantum;"),
    ("write vectors exported after their rounding",
     "        if (u_raw) u_raw[i] = u;\n        if (c->round_storage)\n"
     "            u = (u_flip && u_flip[i]) ? orc_round_other(c->buf_round, u) : round_to(c->buf_round, u);",
     "        if (c->round_storage)\n"
     "            u = (u_flip && u_flip[i]) ? orc_round_other(c->buf_round, u) : round_to(c->buf_round, u);\n"
     "        if (u_raw) u_raw[i] = u;"),
    ("flipped write vector rounded as usual",
     "u = (u_flip && u_flip[i]) ? orc_round_other",
     "u = (0) ? orc_round_other"),
    ("FP8 vector: scale for a largest value of 240",
     "double s = m / 448.0;",
     "double s = m / 240.0;"),
]


def _build_mutant(tmp_path, original, replacement):
    src = open(orc_build.SRC).read()
    assert src.count(original) == 1, f"mutation anchor not unique: {original!r}"
    path = os.path.join(tmp_path, "mutant.c")
    with open(path, "w") as f:
        f.write(src.replace(original, replacement))
    return orc_build.compile_oracle(path, os.path.join(tmp_path, "libmutant.so"))


@pytest.mark.parametrize("name,original,replacement", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, original, replacement, tmp_path):
    lib = oracle.load(_build_mutant(str(tmp_path), original, replacement))
    caught = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches: {name}"
