"""fp64 CPU oracle for windowed low-bit GDN / KDA decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline / reference legs
may import this package. It never touches the CUDA library and the CUDA library never touches
it: both sides only share the seeded inputs made by ``workloads``.

This module is argument marshalling around ``gdn_oracle.c`` (numpy <-> C pointers). Every
function of the method lives in the C file, which states what it restates from the pages
("LeapQuant: Efficient Linear Attention with Accurate Recurrent State Quantization", Abstract;
"Low-Bit GDN Recurrent-State Quantization: ... Pure-Write Sliding Windows", Abstract).

Parity unpinned against the pages (pinned only to the mathematics): the FP8 format of the
pure-write pairs (e4m3, one fp32 scale absmax / 448 per vector). The page says "FP8 vector
pairs" and nothing more; the tests pin the e4m3 rounding to torch's float8_e4m3fn and the
window's algebra to the plain recurrence, not the format choice.

Parity unpinned: the compensator column-selection rule (top-r columns by max-abs). The pages
name compensator tokens but give no selection rule and no numbers; the tests pin only that the
taken-out columns plus the residual reproduce the state exactly.

Parity unpinned: the "power" compensator rule (keys from six steps of subspace iteration started
at the largest-norm key columns, values S x_c). The pages give no rule; the tests pin it to the
mathematics (exact low-rank states, a planted dominant direction against LAPACK's singular
vectors, the truncated SVD's energy), not to the pages.

Conventions: a state S is [D][D] with row i = value channel, column j = key channel. Per-step
arrays are time-major, ``[T][nh][D]``; the gate ``g = log a`` is ``[T][nh]`` (scalar, GDN) or
``[T][nh][D]`` (per key channel, KDA).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

FMT_NONE, FMT_INT8, FMT_INT4 = 0, 1, 2
COMP_RULES = {"columns": 0, "power": 1}
ROUND_NONE, ROUND_F32, ROUND_BF16 = 0, 1, 2
_FMT = {"none": FMT_NONE, "int8": FMT_INT8, "int4_g32": FMT_INT4, "int4": FMT_INT4}
_ROUND = {"none": ROUND_NONE, "f32": ROUND_F32, "bf16": ROUND_BF16}

_lib = None
_lib_path = None

_d = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i8 = np.ctypeslib.ndpointer(dtype=np.int8, flags="C_CONTIGUOUS")
_u8 = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_i32 = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p
_int = ctypes.c_int


def load(path: Optional[str] = None):
    """Load (building if needed) the oracle library. ``path`` selects another build of the
    same source, e.g. a deliberately broken copy in a mutation test."""
    global _lib, _lib_path
    if path is None:
        if _lib is not None and _lib_path == _build.OUT:
            return _lib
        path = _build.build()
    lib = ctypes.CDLL(path)
    lib.orc_num_threads.restype = _int
    lib.orc_round_bf16.restype = ctypes.c_double
    lib.orc_round_bf16.argtypes = [ctypes.c_double]
    lib.orc_round_f32.restype = ctypes.c_double
    lib.orc_round_f32.argtypes = [ctypes.c_double]
    lib.orc_num_groups.restype = _int
    lib.orc_num_groups.argtypes = [_int, _int]
    lib.orc_quantize.restype = _int
    lib.orc_quantize.argtypes = [_int, _int, _int, _d, _i8, _d]
    lib.orc_dequantize.restype = None
    lib.orc_dequantize.argtypes = [_int, _int, _i8, _d, _d]
    lib.orc_pack_int4.restype = None
    lib.orc_pack_int4.argtypes = [_int, _i8, _u8]
    lib.orc_unpack_int4.restype = None
    lib.orc_unpack_int4.argtypes = [_int, _u8, _i8]
    lib.orc_select_columns.restype = _int
    lib.orc_select_columns.argtypes = [_int, _int, _d, _i32]
    lib.orc_plain_run.restype = None
    lib.orc_plain_run.argtypes = [_int] * 5 + [_vp] * 8
    lib.orc_o1_run.restype = _int
    lib.orc_o1_run.argtypes = [_int] * 9 + [_vp] * 8
    lib.orc_o2_run.restype = _int
    lib.orc_o2_run.argtypes = [_int] * 11 + [_vp] * 22
    lib.orc_round_other.restype = ctypes.c_double
    lib.orc_round_other.argtypes = [_int, ctypes.c_double]
    lib.orc_smooth_exponent.restype = _int
    lib.orc_smooth_exponent.argtypes = [ctypes.c_double]
    lib.orc_window_end.restype = _int
    lib.orc_window_end.argtypes = [_int] * 6 + [_vp] * 7
    lib.orc_round_e4m3.restype = ctypes.c_double
    lib.orc_round_e4m3.argtypes = [ctypes.c_double]
    lib.orc_fp8_vector.restype = ctypes.c_double
    lib.orc_fp8_vector.argtypes = [_int, _int, _d, _d]
    lib.orc_pw_run.restype = _int
    lib.orc_pw_run.argtypes = [_int] * 9 + [_vp] * 12
    if path == _build.OUT:
        _lib, _lib_path = lib, path
    return lib


def num_threads(lib=None) -> int:
    return (lib or load()).orc_num_threads()


def _p(a):
    return None if a is None else a.ctypes.data_as(_vp)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------------------------
# Roundings and the quantizer
# ---------------------------------------------------------------------------------------------
def round_bf16(x: float, lib=None) -> float:
    return (lib or load()).orc_round_bf16(float(x))


def round_other(x: float, mode: str = "bf16", lib=None) -> float:
    """The neighbour of x in the storage format on the other side from its rounding."""
    return (lib or load()).orc_round_other(_ROUND[mode], float(x))


def round_bf16_array(a: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    flat = np.asarray(a, dtype=np.float64).ravel()
    return np.array([lib.orc_round_bf16(float(x)) for x in flat]).reshape(np.shape(a))


def quantize(S: np.ndarray, fmt: str = "int8", prec32: bool = False, lib=None):
    """S [D][D] -> (codes int8 [D][D], scales f64 [D][groups])."""
    lib = lib or load()
    S = _f64(S)
    D = S.shape[0]
    f = _FMT[fmt]
    ng = lib.orc_num_groups(f, D)
    codes = np.zeros((D, D), np.int8)
    scales = np.zeros((D, ng), np.float64)
    if lib.orc_quantize(D, f, int(prec32), S, codes, scales) != 0:
        raise ValueError(f"bad format {fmt}")
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, fmt: str = "int8", lib=None) -> np.ndarray:
    lib = lib or load()
    D = codes.shape[0]
    out = np.zeros((D, D), np.float64)
    lib.orc_dequantize(D, _FMT[fmt], np.ascontiguousarray(codes, np.int8), _f64(scales), out)
    return out


def pack_int4(codes: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    D = codes.shape[0]
    out = np.zeros((D, D // 2), np.uint8)
    lib.orc_pack_int4(D, np.ascontiguousarray(codes, np.int8), out)
    return out


def unpack_int4(packed: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    D = packed.shape[0]
    out = np.zeros((D, D), np.int8)
    lib.orc_unpack_int4(D, np.ascontiguousarray(packed, np.uint8), out)
    return out


def select_columns(S: np.ndarray, r: int, lib=None):
    """Compensator choice: (column indices in pick order, near-tie flag)."""
    lib = lib or load()
    S = _f64(S)
    idx = np.zeros(max(r, 1), np.int32)
    near = lib.orc_select_columns(S.shape[0], r, S, idx)
    return idx[:r].copy(), bool(near)


# ---------------------------------------------------------------------------------------------
# The three formulations
# ---------------------------------------------------------------------------------------------
def smooth_exponent(colmax: float, lib=None) -> int:
    """e = floor(floor(log2 colmax) / 2) clamped to [-63, 63]; 0 for a zero column."""
    return (lib or load()).orc_smooth_exponent(float(colmax))


@dataclass
class WindowEnd:
    residual: np.ndarray   # [D][D] the rescaled residual that was quantized
    codes: np.ndarray      # [D][D] int8
    scales: np.ndarray     # [D][groups]
    cidx: np.ndarray       # [r] column rule's columns (-1 for the power rule)
    cu: np.ndarray         # [r][D] compensator token values
    ck: np.ndarray         # [r][D] compensator token keys (e_j for the column rule)
    sexp: np.ndarray       # [D] int8 smoothing exponents
    near_tie: int


def window_end(S: np.ndarray, fmt: str = "int8", r: int = 0, smooth: bool = False,
               prec32: bool = False, comp_rule: str = "columns", lib=None) -> WindowEnd:
    """The window-end operation on one [D][D] state: compensator tokens out (``comp_rule``
    "columns" or "power"), residual smoothing, quantization. The state it leaves is
    dequant(codes, scales) Diag(2^sexp) plus sum_c cu_c ck_c^T."""
    lib = lib or load()
    R = _f64(S).copy()
    D = R.shape[0]
    f = _FMT[fmt]
    ng = lib.orc_num_groups(FMT_INT8 if f == FMT_NONE else f, D)
    out = WindowEnd(R, np.zeros((D, D), np.int8), np.zeros((D, ng)), np.zeros(max(r, 1), np.int32),
                    np.zeros((max(r, 1), D)), np.zeros((max(r, 1), D)), np.zeros(D, np.int8), 0)
    out.near_tie = lib.orc_window_end(D, f, r, int(prec32), int(smooth), COMP_RULES[comp_rule],
                                      _p(R), _p(out.codes), _p(out.scales), _p(out.cidx),
                                      _p(out.cu), _p(out.ck), _p(out.sexp))
    out.cidx, out.cu, out.ck = out.cidx[:r], out.cu[:r], out.ck[:r]
    return out


def _gate(g, T, nh, D):
    g = _f64(g)
    if g.ndim == 2:
        return g.reshape(T, nh, 1), 1
    return g.reshape(T, nh, D), D


def plain_run(q, k, v, g, beta, S0=None, state_round: str = "none", want_o: bool = True, lib=None):
    """fp64 recurrence. Returns (o [T][nh][D] or None, S_T [nh][D][D])."""
    lib = lib or load()
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    T, nh, D = k.shape
    g, Dg = _gate(g, T, nh, D)
    S0 = _f64(S0)
    o = np.zeros((T, nh, D)) if want_o else None
    S = np.zeros((nh, D, D))
    lib.orc_plain_run(D, T, nh, Dg, _ROUND[state_round], _p(S0), _p(q), _p(k), _p(v), _p(g),
                      _p(beta), _p(o), _p(S))
    return o, S


def o1_run(q, k, v, g, beta, W: int, r: int = 0, fmt: str = "int8", S0=None,
           smooth: bool = False, comp_rule: str = "columns", lib=None):
    """Literal matrix-form recurrence with window-end requantisation (fp64 decisions; ``smooth``
    adds the residual smoothing). Returns (o, S_T, near_ties)."""
    lib = lib or load()
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    T, nh, D = k.shape
    g, Dg = _gate(g, T, nh, D)
    S0 = _f64(S0)
    o = np.zeros((T, nh, D))
    S = np.zeros((nh, D, D))
    ties = lib.orc_o1_run(D, T, W, r, _FMT[fmt], nh, Dg, int(smooth), COMP_RULES[comp_rule],
                          _p(S0), _p(q), _p(k),
                          _p(v), _p(g), _p(beta), _p(o), _p(S))
    return o, S, ties


@dataclass
class O2Result:
    o: np.ndarray          # [T][nh][D] fp64, unrounded
    codes: np.ndarray      # [nh][D][D] int8 (int4 codes unpacked, in [-7, 7])
    scales: np.ndarray     # [nh][D][groups]
    cidx: np.ndarray       # [nh][r]
    cu: np.ndarray         # [nh][r][D]
    ck: np.ndarray         # [nh][r][D] compensator keys
    pos: np.ndarray        # [nh]
    bk: np.ndarray         # [nh][W][D]
    bu: np.ndarray         # [nh][W][D]
    bL: np.ndarray         # [nh][W][D]
    S: np.ndarray          # [nh][D][D] logical state at the end
    near_ties: int
    ties: np.ndarray       # [nh] near ties per head
    sexp: np.ndarray       # [nh][D] int8 smoothing exponents (zeros without smoothing)
    u_raw: Optional[np.ndarray] = None  # [T][nh][D] write vectors before storage rounding


def o2_run(q, k, v, g, beta, W: int, r: int = 0, fmt: str = "int8", S0=None,
           round_storage: bool = False, buf_round: str = "bf16", flush_mask=None,
           smooth: bool = False, want_u_raw: bool = False, u_flip=None,
           comp_rule: str = "columns", lib=None) -> O2Result:
    """Buffered-window form. ``round_storage`` mirrors GPU storage (fp32 state / L / scales,
    ``buf_round`` write vectors, fp32 quantizer decisions); ``smooth`` adds the residual
    smoothing at every quantization. ``want_u_raw`` returns every write vector before its
    storage rounding; ``u_flip`` ([T][nh][D], nonzero entries) stores those write-vector entries
    rounded to the other neighbour (an alternative result for entries on a rounding midpoint)."""
    lib = lib or load()
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    T, nh, D = k.shape
    g, Dg = _gate(g, T, nh, D)
    S0 = _f64(S0)
    f = _FMT[fmt]
    ng = lib.orc_num_groups(FMT_INT8 if f == FMT_NONE else f, D)
    res = O2Result(
        o=np.zeros((T, nh, D)), codes=np.zeros((nh, D, D), np.int8),
        scales=np.zeros((nh, D, ng)), cidx=np.zeros((nh, max(r, 0)), np.int32),
        cu=np.zeros((nh, max(r, 0), D)), ck=np.zeros((nh, max(r, 0), D)),
        pos=np.zeros(nh, np.int32),
        bk=np.zeros((nh, W, D)), bu=np.zeros((nh, W, D)), bL=np.zeros((nh, W, D)),
        S=np.zeros((nh, D, D)), near_ties=0, ties=np.zeros(nh, np.int32),
        sexp=np.zeros((nh, D), np.int8))
    fm = None if flush_mask is None else np.ascontiguousarray(flush_mask, np.uint8).reshape(T, nh)
    if want_u_raw:
        res.u_raw = np.zeros((T, nh, D))
    uf = None if u_flip is None else np.ascontiguousarray(u_flip, np.uint8).reshape(T, nh, D)
    res.near_ties = lib.orc_o2_run(
        D, T, W, r, f, nh, Dg, int(round_storage), _ROUND[buf_round], int(smooth),
        COMP_RULES[comp_rule], _p(S0),
        _p(q), _p(k), _p(v), _p(g), _p(beta), _p(fm), _p(res.o), _p(res.codes), _p(res.scales),
        _p(res.cidx) if r > 0 else None, _p(res.cu) if r > 0 else None,
        _p(res.ck) if r > 0 else None, _p(res.pos),
        _p(res.bk), _p(res.bu), _p(res.bL), _p(res.S), _p(res.ties), _p(res.sexp),
        _p(res.u_raw), _p(uf))
    return res


# ---------------------------------------------------------------------------------------------
# PW: the pure-write sliding window
# ---------------------------------------------------------------------------------------------
def round_e4m3(x: float, lib=None) -> float:
    return (lib or load()).orc_round_e4m3(float(x))


def fp8_vector(x: np.ndarray, prec32: bool = False, lib=None):
    """FP8 round trip of a vector with one scale. Returns (values, scale)."""
    lib = lib or load()
    x = _f64(x).ravel()
    out = np.zeros_like(x)
    s = lib.orc_fp8_vector(x.size, int(prec32), x, out)
    return out, s


@dataclass
class PWResult:
    o: np.ndarray          # [T][nh][D] fp64, before storage rounding
    codes: np.ndarray      # [nh][D][D] int8 history codes (int4 unpacked, in [-7, 7])
    scales: np.ndarray     # [nh][D][groups]
    px: np.ndarray         # [nh][Wp][D] pair value vectors as stored, by ring slot
    py: np.ndarray         # [nh][Wp][D] pair key vectors as stored, by ring slot
    S: np.ndarray          # [nh][D][D] logical state: history + the pairs in the window


def pw_run(q, k, v, g, beta, Wp: int, fmt: str = "int8", S0=None, quant: bool = True,
           fp8: bool = True, prec32: bool = False, lib=None) -> PWResult:
    """Pure-write sliding window of Wp FP8 pairs over a low-bit history (``quant``; else an
    exact history). ``prec32`` mirrors GPU storage and single-precision decisions."""
    lib = lib or load()
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    T, nh, D = k.shape
    g, Dg = _gate(g, T, nh, D)
    S0 = _f64(S0)
    f = _FMT[fmt]
    ng = lib.orc_num_groups(FMT_INT4 if f == FMT_INT4 else FMT_INT8, D)
    res = PWResult(o=np.zeros((T, nh, D)), codes=np.zeros((nh, D, D), np.int8),
                   scales=np.zeros((nh, D, ng)), px=np.zeros((nh, Wp, D)),
                   py=np.zeros((nh, Wp, D)), S=np.zeros((nh, D, D)))
    rc = lib.orc_pw_run(D, T, Wp, f, nh, Dg, int(quant), int(fp8), int(prec32), _p(S0), _p(q),
                        _p(k), _p(v), _p(g), _p(beta), _p(res.o), _p(res.codes),
                        _p(res.scales), _p(res.px), _p(res.py), _p(res.S))
    if rc != 0:
        raise ValueError("pw_run: bad window length or history format")
    return res
