"""Argument marshalling for libgdnq: torch tensors -> pointers, status codes -> exceptions.

Shapes follow include/gdnq.h. Each function checks that the tensors it is given are contiguous,
on the right device, of the right dtype and size (the C ABI only sees pointers), then calls the
C entry point of the same name on the current CUDA stream (or ``stream``).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, fields
from typing import Optional

import torch

from . import _abi

_DT = {"f32": _abi.GDN_DTYPE_F32, "bf16": _abi.GDN_DTYPE_BF16}
_TORCH_DT = {_abi.GDN_DTYPE_F32: torch.float32, _abi.GDN_DTYPE_BF16: torch.bfloat16}
_FMT = {"int8": _abi.GDN_FMT_INT8, "int4_g32": _abi.GDN_FMT_INT4_G32, "bf16": _abi.GDN_FMT_BF16,
        "fp32": _abi.GDN_FMT_FP32, "mixed": _abi.GDN_FMT_MIXED}
_GATE = {"scalar": _abi.GDN_GATE_SCALAR, "diag": _abi.GDN_GATE_DIAG}


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _abi.load()
        self.status = status
        name = lib.gdn_status_string(status).decode()
        detail = lib.gdn_last_error().decode()
        super().__init__(f"{where}: {name}: {detail}")


_COMP = {"columns": 0, "power": 1}


def make_config(B: int, H: int, D: int, W: int = 1, r: int = 0, gate: str = "scalar",
                fmt: str = "int8", act: str = "bf16", buf: str = "bf16",
                smooth: bool = False, comp_rule: str = "columns") -> _abi.gdn_config:
    """smooth: residual smoothing (per-key-column power-of-two factors) at every quantization.
    comp_rule: "columns" or "power" compensator tokens."""
    return _abi.gdn_config(B, H, D, D, W, r, _GATE[gate], _FMT[fmt], _DT[act], _DT[buf],
                           _abi.GDN_SMOOTH_POW2_COLUMNS if smooth else _abi.GDN_SMOOTH_NONE,
                           _COMP[comp_rule])


def _check(status: int, where: str):
    if status != _abi.GDN_OK:
        raise GdnError(status, where)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream if isinstance(stream, int) else stream.cuda_stream


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, numel=None, device=None):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return t.data_ptr() or None


def gdn_state_sizes(cfg: _abi.gdn_config) -> _abi.gdn_sizes:
    out = _abi.gdn_sizes()
    _check(_abi.load().gdn_state_sizes(ctypes.byref(cfg), ctypes.byref(out)), "gdn_state_sizes")
    return out


def gdn_host_staging_bytes(cfg: _abi.gdn_config) -> int:
    return int(_abi.load().gdn_host_staging_bytes(ctypes.byref(cfg)))


@dataclass
class GdnState:
    """Caller-owned device buffers of a windowed low-bit state (layouts in include/gdnq.h)."""
    codes: torch.Tensor
    scales: torch.Tensor
    buf_k: torch.Tensor
    buf_u: torch.Tensor
    buf_L: torch.Tensor
    comp_idx: torch.Tensor
    comp_u: torch.Tensor
    pos: torch.Tensor
    status: torch.Tensor
    head_fmt: torch.Tensor  # int8 [B*H]: each head's format (mixed-format states only)
    smooth_exp: torch.Tensor  # int8 [B*H*D]: smoothing exponents (smoothed states only)
    comp_k: torch.Tensor  # fp32 [B*H*r*D]: compensator token keys (power rule only)

    @staticmethod
    def allocate(cfg: _abi.gdn_config, device="cuda", head_fmt=None) -> "GdnState":
        """Zeroed buffers for cfg. head_fmt (mixed states): one format name ("int8" /
        "int4_g32") or gdn_state_format value per head, in [B][H] order."""
        sz = gdn_state_sizes(cfg)
        dev = torch.device(device)

        def buf(nbytes, dtype):
            n = max(nbytes // torch.empty((), dtype=dtype).element_size(), 1)
            return torch.zeros(n, dtype=dtype, device=dev)

        return GdnState(
            codes=buf(sz.codes, torch.uint8), scales=buf(sz.scales, torch.float32),
            buf_k=buf(sz.buf_k, torch.uint8), buf_u=buf(sz.buf_u, torch.uint8),
            buf_L=buf(sz.buf_L, torch.float32), comp_idx=buf(sz.comp_idx, torch.int32),
            comp_u=buf(sz.comp_u, torch.float32), pos=buf(sz.pos, torch.int32),
            status=torch.zeros(4, dtype=torch.int32, device=dev),
            head_fmt=_head_fmt(cfg, head_fmt, sz.head_fmt, dev),
            smooth_exp=torch.zeros(max(sz.smooth_exp, 16), dtype=torch.int8, device=dev),
            comp_k=torch.zeros(max(sz.comp_k // 4, 4), dtype=torch.float32, device=dev))

    def c_struct(self) -> _abi.gdn_state:
        return _abi.gdn_state(*[getattr(self, n).data_ptr() for n in _abi.STATE_FIELDS])

    def tensors(self) -> dict:
        return {f.name: getattr(self, f.name) for f in fields(self)}

    def clone(self) -> "GdnState":
        return GdnState(**{n: t.clone() for n, t in self.tensors().items()})

    def copy_(self, other: "GdnState") -> "GdnState":
        for n, t in self.tensors().items():
            t.copy_(getattr(other, n))
        return self


def _head_fmt(cfg, head_fmt, nbytes, dev) -> torch.Tensor:
    if cfg.fmt != _abi.GDN_FMT_MIXED:
        return torch.zeros(1, dtype=torch.int8, device=dev)
    if head_fmt is None or len(head_fmt) != nbytes:
        raise ValueError(f"a mixed-format state needs head_fmt with {nbytes} entries")
    vals = [_FMT[f] if isinstance(f, str) else int(f) for f in head_fmt]
    if any(v not in (_abi.GDN_FMT_INT8, _abi.GDN_FMT_INT4_G32) for v in vals):
        raise ValueError("head_fmt entries must be int8 or int4_g32")
    return torch.tensor(vals, dtype=torch.int8, device=dev)


def _heads(cfg):
    return cfg.B * cfg.H


def _act(cfg):
    return _TORCH_DT[cfg.act_dtype]


def _gate_numel(cfg):
    return _heads(cfg) * (cfg.d_k if cfg.gate == _abi.GDN_GATE_DIAG else 1)


def gdn_state_quantize(cfg, S: torch.Tensor, state: GdnState, stream=None):
    n = _heads(cfg) * cfg.d_k * cfg.d_v
    st = state.c_struct()
    _check(_abi.load().gdn_state_quantize(ctypes.byref(cfg), _ptr(S, "S", torch.float32, n),
                                          ctypes.byref(st), _stream(stream)),
           "gdn_state_quantize")


def gdn_decode_window_step(cfg, state: GdnState, q, k, v, g, beta, o, stream=None):
    n, act = _heads(cfg) * cfg.d_v, _act(cfg)
    st = state.c_struct()
    _check(_abi.load().gdn_decode_window_step(
        ctypes.byref(cfg), ctypes.byref(st), _ptr(q, "q", act, n), _ptr(k, "k", act, n),
        _ptr(v, "v", act, n), _ptr(g, "g", torch.float32, _gate_numel(cfg)),
        _ptr(beta, "beta", torch.float32, _heads(cfg)), _ptr(o, "o", act, n), _stream(stream)),
        "gdn_decode_window_step")


def gdn_decode_window_steps(cfg, state: GdnState, q, k, v, g, beta, o, stream=None):
    """q, k, v, o [T][B][H][D]; g [T][B][H](/[D]); beta [T][B][H]."""
    T = q.shape[0]
    n, act = T * _heads(cfg) * cfg.d_v, _act(cfg)
    st = state.c_struct()
    _check(_abi.load().gdn_decode_window_steps(
        ctypes.byref(cfg), ctypes.byref(st), T, _ptr(q, "q", act, n), _ptr(k, "k", act, n),
        _ptr(v, "v", act, n), _ptr(g, "g", torch.float32, T * _gate_numel(cfg)),
        _ptr(beta, "beta", torch.float32, T * _heads(cfg)), _ptr(o, "o", act, n),
        _stream(stream)), "gdn_decode_window_steps")


def gdn_decode_window_steps_host(cfg, state: GdnState, q, k, v, g, beta, o,
                                 staging: torch.Tensor, stream=None):
    """Host (pinned CPU) tensors q, k, v, o [T][B][H][D], g, beta; device ``staging`` of at
    least gdn_host_staging_bytes(cfg) bytes."""
    T = q.shape[0]
    n, act, cpu = T * _heads(cfg) * cfg.d_v, _act(cfg), torch.device("cpu")
    st = state.c_struct()
    _check(_abi.load().gdn_decode_window_steps_host(
        ctypes.byref(cfg), ctypes.byref(st), T, _ptr(q, "q", act, n, cpu),
        _ptr(k, "k", act, n, cpu), _ptr(v, "v", act, n, cpu),
        _ptr(g, "g", torch.float32, T * _gate_numel(cfg), cpu),
        _ptr(beta, "beta", torch.float32, T * _heads(cfg), cpu), _ptr(o, "o", act, n, cpu),
        _ptr(staging, "staging"), staging.numel() * staging.element_size(), _stream(stream)),
        "gdn_decode_window_steps_host")


def gdn_decode_window_steps_host_fixed(cfg, state: GdnState, q, k, v, g, beta, o, stream=None):
    """As gdn_decode_window_steps_host, staging through the library's fixed device array
    (no staging argument; the call allocates nothing)."""
    T = q.shape[0]
    n, act, cpu = T * _heads(cfg) * cfg.d_v, _act(cfg), torch.device("cpu")
    st = state.c_struct()
    _check(_abi.load().gdn_decode_window_steps_host_fixed(
        ctypes.byref(cfg), ctypes.byref(st), T, _ptr(q, "q", act, n, cpu),
        _ptr(k, "k", act, n, cpu), _ptr(v, "v", act, n, cpu),
        _ptr(g, "g", torch.float32, T * _gate_numel(cfg), cpu),
        _ptr(beta, "beta", torch.float32, T * _heads(cfg), cpu), _ptr(o, "o", act, n, cpu),
        _stream(stream)), "gdn_decode_window_steps_host_fixed")


def gdn_window_flush(cfg, state: GdnState, seq_mask: Optional[torch.Tensor] = None, stream=None):
    st = state.c_struct()
    _check(_abi.load().gdn_window_flush(
        ctypes.byref(cfg), ctypes.byref(st), _ptr(seq_mask, "seq_mask", torch.int32, cfg.B),
        _stream(stream)), "gdn_window_flush")


def gdn_state_materialize(cfg, state: GdnState, S: torch.Tensor, stream=None):
    n = _heads(cfg) * cfg.d_k * cfg.d_v
    st = state.c_struct()
    _check(_abi.load().gdn_state_materialize(ctypes.byref(cfg), ctypes.byref(st),
                                             _ptr(S, "S", torch.float32, n), _stream(stream)),
           "gdn_state_materialize")


def gdn_baseline_step(cfg, S: torch.Tensor, q, k, v, g, beta, o, stream=None):
    n, act = _heads(cfg) * cfg.d_v, _act(cfg)
    sdt = torch.float32 if cfg.fmt == _abi.GDN_FMT_FP32 else torch.bfloat16
    _check(_abi.load().gdn_baseline_step(
        ctypes.byref(cfg), _ptr(S, "S", sdt, n * cfg.d_k), _ptr(q, "q", act, n),
        _ptr(k, "k", act, n), _ptr(v, "v", act, n),
        _ptr(g, "g", torch.float32, _gate_numel(cfg)),
        _ptr(beta, "beta", torch.float32, _heads(cfg)), _ptr(o, "o", act, n), _stream(stream)),
        "gdn_baseline_step")
