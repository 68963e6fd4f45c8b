"""Argument marshalling for the pure-write sliding window entry points (include/gdnq_pw.h):
torch tensors -> pointers, status codes -> exceptions. Same conventions as ``api``."""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, fields

import torch

from . import _abi
from .api import _DT, _FMT, _GATE, _TORCH_DT, _check, _ptr, _stream


def make_pw_config(B: int, H: int, D: int = 128, Wp: int = 8, gate: str = "scalar",
                   fmt: str = "int4_g32", act: str = "bf16") -> _abi.gdn_pw_config:
    return _abi.gdn_pw_config(B, H, D, Wp, _GATE[gate], _FMT[fmt], _DT[act])


def gdn_pw_state_sizes(cfg: _abi.gdn_pw_config) -> _abi.gdn_pw_sizes:
    out = _abi.gdn_pw_sizes()
    _check(_abi.load().gdn_pw_state_sizes(ctypes.byref(cfg), ctypes.byref(out)),
           "gdn_pw_state_sizes")
    return out


@dataclass
class PwState:
    """Caller-owned device buffers of a pure-write window state (layouts in gdnq_pw.h)."""
    codes: torch.Tensor
    scales: torch.Tensor
    pairs: torch.Tensor
    pscales: torch.Tensor
    count: torch.Tensor
    status: torch.Tensor

    @staticmethod
    def allocate(cfg: _abi.gdn_pw_config, device="cuda") -> "PwState":
        sz = gdn_pw_state_sizes(cfg)
        dev = torch.device(device)

        def buf(nbytes, dtype):
            n = max(nbytes // torch.empty((), dtype=dtype).element_size(), 1)
            return torch.zeros(n, dtype=dtype, device=dev)

        return PwState(codes=buf(sz.codes, torch.uint8), scales=buf(sz.scales, torch.float32),
                       pairs=buf(sz.pairs, torch.uint8), pscales=buf(sz.pscales, torch.float32),
                       count=buf(sz.count, torch.int32),
                       status=torch.zeros(4, dtype=torch.int32, device=dev))

    def c_struct(self) -> _abi.gdn_pw_state:
        return _abi.gdn_pw_state(*[getattr(self, n).data_ptr() for n in _abi.PW_STATE_FIELDS])

    def tensors(self) -> dict:
        return {f.name: getattr(self, f.name) for f in fields(self)}

    def clone(self) -> "PwState":
        return PwState(**{n: t.clone() for n, t in self.tensors().items()})


def _heads(cfg):
    return cfg.B * cfg.H


def _gate_numel(cfg):
    return _heads(cfg) * (cfg.d if cfg.gate == _abi.GDN_GATE_DIAG else 1)


def gdn_pw_quantize(cfg, S: torch.Tensor, state: PwState, stream=None):
    st = state.c_struct()
    _check(_abi.load().gdn_pw_quantize(
        ctypes.byref(cfg), _ptr(S, "S", torch.float32, _heads(cfg) * cfg.d * cfg.d),
        ctypes.byref(st), _stream(stream)), "gdn_pw_quantize")


def gdn_pw_decode_step(cfg, state: PwState, q, k, v, g, beta, o, stream=None):
    n, act = _heads(cfg) * cfg.d, _TORCH_DT[cfg.act_dtype]
    st = state.c_struct()
    _check(_abi.load().gdn_pw_decode_step(
        ctypes.byref(cfg), ctypes.byref(st), _ptr(q, "q", act, n), _ptr(k, "k", act, n),
        _ptr(v, "v", act, n), _ptr(g, "g", torch.float32, _gate_numel(cfg)),
        _ptr(beta, "beta", torch.float32, _heads(cfg)), _ptr(o, "o", act, n), _stream(stream)),
        "gdn_pw_decode_step")


def gdn_pw_decode_steps(cfg, state: PwState, q, k, v, g, beta, o, stream=None):
    """q, k, v, o [T][B][H][D]; g [T][B][H](/[D]); beta [T][B][H]."""
    T = q.shape[0]
    n, act = T * _heads(cfg) * cfg.d, _TORCH_DT[cfg.act_dtype]
    st = state.c_struct()
    _check(_abi.load().gdn_pw_decode_steps(
        ctypes.byref(cfg), ctypes.byref(st), T, _ptr(q, "q", act, n), _ptr(k, "k", act, n),
        _ptr(v, "v", act, n), _ptr(g, "g", torch.float32, T * _gate_numel(cfg)),
        _ptr(beta, "beta", torch.float32, T * _heads(cfg)), _ptr(o, "o", act, n),
        _stream(stream)), "gdn_pw_decode_steps")


def gdn_pw_materialize(cfg, state: PwState, S: torch.Tensor, stream=None):
    st = state.c_struct()
    _check(_abi.load().gdn_pw_materialize(
        ctypes.byref(cfg), ctypes.byref(st),
        _ptr(S, "S", torch.float32, _heads(cfg) * cfg.d * cfg.d), _stream(stream)),
        "gdn_pw_materialize")
