"""Argument marshalling for the chunkwise prefill entry point (include/gdnq_prefill.h): torch
tensors -> pointers, status codes -> exceptions. Same conventions as ``api``."""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from .api import _check, _ptr, _stream


def gdn_prefill_workspace_bytes(cfg, L: int) -> int:
    return int(_abi.load().gdn_prefill_workspace_bytes(ctypes.byref(cfg), L))


def gdn_prefill(cfg, q, k, v, g, beta, o, S, workspace=None, stream=None):
    """q, k, v, o bf16 [B][H][L][D]; beta fp32 [B][H][L]; g fp32 [B][H][L] (scalar gate) or
    [B][H][L][D] (per-key-channel gate); S fp32 [B][H][D][D] (in place). workspace: a uint8
    device tensor of at least gdn_prefill_workspace_bytes(cfg, L) bytes, made here when None."""
    L = q.shape[2] if q.dim() == 4 else 0
    nh, D = cfg.B * cfg.H, cfg.d_k
    n = nh * L * D
    ng = n if cfg.gate == _abi.GDN_GATE_DIAG else nh * L
    need = gdn_prefill_workspace_bytes(cfg, L)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=S.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_abi.load().gdn_prefill(
        ctypes.byref(cfg), L, _ptr(q, "q", torch.bfloat16, n), _ptr(k, "k", torch.bfloat16, n),
        _ptr(v, "v", torch.bfloat16, n), _ptr(g, "g", torch.float32, ng),
        _ptr(beta, "beta", torch.float32, nh * L), _ptr(o, "o", torch.bfloat16, n),
        _ptr(S, "S", torch.float32, nh * D * D), _ptr(workspace, "workspace"), ws_bytes,
        _stream(stream)), "gdn_prefill")
