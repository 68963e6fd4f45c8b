"""Seeded input generators (no arithmetic of the method itself).

Recipe, per (sequence, head) and step:
  q, k ~ N(0, 1)^D, each scaled to unit L2 norm; v ~ N(0, 1)^D;
  beta = sigmoid(N(0, 1)); log-gate g = -softplus(N(0, 1)) (one per head for the scalar gate,
  one per key channel for the diagonal gate);
  with outliers: round(0.02 * D) key channels and as many value channels per head, fixed for the
  whole run, are multiplied by 20 -- keys before the L2 normalisation.
q, k, v are stored in the workload's activation dtype; g and beta in fp32.

Every step has its own generator seeded from (workload seed, phase, step), so any step can be
made on its own and on either device; draws on CPU and on CUDA differ, so a parity check makes
the inputs once and hands the same bytes to both sides.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.nn.functional as F

from .configs import Workload

_PHASE = {"warmup": 1, "decode": 2, "outliers": 3}
OUTLIER_FACTOR = 20.0
OUTLIER_FRACTION = 0.02


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _generator(device, seed: int, phase: str, t: int) -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed((seed * 1_000_003 + _PHASE[phase] * 7_919 + t) & 0x7FFF_FFFF_FFFF_FFFF)
    return gen


def n_outlier_channels(D: int) -> int:
    return int(round(OUTLIER_FRACTION * D))


def outlier_scales(wl: Workload, device="cpu"):
    """(key_scale, value_scale), each fp32 [B][H][D] with entries 1 or 20 (all 1 if the workload
    has no outliers)."""
    shape = (wl.B, wl.H, wl.D)
    ks = torch.ones(shape, dtype=torch.float32, device=device)
    vs = torch.ones(shape, dtype=torch.float32, device=device)
    n = n_outlier_channels(wl.D)
    if not wl.outliers or n == 0 or wl.heads == 0:
        return ks, vs
    gen = _generator(device, wl.seed, "outliers", 0)
    kidx = torch.rand(shape, generator=gen, device=device).argsort(dim=-1)[..., :n]
    vidx = torch.rand(shape, generator=gen, device=device).argsort(dim=-1)[..., :n]
    ks.scatter_(-1, kidx, OUTLIER_FACTOR)
    vs.scatter_(-1, vidx, OUTLIER_FACTOR)
    return ks, vs


@dataclass
class StepInputs:
    q: torch.Tensor      # [B][H][D] act dtype
    k: torch.Tensor      # [B][H][D] act dtype
    v: torch.Tensor      # [B][H][D] act dtype
    g: torch.Tensor      # [B][H] or [B][H][D] fp32, log of the gate
    beta: torch.Tensor   # [B][H] fp32


def step_inputs(wl: Workload, phase: str, t: int, device="cpu", scales=None) -> StepInputs:
    """Inputs of step ``t`` of ``phase`` ("warmup" or "decode"). ``scales`` is the result of
    ``outlier_scales`` (made once per run and passed in to save work)."""
    B, H, D = wl.B, wl.H, wl.D
    if scales is None:
        scales = outlier_scales(wl, device)
    ks, vs = scales
    gen = _generator(device, wl.seed, phase, t)
    q = torch.randn((B, H, D), generator=gen, device=device)
    k = torch.randn((B, H, D), generator=gen, device=device) * ks
    v = torch.randn((B, H, D), generator=gen, device=device) * vs
    q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    beta = torch.sigmoid(torch.randn((B, H), generator=gen, device=device))
    gshape = (B, H) if wl.gate == "scalar" else (B, H, D)
    g = -F.softplus(torch.randn(gshape, generator=gen, device=device))
    act = torch_dtype(wl.act)
    return StepInputs(q.to(act), k.to(act), v.to(act), g.float().contiguous(),
                      beta.float().contiguous())


def decode_inputs(wl: Workload, device="cpu", T: int | None = None, phase: str = "decode"):
    """All ``T`` steps stacked: dict of q, k, v [T][B][H][D], g [T][B][H](/[D]), beta [T][B][H]."""
    T = wl.T if T is None else T
    scales = outlier_scales(wl, device)
    act = torch_dtype(wl.act)
    B, H, D = wl.B, wl.H, wl.D
    gshape = (T, B, H) if wl.gate == "scalar" else (T, B, H, D)
    out = {
        "q": torch.empty((T, B, H, D), dtype=act, device=device),
        "k": torch.empty((T, B, H, D), dtype=act, device=device),
        "v": torch.empty((T, B, H, D), dtype=act, device=device),
        "g": torch.empty(gshape, dtype=torch.float32, device=device),
        "beta": torch.empty((T, B, H), dtype=torch.float32, device=device),
    }
    for t in range(T):
        s = step_inputs(wl, phase, t, device, scales)
        out["q"][t], out["k"][t], out["v"][t] = s.q, s.k, s.v
        out["g"][t], out["beta"][t] = s.g, s.beta
    return out
