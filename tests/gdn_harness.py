"""Test harness: runs a workload through the CUDA library and through the CPU oracle on the
same seeded inputs, and compares the two.

GPU side: the initial state is the fp32 recurrence over the workload's warm-up tokens, run by the
library's fp32-state baseline kernel; then initial quantization and T windowed decode steps.
Oracle side: the same warm-up tokens through the oracle's plain recurrence (fp32 state storage),
then the buffered-window form with GPU storage roundings (fp32 state / gates / scales, write
vectors in the buffer dtype, single-precision quantizer decisions). Both sides make their own
initial state; nothing the GPU computed is handed to the oracle.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import bit_recurrent_state_gdn_b200 as gdn
import oracle
from workloads import Workload, decode_inputs, outlier_scales, step_inputs, torch_dtype


def cfg_of(wl: Workload):
    return gdn.make_config(wl.B, wl.H, wl.D, wl.W, wl.r, wl.gate, wl.fmt, wl.act, wl.buf,
                           smooth=wl.smooth, comp_rule=wl.comp_rule)


def gpu_warmup(wl: Workload, device="cuda", draw=None) -> torch.Tensor:
    """fp32 [B][H][D][D] initial states from the library's fp32-state baseline kernel. The
    warm-up inputs are drawn on ``draw`` (default: ``device``) and copied to ``device``; the
    oracle's initial state must be drawn on the same device (the generators differ)."""
    draw = draw or device
    S = torch.zeros((wl.B, wl.H, wl.D, wl.D), dtype=torch.float32, device=device)
    if wl.warmup == 0:
        return S
    cfg = gdn.make_config(wl.B, wl.H, wl.D, gate=wl.gate, fmt="fp32", act=wl.act)
    scales = outlier_scales(wl, draw)
    o = torch.empty((wl.B, wl.H, wl.D), dtype=torch_dtype(wl.act), device=device)
    for t in range(wl.warmup):
        s = step_inputs(wl, "warmup", t, draw, scales)
        q, k, v, g, beta = (x.to(device) for x in (s.q, s.k, s.v, s.g, s.beta))
        gdn.gdn_baseline_step(cfg, S, q, k, v, g, beta, o)
    return S


def _heads_np(x: torch.Tensor, heads: np.ndarray) -> np.ndarray:
    """[T][B][H](...) device tensor -> [T][n](...) float64 numpy for the flat head indices."""
    T, nh = x.shape[0], x.shape[1] * x.shape[2]
    flat = x.reshape(T, nh, *x.shape[3:])
    idx = torch.as_tensor(heads, device=x.device, dtype=torch.long)
    return flat.index_select(1, idx).double().cpu().numpy()


def warmup_inputs_np(wl: Workload, heads: np.ndarray, device="cuda") -> dict:
    scales = outlier_scales(wl, device)
    idx = torch.as_tensor(heads, device=device, dtype=torch.long)
    acc = {n: [] for n in ("q", "k", "v", "g", "beta")}
    for t in range(wl.warmup):
        s = step_inputs(wl, "warmup", t, device, scales)
        for n in acc:
            x = getattr(s, n)
            flat = x.reshape(-1, *x.shape[2:]) if x.dim() > 2 else x.reshape(-1)
            acc[n].append(flat.index_select(0, idx).double().cpu().numpy())
    return {n: np.stack(v) if v else np.zeros((0,)) for n, v in acc.items()}


def oracle_initial_state(wl: Workload, heads: np.ndarray, device="cuda") -> np.ndarray:
    n = len(heads)
    if wl.warmup == 0:
        return np.zeros((n, wl.D, wl.D))
    w = warmup_inputs_np(wl, heads, device)
    _, S = oracle.plain_run(w["q"], w["k"], w["v"], w["g"], w["beta"], state_round="f32",
                            want_o=False)
    return S


@dataclass
class GpuRun:
    o: torch.Tensor            # [T][B][H][D] act dtype
    state: gdn.GdnState
    S0: torch.Tensor           # fp32 initial states
    inputs: dict


def gpu_run(wl: Workload, device="cuda", T: int | None = None, inputs=None, S0=None) -> GpuRun:
    cfg = cfg_of(wl)
    T = wl.T if T is None else T
    if inputs is None:
        inputs = decode_inputs(wl, device, T)
    if S0 is None:
        S0 = gpu_warmup(wl, device)
    state = gdn.GdnState.allocate(cfg, device)
    gdn.gdn_state_quantize(cfg, S0, state)
    o = torch.empty_like(inputs["q"])
    if T > 0:
        gdn.gdn_decode_window_steps(cfg, state, inputs["q"], inputs["k"], inputs["v"],
                                    inputs["g"], inputs["beta"], o)
    torch.cuda.synchronize()
    return GpuRun(o, state, S0, inputs)


def _o2(wl: Workload, q, k, v, g, beta, S0, flush_mask, **kw):
    return oracle.o2_run(q, k, v, g, beta, W=wl.W, r=wl.r, fmt=wl.fmt, S0=S0,
                         round_storage=True, buf_round=wl.buf, flush_mask=flush_mask,
                         smooth=wl.smooth, comp_rule=wl.comp_rule, **kw)


def oracle_run(wl: Workload, heads: np.ndarray, inputs: dict, S0: np.ndarray, flush_mask=None):
    q, k, v, g, beta = (_heads_np(inputs[n], heads) for n in ("q", "k", "v", "g", "beta"))
    res = _o2(wl, q, k, v, g, beta, S0, flush_mask)
    # what a re-run of single heads needs (loose scale rows are explained by re-running)
    fm = None if flush_mask is None else np.asarray(flush_mask).reshape(q.shape[0], -1)
    res.rerun = (q, k, v, g, beta, np.asarray(S0), fm)
    return res


# ---------------------------------------------------------------------------------------------
# Reading the GPU state back per head
# ---------------------------------------------------------------------------------------------
def unswizzle(tiles: np.ndarray) -> np.ndarray:
    """[n][rows][RB] bytes of swizzled tiles -> row-major bytes. Chunk c (16 bytes) of row i is
    stored at chunk c ^ x(i): x(i) = i & 7 for rows of 128 bytes or more, else
    (i * RB / 128) & (RB / 16 - 1) (the layout include/gdnq.h documents)."""
    n, rows, RB = tiles.shape
    nch = RB // 16
    i = np.arange(rows)
    x = (i & 7) if RB >= 128 else ((i * RB // 128) & (nch - 1))
    src = np.arange(nch)[None, :] ^ x[:, None]             # [rows][nch] physical chunk
    t = tiles.reshape(n, rows, nch, 16)
    return np.take_along_axis(t, src[None, :, :, None], axis=2).reshape(n, rows, RB)


def gpu_codes(wl: Workload, st: gdn.GdnState, heads: np.ndarray) -> np.ndarray:
    """Unpacked int8 codes [n][D][D] of the chosen heads, in row-major order."""
    D = wl.D
    h = torch.as_tensor(heads, device=st.codes.device)
    if wl.fmt == "int4_g32":
        packed = unswizzle(st.codes.view(-1, D, D // 2)[h].cpu().numpy())
        return np.stack([oracle.unpack_int4(p) for p in packed])
    return unswizzle(st.codes.view(-1, D, D)[h].cpu().numpy()).view(np.int8)


def gpu_scales(wl: Workload, st: gdn.GdnState, heads: np.ndarray) -> np.ndarray:
    ng = wl.D // 32 if wl.fmt == "int4_g32" else 1
    return st.scales.view(-1, wl.D, ng)[torch.as_tensor(heads, device=st.scales.device)] \
        .double().cpu().numpy()


def gpu_comps(wl: Workload, st: gdn.GdnState, heads: np.ndarray):
    rp = (wl.r + 3) // 4 * 4
    h = torch.as_tensor(heads, device=st.pos.device)
    cidx = st.comp_idx.view(-1, rp)[h][:, : wl.r].cpu().numpy()
    cu = st.comp_u.view(-1, wl.r, wl.D)[h].double().cpu().numpy()
    return cidx, cu


def round_act(x: np.ndarray, act: str) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch_dtype(act)).double().numpy()


def rel_l2(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------------------------------------
# Acceptance bars (output rel-L2 2e-3; codes equal but for 1-LSB flips on <= 0.1% of entries;
# scales and compensators to fp32 rounding; near-tie compensator heads reported apart)
# ---------------------------------------------------------------------------------------------
O_TOL = 2e-3
FLIP_FRAC = 1e-3
# Scales: the largest scale error measured over every parity case is about 1e-5 of the row's
# largest scale (the fp32 materialisation sums up to W + r terms in another order than the
# oracle), so a 1e-5 bar would sit at the measured edge; 1e-4 keeps a 10x margin. Compensator
# columns are single fp32 entries of the materialised state: measured <= 1.5e-7 rel-L2, bar 1e-5.
SCALE_TOL = 1e-4
COMP_TOL = 1e-5
# Both sides round each buffered write u to the buffer dtype from their own w (fp64 in the
# oracle, fp32 on the GPU). A u whose unrounded value lies within the GPU's fp32 noise of a
# rounding midpoint may land on either neighbour, and the later values of its state row follow
# (a valid alternative result, like a 1-LSB code flip). A row whose scale misses SCALE_TOL is
# accepted only when it is explained: some step's unrounded oracle u of that row lies within
# U_MIDPOINT_NOISE quanta of a midpoint, and the oracle re-run with that one entry rounded to
# its other neighbour reproduces the GPU's scale row within SCALE_TOL. Explained rows stay
# within one bf16 ulp (SCALE_TOL_ROUNDING) and on at most FLIP_FRAC of the compared rows.
SCALE_TOL_ROUNDING = 2.0 ** -8
U_MIDPOINT_NOISE = 2.0 ** -8   # distance to a midpoint, in quanta of the buffer format
EXPLAIN_CANDIDATES = 8         # the closest candidate entries tried per loose row


def _midpoint_distance(u: np.ndarray, buf: str) -> np.ndarray:
    """|u / q - (floor(u / q) + 1/2)|: distance of u to the midpoint between its two storage
    neighbours, in quanta q of u's binade (bf16: 2^(e-8), fp32: 2^(e-24))."""
    bits = 8 if buf == "bf16" else 24
    _, e = np.frexp(u)
    q = np.ldexp(1.0, e - bits)
    f = u / q
    d = np.abs(f - np.floor(f) - 0.5)
    return np.where(u == 0, 1.0, d)


def explain_loose_row(wl: Workload, res, a: int, v: int, gpu_row: np.ndarray) -> bool:
    """Whether the GPU's scale row ``gpu_row`` of compared head ``a`` (index into the compared
    heads), state row ``v``, is the oracle's alternative result of one write-vector entry of
    that row rounded to its other neighbour (see U_MIDPOINT_NOISE)."""
    q, k, vv, g, beta, S0, fm = res.rerun
    one = slice(a, a + 1)
    args = (q[:, one], k[:, one], vv[:, one], g[:, one], beta[:, one], S0[one],
            None if fm is None else np.ascontiguousarray(fm[:, one]))
    base = _o2(wl, *args, want_u_raw=True)
    u = base.u_raw[:, 0, v]
    d = _midpoint_distance(u, wl.buf)
    cands = [t for t in np.argsort(d, kind="stable")[:EXPLAIN_CANDIDATES]
             if d[t] <= U_MIDPOINT_NOISE]
    T = q.shape[0]
    for t in cands:
        flip = np.zeros((T, 1, wl.D), np.uint8)
        flip[t, 0, v] = 1
        alt = _o2(wl, *args, u_flip=flip)
        ref = alt.scales[0, v]
        den = max(float(np.abs(ref).max()), 1e-30)
        if float(np.abs(gpu_row - ref).max()) / den <= SCALE_TOL:
            return True
    return False


@dataclass
class Parity:
    o_rel: float
    o_rel_unrounded: float
    flip_frac: float
    max_code_diff: int
    scale_rel: float
    scale_loose_rows: int
    scale_unexplained: int
    scale_rows: int
    comp_rel: float
    tie_heads: int
    n_heads: int
    pos_equal: bool

    def check(self):
        assert self.o_rel <= O_TOL, self
        assert self.max_code_diff <= 1, self
        assert self.flip_frac <= FLIP_FRAC, self
        assert self.scale_rel <= SCALE_TOL_ROUNDING, self
        assert self.scale_loose_rows <= max(1, int(FLIP_FRAC * self.scale_rows)), self
        assert self.scale_unexplained == 0, self
        assert self.comp_rel <= COMP_TOL, self
        assert self.tie_heads <= max(1, int(FLIP_FRAC * self.n_heads)), self
        assert self.pos_equal, self


def compare(wl: Workload, run: GpuRun, heads: np.ndarray, res) -> Parity:
    T = run.o.shape[0]
    o_gpu = _heads_np(run.o, heads) if T else np.zeros((0, len(heads), wl.D))
    o_ref = round_act(res.o, wl.act)
    ok = res.ties == 0
    codes = gpu_codes(wl, run.state, heads)
    diff = np.abs(codes[ok].astype(int) - res.codes[ok].astype(int))
    sc = gpu_scales(wl, run.state, heads)
    # A scale is absmax / qmax of fp32-materialised entries whose rounding error scales with the
    # magnitude of the row's terms (u_i[v] k_i[j] products, the row's codes), not with the
    # group's own absmax: a small int4 group next to large ones in the same row carries the
    # row's absolute error. Scale errors are therefore measured against the row's largest
    # scale (for int8, one scale per row, this is the plain relative error).
    ref = res.scales[ok].reshape(-1, wl.D, sc.shape[-1] if sc.ndim == 3 else 1)
    row_max = np.maximum(np.abs(ref).max(axis=-1, keepdims=True), 1e-30)
    srel = (np.abs(sc[ok].reshape(ref.shape) - ref) / row_max).reshape(res.scales[ok].shape)
    crel = 0.0
    if wl.r > 0:
        cidx, cu = gpu_comps(wl, run.state, heads)
        assert np.array_equal(cidx[ok], res.cidx[ok]), "compensator columns differ"
        crel = rel_l2(cu[ok], res.cu[ok]) if ok.any() else 0.0
    pos = run.state.pos[torch.as_tensor(heads, device=run.state.pos.device)].cpu().numpy()
    if wl.smooth:  # smoothing exponents are integer decisions: equal away from near ties
        sexp = run.state.smooth_exp[: wl.heads * wl.D].view(-1, wl.D)[
            torch.as_tensor(heads, device=run.state.pos.device)].cpu().numpy()
        assert np.array_equal(sexp[ok], res.sexp[ok]), "smoothing exponents differ"
    # a flipped code changes that row's scale only when the flip is the absmax entry; scales are
    # compared where every code of the row agrees
    rows_same = (diff.reshape(diff.shape[0], wl.D, -1).max(axis=-1) == 0) if diff.size else diff
    srel_cmp = srel.reshape(srel.shape[0], wl.D, -1)
    unexplained = 0
    if np.any(rows_same):
        loose = rows_same & (srel_cmp.max(axis=-1) > SCALE_TOL)
        ok_idx = np.flatnonzero(ok)
        sc_ok = sc[ok].reshape(-1, wl.D, ref.shape[-1])
        for ai, v in zip(*np.nonzero(loose)):
            if not explain_loose_row(wl, res, int(ok_idx[ai]), int(v), sc_ok[ai, v]):
                unexplained += 1
    return Parity(
        o_rel=rel_l2(o_gpu, o_ref), o_rel_unrounded=rel_l2(o_gpu, res.o),
        flip_frac=float((diff > 0).mean()) if diff.size else 0.0,
        max_code_diff=int(diff.max()) if diff.size else 0,
        scale_rel=float(srel_cmp[rows_same].max()) if np.any(rows_same) else 0.0,
        scale_loose_rows=int((srel_cmp[rows_same].max(axis=-1) > SCALE_TOL).sum())
        if np.any(rows_same) else 0,
        scale_unexplained=unexplained,
        scale_rows=int(np.sum(rows_same)),
        comp_rel=crel, tie_heads=int((~ok).sum()), n_heads=len(heads),
        pos_equal=bool(np.array_equal(pos, res.pos)))


def sample_heads(wl: Workload, n: int, seed: int = 0) -> np.ndarray:
    """Every head of the first and the last sequence, plus random others (sorted, unique)."""
    H, Bh = wl.H, wl.heads
    first = np.arange(min(H, Bh))
    last = np.arange(max(Bh - H, 0), Bh)
    rng = np.random.default_rng(seed)
    extra = rng.choice(Bh, size=min(max(n - len(first) - len(last), 0), Bh), replace=False)
    return np.unique(np.concatenate([first, last, extra])).astype(np.int64)
