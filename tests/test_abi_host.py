"""The C ABI on the host: the library loads, exports every symbol include/*.h declares, sizes
its buffers, and rejects bad arguments before touching a device. Every call here fails argument
checks (or is an empty batch), so no kernel is launched and no pointer is dereferenced."""
import ctypes
import glob
import os
import re

import pytest

import bit_recurrent_state_gdn_b200 as gdn
from bit_recurrent_state_gdn_b200 import _abi, build
from workloads import WORKLOADS

HEADERS = sorted(glob.glob(os.path.join(os.path.dirname(build.PKG), "include", "*.h")))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(gdn_[a-z_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported_and_bound(lib):
    assert len(HEADERS) >= 2
    names = declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
        assert n in _abi.SIGNATURES, f"{n} not bound in the Python layer"
    assert set(_abi.SIGNATURES) == set(names)


def test_status_strings(lib):
    assert lib.gdn_status_string(0) == b"GDN_OK"
    assert lib.gdn_status_string(1) == b"GDN_ERR_INVALID_ARG"
    assert lib.gdn_status_string(2) == b"GDN_ERR_UNSUPPORTED"
    assert lib.gdn_status_string(3) == b"GDN_ERR_CUDA"
    assert lib.gdn_status_string(4) == b"GDN_ERR_TIMEOUT"
    assert lib.gdn_status_string(99) == b"GDN_UNKNOWN_STATUS"


def _cfg(**kw):
    base = dict(B=2, H=3, D=128, W=64, r=0, gate="scalar", fmt="int8", act="bf16", buf="bf16")
    base.update(kw)
    return gdn.make_config(**base)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_state_sizes_of_the_workloads(name, lib):
    wl = WORKLOADS[name]
    cfg = gdn.make_config(wl.B, wl.H, wl.D, wl.W, wl.r, wl.gate, wl.fmt, wl.act, wl.buf)
    s = gdn.gdn_state_sizes(cfg)
    n, D, W = wl.heads, wl.D, wl.W
    act = 4 if wl.act == "f32" else 2
    buf = 4 if wl.buf == "f32" else 2
    if wl.fmt == "int8":
        assert s.codes == n * D * D and s.scales == n * D * 4
    else:
        assert s.codes == n * D * D // 2 and s.scales == n * D * (D // 32) * 4
    assert s.buf_k == n * W * D * act and s.buf_u == n * W * D * buf
    assert s.buf_L == n * 4 * (W * D if wl.gate == "diag" else (W + 3) // 4 * 4)
    assert s.comp_idx == (n * 4 * ((wl.r + 3) // 4 * 4) if wl.r else 0)
    assert s.comp_u == n * wl.r * D * 4
    assert s.pos == n * 4
    assert 0 < s.smem_step <= 227 * 1024


BAD_CONFIGS = [
    ("W=0", dict(W=0), _abi.GDN_ERR_INVALID_ARG),
    ("r<0", dict(r=-1), _abi.GDN_ERR_INVALID_ARG),
    ("r>d", dict(D=16, r=17), _abi.GDN_ERR_INVALID_ARG),
    ("r>max", dict(r=17), _abi.GDN_ERR_UNSUPPORTED),
    ("D=64", dict(D=64), _abi.GDN_ERR_UNSUPPORTED),
    ("int4 D=16", dict(D=16, fmt="int4_g32"), _abi.GDN_ERR_UNSUPPORTED),
    ("baseline fmt", dict(fmt="bf16"), _abi.GDN_ERR_INVALID_ARG),
    ("window too big", dict(W=5000), _abi.GDN_ERR_UNSUPPORTED),
    ("B<0", dict(B=-1), _abi.GDN_ERR_INVALID_ARG),
    ("smoothing of a mixed state", dict(fmt="mixed", smooth=True), _abi.GDN_ERR_UNSUPPORTED),
    ("power tokens with smoothing", dict(r=4, comp_rule="power", smooth=True),
     _abi.GDN_ERR_UNSUPPORTED),
    ("power tokens, W = 65", dict(r=4, comp_rule="power", W=65), _abi.GDN_ERR_UNSUPPORTED),
    ("power tokens, D = 16", dict(D=16, r=2, comp_rule="power"), _abi.GDN_ERR_UNSUPPORTED),
    ("power tokens, fp32 buffers", dict(r=2, comp_rule="power", buf="f32"),
     _abi.GDN_ERR_UNSUPPORTED),
    ("power tokens, mixed widths", dict(r=2, comp_rule="power", fmt="mixed"),
     _abi.GDN_ERR_UNSUPPORTED),
]


@pytest.mark.parametrize("name,kw,want", BAD_CONFIGS, ids=[c[0] for c in BAD_CONFIGS])
def test_bad_config_rejected(name, kw, want, lib):
    cfg = _cfg(**kw)
    out = _abi.gdn_sizes()
    assert lib.gdn_state_sizes(ctypes.byref(cfg), ctypes.byref(out)) == want
    assert lib.gdn_last_error() != b""
    st = _abi.gdn_state()
    assert lib.gdn_decode_window_step(ctypes.byref(cfg), ctypes.byref(st), *[None] * 7) == want


def test_raw_field_errors(lib):
    out = _abi.gdn_sizes()
    assert lib.gdn_state_sizes(None, ctypes.byref(out)) == _abi.GDN_ERR_INVALID_ARG
    cfg = _cfg()
    assert lib.gdn_state_sizes(ctypes.byref(cfg), None) == _abi.GDN_ERR_INVALID_ARG
    for field, val in (("gate", 7), ("fmt", 9), ("act_dtype", 3), ("buf_dtype", -1),
                       ("smooth", 2), ("smooth", -1), ("comp_rule", 2), ("comp_rule", -1)):
        c = _cfg()
        setattr(c, field, val)
        assert lib.gdn_state_sizes(ctypes.byref(c), ctypes.byref(out)) == _abi.GDN_ERR_INVALID_ARG
    c = _cfg()
    c.d_v = 64
    assert lib.gdn_state_sizes(ctypes.byref(c), ctypes.byref(out)) == _abi.GDN_ERR_UNSUPPORTED


def _fake_state(misalign=None, null=None):
    vals = {n: 0x10000 * (i + 1) for i, n in enumerate(_abi.STATE_FIELDS)}
    vals["status"] = 0
    if misalign:
        vals[misalign] += 8
    if null:
        vals[null] = 0
    return _abi.gdn_state(**vals)


@pytest.mark.parametrize("field", ["codes", "scales", "buf_k", "buf_u", "buf_L", "pos"])
def test_state_pointer_checks(field, lib):
    cfg = _cfg()
    q = ctypes.c_void_p(0x900000)
    for st in (_fake_state(null=field), _fake_state(misalign=field)):
        rc = lib.gdn_decode_window_step(ctypes.byref(cfg), ctypes.byref(st), q, q, q, q, q, q, None)
        assert rc == _abi.GDN_ERR_INVALID_ARG
        assert field.encode() in lib.gdn_last_error()


@pytest.mark.parametrize("fmt", ["int8", "int4_g32"])
def test_smoothing_sizes_and_exponent_pointer(fmt, lib):
    """A smoothed state has D exponent bytes per head; its pointer is required (16-byte
    aligned) only when smoothing is on, and checked before anything is enqueued."""
    cfg = _cfg(fmt=fmt, smooth=True)
    assert gdn.gdn_state_sizes(cfg).smooth_exp == 6 * 128
    assert gdn.gdn_state_sizes(_cfg(fmt=fmt)).smooth_exp == 0
    q = ctypes.c_void_p(0x900000)
    for st in (_fake_state(null="smooth_exp"), _fake_state(misalign="smooth_exp")):
        rc = lib.gdn_decode_window_step(ctypes.byref(cfg), ctypes.byref(st), q, q, q, q, q, q, None)
        assert rc == _abi.GDN_ERR_INVALID_ARG
        assert b"smooth_exp" in lib.gdn_last_error()


def test_power_token_keys_sized_and_required(lib):
    """Power tokens keep r keys of D floats per head next to the values; the key pointer is
    required (16-byte aligned) only for the power rule with r > 0."""
    cfg = _cfg(r=4, comp_rule="power")
    sz = gdn.gdn_state_sizes(cfg)
    assert sz.comp_k == 6 * 4 * 128 * 4 and sz.comp_u == sz.comp_k
    assert gdn.gdn_state_sizes(_cfg(r=4)).comp_k == 0
    assert gdn.gdn_state_sizes(_cfg(r=0, comp_rule="power")).comp_k == 0
    q = ctypes.c_void_p(0x900000)
    for st in (_fake_state(null="comp_k"), _fake_state(misalign="comp_k")):
        rc = lib.gdn_decode_window_step(ctypes.byref(cfg), ctypes.byref(st), q, q, q, q, q, q, None)
        assert rc == _abi.GDN_ERR_INVALID_ARG
        assert b"comp_k" in lib.gdn_last_error()


def test_compensator_pointers_needed_only_with_r(lib):
    st = _fake_state(null="comp_u")
    cfg = _cfg(r=4)
    rc = lib.gdn_window_flush(ctypes.byref(cfg), ctypes.byref(st), None, None)
    assert rc == _abi.GDN_ERR_INVALID_ARG and b"comp_u" in lib.gdn_last_error()


def test_input_pointer_checks(lib):
    cfg = _cfg()
    st = _fake_state()
    good = ctypes.c_void_p(0x900000)
    odd = ctypes.c_void_p(0x900008)       # bulk-copied q must be 16-byte aligned
    args = [good] * 6
    for i in range(6):
        a = list(args)
        a[i] = None
        assert lib.gdn_decode_window_step(ctypes.byref(cfg), ctypes.byref(st), *a, None) \
            == _abi.GDN_ERR_INVALID_ARG
    a = list(args)
    a[0] = odd
    assert lib.gdn_decode_window_step(ctypes.byref(cfg), ctypes.byref(st), *a, None) \
        == _abi.GDN_ERR_INVALID_ARG
    assert lib.gdn_decode_window_steps(ctypes.byref(cfg), ctypes.byref(st), -1, *args, None) \
        == _abi.GDN_ERR_INVALID_ARG


def test_host_pipeline_checks(lib):
    cfg = _cfg()
    st = _fake_state()
    need = lib.gdn_host_staging_bytes(ctypes.byref(cfg))
    assert need > 0
    h = ctypes.c_void_p(0x900000)
    rc = lib.gdn_decode_window_steps_host(ctypes.byref(cfg), ctypes.byref(st), 3, h, h, h, h, h, h,
                                          ctypes.c_void_p(0x800000), need - 1, None)
    assert rc == _abi.GDN_ERR_INVALID_ARG and b"staging" in lib.gdn_last_error()
    bad = _cfg(W=0)
    assert lib.gdn_host_staging_bytes(ctypes.byref(bad)) == 0


def test_empty_batch_needs_no_buffers(lib):
    cfg = _cfg(B=0)
    st = _abi.gdn_state()
    assert lib.gdn_decode_window_step(ctypes.byref(cfg), ctypes.byref(st), *[None] * 7) == 0
    assert lib.gdn_state_quantize(ctypes.byref(cfg), None, ctypes.byref(st), None) == 0
    assert lib.gdn_window_flush(ctypes.byref(cfg), ctypes.byref(st), None, None) == 0
    assert lib.gdn_state_materialize(ctypes.byref(cfg), ctypes.byref(st), None, None) == 0
    base = _cfg(B=0, fmt="fp32")
    assert lib.gdn_baseline_step(ctypes.byref(base), *[None] * 8) == 0


def test_baseline_format_checks(lib):
    cfg = _cfg(fmt="int8")
    assert lib.gdn_baseline_step(ctypes.byref(cfg), *[None] * 8) == _abi.GDN_ERR_INVALID_ARG
    cfg = _cfg(fmt="fp32")
    s = ctypes.c_void_p(0x900008)         # state array must be 16-byte aligned
    g = ctypes.c_void_p(0x900000)
    assert lib.gdn_baseline_step(ctypes.byref(cfg), s, g, g, g, g, g, g, None) \
        == _abi.GDN_ERR_INVALID_ARG


def test_python_layer_raises_with_detail(lib):
    with pytest.raises(gdn.GdnError, match="GDN_ERR_UNSUPPORTED.*head size"):
        gdn.gdn_state_sizes(_cfg(D=64))


# ---- pure-write sliding window ----------------------------------------------------------------
def _pw(**kw):
    base = dict(B=2, H=3, D=128, Wp=8, gate="scalar", fmt="int4_g32", act="bf16")
    base.update(kw)
    return gdn.make_pw_config(**base)


@pytest.mark.parametrize("fmt,Wp", [("int8", 8), ("int4_g32", 8), ("int4_g32", 0), ("int8", 5)])
def test_pw_state_sizes(fmt, Wp, lib):
    cfg = _pw(fmt=fmt, Wp=Wp)
    s = gdn.gdn_pw_state_sizes(cfg)
    n, D = 6, 128
    if fmt == "int8":
        assert s.codes == n * D * D and s.scales == n * D * 4
    else:
        assert s.codes == n * D * D // 2 and s.scales == n * D * 4 * 4
    assert s.pairs == n * 2 * Wp * D
    assert s.pscales == (n * 8 * ((Wp + 3) // 4 * 4) if Wp else 0)
    assert s.count == n * 4


PW_BAD = [
    ("Wp<0", dict(Wp=-1), _abi.GDN_ERR_INVALID_ARG),
    ("Wp>max", dict(Wp=17), _abi.GDN_ERR_UNSUPPORTED),
    ("D=64", dict(D=64), _abi.GDN_ERR_UNSUPPORTED),
    ("fmt mixed", dict(fmt="mixed"), _abi.GDN_ERR_INVALID_ARG),
    ("fmt fp32", dict(fmt="fp32"), _abi.GDN_ERR_INVALID_ARG),
    ("B<0", dict(B=-1), _abi.GDN_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("name,kw,status", PW_BAD, ids=[b[0] for b in PW_BAD])
def test_pw_bad_configs(name, kw, status, lib):
    out = _abi.gdn_pw_sizes()
    assert lib.gdn_pw_state_sizes(ctypes.byref(_pw(**kw)), ctypes.byref(out)) == status
    assert lib.gdn_last_error() != b""


def test_pw_calls_reject_missing_buffers(lib):
    cfg = _pw()
    st = _abi.gdn_pw_state()  # all null
    assert lib.gdn_pw_quantize(ctypes.byref(cfg), None, ctypes.byref(st), None) == \
        _abi.GDN_ERR_INVALID_ARG
    assert lib.gdn_pw_decode_steps(ctypes.byref(cfg), ctypes.byref(st), 1, *([None] * 7)) == \
        _abi.GDN_ERR_INVALID_ARG
    assert lib.gdn_pw_materialize(ctypes.byref(cfg), ctypes.byref(st), None, None) == \
        _abi.GDN_ERR_INVALID_ARG
    assert lib.gdn_pw_decode_steps(ctypes.byref(cfg), ctypes.byref(st), -1, *([None] * 7)) == \
        _abi.GDN_ERR_INVALID_ARG


def test_pw_empty_batch_and_zero_steps_are_noops(lib):
    st = _abi.gdn_pw_state()
    empty = _pw(B=0)
    assert lib.gdn_pw_quantize(ctypes.byref(empty), None, ctypes.byref(st), None) == _abi.GDN_OK
    assert lib.gdn_pw_decode_steps(ctypes.byref(empty), ctypes.byref(st), 3, *([None] * 7)) == \
        _abi.GDN_OK
    assert lib.gdn_pw_decode_steps(ctypes.byref(_pw()), ctypes.byref(st), 0, *([None] * 7)) == \
        _abi.GDN_OK


# ---- chunkwise prefill ------------------------------------------------------------------------
PF_BAD = [
    ("diag gate, null buffers", dict(gate="diag"), 8, _abi.GDN_ERR_INVALID_ARG),
    ("fp32 activations", dict(act="f32"), 8, _abi.GDN_ERR_UNSUPPORTED),
    ("D=16", dict(D=16), 8, _abi.GDN_ERR_UNSUPPORTED),
    ("L<0", dict(), -1, _abi.GDN_ERR_INVALID_ARG),
    ("null buffers", dict(), 8, _abi.GDN_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("name,kw,L,status", PF_BAD, ids=[b[0] for b in PF_BAD])
def test_prefill_rejects_bad_arguments(name, kw, L, status, lib):
    cfg = _cfg(**kw)
    assert lib.gdn_prefill(ctypes.byref(cfg), L, *([None] * 8), 0, None) == status
    assert lib.gdn_last_error() != b""


def test_prefill_diag_gate_wants_16_byte_aligned_gates(lib):
    """The per-channel gate rows are copied 16 bytes at a time: an 8-byte aligned g is refused
    before anything is enqueued (the other pointers are aligned placeholders, never touched)."""
    p = ctypes.c_void_p(1 << 20)
    args = [p, p, p, ctypes.c_void_p((1 << 20) + 8), p, p, p]
    cfg = _cfg(gate="diag")
    assert lib.gdn_prefill(ctypes.byref(cfg), 8, *args, None, 0, None) == _abi.GDN_ERR_INVALID_ARG
    assert b"g is not 16-byte aligned" in lib.gdn_last_error()


def test_prefill_workspace_size_and_checks(lib):
    """The scalar gate needs one 33,792-byte record per 64-token chunk of every head; the
    per-channel gate none. A missing, misaligned or short workspace is refused before anything
    is enqueued."""
    cfg = _cfg(B=2, H=3)
    assert lib.gdn_prefill_workspace_bytes(ctypes.byref(cfg), 200) == 6 * 4 * 33792
    assert lib.gdn_prefill_workspace_bytes(ctypes.byref(cfg), 0) == 0
    assert lib.gdn_prefill_workspace_bytes(ctypes.byref(_cfg(gate="diag")), 200) == 0
    assert lib.gdn_prefill_workspace_bytes(ctypes.byref(_cfg(D=16)), 200) == 0
    p = ctypes.c_void_p(1 << 20)
    args = [p] * 7
    need = 6 * 4 * 33792
    for ws, size, msg in ((None, need, b"workspace is null"),
                          (ctypes.c_void_p((1 << 20) + 8), need, b"workspace is not"),
                          (p, need - 16, b"workspace holds")):
        rc = lib.gdn_prefill(ctypes.byref(cfg), 200, *args, ws, size, None)
        assert rc == _abi.GDN_ERR_INVALID_ARG
        assert msg in lib.gdn_last_error(), lib.gdn_last_error()


def test_prefill_empty_batch_is_a_noop(lib):
    assert lib.gdn_prefill(ctypes.byref(_cfg(B=0)), 100, *([None] * 8), 0, None) == _abi.GDN_OK
