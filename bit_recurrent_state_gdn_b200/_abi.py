"""ctypes declarations of libgdnq's C ABI (include/gdnq.h, gdnq_pw.h, gdnq_prefill.h). Loading fails loudly when the
library has not been built: there is no fallback path."""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdnq.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT = range(5)
GDN_DEVICE_WAIT_TIMEOUT, GDN_DEVICE_BAD_POS = 0x1, 0x2
GDN_GATE_SCALAR, GDN_GATE_DIAG = 0, 1
GDN_SMOOTH_NONE, GDN_SMOOTH_POW2_COLUMNS = 0, 1
GDN_FMT_INT8, GDN_FMT_INT4_G32, GDN_FMT_BF16, GDN_FMT_FP32, GDN_FMT_MIXED = 0, 1, 2, 3, 4
GDN_DTYPE_F32, GDN_DTYPE_BF16 = 0, 1
GDN_MAX_COMPENSATORS = 16
GDN_PW_MAX_WINDOW = 16

_i32 = ctypes.c_int32
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t


class gdn_config(ctypes.Structure):
    _fields_ = [(n, _i32) for n in
                ("B", "H", "d_k", "d_v", "W", "r", "gate", "fmt", "act_dtype", "buf_dtype",
                 "smooth", "comp_rule")]


STATE_FIELDS = ("codes", "scales", "buf_k", "buf_u", "buf_L", "comp_idx", "comp_u", "pos",
                "status", "head_fmt", "smooth_exp", "comp_k")


class gdn_state(ctypes.Structure):
    _fields_ = [(n, _vp) for n in STATE_FIELDS]


SIZE_FIELDS = ("codes", "scales", "buf_k", "buf_u", "buf_L", "comp_idx", "comp_u", "pos",
               "smem_step", "head_fmt", "smooth_exp", "comp_k")


class gdn_sizes(ctypes.Structure):
    _fields_ = [(n, _sz) for n in SIZE_FIELDS]


class gdn_pw_config(ctypes.Structure):
    _fields_ = [(n, _i32) for n in ("B", "H", "d", "Wp", "gate", "fmt", "act_dtype")]


PW_STATE_FIELDS = ("codes", "scales", "pairs", "pscales", "count", "status")


class gdn_pw_state(ctypes.Structure):
    _fields_ = [(n, _vp) for n in PW_STATE_FIELDS]


PW_SIZE_FIELDS = ("codes", "scales", "pairs", "pscales", "count")


class gdn_pw_sizes(ctypes.Structure):
    _fields_ = [(n, _sz) for n in PW_SIZE_FIELDS]


_PWC, _PWS = ctypes.POINTER(gdn_pw_config), ctypes.POINTER(gdn_pw_state)

# name -> (restype, argtypes); every symbol the headers under include/ declare
SIGNATURES = {
    "gdn_state_sizes": (_i32, [ctypes.POINTER(gdn_config), ctypes.POINTER(gdn_sizes)]),
    "gdn_state_quantize": (_i32, [ctypes.POINTER(gdn_config), _vp, ctypes.POINTER(gdn_state), _vp]),
    "gdn_decode_window_step": (_i32, [ctypes.POINTER(gdn_config), ctypes.POINTER(gdn_state)]
                               + [_vp] * 7),
    "gdn_decode_window_steps": (_i32, [ctypes.POINTER(gdn_config), ctypes.POINTER(gdn_state), _i32]
                                + [_vp] * 7),
    "gdn_host_staging_bytes": (_sz, [ctypes.POINTER(gdn_config)]),
    "gdn_decode_window_steps_host": (_i32, [ctypes.POINTER(gdn_config), ctypes.POINTER(gdn_state),
                                            _i32] + [_vp] * 7 + [_sz, _vp]),
    "gdn_decode_window_steps_host_fixed": (_i32, [ctypes.POINTER(gdn_config),
                                                  ctypes.POINTER(gdn_state), _i32] + [_vp] * 7),
    "gdn_window_flush": (_i32, [ctypes.POINTER(gdn_config), ctypes.POINTER(gdn_state), _vp, _vp]),
    "gdn_state_materialize": (_i32, [ctypes.POINTER(gdn_config), ctypes.POINTER(gdn_state), _vp,
                                     _vp]),
    "gdn_baseline_step": (_i32, [ctypes.POINTER(gdn_config)] + [_vp] * 8),
    "gdn_pw_state_sizes": (_i32, [_PWC, ctypes.POINTER(gdn_pw_sizes)]),
    "gdn_pw_quantize": (_i32, [_PWC, _vp, _PWS, _vp]),
    "gdn_pw_decode_step": (_i32, [_PWC, _PWS] + [_vp] * 7),
    "gdn_pw_decode_steps": (_i32, [_PWC, _PWS, _i32] + [_vp] * 7),
    "gdn_pw_materialize": (_i32, [_PWC, _PWS, _vp, _vp]),
    "gdn_prefill": (_i32, [ctypes.POINTER(gdn_config), _i32] + [_vp] * 8 + [_sz, _vp]),
    "gdn_prefill_workspace_bytes": (_sz, [ctypes.POINTER(gdn_config), _i32]),
    "gdn_status_string": (ctypes.c_char_p, [_i32]),
    "gdn_last_error": (ctypes.c_char_p, []),
}

_lib = None


def load(path: str = LIB_PATH):
    """The loaded library (cached). Raises if it has not been built."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build the CUDA library first "
            "(python -m bit_recurrent_state_gdn_b200.build)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib
