"""Windowed low-bit recurrent-state GDN / KDA decode for B200 (sm_100a).

Python face of libgdnq (include/gdnq.h, gdnq_pw.h, gdnq_prefill.h): the functions here carry the C ABI's names and only
marshal arguments -- torch tensors to device pointers, the current CUDA stream, status codes to
exceptions. Every step of the computation runs in the library's CUDA kernels.
"""
from .api import (  # noqa: F401
    GdnError,
    GdnState,
    gdn_baseline_step,
    gdn_decode_window_step,
    gdn_decode_window_steps,
    gdn_decode_window_steps_host,
    gdn_decode_window_steps_host_fixed,
    gdn_host_staging_bytes,
    gdn_state_materialize,
    gdn_state_quantize,
    gdn_state_sizes,
    gdn_window_flush,
    make_config,
)
from .pw import (  # noqa: F401
    PwState,
    gdn_pw_decode_step,
    gdn_pw_decode_steps,
    gdn_pw_materialize,
    gdn_pw_quantize,
    gdn_pw_state_sizes,
    make_pw_config,
)
from .prefill import gdn_prefill, gdn_prefill_workspace_bytes  # noqa: F401,E402
