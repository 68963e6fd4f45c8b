// Window kernels instantiated for int8 codes with per-row scales.
#include "window_dispatch.cuh"

namespace gdnq {

cudaError_t launch_window_int8(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                               cudaStream_t st) {
  switch (cfg.d_k) {
    case 16: return launch_window_gate<16, false>(op, cfg, a, heads, st);
    case 128: return launch_window_gate<128, false>(op, cfg, a, heads, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace gdnq
