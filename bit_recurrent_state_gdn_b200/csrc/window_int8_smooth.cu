// Window kernels instantiated for int8 codes with per-row scales and residual smoothing.
#include "window_dispatch.cuh"

namespace gdnq {

cudaError_t launch_window_int8_smooth(WinOp op, const gdn_config& cfg, const WinArgs& a,
                                      int heads, cudaStream_t st) {
  switch (cfg.d_k) {
    case 16: return launch_window_gate<16, false, false, true>(op, cfg, a, heads, st);
    case 128: return launch_window_gate<128, false, false, true>(op, cfg, a, heads, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace gdnq
