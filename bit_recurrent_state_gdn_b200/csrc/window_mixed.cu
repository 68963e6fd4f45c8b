// Window kernels instantiated for states whose heads mix int8 and packed int4 (group 32) codes,
// each head in its own format within one launch.
#include "window_dispatch.cuh"

namespace gdnq {

cudaError_t launch_window_mixed(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                                cudaStream_t st) {
  switch (cfg.d_k) {
    case 128: return launch_window_gate<128, false, true>(op, cfg, a, heads, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace gdnq
