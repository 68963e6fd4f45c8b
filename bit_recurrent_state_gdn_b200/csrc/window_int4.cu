// Window kernels instantiated for packed int4 codes with one scale per 32 key channels.
#include "window_dispatch.cuh"

namespace gdnq {

cudaError_t launch_window_int4(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                               cudaStream_t st) {
  switch (cfg.d_k) {
    case 128: return launch_window_gate<128, true>(op, cfg, a, heads, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace gdnq
