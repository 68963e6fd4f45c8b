// Window kernels instantiated for packed int4 codes (group-32 scales) with residual smoothing.
#include "window_dispatch.cuh"

namespace gdnq {

cudaError_t launch_window_int4_smooth(WinOp op, const gdn_config& cfg, const WinArgs& a,
                                      int heads, cudaStream_t st) {
  if (cfg.d_k != 128) return cudaErrorNotSupported;
  return launch_window_gate<128, true, false, true>(op, cfg, a, heads, st);
}

}  // namespace gdnq
