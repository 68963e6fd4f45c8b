// Baseline (fp32 / bf16 state) kernels and their dispatch.
#include "baseline_kernels.cuh"
#include "launch.h"

namespace gdnq {

template <int D, bool DIAG, typename State>
static cudaError_t launch_base_act(const gdn_config& cfg, const BaseArgs& a, int heads,
                                   cudaStream_t st) {
  if (cfg.act_dtype == GDN_DTYPE_F32)
    baseline_step_kernel<BaseCfg<D, DIAG, State, float>><<<heads, 256, 0, st>>>(a);
  else
    baseline_step_kernel<BaseCfg<D, DIAG, State, __nv_bfloat16>><<<heads, 256, 0, st>>>(a);
  return cudaGetLastError();
}

template <int D, bool DIAG>
static cudaError_t launch_base_state(const gdn_config& cfg, const BaseArgs& a, int heads,
                                     cudaStream_t st) {
  if (cfg.fmt == GDN_FMT_FP32) return launch_base_act<D, DIAG, float>(cfg, a, heads, st);
  return launch_base_act<D, DIAG, __nv_bfloat16>(cfg, a, heads, st);
}

template <int D>
static cudaError_t launch_base_gate(const gdn_config& cfg, const BaseArgs& a, int heads,
                                    cudaStream_t st) {
  if (cfg.gate == GDN_GATE_DIAG) return launch_base_state<D, true>(cfg, a, heads, st);
  return launch_base_state<D, false>(cfg, a, heads, st);
}

cudaError_t launch_baseline(const gdn_config& cfg, const BaseArgs& a, int heads,
                            cudaStream_t st) {
  switch (cfg.d_k) {
    case 16: return launch_base_gate<16>(cfg, a, heads, st);
    case 128: return launch_base_gate<128>(cfg, a, heads, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace gdnq
