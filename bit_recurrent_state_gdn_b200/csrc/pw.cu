// Pure-write sliding window: launch configuration and dispatch to the kernel instantiations.
#include "launch.h"
#include "pw_kernels.cuh"
#include "window_dispatch.cuh"

namespace gdnq {

namespace {

template <class P>
cudaError_t pw_launch_cfg(PwOp op, const PwArgs& a, int heads, cudaStream_t st) {
  if (heads <= 0) return cudaSuccess;
  if (op == PwOp::Materialize) {
    pw_materialize_kernel<P><<<heads, kPwThreads, 0, st>>>(a);
    return cudaGetLastError();
  }
  // pw_ctas_per_sm CTAs per SM, each walking a contiguous range of heads with up to
  // kPwMaxStages stages in its share of the SM's shared memory
  constexpr int cps = pw_ctas_per_sm<P>();
  const int sms = num_sms();
  int per_cta = (heads + cps * sms - 1) / (cps * sms);
  if (per_cta > kPwMaxHeadsPerCta) per_cta = kPwMaxHeadsPerCta;
  const int grid = (heads + per_cta - 1) / per_cta;
  const size_t budget = (size_t)228 * 1024 / cps - 1024;
  // at least two stages (the loop's refill order needs them; two always fit)
  int nstages = kPwMaxStages;
  while (nstages > 2 && pw_layout<P>(a.Wp, nstages, per_cta).total > budget) --nstages;
  const size_t smem = pw_layout<P>(a.Wp, nstages, per_cta).total;
  cudaError_t e = ensure_smem<pw_step_kernel<P>>(smem);
  if (e != cudaSuccess) return e;
  pw_step_kernel<P><<<grid, kPwThreads, smem, st>>>(a, heads, per_cta, nstages);
  return cudaGetLastError();
}

template <bool DIAG, bool INT4>
cudaError_t pw_launch_act(PwOp op, const gdn_pw_config& c, const PwArgs& a, int heads,
                          cudaStream_t st) {
  if (c.act_dtype == GDN_DTYPE_F32)
    return pw_launch_cfg<PwCfg<DIAG, INT4, float>>(op, a, heads, st);
  return pw_launch_cfg<PwCfg<DIAG, INT4, __nv_bfloat16>>(op, a, heads, st);
}

}  // namespace

cudaError_t launch_pw(PwOp op, const gdn_pw_config& c, const PwArgs& a, int heads,
                      cudaStream_t st) {
  const bool diag = c.gate == GDN_GATE_DIAG, int4 = c.fmt == GDN_FMT_INT4_G32;
  if (diag) return int4 ? pw_launch_act<true, true>(op, c, a, heads, st)
                        : pw_launch_act<true, false>(op, c, a, heads, st);
  return int4 ? pw_launch_act<false, true>(op, c, a, heads, st)
              : pw_launch_act<false, false>(op, c, a, heads, st);
}

}  // namespace gdnq
