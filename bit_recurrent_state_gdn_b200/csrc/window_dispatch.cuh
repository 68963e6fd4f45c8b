// Template dispatch from a runtime gdn_config to an instantiated window kernel configuration.
#pragma once

#include <algorithm>
#include <atomic>

#include "launch.h"
#include "window_kernels.cuh"

namespace gdnq {

// Raises a kernel's dynamic shared-memory limit as needed, once per (kernel, device): the cache
// is a static of this instantiation, so every kernel has its own.
template <auto Kernel>
cudaError_t ensure_smem(size_t bytes) {
  static std::atomic<size_t> granted[64];
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) dev = 63;
  if (granted[dev].load() >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) granted[dev].store(bytes);
  return e;
}

// Streaming multiprocessors of the current device (cached per device).
inline int num_sms() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load();
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n);
  }
  return n;
}

// Shape of a persistent step launch: two CTAs per SM when one stage of the largest window
// position fits into half of an SM's shared memory, else one CTA per SM. Each CTA gets all the
// shared memory that allows and sizes its stages itself (up to kMaxStages). Two CTAs with one
// stage each late in a window (the per-channel gate's stages hold fp32 gates per pair) beat one
// CTA with two stages: the other CTA's head runs while a CTA waits for its copies.
struct StepPlan {
  int grid, per_cta;
  size_t smem;
};

template <class C, bool MIX>
StepPlan plan_step(int W, int r, int heads, bool power = false) {
  constexpr int kSmemPerSm = 228 * 1024, kReserved = 1024;
  const int sms = num_sms();
  const bool red = !step_uses_mma<C>(W);
  auto per = [&](int ctas) { return std::min(kMaxHeadsPerCta, std::max(1, (heads + ctas - 1) / ctas)); };
  StepPlan p;
  const size_t half = (size_t)kSmemPerSm / 2 - kReserved;
  int bps = 2;
  if ((size_t)win_layout_mix<C, MIX>(W, r, 1, per(2 * sms), -1, red, power).total > half) bps = 1;
  p.per_cta = per(bps * sms);
  p.grid = (heads + p.per_cta - 1) / p.per_cta;
  p.smem = bps == 2 ? half
                    : std::min((size_t)kMaxSmemPerCta,
                               (size_t)win_layout_mix<C, MIX>(W, r, kMaxStages, p.per_cta, -1,
                                                              red, power).total);
  return p;
}

// Power compensator tokens: the step leaves full windows to power_end_kernel, launched right
// after it on the same stream; forced flushes and the initial quantization run there too.
template <class C>
cudaError_t launch_power(WinOp op, const WinArgs& a, int heads, cudaStream_t st) {
  const size_t pend = power_end_smem<C>(a.W, a.r, true), pq = power_end_smem<C>(a.W, a.r, false);
  const int pgrid = std::min(heads, 2 * num_sms());
  cudaError_t e = cudaSuccess;
  switch (op) {
    case WinOp::Step: {
      const StepPlan p = plan_step<C, false>(a.W, a.r, heads, true);
      e = ensure_smem<window_step_kernel<C, false>>(p.smem);
      if (e == cudaSuccess)
        window_step_kernel<C, false><<<p.grid, kStepThreads, p.smem, st>>>(a, heads, p.per_cta,
                                                                           (int)p.smem);
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e == cudaSuccess) e = ensure_smem<power_end_kernel<C, 2>>(pend);
      if (e == cudaSuccess) power_end_kernel<C, 2><<<pgrid, kThreads, pend, st>>>(a, heads);
      break;
    }
    case WinOp::Flush:
      e = ensure_smem<power_end_kernel<C, 0>>(pend);
      if (e == cudaSuccess) power_end_kernel<C, 0><<<pgrid, kThreads, pend, st>>>(a, heads);
      break;
    case WinOp::Quantize:
      e = ensure_smem<power_end_kernel<C, 3>>(pq);
      if (e == cudaSuccess) power_end_kernel<C, 3><<<pgrid, kThreads, pq, st>>>(a, heads);
      break;
    case WinOp::Materialize: {
      const size_t sm1 = win_layout<C>(a.W, a.r, 1, 0, -1, true, true).total;
      e = ensure_smem<window_state_kernel<C, 1, false>>(sm1);
      if (e == cudaSuccess) window_state_kernel<C, 1, false><<<heads, kThreads, sm1, st>>>(a);
      break;
    }
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <class C, bool MIX = false>
cudaError_t launch_window_cfg(WinOp op, const WinArgs& a, int heads, cudaStream_t st) {
  if constexpr (!MIX && !C::SMOOTH && C::MMA) {
    if (a.comp_k) return launch_power<C>(op, a, heads, st);
  }
  size_t smem1 = win_layout<C>(a.W, a.r, 1, 0).total;
  if constexpr (MIX) smem1 = std::max(smem1, (size_t)win_layout<Int4Of<C>>(a.W, a.r, 1, 0).total);
  cudaError_t e = cudaSuccess;
  switch (op) {
    case WinOp::Step: {
      const StepPlan p = plan_step<C, MIX>(a.W, a.r, heads);
      e = ensure_smem<window_step_kernel<C, MIX>>(p.smem);
      if (e == cudaSuccess)
        window_step_kernel<C, MIX><<<p.grid, kStepThreads, p.smem, st>>>(a, heads, p.per_cta,
                                                                          (int)p.smem);
      break;
    }
    case WinOp::Flush:
      e = ensure_smem<window_state_kernel<C, 0, MIX>>(smem1);
      if (e == cudaSuccess) window_state_kernel<C, 0, MIX><<<heads, kThreads, smem1, st>>>(a);
      break;
    case WinOp::Materialize:
      e = ensure_smem<window_state_kernel<C, 1, MIX>>(smem1);
      if (e == cudaSuccess) window_state_kernel<C, 1, MIX><<<heads, kThreads, smem1, st>>>(a);
      break;
    case WinOp::Quantize:
      quantize_kernel<C, MIX><<<heads, kThreads, 0, st>>>(a);
      break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// MIX: int8 and int4 heads in one launch (INT4 is then false: the int8 configuration, whose
// int4 companion Int4Of<> takes the int4 heads).
template <int D, bool DIAG, bool INT4, bool MIX = false, bool SMOOTH = false>
cudaError_t launch_window_types(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                                cudaStream_t st) {
  using bf = __nv_bfloat16;
  const bool af = cfg.act_dtype == GDN_DTYPE_F32, bfp = cfg.buf_dtype == GDN_DTYPE_F32;
  if (af && bfp)
    return launch_window_cfg<WinCfg<D, DIAG, INT4, float, float, SMOOTH>, MIX>(op, a, heads, st);
  if (af)
    return launch_window_cfg<WinCfg<D, DIAG, INT4, float, bf, SMOOTH>, MIX>(op, a, heads, st);
  if (bfp)
    return launch_window_cfg<WinCfg<D, DIAG, INT4, bf, float, SMOOTH>, MIX>(op, a, heads, st);
  return launch_window_cfg<WinCfg<D, DIAG, INT4, bf, bf, SMOOTH>, MIX>(op, a, heads, st);
}

template <int D, bool INT4, bool MIX = false, bool SMOOTH = false>
cudaError_t launch_window_gate(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                               cudaStream_t st) {
  if (cfg.gate == GDN_GATE_DIAG)
    return launch_window_types<D, true, INT4, MIX, SMOOTH>(op, cfg, a, heads, st);
  return launch_window_types<D, false, INT4, MIX, SMOOTH>(op, cfg, a, heads, st);
}

}  // namespace gdnq
