// Template dispatch from a runtime gdn_config to an instantiated window kernel configuration.
#pragma once

#include <atomic>

#include "launch.h"
#include "window_kernels.cuh"

namespace gdnq {

// Raises a kernel's dynamic shared-memory limit once per device as needed.
template <class Kernel>
cudaError_t ensure_smem(Kernel k, size_t bytes) {
  static std::atomic<size_t> granted[64];
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) dev = 63;
  if (granted[dev].load() >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) granted[dev].store(bytes);
  return e;
}

template <class C>
cudaError_t launch_window_cfg(WinOp op, const WinArgs& a, int heads, cudaStream_t st) {
  const size_t smem = window_smem_layout<C>(a.W, a.r).total;
  cudaError_t e = cudaSuccess;
  switch (op) {
    case WinOp::Step:
      e = ensure_smem(window_step_kernel<C>, smem);
      if (e == cudaSuccess) window_step_kernel<C><<<heads, kThreads, smem, st>>>(a);
      break;
    case WinOp::Flush:
      e = ensure_smem(window_state_kernel<C, 0>, smem);
      if (e == cudaSuccess) window_state_kernel<C, 0><<<heads, kThreads, smem, st>>>(a);
      break;
    case WinOp::Materialize:
      e = ensure_smem(window_state_kernel<C, 1>, smem);
      if (e == cudaSuccess) window_state_kernel<C, 1><<<heads, kThreads, smem, st>>>(a);
      break;
    case WinOp::Quantize:
      quantize_kernel<C><<<heads, kThreads, 0, st>>>(a);
      break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, bool DIAG, bool INT4>
cudaError_t launch_window_types(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                                cudaStream_t st) {
  using bf = __nv_bfloat16;
  const bool af = cfg.act_dtype == GDN_DTYPE_F32, bfp = cfg.buf_dtype == GDN_DTYPE_F32;
  if (af && bfp) return launch_window_cfg<WinCfg<D, DIAG, INT4, float, float>>(op, a, heads, st);
  if (af) return launch_window_cfg<WinCfg<D, DIAG, INT4, float, bf>>(op, a, heads, st);
  if (bfp) return launch_window_cfg<WinCfg<D, DIAG, INT4, bf, float>>(op, a, heads, st);
  return launch_window_cfg<WinCfg<D, DIAG, INT4, bf, bf>>(op, a, heads, st);
}

template <int D, bool INT4>
cudaError_t launch_window_gate(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                               cudaStream_t st) {
  if (cfg.gate == GDN_GATE_DIAG) return launch_window_types<D, true, INT4>(op, cfg, a, heads, st);
  return launch_window_types<D, false, INT4>(op, cfg, a, heads, st);
}

}  // namespace gdnq
