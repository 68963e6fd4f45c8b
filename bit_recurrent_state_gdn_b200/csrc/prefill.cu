// Chunkwise prefill: launches of the kernels in prefill_kernels.cuh (scalar gate) and
// prefill_kda_kernels.cuh (per-key-channel gate).
#include "launch.h"
#include "prefill_kda_kernels.cuh"
#include "window_dispatch.cuh"

namespace gdnq {

cudaError_t launch_prefill(const PfArgs& a, int heads, bool diag, cudaStream_t st) {
  if (heads <= 0) return cudaSuccess;
  if (diag) {
    cudaError_t e = ensure_smem<prefill_kda_kernel>(KdaLayout::TOTAL);
    if (e != cudaSuccess) return e;
    prefill_kda_kernel<<<heads, kPfThreads, KdaLayout::TOTAL, st>>>(a);
    return cudaGetLastError();
  }
  cudaError_t e = ensure_smem<prefill_kernel>(PfLayout::TOTAL);
  if (e != cudaSuccess) return e;
  prefill_kernel<<<heads, kPfThreads, PfLayout::TOTAL, st>>>(a);
  return cudaGetLastError();
}

size_t prefill_smem_bytes(bool diag) { return diag ? KdaLayout::TOTAL : PfLayout::TOTAL; }

}  // namespace gdnq
