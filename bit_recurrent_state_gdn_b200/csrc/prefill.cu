// Chunkwise prefill: launch of the kernel in prefill_kernels.cuh.
#include "launch.h"
#include "prefill_kernels.cuh"
#include "window_dispatch.cuh"

namespace gdnq {

cudaError_t launch_prefill(const PfArgs& a, int heads, cudaStream_t st) {
  if (heads <= 0) return cudaSuccess;
  cudaError_t e = ensure_smem<prefill_kernel>(PfLayout::TOTAL);
  if (e != cudaSuccess) return e;
  prefill_kernel<<<heads, kPfThreads, PfLayout::TOTAL, st>>>(a);
  return cudaGetLastError();
}

size_t prefill_smem_bytes() { return PfLayout::TOTAL; }

}  // namespace gdnq
