// Chunkwise prefill: launches of the kernels in prefill_tc_kernels.cuh (scalar gate, tcgen05)
// and prefill_kda_kernels.cuh (per-key-channel gate).
#include <cudaTypedefs.h>

#include "launch.h"
#include "prefill_kda_kernels.cuh"
#include "prefill_tc_kernels.cuh"
#include "window_dispatch.cuh"

namespace gdnq {
namespace {

// cuTensorMapEncodeTiled, found once through the runtime (no link against the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// bf16 [heads][L][128] as a 3-D tensor map with boxes of 64 tokens x 64 channels, 128-byte
// swizzle; boxes reaching past a head's last token read zeros.
cudaError_t token_map(CUtensorMap* m, const void* base, int L, int heads) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)kPfD, (cuuint64_t)L, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)kPfD * 2, (cuuint64_t)L * kPfD * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)kPfC, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prefill(const PfArgs& a, int heads, bool diag, cudaStream_t st) {
  if (heads <= 0 || a.L <= 0) return cudaSuccess;
  if (diag) {
    cudaError_t e = ensure_smem<prefill_kda_kernel>(KdaLayout::TOTAL);
    if (e != cudaSuccess) return e;
    prefill_kda_kernel<<<heads, kPfThreads, KdaLayout::TOTAL, st>>>(a);
    return cudaGetLastError();
  }
  PfTcMaps maps;
  cudaError_t e = token_map(&maps.q, a.q, a.L, heads);
  if (e == cudaSuccess) e = token_map(&maps.k, a.k, a.L, heads);
  if (e == cudaSuccess) e = token_map(&maps.v, a.v, a.L, heads);
  if (e == cudaSuccess) e = ensure_smem<prefill_chunk_kernel>(ChunkLayout::ALLOC);
  if (e == cudaSuccess) e = ensure_smem<prefill_tc_kernel>(TcLayout::ALLOC);
  if (e != cudaSuccess) return e;
  // the state-independent part of every chunk (persistent CTAs), then each head's chunks in
  // order
  const int total = heads * ((a.L + kPfC - 1) / kPfC);
  const int grid = std::min(total, kChunkCtasPerSm * num_sms());
  prefill_chunk_kernel<<<grid, kPfThreads, ChunkLayout::ALLOC, st>>>(a, maps, total);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  prefill_tc_kernel<<<heads, kPfThreads, TcLayout::ALLOC, st>>>(a, maps);
  return cudaGetLastError();
}

size_t prefill_smem_bytes(bool diag) { return diag ? KdaLayout::TOTAL : TcLayout::ALLOC; }

size_t prefill_workspace_bytes(bool diag, int64_t heads, int L) {
  if (diag || heads <= 0 || L <= 0) return 0;
  return (size_t)heads * (size_t)((L + kPfC - 1) / kPfC) * kPfRecBytes;
}

}  // namespace gdnq
