// Arguments of the chunkwise prefill kernel (shared by the kernel and the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace gdnq {

struct PfArgs {
  const __nv_bfloat16* q;  // [heads][L][128]
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* g;          // [heads][L] (scalar gate) or [heads][L][128] (per-channel gate)
  const float* beta;
  __nv_bfloat16* o;        // [heads][L][128]
  float* S;                // [heads][128][128], in place
  uint8_t* ws;             // scalar gate: [heads][ceil(L / 64)] chunk records (workspace)
  int L;
};

}  // namespace gdnq
