// High-precision-state baseline: one plain decode step per (sequence, head), the state read
// from HBM once and written back once. The baseline the low-bit windowed state is measured
// against ("LeapQuant: Efficient Linear Attention with Accurate Recurrent State Quantization",
// Abstract: speedups quoted against an FP32-state baseline).
//   w = S Diag(a) k,  z = S Diag(a) q,  u = beta (v - w),
//   S <- S Diag(a) + u k^T,  o = z + u <k, q>
// One CTA of 256 threads per head; thread (rg, cg) holds TR rows x TC columns of S in registers.
// Columns are interleaved in 16-byte vectors so each load / store instruction of a warp covers
// contiguous memory.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "device_util.cuh"

namespace gdnq {

struct BaseArgs {
  void* S;
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  void* o;
};

template <typename T>
__device__ __forceinline__ void store_vec(T* p, const float* x, int n);

template <>
__device__ __forceinline__ void store_vec<float>(float* p, const float* x, int n) {
  if (n == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  } else {
    for (int e = 0; e < n; ++e) p[e] = x[e];
  }
}

template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16>(__nv_bfloat16* p, const float* x, int n) {
  if (n == 8) {
    uint4 w;
    uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
      wv[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = w;
  } else {
    for (int e = 0; e < n; ++e) p[e] = __float2bfloat16_rn(x[e]);
  }
}


template <int D_, bool DIAG_, typename State_, typename Act_>
struct BaseCfg {
  static constexpr int D = D_;
  static constexpr bool DIAG = DIAG_;
  using State = State_;
  using Act = Act_;
  static constexpr int NT = 256, CG = 16, RG = NT / CG;
  static constexpr int TR = D / RG, TC = D / CG;
  static constexpr int VW0 = 16 / (int)sizeof(State);
  static constexpr int VW = VW0 < TC ? VW0 : TC;  // elements per vector access
  static constexpr int NV = TC / VW;              // vector accesses per row
  static_assert(D % 16 == 0, "head size");
  __device__ __forceinline__ static int col(int cg, int m, int e) { return (m * CG + cg) * VW + e; }
};

template <class C>
__global__ void __launch_bounds__(256) baseline_step_kernel(const BaseArgs a) {
  using State = typename C::State;
  using Act = typename C::Act;
  constexpr int D = C::D, TR = C::TR, TC = C::TC, VW = C::VW, NV = C::NV;
  const int head = blockIdx.x, tid = threadIdx.x, cg = tid % C::CG, rg = tid / C::CG;
  State* S = static_cast<State*>(a.S) + (size_t)head * D * D;

  float s[TR][TC];
#pragma unroll
  for (int r = 0; r < TR; ++r) {
    const int row = rg * TR + r;
#pragma unroll
    for (int m = 0; m < NV; ++m) {
      const State* p = S + (size_t)row * D + C::col(cg, m, 0);
      if constexpr (VW * sizeof(State) == 16) {
        Num<State>::template load<VW>(p, &s[r][m * VW]);
      } else {
#pragma unroll
        for (int e = 0; e < VW; ++e) s[r][m * VW + e] = Num<State>::to_f(p[e]);
      }
    }
  }

  const Act* kin = static_cast<const Act*>(a.k) + (size_t)head * D;
  const Act* qin = static_cast<const Act*>(a.q) + (size_t)head * D;
  float kk[TC], x[TC], y[TC], dec[TC];
  float kq = 0.f;
  const float ascalar = C::DIAG ? 1.f : fast_exp(a.g[head]);
#pragma unroll
  for (int m = 0; m < NV; ++m)
#pragma unroll
    for (int e = 0; e < VW; ++e) {
      const int j = C::col(cg, m, e), b = m * VW + e;
      const float kj = Num<Act>::to_f(kin[j]), qj = Num<Act>::to_f(qin[j]);
      dec[b] = C::DIAG ? fast_exp(a.g[(size_t)head * D + j]) : ascalar;
      kk[b] = kj;
      x[b] = dec[b] * kj;
      y[b] = dec[b] * qj;
      kq = fmaf(kj, qj, kq);
    }
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);

  const float bt = a.beta[head];
  const Act* vin = static_cast<const Act*>(a.v) + (size_t)head * D;
  Act* out = static_cast<Act*>(a.o) + (size_t)head * D;
#pragma unroll
  for (int r = 0; r < TR; ++r) {
    float w = 0.f, z = 0.f;
#pragma unroll
    for (int b = 0; b < TC; ++b) {
      w = fmaf(s[r][b], x[b], w);
      z = fmaf(s[r][b], y[b], z);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {
      w += __shfl_xor_sync(0xffffffffu, w, off);
      z += __shfl_xor_sync(0xffffffffu, z, off);
    }
    const int row = rg * TR + r;
    const float u = bt * (Num<Act>::to_f(vin[row]) - w);
    if (cg == 0) out[row] = Num<Act>::from_f(z + u * kq);
    float nv[TC];
#pragma unroll
    for (int b = 0; b < TC; ++b) nv[b] = fmaf(u, kk[b], s[r][b] * dec[b]);
#pragma unroll
    for (int m = 0; m < NV; ++m) store_vec<State>(S + (size_t)row * D + C::col(cg, m, 0), &nv[m * VW], VW);
  }
}

}  // namespace gdnq
