// Chunkwise-parallel GDN prefill ("LinQuant: Functional Invariances for Low-Precision Linear
// Recurrences", Abstract: prefill of a linear recurrence cast as chunked dense matmuls), the
// step before decode: L tokens of the gated delta rule for every head, from an initial fp32
// state, writing every output and the final state.
//
// Per chunk of C = 64 tokens (scalar gate, G_t = cumulative log-gate inside the chunk, state S
// entering the chunk, rows t, s of the chunk):
//   A[t][s] = beta_t e^{G_t - G_s} <k_t, k_s>  (s < t)          T = (I + A)^{-1} Diag(beta)
//   V'      = V - Diag(e^G) K S^T                                 U = T V'
//   O       = Diag(e^G) Q S^T + (M .* Q K^T) U,   M[t][s] = e^{G_t - G_s} (s <= t)
//   S_next  = e^{G_C} S + U^T Diag(e^{G_C - G}) K
// (from u_t = beta_t (v_t - e^{g_t} S_{t-1} k_t), S_t = e^{g_t} S_{t-1} + u_t k_t^T unrolled
// over the chunk: (I + A) U = Diag(beta) V').
//
// This file holds that algebra's shared pieces: the chunk constants, the blocked triangular
// inverse in fp32, the hi / lo bf16 operand splits and small mma.sync helpers. The kernels are
// prefill_tc_kernels.cuh (scalar gate, tcgen05) and prefill_kda_kernels.cuh (per-channel gate).
#pragma once

#include <cuda_bf16.h>

#include "device_util.cuh"
#include "mma_util.cuh"
#include "prefill_args.h"

namespace gdnq {

constexpr int kPfThreads = 256;
constexpr int kPfC = 64;     // chunk length
constexpr int kPfD = 128;    // head size
constexpr int kLd128 = 136;  // bf16 row stride of 128-column tiles (272 B: ldmatrix without conflicts)
constexpr int kLd64 = 72;    // bf16 row stride of 64-column tiles (144 B)
constexpr int kLdF = 65;     // fp32 row stride of 64 x 64 fp32 tiles


// 16-byte asynchronous global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// 2^x on the hardware path (relative error about 2^-22; a result below 2^-126 flushes to 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// The same for two values at once, as packed bf16 pairs (x0 in the low half): hi = RN(x),
// lo = RN(x - hi), with one packed conversion each.
__device__ __forceinline__ void split2_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(x0, x1);
  lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
}

// acc (16 x 8 NT) += A (16 x 16 KS) * B (16 KS x 8 NT) on mma.m16n8k16 bf16.
//   A: rows m0.., columns k0.. of a bf16 tile at a_base (row stride lda elements); A_T: the tile
//      is stored transposed ([k][m]).
//   B: columns n0.. and rows k0..; B_KN: stored [k][n] (row = k), else [n][k].
template <int NT, int KS, bool A_T, bool B_KN>
__device__ __forceinline__ void warp_mma(float (&acc)[NT][4], uint32_t a_base, int lda, int m0,
                                         uint32_t b_base, int ldb, int n0, int k0) {
  static_assert(NT % 2 == 0, "n-tiles in pairs");
  const int lane = threadIdx.x & 31, mi = lane >> 3, r8 = lane & 7;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int kk = k0 + 16 * ks;
    uint32_t a[4];
    if constexpr (A_T) {
      ldsm_x4_t(a_base + 2u * ((kk + r8 + 8 * (mi >> 1)) * lda + m0 + 8 * (mi & 1)), a);
    } else {
      ldsm_x4(a_base + 2u * ((m0 + (lane & 15)) * lda + kk + 8 * (lane >> 4)), a);
    }
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      const int nn = n0 + 16 * np;
      uint32_t b[4];
      if constexpr (B_KN) {
        ldsm_x4_t(b_base + 2u * ((kk + r8 + 8 * (mi & 1)) * ldb + nn + 8 * (mi >> 1)), b);
      } else {
        ldsm_x4(b_base + 2u * ((nn + r8 + 8 * (mi >> 1)) * ldb + kk + 8 * (mi & 1)), b);
      }
      mma_bf16(acc[2 * np], a, b[0], b[1]);
      mma_bf16(acc[2 * np + 1], a, b[2], b[3]);
    }
  }
}

template <int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[NT][4]) {
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
}

// Writes a 16 x 8 NT fp32 accumulator block (rows m0.., columns n0..) split into hi / lo bf16
// tiles, each value first mapped by f(row, column, value).
template <int NT, class F>
__device__ __forceinline__ void store_split(const float (&acc)[NT][4], __nv_bfloat16* hi,
                                            __nv_bfloat16* lo, int ld, int m0, int n0, F f) {
  const int lane = threadIdx.x & 31, gid = lane >> 2, q4 = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int r = m0 + gid + 8 * hh, c = n0 + 8 * nt + 2 * q4;
      uint32_t hv, lv;
      split2_bf16(f(r, c, acc[nt][2 * hh]), f(r, c + 1, acc[nt][2 * hh + 1]), hv, lv);
      *reinterpret_cast<uint32_t*>(hi + r * ld + c) = hv;
      *reinterpret_cast<uint32_t*>(lo + r * ld + c) = lv;
    }
  }
}

// R = (I + A)^{-1} for the strictly lower triangular 64 x 64 A (fp32, stride kLdF), blocked in
// 16 x 16: diagonal blocks by column-oriented substitution (one lane per column: after row k of
// the column is final, every later row takes its -A_tk R_k term, so the 15 updates of a step are
// independent), then R_ij = -R_ii sum_{j <= k < i} A_ik R_kj level by level (i - j = 1, 2, 3),
// each level spread over all threads, its sums split over four partial accumulators.
// xs: 3 x 256 floats of scratch.
__device__ __forceinline__ void unit_lower_inverse(const float* A, float* R, float* xs) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // diagonal blocks: warps 0-1, lanes 0-15 / 16-31 take blocks 2 warp and 2 warp + 1
  if (warp < 2) {
    const int b = 2 * warp + (lane >> 4), c = lane & 15, o = 16 * b;
    float rc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) rc[t] = t == c ? 1.f : 0.f;
#pragma unroll
    for (int k = 0; k < 15; ++k)
#pragma unroll
      for (int t = k + 1; t < 16; ++t) rc[t] = fmaf(-A[(o + t) * kLdF + o + k], rc[k], rc[t]);
#pragma unroll
    for (int t = 0; t < 16; ++t) R[(o + t) * kLdF + o + c] = rc[t];
  }
  __syncthreads();
  // off-diagonal blocks, every thread: level lvl has the blocks (j + lvl, j), j < 4 - lvl;
  // first X_j = sum_{j <= kb < i} A_{i,kb} R_{kb,j}, then R_ij = -R_ii X_j
  for (int lvl = 1; lvl < 4; ++lvl) {
    const int nb = 4 - lvl;
    for (int e = tid; e < 256 * nb; e += kPfThreads) {
      const int j = e >> 8, i = j + lvl, r = (e >> 4) & 15, c = e & 15;
      float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
      for (int kb = j; kb < i; ++kb) {
        const float* ar = A + (16 * i + r) * kLdF + 16 * kb;
        const float* rcol = R + (16 * kb) * kLdF + 16 * j + c;
#pragma unroll
        for (int s = 0; s < 16; s += 4) {
          p0 = fmaf(ar[s], rcol[s * kLdF], p0);
          p1 = fmaf(ar[s + 1], rcol[(s + 1) * kLdF], p1);
          p2 = fmaf(ar[s + 2], rcol[(s + 2) * kLdF], p2);
          p3 = fmaf(ar[s + 3], rcol[(s + 3) * kLdF], p3);
        }
      }
      xs[e] = (p0 + p1) + (p2 + p3);
    }
    __syncthreads();
    for (int e = tid; e < 256 * nb; e += kPfThreads) {
      const int j = e >> 8, i = j + lvl, r = (e >> 4) & 15, c = e & 15;
      const float* rr = R + (16 * i + r) * kLdF + 16 * i;
      const float* xc = xs + (j << 8) + c;
      float p0 = 0.f, p1 = 0.f;
#pragma unroll
      for (int s = 0; s < 16; s += 2) {
        p0 = fmaf(rr[s], xc[s * 16], p0);
        p1 = fmaf(rr[s + 1], xc[(s + 1) * 16], p1);
      }
      R[(16 * i + r) * kLdF + 16 * j + c] = -(p0 + p1);
    }
    __syncthreads();
  }
}

}  // namespace gdnq
