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
// One CTA per head, 256 threads, the state in registers as mma accumulators (warp w: rows
// 16w..16w+15), which also serve, split into hi / lo bf16 on the fly, as the B operand of the
// products with S^T (warp w computes their columns 16w..16w+15). The products run on mma.sync bf16 with fp32 accumulation; q, k, v are exact in
// bf16, and every fp32 operand (S, T, V', P, U) is split into hi + lo bf16 parts, so products
// carry about 16 significant bits of each fp32 operand. The triangular inverse is blocked
// (16 x 16 diagonal blocks by forward substitution, off-diagonal blocks by three levels of
// block products) in fp32.
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


// Shared memory (bytes)
struct PfLayout {
  static constexpr uint32_t Q = 0;
  static constexpr uint32_t K0 = Q + kPfC * kLd128 * 2;        // K of even chunks
  static constexpr uint32_t K1 = K0 + kPfC * kLd128 * 2;       // K of odd chunks
  static constexpr uint32_t V = K1 + kPfC * kLd128 * 2;
  static constexpr uint32_t X_HI = V + kPfC * kLd128 * 2;      // V', then U, then e^{G_C-G} U
  static constexpr uint32_t X_LO = X_HI + kPfC * kLd128 * 2;
  static constexpr uint32_t T_HI = X_LO + kPfC * kLd128 * 2;   // T, then P
  static constexpr uint32_t T_LO = T_HI + kPfC * kLd64 * 2;
  static constexpr uint32_t AF = T_LO + kPfC * kLd64 * 2;      // A (fp32)
  static constexpr uint32_t RF = AF + kPfC * kLdF * 4;         // R = (I + A)^{-1} (fp32)
  static constexpr uint32_t XS = RF + kPfC * kLdF * 4;         // 3 x 256 fp32 scratch
  static constexpr uint32_t GATE = XS + 3 * 256 * 4;           // G, e^G, e^{G_C - G}, beta
  static constexpr uint32_t TOTAL = GATE + 4 * kPfC * 4;
};

// 16-byte asynchronous global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// One 64 x 128 bf16 tile of chunk rows [c0, c0 + 64) of a head (rows >= n zero) into a padded
// shared tile, as asynchronous copies (4 per thread).
__device__ __forceinline__ void load_tile_async(__nv_bfloat16* dst, const __nv_bfloat16* src,
                                                size_t row0, int n) {
  for (int e = threadIdx.x; e < kPfC * 16; e += kPfThreads) {
    const int r = e >> 4, ch = e & 15;
    const __nv_bfloat16* g = src + (row0 + (r < n ? r : 0)) * kPfD + 8 * ch;
    cp_async16(dst + r * kLd128 + 8 * ch, g, r < n ? 16 : 0);
  }
}

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
// 16 x 16: diagonal blocks by forward substitution (one lane per column), then
// R_ij = -R_ii sum_{j <= k < i} A_ik R_kj level by level (i - j = 1, 2, 3), each level spread
// over all threads. xs: 3 x 256 floats of scratch.
__device__ __forceinline__ void unit_lower_inverse(const float* A, float* R, float* xs) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // diagonal blocks: warps 0-1, lanes 0-15 / 16-31 take blocks 2 warp and 2 warp + 1
  if (warp < 2) {
    const int b = 2 * warp + (lane >> 4), c = lane & 15, o = 16 * b;
    float rc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float sum = 0.f;
#pragma unroll
      for (int s = 0; s < t; ++s) sum = fmaf(A[(o + t) * kLdF + o + s], rc[s], sum);
      rc[t] = t < c ? 0.f : (t == c ? 1.f : -sum);
    }
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
      float sum = 0.f;
      for (int kb = j; kb < i; ++kb) {
#pragma unroll
        for (int s = 0; s < 16; ++s)
          sum = fmaf(A[(16 * i + r) * kLdF + 16 * kb + s], R[(16 * kb + s) * kLdF + 16 * j + c], sum);
      }
      xs[e] = sum;
    }
    __syncthreads();
    for (int e = tid; e < 256 * nb; e += kPfThreads) {
      const int j = e >> 8, i = j + lvl, r = (e >> 4) & 15, c = e & 15;
      float sum = 0.f;
#pragma unroll
      for (int s = 0; s < 16; ++s) sum = fmaf(R[(16 * i + r) * kLdF + 16 * i + s], xs[(j << 8) + s * 16 + c], sum);
      R[(16 * i + r) * kLdF + 16 * j + c] = -sum;
    }
    __syncthreads();
  }
}

// acc[2 mt + nn] (rows 16 mt.., columns 8 nn.. of this warp's 16-column slab v0..v0+15)
// += A (64 x 128, a bf16 tile at a_base) * S^T restricted to the slab, S in this warp's
// accumulators: the accumulator layout of the warp's state rows v0..v0+15 is the B-fragment
// layout of those columns of S^T, so each B register is two accumulator entries, split into
// hi and lo bf16 on the fly.
__device__ __forceinline__ void mma_state_slab(float (&acc)[8][4], uint32_t a_base,
                                               const float (&sacc)[16][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    uint32_t bh[2][2], bl[2][2];
#pragma unroll
    for (int nn = 0; nn < 2; ++nn)
#pragma unroll
      for (int half = 0; half < 2; ++half)
        split2_bf16(sacc[2 * ks + half][2 * nn], sacc[2 * ks + half][2 * nn + 1], bh[nn][half],
                    bl[nn][half]);
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      uint32_t a[4];
      ldsm_x4(a_base + 2u * ((16 * mt + (lane & 15)) * kLd128 + 16 * ks + 8 * (lane >> 4)), a);
#pragma unroll
      for (int nn = 0; nn < 2; ++nn) {
        mma_bf16(acc[2 * mt + nn], a, bh[nn][0], bh[nn][1]);
        mma_bf16(acc[2 * mt + nn], a, bl[nn][0], bl[nn][1]);
      }
    }
  }
}

// A slab accumulator (tiles 2 mt + nn: rows 16 mt.., columns v0 + 8 nn..) into hi / lo tiles
// after f(row, column, value).
template <class F>
__device__ __forceinline__ void store_split_slab(const float (&acc)[8][4], __nv_bfloat16* hi,
                                                 __nv_bfloat16* lo, int ld, int v0, F f) {
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const float(&t2)[2][4] = *reinterpret_cast<const float(*)[2][4]>(&acc[2 * mt]);
    store_split(t2, hi, lo, ld, 16 * mt, v0, f);
  }
}

// acc (slab) += A (64 x 64 hi / lo tiles, rows t) * B (64 x 128 hi / lo tiles stored [s][v],
// columns v0..v0+15): the three-term split product.
__device__ __forceinline__ void mma_slab_split3(float (&acc)[8][4], uint32_t ahi, uint32_t alo,
                                                uint32_t bhi, uint32_t blo, int v0) {
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    float(&t2)[2][4] = *reinterpret_cast<float(*)[2][4]>(&acc[2 * mt]);
    warp_mma<2, 4, false, true>(t2, ahi, kLd64, 16 * mt, bhi, kLd128, v0, 0);
    warp_mma<2, 4, false, true>(t2, ahi, kLd64, 16 * mt, blo, kLd128, v0, 0);
    warp_mma<2, 4, false, true>(t2, alo, kLd64, 16 * mt, bhi, kLd128, v0, 0);
  }
}

__global__ void __launch_bounds__(kPfThreads, 1) prefill_kernel(const PfArgs a) {
  using bf = __nv_bfloat16;
  extern __shared__ __align__(128) uint8_t sm[];
  const int head = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, q4 = lane & 3;
  const int L = a.L;
  bf* Qs = reinterpret_cast<bf*>(sm + PfLayout::Q);
  bf* K0s = reinterpret_cast<bf*>(sm + PfLayout::K0);
  bf* K1s = reinterpret_cast<bf*>(sm + PfLayout::K1);
  bf* Vs = reinterpret_cast<bf*>(sm + PfLayout::V);
  bf* Xhi = reinterpret_cast<bf*>(sm + PfLayout::X_HI);
  bf* Xlo = reinterpret_cast<bf*>(sm + PfLayout::X_LO);
  bf* Thi = reinterpret_cast<bf*>(sm + PfLayout::T_HI);
  bf* Tlo = reinterpret_cast<bf*>(sm + PfLayout::T_LO);
  float* Af = reinterpret_cast<float*>(sm + PfLayout::AF);
  float* Rf = reinterpret_cast<float*>(sm + PfLayout::RF);
  float* xs = reinterpret_cast<float*>(sm + PfLayout::XS);
  float* Gs = reinterpret_cast<float*>(sm + PfLayout::GATE);
  float* eG = Gs + kPfC;   // e^{G_t}
  float* eGC = eG + kPfC;  // e^{G_C - G_t}
  float* bet = eGC + kPfC;
  const uint32_t q_b = smem_u32(Qs);
  const uint32_t xhi_b = smem_u32(Xhi), xlo_b = smem_u32(Xlo), thi_b = smem_u32(Thi), tlo_b = smem_u32(Tlo);

  // the state: warp w holds rows 16w..16w+15, all 128 columns, in accumulator layout; it also
  // computes every chunk product whose columns are value channels for the slab v0..v0+15
  float sacc[16][4];
  float* Sg = a.S + (size_t)head * kPfD * kPfD;
  const int v0 = 16 * warp;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int j = 8 * nt + 2 * q4;
    const float2 r0 = *reinterpret_cast<const float2*>(Sg + (v0 + gid) * kPfD + j);
    const float2 r1 = *reinterpret_cast<const float2*>(Sg + (v0 + gid + 8) * kPfD + j);
    sacc[nt][0] = r0.x; sacc[nt][1] = r0.y; sacc[nt][2] = r1.x; sacc[nt][3] = r1.y;
  }

  const int mt = warp & 3, nh = warp >> 2;  // the C x C products: row tile and column half
  const int m0 = 16 * mt;
  if (L > 0) {  // the first chunk's tiles
    const int n = min(kPfC, L);
    load_tile_async(Qs, a.q, (size_t)head * L, n);
    load_tile_async(Vs, a.v, (size_t)head * L, n);
    load_tile_async(K0s, a.k, (size_t)head * L, n);
    cp_async_commit();
  }
  for (int c0 = 0, ci = 0; c0 < L; c0 += kPfC, ++ci) {
    const int n = min(kPfC, L - c0);
    const size_t row0 = (size_t)head * L + c0;
    const int n1 = min(kPfC, L - c0 - kPfC);  // the next chunk (<= 0: none)
    bf* Ks = (ci & 1) ? K1s : K0s;
    const uint32_t k_b = smem_u32(Ks);
    if (warp == 0) {  // cumulative log-gate over the chunk, two tokens per lane
      const int t0 = 2 * lane;
      const float g0 = t0 < n ? a.g[row0 + t0] : 0.f;
      const float g1 = t0 + 1 < n ? a.g[row0 + t0 + 1] : 0.f;
      float incl = g0 + g1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const float excl = incl - (g0 + g1);
      const float GC = __shfl_sync(0xffffffffu, incl, 31);
      const float G0 = excl + g0, G1 = incl;
      Gs[t0] = G0;
      Gs[t0 + 1] = G1;
      eG[t0] = expf(G0);
      eG[t0 + 1] = expf(G1);
      eGC[t0] = expf(GC - G0);
      eGC[t0 + 1] = expf(GC - G1);
      bet[t0] = t0 < n ? a.beta[row0 + t0] : 0.f;
      bet[t0 + 1] = t0 + 1 < n ? a.beta[row0 + t0 + 1] : 0.f;
    }
    cp_async_wait_all();  // this chunk's Q, K, V (rows past the end are zero)
    __syncthreads();
    if (n1 > 0) {  // the next chunk's K, into the other buffer (its last reader, the previous
                   // chunk's state update, is behind the barrier above)
      load_tile_async((ci & 1) ? K0s : K1s, a.k, row0 + kPfC, n1);
      cp_async_commit();
    }

    // ---- A = beta_t e^{G_t - G_s} K K^T (s < t); V' = V - Diag(e^G) K S^T --------------------
    {
      float acc[4][4];
      zero_acc(acc);
      warp_mma<4, 8, false, false>(acc, k_b, kLd128, m0, k_b, kLd128, 32 * nh, 0);
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = m0 + gid + 8 * (e >> 1), s = 32 * nh + 8 * nt + 2 * q4 + (e & 1);
          Af[t * kLdF + s] = s < t ? bet[t] * __expf(Gs[t] - Gs[s]) * acc[nt][e] : 0.f;
        }
      float ks[8][4];
      zero_acc(ks);
      mma_state_slab(ks, k_b, sacc);
      store_split_slab(ks, Xhi, Xlo, kLd128, v0, [&](int t, int vv, float x) {
        return __bfloat162float(Vs[t * kLd128 + vv]) - eG[t] * x;
      });
    }
    __syncthreads();
    if (n1 > 0) {  // V is read out: the next chunk's V
      load_tile_async(Vs, a.v, row0 + kPfC, n1);
      cp_async_commit();
    }

    // ---- T = (I + A)^{-1} Diag(beta), split ---------------------------------------------------
    unit_lower_inverse(Af, Rf, xs);
    for (int e = tid; e < kPfC * kPfC; e += kPfThreads) {
      const int t = e >> 6, s = e & 63;  // (blocks above the diagonal of R are never written)
      split_bf16(s <= t ? Rf[t * kLdF + s] * bet[s] : 0.f, Thi[t * kLd64 + s], Tlo[t * kLd64 + s]);
    }
    __syncthreads();

    // ---- U = T V'; O = Diag(e^G) Q S^T (slabs); P = M .* Q K^T --------------------------------
    float uacc[8][4], oacc[8][4];
    zero_acc(uacc);
    mma_slab_split3(uacc, thi_b, tlo_b, xhi_b, xlo_b, v0);
    zero_acc(oacc);
    mma_state_slab(oacc, q_b, sacc);
#pragma unroll
    for (int tt = 0; tt < 8; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) oacc[tt][e] *= eG[16 * (tt >> 1) + gid + 8 * (e >> 1)];
    float pacc[4][4];
    zero_acc(pacc);
    warp_mma<4, 8, false, false>(pacc, q_b, kLd128, m0, k_b, kLd128, 32 * nh, 0);
    __syncthreads();  // V', T and Q are read out
    if (n1 > 0) {  // the next chunk's Q
      load_tile_async(Qs, a.q, row0 + kPfC, n1);
      cp_async_commit();
    }
    store_split_slab(uacc, Xhi, Xlo, kLd128, v0, [](int, int, float x) { return x; });
    store_split(pacc, Thi, Tlo, kLd64, m0, 32 * nh, [&](int t, int s, float x) {
      return s <= t ? __expf(Gs[t] - Gs[s]) * x : 0.f;
    });
    __syncthreads();

    // ---- O += P U; outputs ----------------------------------------------------------------------
    mma_slab_split3(oacc, thi_b, tlo_b, xhi_b, xlo_b, v0);
#pragma unroll
    for (int tt = 0; tt < 8; ++tt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * (tt >> 1) + gid + 8 * hh, vv = v0 + 8 * (tt & 1) + 2 * q4;
        if (t < n) {
          __nv_bfloat162 ov;
          ov.x = __float2bfloat16_rn(oacc[tt][2 * hh]);
          ov.y = __float2bfloat16_rn(oacc[tt][2 * hh + 1]);
          *reinterpret_cast<__nv_bfloat162*>(a.o + (row0 + t) * kPfD + vv) = ov;
        }
      }
    __syncthreads();  // U is read out

    // ---- S = e^{G_C} S + (Diag(e^{G_C - G}) U)^T K -------------------------------------------
    store_split_slab(uacc, Xhi, Xlo, kLd128, v0, [&](int t, int, float x) { return eGC[t] * x; });
    __syncthreads();
    {
      const float eC = eG[kPfC - 1];
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] *= eC;
      // A = (e^{G_C - G} U)^T: stored [t][v] = [k][m]; B = K stored [t][j] = [k][n]
      warp_mma<16, 4, true, true>(sacc, xhi_b, kLd128, v0, k_b, kLd128, 0, 0);
      warp_mma<16, 4, true, true>(sacc, xlo_b, kLd128, v0, k_b, kLd128, 0, 0);
    }
    __syncthreads();  // every warp is done with X and this chunk's K
  }
  // ---- the final state ---------------------------------------------------------------------
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int j = 8 * nt + 2 * q4;
    *reinterpret_cast<float2*>(Sg + (v0 + gid) * kPfD + j) = make_float2(sacc[nt][0], sacc[nt][1]);
    *reinterpret_cast<float2*>(Sg + (v0 + gid + 8) * kPfD + j) = make_float2(sacc[nt][2], sacc[nt][3]);
  }
}

}  // namespace gdnq
