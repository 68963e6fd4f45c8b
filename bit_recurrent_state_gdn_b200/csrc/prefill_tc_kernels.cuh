// Chunkwise-parallel GDN prefill on the fifth-generation tensor cores (tcgen05) of sm_100a
// ("LinQuant: Functional Invariances for Low-Precision Linear Recurrences", Abstract: prefill of
// a linear recurrence cast as chunked dense products). Scalar gate, 64-token chunks, the UT-form
// chunk algebra of prefill_kernels.cuh (derivation there):
//   A[t][s] = beta_t e^{G_t - G_s} <k_t, k_s> (s < t),   T = (I + A)^{-1} Diag(beta)
//   P[t][s] = e^{G_t - G_s} <q_t, k_s> (s <= t)
//   V' = V - Diag(e^G) K S^T,   U = T V',   O = Diag(e^G) Q S^T + P U
//   S <- e^{G_C} S + U^T Diag(e^{G_C - G}) K
// Two kernels:
//   prefill_chunk_kernel  every chunk of every head in parallel (one CTA each): the gates,
//       [K; Q] K^T on tcgen05 (rows 0-63 K K^T, 64-127 Q K^T), the masks, the triangular
//       inverse in fp32, and T and P as hi + lo bf16 operand planes, written with the gates to
//       a workspace record per chunk. None of this depends on the state.
//   prefill_tc_kernel     one CTA per head, the chunks in order: only the state-dependent work.
//       The state lives in TMEM (fp32, 128 lanes x 128 columns); each chunk reads it once,
//       writes it as hi + lo bf16 planes and stores e^{G_C} S back, onto which the update
//       accumulates. Every product is transposed so that M is the value channel v (TMEM lane):
//       S K^T, S Q^T, V'^T T^T, U^T P^T and S += U~^T K. K, Q and V are staged by 3-D TMA loads
//       with the 128-byte swizzle (zeros past the prompt), the chunk records by bulk copies.
// Thread 0 issues every tcgen05.mma (bf16 operands, fp32 accumulation in TMEM) and commits to
// an mbarrier. fp32 operands enter as two bf16 parts, products of two split operands as three
// terms (hi hi + hi lo + lo hi); q, k, v enter exactly.
#pragma once

#include <cuda_bf16.h>

#include "device_util.cuh"
#include "prefill_args.h"
#include "prefill_kernels.cuh"
#include "tc_util.cuh"

namespace gdnq {

struct PfTcMaps {
  CUtensorMap q, k, v;  // bf16 [heads][L][128], boxes of 64 tokens x 64 channels, 128 B swizzle
};

// A chunk's workspace record: T hi, T lo, P hi, P lo ([64 t][128 B] 128-byte-swizzled planes,
// 8 KB each), then G, e^G, e^{G_C - G}, beta (64 floats each).
constexpr uint32_t kPfRecPlanes = 32768, kPfRecBytes = kPfRecPlanes + 1024;

// Eight consecutive fp32 values as two 16-byte rows of hi and lo bf16 parts.
__device__ __forceinline__ void store_split8(uint32_t hi_addr, uint32_t lo_addr, const float* x) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) split2_bf16(x[2 * i], x[2 * i + 1], h[i], l[i]);
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(hi_addr), "r"(h[0]), "r"(h[1]),
               "r"(h[2]), "r"(h[3])
               : "memory");
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(lo_addr), "r"(l[0]), "r"(l[1]),
               "r"(l[2]), "r"(l[3])
               : "memory");
}

// TMA loads of a chunk's K and Q into one 128-row tile: [2 channel halves][K rows 0-63,
// Q rows 64-127][128 B].
__device__ __forceinline__ void load_kq(uint8_t* t, const PfTcMaps& maps, int chunk, int head,
                                        uint64_t* bar) {
  mbar_arrive_expect_tx(bar, 32768u);
  tma_load_3d(t, &maps.k, 0, kPfC * chunk, head, bar);
  tma_load_3d(t + 16384, &maps.k, 64, kPfC * chunk, head, bar);
  tma_load_3d(t + 8192, &maps.q, 0, kPfC * chunk, head, bar);
  tma_load_3d(t + 16384 + 8192, &maps.q, 64, kPfC * chunk, head, bar);
}

// ---------------------------------------------------------------------------------------------
// The state-independent part of every chunk. Persistent: CTA b takes chunks b, b + grid, ...
// (head-major order); the next chunk's K and Q are loaded while this one is worked on. The
// planes and gates go straight from registers to the chunk's workspace record.
// ---------------------------------------------------------------------------------------------
struct ChunkLayout {
  static constexpr uint32_t KQ = 0;                              // K and Q tile
  static constexpr uint32_t AF = 32768;                          // A (fp32)
  static constexpr uint32_t RF = AF + kPfC * kLdF * 4;           // R (fp32)
  static constexpr uint32_t XS = RF + kPfC * kLdF * 4;           // scratch of the inverse
  static constexpr uint32_t GATE = XS + 3072;                    // G, e^G, e^{G_C - G}, beta
  static constexpr uint32_t BARS = GATE + 1024;
  static constexpr uint32_t TOTAL = BARS + 64;
  static constexpr uint32_t ALLOC = TOTAL + 1024;
};
constexpr uint32_t kChunkCols = 64;
constexpr int kChunkCtasPerSm = 3;

// Eight consecutive fp32 values as hi and lo bf16 parts, 16 bytes each, to global memory.
__device__ __forceinline__ void store_split8_global(uint8_t* hi, uint8_t* lo, const float* x) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) split2_bf16(x[2 * i], x[2 * i + 1], h[i], l[i]);
  *reinterpret_cast<uint4*>(hi) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(lo) = make_uint4(l[0], l[1], l[2], l[3]);
}

__global__ void __launch_bounds__(kPfThreads, kChunkCtasPerSm)
    prefill_chunk_kernel(const PfArgs a, const __grid_constant__ PfTcMaps maps, int total) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = a.L, nch = (L + kPfC - 1) / kPfC;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + ChunkLayout::BARS);
  uint64_t* bar_mma = bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2);
  float* Gs = reinterpret_cast<float*>(sm + ChunkLayout::GATE);
  float* eG = Gs + kPfC;
  float* eGC = eG + kPfC;
  float* bet = eGC + kPfC;
  float* Af = reinterpret_cast<float*>(sm + ChunkLayout::AF);
  float* Rf = reinterpret_cast<float*>(sm + ChunkLayout::RF);
  float* xs = reinterpret_cast<float*>(sm + ChunkLayout::XS);

  if (warp == 0) {
    tmem_alloc(tmem_slot, kChunkCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
    if ((int)blockIdx.x < total)
      load_kq(sm + ChunkLayout::KQ, maps, (int)blockIdx.x % nch, (int)blockIdx.x / nch, bar);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;
  const uint32_t tl = tm + ((uint32_t)(32 * (warp & 3)) << 16);
  constexpr uint32_t ID64 = idesc_bf16(128, 64, false, false);
  uint32_t phase = 0;
  for (int idx = blockIdx.x; idx < total; idx += gridDim.x, phase ^= 1u) {
    const int head = idx / nch, c = idx % nch;
    const int c0 = kPfC * c, n = min(kPfC, L - c0);
    const size_t row0 = (size_t)head * L + c0;
    uint8_t* rec = a.ws + (size_t)idx * kPfRecBytes;  // records are in (head, chunk) order
    bool ok = true;
    if (tid == 0) {  // [K; Q] K^T, then the next chunk's K and Q into the same tile
      tc_fence_after();
      ok = mbar_wait_bounded(bar, phase);
      const uint32_t kq = sb + ChunkLayout::KQ;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
        umma_bf16(tm, kmajor_desc(kq + off), kmajor_desc(kq + off), ID64, kk > 0);
      }
      umma_commit(bar_mma);
    }
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
    if (!mbar_wait_bounded(bar_mma, phase)) ok = false;
    tc_fence_after();
    if (tid == 0 && idx + (int)gridDim.x < total) {
      const int nx = idx + gridDim.x;
      load_kq(sm + ChunkLayout::KQ, maps, nx % nch, nx / nch, bar);
    }
    __syncthreads();  // the gates
    {  // row t of A (TMEM lanes 0-63: warps 0, 1, 4, 5) or P (lanes 64-127: warps 2, 3, 6, 7),
       // columns 32 p .. 32 p + 31 (p = warp / 4)
      const int t = 32 * (warp & 1) + lane, p = warp >> 2;
      float x[32];
      tmem_ld32(tl + 32 * p, x);
      if ((warp & 2) == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int s = 32 * p + i;
          Af[t * kLdF + s] = s < t ? bet[t] * __expf(Gs[t] - Gs[s]) * x[i] : 0.f;
        }
      } else {  // P, to the record
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int s = 32 * p + i;
          x[i] = s <= t ? __expf(Gs[t] - Gs[s]) * x[i] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t off = 16384u + sw128_off(t, 4 * p + q);
          store_split8_global(rec + off, rec + off + 8192u, x + 8 * q);
        }
      }
    }
    if (warp == 4) {  // the gates, to the record
      float* rg = reinterpret_cast<float*>(rec + kPfRecPlanes);
      for (int e = lane; e < 4 * kPfC; e += 32) rg[e] = Gs[e];
    }
    tc_fence_before();
    __syncthreads();
    unit_lower_inverse(Af, Rf, xs);
    for (int e = tid; e < kPfC * 8; e += kPfThreads) {  // T = R Diag(beta), to the record
      const int t = e >> 3, ch = e & 7;
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int s = 8 * ch + i;
        x[i] = s <= t ? Rf[t * kLdF + s] * bet[s] : 0.f;
      }
      const uint32_t off = sw128_off(t, ch);
      store_split8_global(rec + off, rec + off + 8192u, x);
    }
    // a wait that ran out leaves NaN gates: the head's result is not valid
    if (__syncthreads_or(!ok) && tid < 4 * kPfC)
      reinterpret_cast<float*>(rec + kPfRecPlanes)[tid] = __int_as_float(0x7fc00000);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, kChunkCols);
  }
}

// ---------------------------------------------------------------------------------------------
// The chunks of one head in order: the state-dependent part.
// ---------------------------------------------------------------------------------------------
struct TcLayout {
  static constexpr uint32_t KQ0 = 0;            // K and Q tiles of even chunks
  static constexpr uint32_t KQ1 = 32768;        // of odd chunks
  static constexpr uint32_t V = 65536;          // [2 channel halves][64 tokens][128 B]
  static constexpr uint32_t SP = 81920;         // S planes hi / lo, [2 halves][128 v][128 B]
                                                //  each; then U, U~ planes [128 v][128 B]
  static constexpr uint32_t VT = SP + 65536;    // V'^T planes hi / lo, [128 v][128 B]
  static constexpr uint32_t TP = VT + 32768;    // the chunk record: T hi / lo, P hi / lo
  static constexpr uint32_t PP = TP + 16384;
  static constexpr uint32_t GATE = PP + 16384;  // two chunks' gates (G, e^G, e^{G_C - G}, beta)
  static constexpr uint32_t BARS = GATE + 2048; // mbarriers; TMEM address
  static constexpr uint32_t TOTAL = BARS + 128;
  static constexpr uint32_t ALLOC = TOTAL + 1024;  // dynamic size (base aligned inside)
};

constexpr uint32_t kTcColS = 0, kTcColSK = 128, kTcColSQ = 192, kTcColU = 256, kTcColO = 320,
                   kTcCols = 512;

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_tc_kernel(const PfArgs a, const __grid_constant__ PfTcMaps maps) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int head = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = a.L, nch = (L + kPfC - 1) / kPfC;
  uint64_t* bar_kq = reinterpret_cast<uint64_t*>(sm + TcLayout::BARS);  // [2]
  uint64_t* bar_v = bar_kq + 2;
  uint64_t* bar_mma = bar_kq + 3;
  uint64_t* bar_g = bar_kq + 4;   // [2] gates of even / odd chunks
  uint64_t* bar_tp = bar_kq + 6;  // T and P planes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_kq + 7);
  int* fail = reinterpret_cast<int*>(tmem_slot + 1);
  const uint8_t* rec0 = a.ws + (size_t)head * nch * kPfRecBytes;

  if (warp == 0) {
    tmem_alloc(tmem_slot, kTcCols);
    tmem_relinquish();
  }
  auto issue_v = [&](int cc) {
    mbar_arrive_expect_tx(bar_v, 16384u);
    tma_load_3d(sm + TcLayout::V, &maps.v, 0, kPfC * cc, head, bar_v);
    tma_load_3d(sm + TcLayout::V + 8192, &maps.v, 64, kPfC * cc, head, bar_v);
  };
  auto issue_gates = [&](int cc) {
    uint64_t* b = &bar_g[cc & 1];
    mbar_arrive_expect_tx(b, 1024u);
    bulk_g2s(sm + TcLayout::GATE + 1024u * (cc & 1), rec0 + (size_t)cc * kPfRecBytes + kPfRecPlanes,
             1024u, b);
  };
  auto issue_planes = [&](int cc) {
    mbar_arrive_expect_tx(bar_tp, kPfRecPlanes);
    bulk_g2s(sm + TcLayout::TP, rec0 + (size_t)cc * kPfRecBytes, kPfRecPlanes, bar_tp);
  };
  if (tid == 0) {
    for (int i = 0; i < 7; ++i) mbar_init(&bar_kq[i], 1);
    *fail = 0;
    fence_barrier_init();
    if (nch > 0) {
      load_kq(sm + TcLayout::KQ0, maps, 0, head, &bar_kq[0]);
      issue_v(0);
      issue_gates(0);
      issue_planes(0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;
  // this thread's TMEM lane (value channel v) and column half
  const int v = 32 * (warp & 3) + lane, half = warp >> 2;
  const uint32_t tl = tm + ((uint32_t)(32 * (warp & 3)) << 16);
  float* Sg = a.S + (size_t)head * kPfD * kPfD;

  // the initial state into TMEM (row v, columns 64 half ..)
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    float x[32];
    const float4* src = reinterpret_cast<const float4*>(Sg + v * kPfD + 64 * half + 32 * p);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 f = src[i];
      x[4 * i] = f.x; x[4 * i + 1] = f.y; x[4 * i + 2] = f.z; x[4 * i + 3] = f.w;
    }
    tmem_st32(tl + kTcColS + 64 * half + 32 * p, x);
  }
  tc_wait_st();

  uint32_t mma_phase = 0;
  auto wait_products = [&]() {
    if (!mbar_wait_bounded(bar_mma, mma_phase)) *fail = 1;
    mma_phase ^= 1u;
    tc_fence_after();
  };
  constexpr uint32_t ID64 = idesc_bf16(128, 64, false, false);
  constexpr uint32_t ID128 = idesc_bf16(128, 128, false, false);
  constexpr uint32_t ID128_BMN = idesc_bf16(128, 128, false, true);
  static_assert(kTcColSQ == kTcColSK + 64, "S Q^T follows S K^T");

  int c_stop = nch;  // the chunk a failed run stopped at (its copies are in flight)
  for (int c = 0; c < nch; ++c) {
    const int c0 = kPfC * c, n = min(kPfC, L - c0), buf = c & 1;
    const size_t row0 = (size_t)head * L + c0;
    const uint32_t kq = sb + (buf ? TcLayout::KQ1 : TcLayout::KQ0);
    const float* Gs = reinterpret_cast<const float*>(sm + TcLayout::GATE + 1024u * buf);
    const float* eG = Gs + kPfC;
    const float* eGC = eG + kPfC;
    tc_fence_before();
    __syncthreads();  // every thread is done with the previous chunk
    if (*fail) {
      c_stop = c;
      break;
    }
    if (tid == 0 && c + 1 < nch) issue_gates(c + 1);
    if (!mbar_wait_bounded(&bar_g[buf], (uint32_t)(c >> 1) & 1u)) *fail = 1;

    // ---- the state: split operand planes of S; e^{G_C} S back into TMEM ----------------------
    {
      const float eC = eG[kPfC - 1];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        float x[32];
        tmem_ld32(tl + kTcColS + 64 * half + 32 * p, x);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t off = TcLayout::SP + 16384u * half + sw128_off(v, 4 * p + q);
          store_split8(sb + off, sb + off + 32768u, x + 8 * q);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] *= eC;
        tmem_st32(tl + kTcColS + 64 * half + 32 * p, x);
      }
    }
    fence_async_smem();
    tc_wait_st();
    tc_fence_before();
    __syncthreads();

    // ---- products S K^T, S Q^T; the next chunk's K and Q ----------------------------------------
    if (tid == 0) {
      tc_fence_after();
      if (!mbar_wait_bounded(&bar_kq[buf], (uint32_t)(c >> 1) & 1u)) *fail = 1;
      // one N = 128 product: the tile's rows 0-63 are K, 64-127 Q, so [S K^T | S Q^T] lands in
      // the adjacent column blocks kTcColSK, kTcColSQ
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
          umma_bf16(tm + kTcColSK, kmajor_desc(sb + TcLayout::SP + 32768u * p + off),
                    kmajor_desc(kq + off), ID128, (p | kk) != 0);
        }
      umma_commit(bar_mma);
      if (c + 1 < nch) load_kq(sm + (buf ? TcLayout::KQ0 : TcLayout::KQ1), maps, c + 1, head, &bar_kq[buf ^ 1]);
    }
    wait_products();
    if (!mbar_wait_bounded(bar_v, (uint32_t)c & 1u)) *fail = 1;

    // ---- V'^T[v][t] = V[t][v] - e^{G_t} (S K^T)[v][t], tokens 32 half .. ----------------------
    {
      const __nv_bfloat16* Vs = reinterpret_cast<const __nv_bfloat16*>(sm + TcLayout::V);
      const uint32_t vb = (uint32_t)(v >> 6) * 8192u, vc = (uint32_t)((v & 63) >> 3), ve = v & 7;
      float x[32];
      tmem_ld32(tl + kTcColSK + 32 * half, x);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int t = 32 * half + i;
        const float vt = __bfloat162float(Vs[(vb + sw128_off(t, (int)vc)) / 2 + ve]);
        x[i] = vt - eG[t] * x[i];
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t off = TcLayout::VT + sw128_off(v, 4 * half + q);
        store_split8(sb + off, sb + off + 16384u, x + 8 * q);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && c + 1 < nch) issue_v(c + 1);  // V is read out

    // ---- U^T = V'^T T^T (three terms) ----------------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      if (!mbar_wait_bounded(bar_tp, (uint32_t)c & 1u)) *fail = 1;
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        const uint32_t va = sb + TcLayout::VT + (term == 2 ? 16384u : 0u);
        const uint32_t tb = sb + TcLayout::TP + (term == 1 ? 8192u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tm + kTcColU, kmajor_desc(va + 32u * kk), kmajor_desc(tb + 32u * kk), ID64,
                    (term | kk) != 0);
      }
      umma_commit(bar_mma);
    }
    wait_products();

    // ---- U and U~ = U Diag(e^{G_C - G}) as split planes ---------------------------------------
    {
      float x[32];
      tmem_ld32(tl + kTcColU + 32 * half, x);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t off = sw128_off(v, 4 * half + q);
        store_split8(sb + TcLayout::SP + off, sb + TcLayout::SP + 16384u + off, x + 8 * q);
        float y[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = x[8 * q + i] * eGC[32 * half + 8 * q + i];
        store_split8(sb + TcLayout::SP + 32768u + off, sb + TcLayout::SP + 49152u + off, y);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O^T = U^T P^T (three terms); S += U~^T K (two terms); the next chunk's T and P ------
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        const uint32_t ua = sb + TcLayout::SP + (term == 2 ? 16384u : 0u);
        const uint32_t pb = sb + TcLayout::PP + (term == 1 ? 8192u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tm + kTcColO, kmajor_desc(ua + 32u * kk), kmajor_desc(pb + 32u * kk), ID64,
                    (term | kk) != 0);
      }
#pragma unroll
      for (int term = 0; term < 2; ++term) {
        const uint32_t ua = sb + TcLayout::SP + 32768u + 16384u * term;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tm + kTcColS, kmajor_desc(ua + 32u * kk),
                    sw128_desc(kq + 2048u * kk, 16384u, 1024u), ID128_BMN, 1u);
      }
      umma_commit(bar_mma);
    }
    wait_products();
    if (tid == 0 && c + 1 < nch) issue_planes(c + 1);  // T and P are read out

    // ---- outputs o_t = e^{G_t} (S Q^T)[v][t] + O^T[v][t] -------------------------------------
    {
      float sq[32], oo[32];
      tmem_ld32(tl + kTcColSQ + 32 * half, sq);
      tmem_ld32(tl + kTcColO + 32 * half, oo);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int t = 32 * half + i;
        if (t < n) a.o[(row0 + t) * kPfD + v] = __float2bfloat16_rn(eG[t] * sq[i] + oo[i]);
      }
    }
  }

  // ---- the final state (NaN on a wait that ran out: the head's result is not valid) --------
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const bool bad = *fail != 0;
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    float x[32];
    tmem_ld32(tl + kTcColS + 64 * half + 32 * p, x);
    float4* dst = reinterpret_cast<float4*>(Sg + v * kPfD + 64 * half + 32 * p);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = bad ? make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                 __int_as_float(0x7fc00000), __int_as_float(0x7fc00000))
                   : make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
  }
  if (bad && tid == 0) {  // products and the stopped chunk's copies still in flight
    mbar_wait_bounded(bar_mma, mma_phase);
    if (c_stop < nch) {
      const int b = c_stop & 1;
      (void)mbar_wait_bounded(&bar_g[b], (uint32_t)(c_stop >> 1) & 1u);
      (void)mbar_wait_bounded(&bar_kq[b], (uint32_t)(c_stop >> 1) & 1u);
      (void)mbar_wait_bounded(bar_v, (uint32_t)c_stop & 1u);
      (void)mbar_wait_bounded(bar_tp, (uint32_t)c_stop & 1u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, kTcCols);
  }
}

}  // namespace gdnq
