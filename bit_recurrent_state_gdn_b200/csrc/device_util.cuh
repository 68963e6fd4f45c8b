// Device helpers for the sm_100a kernels: bulk async copies (TMA, 1-D form) completing on an
// mbarrier, a bounded mbarrier wait, and exact code / bf16 conversions.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace gdnq {

// Upper bound on mbarrier polls before a kernel gives up on a staging copy and reports
// GDN_DEVICE_WAIT_TIMEOUT instead of spinning forever.
constexpr uint32_t kWaitPollLimit = 1u << 24;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes the initialised barrier visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Global -> shared bulk copy. dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for the phase with the given parity to complete; false after kWaitPollLimit polls.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitPollLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Tile swizzle of the stored state. A tile with RB-byte rows keeps its 16-byte chunks permuted
// within each row: chunk c of row `row` lives at chunk c ^ x(row), x(row) = row & 7 for rows of
// 128 bytes or more, (row * RB / 128) & (RB / 16 - 1) for shorter rows. Eight consecutive rows
// read at one column then fall in distinct shared-memory banks, and a plain 1-D bulk copy of
// the tile keeps the property. Returns the byte offset of logical byte b of the row.
template <int RB>
__host__ __device__ constexpr uint32_t swz(int row, int b) {
  static_assert(RB >= 16 && (RB & (RB - 1)) == 0, "row bytes: a power of two >= 16");
  if constexpr (RB >= 128) {
    return (uint32_t)row * RB + ((((b >> 4) ^ (row & 7)) << 4) | (b & 15));
  } else {
    return (uint32_t)row * RB + ((((b >> 4) ^ ((row * RB / 128) & (RB / 16 - 1))) << 4) | (b & 15));
  }
}

// Element offset of element `col` of row `row` in a swizzled tile of T with D columns.
template <typename T, int D>
__host__ __device__ constexpr uint32_t swz_el(int row, int col) {
  return swz<D * (int)sizeof(T)>(row, col * (int)sizeof(T)) / (uint32_t)sizeof(T);
}

// Barrier among the 256 computing threads of a CTA (named barrier 1): in the persistent step
// kernel a 9th warp stages data and never joins; in the other kernels it is every thread.
constexpr int kComputeThreads = 256;

__device__ __forceinline__ void csync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(kComputeThreads) : "memory");
}

// Barrier of warps 0-3 only (named barrier 2), for work split between two warp groups.
__device__ __forceinline__ void xsync() {
  asm volatile("bar.sync 2, %0;\n" ::"n"(kComputeThreads / 2) : "memory");
}

// Barrier of warps 4-7 only (named barrier 3).
__device__ __forceinline__ void ysync() {
  asm volatile("bar.sync 3, %0;\n" ::"n"(kComputeThreads / 2) : "memory");
}

// csync() that also returns whether any computing thread passed a nonzero `pred`.
__device__ __forceinline__ int csync_or(int pred) {
  int out;
  asm volatile(
      "{\n"
      " .reg .pred p, q;\n"
      " setp.ne.s32 p, %1, 0;\n"
      " barrier.cta.red.or.pred q, 1, %2, p;\n"
      " selp.s32 %0, 1, 0, q;\n"
      "}\n"
      : "=r"(out)
      : "r"(pred), "n"(kComputeThreads)
      : "memory");
  return out;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// 2^x on the hardware path (flushes results below 2^-126 to zero).
__device__ __forceinline__ float exp2_hw(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// e^x through the hardware base-2 exponential (flushes results below 2^-126 to zero).
__device__ __forceinline__ float fast_exp(float x) { return exp2_hw(x * 1.4426950408889634f); }

// rint of the correctly rounded quotient x / s (|x / s| <= 128), given inv = the correctly
// rounded 1 / s. q = x * inv differs from x / s by at most 2 rounding errors of size
// 2^-24 * 128 = 2^-17, and the rounded quotient from x / s by one more, so q and the rounded
// quotient lie on the same side of every half-integer unless q is within 2^-15 of one; only
// there is the quotient formed by a correctly rounded division.
// |q - rint(q)| is the distance to the nearest integer, near 1/2 only near a half-integer; a
// non-finite q (a reciprocal that overflowed) also takes the division.
__device__ __forceinline__ float rint_quotient(float x, float s, float inv) {
  const float q = x * inv;
  const float r = rintf(q);
  if (!(fabsf(q - r) <= 0.5f - 0x1p-14f)) return rintf(__fdiv_rn(x, s));
  return r;
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic, round to nearest) -------------------------
struct F2 {
  uint64_t v;
};
__device__ __forceinline__ F2 f2(float lo, float hi) {
  F2 r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(r.v) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_get(F2 a, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(lo), "=f"(hi) : "l"(a.v));
}
__device__ __forceinline__ F2 f2_fma(F2 a, F2 b, F2 c) {
  F2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(d.v) : "l"(a.v), "l"(b.v), "l"(c.v));
  return d;
}
__device__ __forceinline__ F2 f2_mul(F2 a, F2 b) {
  F2 d;
  asm("mul.rn.f32x2 %0, %1, %2;\n" : "=l"(d.v) : "l"(a.v), "l"(b.v));
  return d;
}
__device__ __forceinline__ F2 f2_add(F2 a, F2 b) {
  F2 d;
  asm("add.rn.f32x2 %0, %1, %2;\n" : "=l"(d.v) : "l"(a.v), "l"(b.v));
  return d;
}

// Correctly rounded quotients x / s of a pair, from inv = the correctly rounded 1 / s and
// ninv_s = -s: q1 = x * inv is within one ulp of x / s, the remainder x - q1 s is exact in one
// fma, and q1 + remainder * inv rounded once is the correctly rounded quotient (Markstein's
// correction: P. Markstein, IBM J. Res. Dev. 34(1), 1990; also Muller et al., Handbook of
// Floating-Point Arithmetic, the theorem on correcting a quotient with an fma). Valid while
// x / s and 1 / s are normal and finite.
__device__ __forceinline__ F2 f2_quot(F2 x, F2 inv, F2 neg_s) {
  const F2 q1 = f2_mul(x, inv);
  const F2 r = f2_fma(q1, neg_s, x);
  return f2_fma(r, inv, q1);
}

// The correctly rounded quotient x / d given inv_d = the correctly rounded 1 / d (the same
// correction, scalar; d a constant or not). Valid while x / d is normal or zero and 1 / d is
// finite and normal.
__device__ __forceinline__ float quot_const(float x, float d, float inv_d) {
  const float q1 = x * inv_d;
  const float r = fmaf(-q1, d, x);
  return fmaf(r, inv_d, q1);
}

// ---- exact conversions -------------------------------------------------------------------
// Four int8 codes (two's complement, byte e = code e) to fp32: bias each byte to b + 128,
// place it in the mantissa of 2^23 (0x4B0000xx = 2^23 + xx) and subtract 2^23 + 128.
__device__ __forceinline__ void i8x4_to_f32(uint32_t w, float* f) {
  const uint32_t x = w ^ 0x80808080u;
  f[0] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7650)) - 8388736.f;
  f[1] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7651)) - 8388736.f;
  f[2] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7652)) - 8388736.f;
  f[3] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7653)) - 8388736.f;
}

// Eight int4 codes (one 32-bit word: byte m holds column 2m low, 2m+1 high; 4-bit two's
// complement) to fp32 in column order: bias each nibble to c + 8 and use the same 2^23 trick.
__device__ __forceinline__ void i4x8_to_f32(uint32_t w, float* f) {
  const uint32_t x = w ^ 0x88888888u;
  const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    f[2 * m] = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650 + m)) - 8388616.f;
    f[2 * m + 1] = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650 + m)) - 8388616.f;
  }
}

// The same two conversions with the bias subtractions done on packed pairs.
__device__ __forceinline__ void i8x4_to_f32_2(uint32_t w, float* f) {
  const uint32_t x = w ^ 0x80808080u;
  const F2 bias = f2(-8388736.f, -8388736.f);
  const F2 a = f2_add(f2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7650)),
                         __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7651))), bias);
  const F2 b = f2_add(f2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7652)),
                         __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7653))), bias);
  f2_get(a, f[0], f[1]);
  f2_get(b, f[2], f[3]);
}

__device__ __forceinline__ void i4x8_to_f32_2(uint32_t w, float* f) {
  const uint32_t x = w ^ 0x88888888u;
  const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
  const F2 bias = f2(-8388616.f, -8388616.f);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const F2 v = f2_add(f2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650 + m)),
                           __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650 + m))), bias);
    f2_get(v, f[2 * m], f[2 * m + 1]);
  }
}

// Packed-pair forms: int8 codes of one word as (c0, c1), (c2, c3); int4 codes of one word as
// (c0, c1) .. (c6, c7).
__device__ __forceinline__ void i8x4_to_f2(uint32_t w, F2* out) {
  const uint32_t x = w ^ 0x80808080u;
  const F2 bias = f2(-8388736.f, -8388736.f);
  out[0] = f2_add(f2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7650)),
                     __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7651))), bias);
  out[1] = f2_add(f2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7652)),
                     __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7653))), bias);
}

__device__ __forceinline__ void i4x8_to_f2(uint32_t w, F2* out) {
  const uint32_t x = w ^ 0x88888888u;
  const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
  const F2 bias = f2(-8388616.f, -8388616.f);
#pragma unroll
  for (int m = 0; m < 4; ++m)
    out[m] = f2_add(f2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650 + m)),
                       __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650 + m))), bias);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <typename T>
struct Num;

template <>
struct Num<float> {
  __device__ __forceinline__ static float to_f(float x) { return x; }
  __device__ __forceinline__ static float from_f(float x) { return x; }
  // n consecutive elements (n a multiple of 4, p 16-byte aligned) to fp32
  template <int N>
  __device__ __forceinline__ static void load(const float* p, float* out) {
#pragma unroll
    for (int e = 0; e < N; e += 4) {
      const float4 t = *reinterpret_cast<const float4*>(p + e);
      out[e] = t.x;
      out[e + 1] = t.y;
      out[e + 2] = t.z;
      out[e + 3] = t.w;
    }
  }
};

template <>
struct Num<__nv_bfloat16> {
  __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
  template <int N>
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int e = 0; e < N; e += 8) {
        const uint4 t = *reinterpret_cast<const uint4*>(p + e);
        out[e] = bf16_lo(t.x);
        out[e + 1] = bf16_hi(t.x);
        out[e + 2] = bf16_lo(t.y);
        out[e + 3] = bf16_hi(t.y);
        out[e + 4] = bf16_lo(t.z);
        out[e + 5] = bf16_hi(t.z);
        out[e + 6] = bf16_lo(t.w);
        out[e + 7] = bf16_hi(t.w);
      }
    } else {
#pragma unroll
      for (int e = 0; e < N; ++e) out[e] = __bfloat162float(p[e]);
    }
  }
};

}  // namespace gdnq
