// Warp-level tensor-core helpers shared by the window and pure-write kernels: ldmatrix loads,
// mma.sync (int8 and bf16), bf16 splitting of fp32 operands, and the digit layout of an exact
// integer mat-vec (an fp32 vector written as a block exponent and three signed 8-bit digits).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "device_util.cuh"

namespace gdnq {

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// x = hi + mid + lo with each part a bf16 (nearest): the three parts carry x's 24 bits.
__device__ __forceinline__ void split3(float x, float& hi, float& mid, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  const float r1 = x - hi;
  mid = __bfloat162float(__float2bfloat16_rn(r1));
  lo = r1 - mid;
}

// Splits a packed bf16 pair scaled by (f0, f1) into three packed bf16 pairs.
__device__ __forceinline__ void split3_pair(uint32_t w, float f0, float f1, uint32_t& h,
                                            uint32_t& m, uint32_t& l) {
  float h0, m0, l0, h1, m1, l1;
  split3(bf16_lo(w) * f0, h0, m0, l0);
  split3(bf16_hi(w) * f1, h1, m1, l1);
  h = pack_bf16(h0, h1);
  m = pack_bf16(m0, m1);
  l = pack_bf16(l0, l1);
}

// Positions of the digit matrix: for int4 codes a 32-column chunk is loaded as 8 consecutive
// columns per lane, which the s8 mma reads as logical k = 4q+e (first 4) and 16+4q+e (next 4).
template <bool INT4>
__device__ __forceinline__ int digit_pos(int j) {
  if constexpr (!INT4) {
    return j;
  } else {
    const int c = j >> 5, jj = j & 31, q = jj >> 3, e = jj & 7;
    return 32 * c + (e < 4 ? 4 * q + e : 16 + 4 * q + e - 4);
  }
}

// Eight int4 codes of one 32-bit word (byte m: column 2m low nibble, 2m+1 high) as 16 x code
// in int8 lanes: e0 = columns 0..3, e1 = columns 4..7.
__device__ __forceinline__ void i4x8_to_s8x16(uint32_t w, uint32_t& e0, uint32_t& e1) {
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;  // even columns, nibble in the high half
  const uint32_t hi = w & 0xF0F0F0F0u;         // odd columns
  e0 = __byte_perm(lo, hi, 0x5140);
  e1 = __byte_perm(lo, hi, 0x7362);
}

// Byte offset of digit (row n, logical k) in the fragment-ordered phase-1 right-hand side: lane
// (n, q4) finds its eight 32-bit b-registers (b0, b1 of the four 32-column chunks) contiguous.
__device__ __forceinline__ int digit_off(int n, int k) {
  const int c = k >> 5, kk = k & 31, half = kk >> 4, q4 = (kk & 15) >> 2, e = kk & 3;
  return ((n * 4 + q4) * 8 + c * 2 + half) * 4 + e;
}

// Writes column j of a vector (entry val, vector absmax m) into the fragment-ordered right-hand
// side as the three signed 8-bit digits of X = rint(val 2^(22-e)), m = f 2^e (0.5 <= f < 1),
// at digit columns n0, n0 + 1, n0 + 2 (X = d1 2^16 + d2 2^8 + d3, |X| <= 2^22). Returns
// 2^(e-22), the value of one unit of X (0 for a negligible vector, whose digits are all 0).
template <bool INT4>
__device__ __forceinline__ float put_digits(uint8_t* Bfrag, int n0, int j, float val, float m) {
  float mul = 0.f, scale = 0.f;
  if (m >= 0x1p-100f) {
    const int e2 = ((__float_as_int(m) >> 23) & 0xFF) - 126;
    mul = __int_as_float((22 - e2 + 127) << 23);
    scale = __int_as_float((e2 - 22 + 127) << 23);
  }
  const int X = __float2int_rn(val * mul);
  const int d3 = (int)(int8_t)(X & 0xFF);
  const int X1 = (X - d3) >> 8;  // exact: X - d3 is a multiple of 256
  const int d2 = (int)(int8_t)(X1 & 0xFF);
  const int d1 = (X1 - d2) >> 8;
  const int k = digit_pos<INT4>(j);
  Bfrag[digit_off(n0, k)] = (uint8_t)d1;
  Bfrag[digit_off(n0 + 1, k)] = (uint8_t)d2;
  Bfrag[digit_off(n0 + 2, k)] = (uint8_t)d3;
  return scale;
}

}  // namespace gdnq
