// Blackwell tensor-core (tcgen05) and tensor-memory-accelerator helpers, inline PTX for sm_100a.
//
//  - Tensor memory (TMEM): 128 lanes x 512 32-bit columns per SM. One warp allocates a power of
//    two of columns (>= 32) and frees them before the CTA exits; a warp may only move lanes
//    32 (w % 4) .. 32 (w % 4) + 31 to and from its registers.
//  - tcgen05.mma (kind::f16, bf16 operands, fp32 accumulate, cta_group::1): D [TMEM] (+)= A B,
//    A an M x 16 and B an N x 16 operand in shared memory, described by 64-bit descriptors; one
//    thread issues, tcgen05.commit makes an mbarrier arrive once the issued products are done.
//    With M = 128 row m of D is TMEM lane m, column n its column base + n.
//  - Shared-memory operand tiles use the 128-byte swizzle: a tile is made of 8-row x 128-byte
//    atoms (1024 bytes, 1024-byte aligned), and 16-byte chunk c of row r of an atom sits at chunk
//    c ^ (r & 7). K-major: rows are M (or N) indices, the 64 bf16 of a row are K; the next 8 rows
//    are SBO bytes on, the next 64 K elements are a separate block. MN-major: rows are K indices,
//    the 64 bf16 of a row are M (or N); 8 rows on is SBO, the next 64 M/N elements LBO on.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "device_util.cuh"

namespace gdnq {

// ---- TMEM allocation (called by one whole warp) ---------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// ---- ordering of tensor-core work against thread barriers ----------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
// generic-proxy shared-memory writes made visible to the tensor cores / bulk copies
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// ---- shared-memory operand descriptors -------------------------------------------------------
// 128-byte-swizzled operand starting at shared address `saddr`; lbo / sbo in bytes.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version of sm_100
  d |= (uint64_t)2 << 61;  // 128-byte swizzle
  return d;
}
// K-major operand (8-row groups 1024 bytes apart; the leading offset is unused when swizzled)
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) { return sw128_desc(saddr, 16, 1024); }

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 D, an M x N tile; a_mn / b_mn
// select MN-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled block whose
// base is 1024-byte aligned.
__host__ __device__ constexpr uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)row * 128u + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

// ---- tensor-core products -----------------------------------------------------------------------
// D (+)= A B for one K = 16 step (accumulate = 0 overwrites D). Issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The mbarrier gets one arrival once every product this thread issued so far is complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
          smem_u32(bar))
      : "memory");
}

// ---- TMEM <-> registers (32 lanes x 32 columns per warp; this thread: its lane, 32 columns) ----
// The load waits for its own completion, so the values are ready when it returns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];\ntcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// Store; tc_wait_st() before the values may be used by products.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// ---- TMEM <-> registers in the mma.sync accumulator layout (16 lanes x 8 columns per step) ----
// Shape 16x256b: lane l of the warp holds TMEM lanes base + l / 4 and base + l / 4 + 8, columns
// 2 (l % 4) and 2 (l % 4) + 1 of each 8-column step: acc[n][0..3] = (row l/4, col 8n + 2(l%4)),
// (row l/4, +1), (row l/4 + 8, col), (row l/4 + 8, +1), the C fragment of an m16n8 product.
__device__ __forceinline__ void tmem_st_frag8(uint32_t taddr, const float (&acc)[8][4]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};\n" ::"r"(taddr),
      "f"(acc[0][0]), "f"(acc[0][1]), "f"(acc[0][2]), "f"(acc[0][3]), "f"(acc[1][0]),
      "f"(acc[1][1]), "f"(acc[1][2]), "f"(acc[1][3]), "f"(acc[2][0]), "f"(acc[2][1]),
      "f"(acc[2][2]), "f"(acc[2][3]), "f"(acc[3][0]), "f"(acc[3][1]), "f"(acc[3][2]),
      "f"(acc[3][3]), "f"(acc[4][0]), "f"(acc[4][1]), "f"(acc[4][2]), "f"(acc[4][3]),
      "f"(acc[5][0]), "f"(acc[5][1]), "f"(acc[5][2]), "f"(acc[5][3]), "f"(acc[6][0]),
      "f"(acc[6][1]), "f"(acc[6][2]), "f"(acc[6][3]), "f"(acc[7][0]), "f"(acc[7][1]),
      "f"(acc[7][2]), "f"(acc[7][3])
      : "memory");
}
// Load (waits for completion).
__device__ __forceinline__ void tmem_ld_frag8(uint32_t taddr, float (&acc)[8][4]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31}, [%32];\ntcgen05.wait::ld.sync.aligned;\n"
      : "=f"(acc[0][0]), "=f"(acc[0][1]), "=f"(acc[0][2]), "=f"(acc[0][3]), "=f"(acc[1][0]),
        "=f"(acc[1][1]), "=f"(acc[1][2]), "=f"(acc[1][3]), "=f"(acc[2][0]), "=f"(acc[2][1]),
        "=f"(acc[2][2]), "=f"(acc[2][3]), "=f"(acc[3][0]), "=f"(acc[3][1]), "=f"(acc[3][2]),
        "=f"(acc[3][3]), "=f"(acc[4][0]), "=f"(acc[4][1]), "=f"(acc[4][2]), "=f"(acc[4][3]),
        "=f"(acc[5][0]), "=f"(acc[5][1]), "=f"(acc[5][2]), "=f"(acc[5][3]), "=f"(acc[6][0]),
        "=f"(acc[6][1]), "=f"(acc[6][2]), "=f"(acc[6][3]), "=f"(acc[7][0]), "=f"(acc[7][1]),
        "=f"(acc[7][2]), "=f"(acc[7][3])
      : "r"(taddr)
      : "memory");
}
// One 8-column step of packed 32-bit values (4 per thread) in the same layout.
__device__ __forceinline__ void tmem_st_frag1(uint32_t taddr, uint32_t r0, uint32_t r1,
                                              uint32_t r2, uint32_t r3) {
  asm volatile("tcgen05.st.sync.aligned.16x256b.x1.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(taddr),
               "r"(r0), "r"(r1), "r"(r2), "r"(r3)
               : "memory");
}

// D [TMEM] (+)= A [TMEM, 16-bit values packed two per column, K-consecutive] x B [smem
// descriptor], kind::f16, one K = 16 step. Issued by one thread.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Operand without swizzle: 8 x 16-byte core matrices; lbo / sbo the byte strides between core
// matrices along K and along M / N (MN-major) -- see the canonical layouts above.
__device__ __forceinline__ uint64_t interleave_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version of sm_100; layout type 0: no swizzle
  return d;
}

// ---- tensor-map (TMA) tile loads -------------------------------------------------------------
// Box at coordinates (x, y, z) of a 3-D tensor map into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3, %4}], [%5];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace gdnq
