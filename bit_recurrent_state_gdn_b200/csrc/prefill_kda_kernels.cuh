// Chunkwise-parallel prefill with a per-key-channel gate (Kimi Delta Attention, KDA, which
// "LeapQuant: Efficient Linear Attention with Accurate Recurrent State Quantization", Abstract,
// names beside GDN), the counterpart of the scalar-gate kernels in prefill_tc_kernels.cuh
// ("LinQuant: Functional Invariances for Low-Precision Linear Recurrences", Abstract: prefill of
// a linear recurrence cast as chunked dense matmuls), on the fifth-generation tensor cores.
//
// The recurrence S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, a_t = e^{g_t}
// per key channel, unrolled over a chunk with the per-channel cumulative log-gate G_t (a vector):
//   u_t     = beta_t (v_t - S (e^{G_t} .* k_t) - sum_{s<t} u_s <e^{G_t - G_s} .* k_s, k_t>)
//   o_t     = S (e^{G_t} .* q_t) + sum_{s<=t} u_s <e^{G_t - G_s} .* k_s, q_t>
//   S_next  = S Diag(e^{G_C}) + sum_s u_s (e^{G_C - G_s} .* k_s)^T
// The pairwise decays e^{G_t - G_s} factor through a reference token r of the chunk,
// e^{G_t - G_r} e^{G_r - G_s}, which turns both C x C matrices into products of decayed key and
// query tiles (Kt = K e^{G - G_r}, Qt = Q e^{G - G_r}, Kh = K e^{G_r - G}):
//   A = beta_t (Kt Kh^T)[t][s] (s < t),   P = (Qt Kh^T)[t][s] (s <= t),   T = (I + A)^{-1} Diag(beta)
//   V' = V - Kt S_r^T,  O = Qt S_r^T + P U,  U = T V',  S_r = S Diag(e^{G_r})
//   S_next = S Diag(e^{G_C}) + U^T (K e^{G_C - G}).
// Chunks are 16 tokens with r the eighth, so every factor spans at most 8 tokens of decay: the
// factors stay finite in fp32 (and in bf16, which has fp32's exponent range) while every
// channel's log-gate summed over 8 consecutive tokens is above -80. The triangular inverse is a
// single 16 x 16 forward substitution.
//
// One CTA per head, 256 threads. The state lives in TMEM (fp32, lane = value channel v, column
// = key channel j). Every state product is transposed so that M is the value channel: per chunk
//   [S_r Kt^T | S_r Qt^T]  (M = 128, N = 32, K = 128),   U^T = V'^T T^T  (N = 16, K = 16),
//   O^T = S_r Qt^T + U^T P^T  (N = 16, K = 16),          S += U^T Kc     (N = 128, K = 16),
// on tcgen05.mma (bf16 operands, fp32 in TMEM) issued by thread 0; fp32 operands enter as hi + lo
// bf16 parts (three products: hi hi, hi lo, lo hi). The small state-independent products A and P
// (16 x 16 x 128) run on mma.sync beside the first state product.
#pragma once

#include "prefill_kernels.cuh"
#include "prefill_tc_kernels.cuh"

namespace gdnq {

constexpr int kKc = 16;       // chunk length
constexpr int kKref = 7;      // the chunk's reference token
constexpr int kLd16 = 24;     // bf16 row stride of 16 x 16 tiles (48 B)

// Shared memory (bytes, from a 1024-byte aligned base). Two stages of raw chunk inputs, then
// the operand planes of the tensor-core products and the small tiles of A and P.
struct KdaLayout {
  static constexpr uint32_t T128 = kKc * kLd128 * 2;  // a padded 16 x 128 bf16 tile
  static constexpr uint32_t RQ = 0;                    // q, k, v (bf16), g (fp32), beta (fp32)
  static constexpr uint32_t RK = RQ + T128;
  static constexpr uint32_t RV = RK + T128;
  static constexpr uint32_t RG = RV + T128;
  static constexpr uint32_t RB = RG + kKc * kPfD * 4;
  static constexpr uint32_t STAGE = RB + kKc * 4;
  static constexpr uint32_t SP = (2 * STAGE + 1023u) & ~1023u;  // S_r hi / lo: [2 j-halves][128 v][128 B]
  static constexpr uint32_t KQT = SP + 65536;   // [Kt; Qt] hi / lo: [2 j-halves][32 rows][128 B]
  static constexpr uint32_t KCS = KQT + 16384;  // Kc hi / lo, MN-major: [2 j-halves][16 s][128 B]
  static constexpr uint32_t VPC = KCS + 8192;   // V'^T hi / lo, core matrices [16][2][8 x 16 B]
  static constexpr uint32_t UPC = VPC + 8192;   // U^T hi / lo, the same
  static constexpr uint32_t TPC = UPC + 8192;   // T hi / lo, core matrices [2][2][8 x 16 B]
  static constexpr uint32_t PPC = TPC + 1024;   // P hi / lo, the same
  static constexpr uint32_t KT = PPC + 1024;    // padded Kt, Qt, Kh hi / lo (the A / P partials)
  static constexpr uint32_t QT = KT + 2 * T128;
  static constexpr uint32_t KH = QT + 2 * T128;
  static constexpr uint32_t AF = KH + 2 * T128;        // A, fp32 16 x 17
  static constexpr uint32_t PART = AF + kKc * 17 * 4;  // per-warp partial A / P, 8 x 256 fp32
  static constexpr uint32_t ER = PART + 8 * 256 * 4;   // e^{G_r}, 128 fp32
  static constexpr uint32_t EC = ER + kPfD * 4;        // e^{G_C}, 128 fp32
  static constexpr uint32_t BARS = EC + kPfD * 4;      // the products' mbarrier; TMEM address
  static constexpr uint32_t TOTAL = BARS + 64;
  static constexpr uint32_t ALLOC = TOTAL + 1024;      // dynamic size (base aligned inside)
};
static_assert(KdaLayout::STAGE % 16 == 0 && KdaLayout::AF % 16 == 0, "16-byte aligned tiles");
static_assert(KdaLayout::KQT % 1024 == 0 && KdaLayout::KCS % 1024 == 0, "swizzle atoms aligned");
static_assert(KdaLayout::ALLOC <= 227 * 1024, "one CTA per SM");
constexpr uint32_t kKdaColS = 0, kKdaColSK = 128, kKdaColSQ = 144, kKdaColU = 160, kKdaCols = 256;

// Byte offset of element (m, k) of an M x 16 bf16 K-major operand of 8 x 16-byte core matrices
// (no swizzle): core matrix (m / 8, k / 8), 256 bytes per 8 rows, 128 bytes per 8 k.
__host__ __device__ constexpr uint32_t core16_off(int m, int k) {
  return (uint32_t)(m >> 3) * 256u + (uint32_t)(k >> 3) * 128u + (uint32_t)(m & 7) * 16u +
         (uint32_t)(k & 7) * 2u;
}
// Descriptor of such an operand (K-major: core matrices 128 bytes apart along K, 256 along M).
__device__ __forceinline__ uint64_t core16_desc(uint32_t saddr) {
  return interleave_desc(saddr, 128u, 256u);
}

// Eight TMEM columns of this thread's lane (waits for completion).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Raw inputs of chunk rows [row0, row0 + n) of the flattened [head][L] token index into a stage
// (rows >= n zero-filled): q, k, v one 16-byte piece per thread per tile, g two, beta one float
// for threads 0-15.
__device__ __forceinline__ void kda_load_chunk(uint8_t* st, const PfArgs& a, size_t row0, int n) {
  const int tid = threadIdx.x;
  {
    const int r = tid >> 4, ch = tid & 15, ok = r < n;
    const size_t off = (row0 + (ok ? r : 0)) * kPfD + 8 * ch;
    const uint32_t d = 2u * (r * kLd128 + 8 * ch);
    cp_async16(st + KdaLayout::RQ + d, a.q + off, ok ? 16 : 0);
    cp_async16(st + KdaLayout::RK + d, a.k + off, ok ? 16 : 0);
    cp_async16(st + KdaLayout::RV + d, a.v + off, ok ? 16 : 0);
  }
#pragma unroll
  for (int e = tid; e < kKc * 32; e += kPfThreads) {
    const int r = e >> 5, ch = e & 31, ok = r < n;
    cp_async16(st + KdaLayout::RG + 4u * (r * kPfD + 4 * ch),
               a.g + (row0 + (ok ? r : 0)) * kPfD + 4 * ch, ok ? 16 : 0);
  }
  if (tid < kKc) cp_async4(st + KdaLayout::RB + 4 * tid, a.beta + row0 + (tid < n ? tid : 0), tid < n ? 4 : 0);
}

// Two adjacent fp32 values as hi / lo bf16 pairs at element idx of the tiles hi and lo.
__device__ __forceinline__ void put_split2(uint8_t* hi, uint8_t* lo, int idx, float x, float y) {
  uint32_t h, l;
  split2_bf16(x, y, h, l);
  reinterpret_cast<uint32_t*>(hi)[idx >> 1] = h;
  reinterpret_cast<uint32_t*>(lo)[idx >> 1] = l;
}

__global__ void __launch_bounds__(kPfThreads, 1) prefill_kda_kernel(const PfArgs a) {
  using L_ = KdaLayout;
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int head = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, q4 = lane & 3;
  const int L = a.L;
  const float* ER = reinterpret_cast<const float*>(sm + L_::ER);
  const float* EC = reinterpret_cast<const float*>(sm + L_::EC);
  float* PART = reinterpret_cast<float*>(sm + L_::PART);
  uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + L_::BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
  int* fail = reinterpret_cast<int*>(tmem_slot + 1);

  if (warp == 0) {
    tmem_alloc(tmem_slot, kKdaCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_mma, 1);
    *fail = 0;
    fence_barrier_init();
  }
  if (L > 0) kda_load_chunk(sm, a, (size_t)head * L, min(kKc, L));
  cp_async_commit();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;
  // this thread's TMEM lane (value channel v) and column half
  const int v = 32 * (warp & 3) + lane, half = warp >> 2;
  const uint32_t tl = tm + ((uint32_t)(32 * (warp & 3)) << 16);
  float* Sg = a.S + (size_t)head * kPfD * kPfD;
#pragma unroll
  for (int p = 0; p < 2; ++p) {  // the initial state into TMEM (row v, columns 64 half ..)
    float x[32];
    const float4* src = reinterpret_cast<const float4*>(Sg + v * kPfD + 64 * half + 32 * p);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 f = src[i];
      x[4 * i] = f.x; x[4 * i + 1] = f.y; x[4 * i + 2] = f.z; x[4 * i + 3] = f.w;
    }
    tmem_st32(tl + kKdaColS + 64 * half + 32 * p, x);
  }
  tc_wait_st();

  uint32_t mma_phase = 0;
  auto wait_products = [&]() {
    if (!mbar_wait_bounded(bar_mma, mma_phase)) *fail = 1;
    mma_phase ^= 1u;
    tc_fence_after();
  };
  constexpr uint32_t ID32 = idesc_bf16(128, 32, false, false);
  constexpr uint32_t ID16 = idesc_bf16(128, 16, false, false);
  constexpr uint32_t ID128_BMN = idesc_bf16(128, 128, false, true);

  for (int c0 = 0, ci = 0; c0 < L; c0 += kKc, ++ci) {
    const int n = min(kKc, L - c0);
    const size_t row0 = (size_t)head * L + c0;
    const uint32_t so = (ci & 1) * L_::STAGE;
    const uint8_t* st = sm + so;
    // the next chunk's inputs into the other stage (its last reader, the previous chunk's
    // V' step, is behind that chunk's later barriers)
    if (c0 + kKc < L) kda_load_chunk(sm + (L_::STAGE - so), a, row0 + kKc, min(kKc, L - c0 - kKc));
    cp_async_commit();
    cp_async_wait_one();
    tc_fence_before();
    __syncthreads();  // this chunk's inputs; every thread done with the previous chunk
    tc_fence_after();
    if (*fail) break;

    // ---- decayed operands: thread = (channels 2 jp, 2 jp + 1; tokens 4 tq..4 tq + 3) ----------
    // (cumulative log-gates in base 2, G log2(e), so each factor is one hardware exp2)
    {
      constexpr float kLog2e = 1.4426950408889634f;
      const int jp = tid & 63, tq = tid >> 6, j0 = 2 * jp;
      const int jh = j0 >> 6, jc = (j0 & 63) >> 3, je = j0 & 7;
      const float* G = reinterpret_cast<const float*>(st + L_::RG);
      float2 run = make_float2(0.f, 0.f), gr = run, gt[4];
#pragma unroll
      for (int t = 0; t < kKc; ++t) {
        const float2 gg = *reinterpret_cast<const float2*>(G + t * kPfD + j0);
        run.x = fmaf(gg.x, kLog2e, run.x);
        run.y = fmaf(gg.y, kLog2e, run.y);
        if (t == kKref) gr = run;
        if ((t >> 2) == tq) gt[t & 3] = run;
      }
      const float2 gc = run;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 4 * tq + i, idx = t * kLd128 + j0;
        const float dx = gt[i].x - gr.x, dy = gt[i].y - gr.y;
        const float tx = fast_exp2(dx), ty = fast_exp2(dy);    // e^{G_t - G_r}
        const float hx = fast_exp2(-dx), hy = fast_exp2(-dy);  // e^{G_r - G_t}
        const float cx = fast_exp2(gc.x - gt[i].x), cy = fast_exp2(gc.y - gt[i].y);  // e^{G_C - G_t}
        const float2 kk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(st + L_::RK + 2 * idx));
        const float2 qq = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(st + L_::RQ + 2 * idx));
        const float ktx = kk.x * tx, kty = kk.y * ty, qtx = qq.x * tx, qty = qq.y * ty;
        put_split2(sm + L_::KT, sm + L_::KT + L_::T128, idx, ktx, kty);
        put_split2(sm + L_::QT, sm + L_::QT + L_::T128, idx, qtx, qty);
        put_split2(sm + L_::KH, sm + L_::KH + L_::T128, idx, kk.x * hx, kk.y * hy);
        // the tensor-core operands: [Kt; Qt] rows t and 16 + t, Kc row t (128-byte swizzle)
        const uint32_t okt = (uint32_t)jh * 4096u + sw128_off(t, jc) + 2u * je;
        const uint32_t oqt = (uint32_t)jh * 4096u + sw128_off(kKc + t, jc) + 2u * je;
        const uint32_t okc = (uint32_t)jh * 2048u + sw128_off(t, jc) + 2u * je;
        uint32_t h, l;
        split2_bf16(ktx, kty, h, l);
        *reinterpret_cast<uint32_t*>(sm + L_::KQT + okt) = h;
        *reinterpret_cast<uint32_t*>(sm + L_::KQT + 8192u + okt) = l;
        split2_bf16(qtx, qty, h, l);
        *reinterpret_cast<uint32_t*>(sm + L_::KQT + oqt) = h;
        *reinterpret_cast<uint32_t*>(sm + L_::KQT + 8192u + oqt) = l;
        split2_bf16(kk.x * cx, kk.y * cy, h, l);
        *reinterpret_cast<uint32_t*>(sm + L_::KCS + okc) = h;
        *reinterpret_cast<uint32_t*>(sm + L_::KCS + 4096u + okc) = l;
      }
      if (tq == 0) {
        *reinterpret_cast<float2*>(sm + L_::ER + 4 * j0) = make_float2(fast_exp2(gr.x), fast_exp2(gr.y));
        *reinterpret_cast<float2*>(sm + L_::EC + 4 * j0) = make_float2(fast_exp2(gc.x), fast_exp2(gc.y));
      }
    }
    __syncthreads();

    // ---- the state: split planes of S_r = S Diag(e^{G_r}); S Diag(e^{G_C}) back into TMEM ------
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      float x[32];
      const int jb = 64 * half + 32 * p;
      tmem_ld32(tl + kKdaColS + jb, x);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float y[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = x[8 * q + i] * ER[jb + 8 * q + i];
        const uint32_t off = L_::SP + 16384u * half + sw128_off(v, 4 * p + q);
        store_split8(sb + off, sb + off + 32768u, y);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] *= EC[jb + i];
      tmem_st32(tl + kKdaColS + jb, x);
    }
    fence_async_smem();
    tc_wait_st();
    tc_fence_before();
    __syncthreads();

    // ---- [S_r Kt^T | S_r Qt^T] on tcgen05 while the warps form A and P on mma.sync -----------
    if (tid == 0) {
      tc_fence_after();
      int first = 1;
#pragma unroll
      for (int term = 0; term < 3; ++term) {  // (S hi, B hi), (S hi, B lo), (S lo, B hi)
        const uint32_t sa = sb + L_::SP + (term == 2 ? 32768u : 0u);
        const uint32_t kb = sb + L_::KQT + (term == 1 ? 8192u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          umma_bf16(tm + kKdaColSK,
                    kmajor_desc(sa + (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u),
                    kmajor_desc(kb + (uint32_t)(kk >> 2) * 4096u + (uint32_t)(kk & 3) * 32u), ID32,
                    first ? 0u : 1u);
          first = 0;
        }
      }
      umma_commit(bar_mma);
    }
    __syncwarp();
    {  // a partial of A (warps 0-3) or P (warps 4-7) over key channels 32 (w & 3)..+31
      const uint32_t kt = sb + L_::KT, qt = sb + L_::QT;
      const uint32_t ax = warp < 4 ? kt : qt, kh = sb + L_::KH;
      const int k0 = 32 * (warp & 3);
      float pacc[2][4];
      zero_acc(pacc);
      warp_mma<2, 2, false, false>(pacc, ax, kLd128, 0, kh, kLd128, 0, k0);
      warp_mma<2, 2, false, false>(pacc, ax, kLd128, 0, kh + L_::T128, kLd128, 0, k0);
      warp_mma<2, 2, false, false>(pacc, ax + L_::T128, kLd128, 0, kh, kLd128, 0, k0);
      float* pw = PART + 256 * warp;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<float2*>(pw + (gid + 8 * hh) * 16 + 8 * nt + 2 * q4) =
              make_float2(pacc[nt][2 * hh], pacc[nt][2 * hh + 1]);
    }
    __syncthreads();
    // warp 0 sums A and forms T = (I + A)^{-1} Diag(beta); warp 1 sums P; both as core-matrix
    // planes (B operands: row = the output token t, K = the token s)
    if (warp == 0) {
      const float* bet = reinterpret_cast<const float*>(st + L_::RB);
      float* Af = reinterpret_cast<float*>(sm + L_::AF);
#pragma unroll
      for (int e = lane; e < 256; e += 32) {
        const int t = e >> 4, s2 = e & 15;
        const float x = (PART[e] + PART[256 + e]) + (PART[512 + e] + PART[768 + e]);
        Af[t * 17 + s2] = s2 < t ? bet[t] * x : 0.f;
      }
      __syncwarp();
      if (lane < kKc) {  // column c of (I + A)^{-1} by forward substitution
        const int c = lane;
        float rc[kKc];
#pragma unroll
        for (int t = 0; t < kKc; ++t) {
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int s2 = 0; s2 < t; ++s2) {
            if (s2 & 1) s1 = fmaf(Af[t * 17 + s2], rc[s2], s1);
            else s0 = fmaf(Af[t * 17 + s2], rc[s2], s0);
          }
          rc[t] = t < c ? 0.f : (t == c ? 1.f : -(s0 + s1));
        }
        const float bc = bet[c];
        __nv_bfloat16* th = reinterpret_cast<__nv_bfloat16*>(sm + L_::TPC);
        __nv_bfloat16* tlo = reinterpret_cast<__nv_bfloat16*>(sm + L_::TPC + 512);
#pragma unroll
        for (int t = 0; t < kKc; ++t) {
          const uint32_t o = core16_off(t, c) / 2;
          split_bf16(rc[t] * bc, th[o], tlo[o]);
        }
      }
      fence_async_smem();
    } else if (warp == 1) {
      __nv_bfloat16* ph = reinterpret_cast<__nv_bfloat16*>(sm + L_::PPC);
      __nv_bfloat16* pl = reinterpret_cast<__nv_bfloat16*>(sm + L_::PPC + 512);
#pragma unroll
      for (int e = lane; e < 256; e += 32) {
        const int t = e >> 4, s2 = e & 15;
        const float x = (PART[1024 + e] + PART[1280 + e]) + (PART[1536 + e] + PART[1792 + e]);
        const uint32_t o = core16_off(t, s2) / 2;
        split_bf16(s2 <= t ? x : 0.f, ph[o], pl[o]);
      }
      fence_async_smem();
    }
    wait_products();

    // ---- V'^T[v][t] = V[t][v] - (S_r Kt^T)[v][t], tokens 8 half .. 8 half + 7 --------------------
    {
      const __nv_bfloat16* Vr = reinterpret_cast<const __nv_bfloat16*>(st + L_::RV);
      float x[8];
      tmem_ld8(tl + kKdaColSK + 8 * half, x);
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = __bfloat162float(Vr[(8 * half + i) * kLd128 + v]) - x[i];
      const uint32_t off = L_::VPC + core16_off(v, 8 * half);
      store_split8(sb + off, sb + off + 4096u, x);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- U^T = V'^T T^T (three terms) -----------------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int term = 0; term < 3; ++term)
        umma_bf16(tm + kKdaColU, core16_desc(sb + L_::VPC + (term == 2 ? 4096u : 0u)),
                  core16_desc(sb + L_::TPC + (term == 1 ? 512u : 0u)), ID16, term != 0);
      umma_commit(bar_mma);
    }
    __syncwarp();
    wait_products();

    // ---- U^T as split planes (the A operand of both remaining products) -----------------------
    {
      float x[8];
      tmem_ld8(tl + kKdaColU + 8 * half, x);
      const uint32_t off = L_::UPC + core16_off(v, 8 * half);
      store_split8(sb + off, sb + off + 4096u, x);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O^T = S_r Qt^T + U^T P^T; S += U^T Kc (three terms each) --------------------------------
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        const uint64_t ua = core16_desc(sb + L_::UPC + (term == 2 ? 4096u : 0u));
        umma_bf16(tm + kKdaColSQ, ua, core16_desc(sb + L_::PPC + (term == 1 ? 512u : 0u)), ID16, 1u);
        umma_bf16(tm + kKdaColS, ua, sw128_desc(sb + L_::KCS + (term == 1 ? 4096u : 0u), 2048u, 1024u),
                  ID128_BMN, 1u);
      }
      umma_commit(bar_mma);
    }
    __syncwarp();
    wait_products();

    // ---- outputs o_t = O^T[v][t] ------------------------------------------------------------------
    {
      float x[8];
      tmem_ld8(tl + kKdaColSQ + 8 * half, x);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = 8 * half + i;
        if (t < n) a.o[(row0 + t) * kPfD + v] = __float2bfloat16_rn(x[i]);
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
    tmem_ld32(tl + kKdaColS + 64 * half + 32 * p, x);
    float4* dst = reinterpret_cast<float4*>(Sg + v * kPfD + 64 * half + 32 * p);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = bad ? make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                 __int_as_float(0x7fc00000), __int_as_float(0x7fc00000))
                   : make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
  }
  if (bad && tid == 0) mbar_wait_bounded(bar_mma, mma_phase);  // products still in flight
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, kKdaCols);
  }
}

}  // namespace gdnq
