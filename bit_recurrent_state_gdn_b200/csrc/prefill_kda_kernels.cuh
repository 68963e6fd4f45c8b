// Chunkwise-parallel prefill with a per-key-channel gate (Kimi Delta Attention, KDA, which
// "LeapQuant: Efficient Linear Attention with Accurate Recurrent State Quantization", Abstract,
// names beside GDN), the counterpart of prefill_kernels.cuh's scalar-gate kernel ("LinQuant:
// Functional Invariances for Low-Precision Linear Recurrences", Abstract: prefill of a linear
// recurrence cast as chunked dense matmuls).
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
// One CTA per head, 256 threads, two CTAs per SM. The state sits in registers as mma
// accumulators (warp w: value rows 16w..16w+15); scaled by e^{G_r} per column and split into hi /
// lo bf16 on the fly it is the B operand of the products with S_r^T, whose value columns
// 16w..16w+15 warp w computes. Every fp32 operand enters the bf16 mma as hi + lo parts (three
// products: hi hi, hi lo, lo hi), accumulation in fp32.
#pragma once

#include "prefill_kernels.cuh"

namespace gdnq {

constexpr int kKc = 16;       // chunk length
constexpr int kKref = 7;      // the chunk's reference token
constexpr int kLd16 = 24;     // bf16 row stride of 16 x 16 tiles (48 B: ldmatrix without conflicts)
constexpr int kKdaCtas = 2;   // CTAs per SM

// Shared memory (bytes). Two stages of raw chunk inputs, then the chunk's working tiles.
struct KdaLayout {
  static constexpr uint32_t T128 = kKc * kLd128 * 2;  // a 16 x 128 bf16 tile
  static constexpr uint32_t T16 = kKc * kLd16 * 2;    // a 16 x 16 bf16 tile
  static constexpr uint32_t RQ = 0;                    // q, k, v (bf16), g (fp32), beta (fp32)
  static constexpr uint32_t RK = RQ + T128;
  static constexpr uint32_t RV = RK + T128;
  static constexpr uint32_t RG = RV + T128;
  static constexpr uint32_t RB = RG + kKc * kPfD * 4;
  static constexpr uint32_t STAGE = RB + kKc * 4;
  static constexpr uint32_t KT = 2 * STAGE;            // hi, lo pairs of tiles from here
  static constexpr uint32_t QT = KT + 2 * T128;
  static constexpr uint32_t KH = QT + 2 * T128;
  static constexpr uint32_t KC = KH + 2 * T128;        // K e^{G_C - G}
  static constexpr uint32_t VP = KC + 2 * T128;        // V'
  static constexpr uint32_t U = VP + 2 * T128;
  static constexpr uint32_t TT = U + 2 * T128;         // T
  static constexpr uint32_t PP = TT + 2 * T16;         // P
  static constexpr uint32_t AF = PP + 2 * T16;         // A, fp32 16 x 17
  static constexpr uint32_t PART = AF + kKc * 17 * 4;  // per-warp partial A / P, 8 x 256 fp32
  static constexpr uint32_t ER = PART + 8 * 256 * 4;   // e^{G_r}, 128 fp32
  static constexpr uint32_t EC = ER + kPfD * 4;        // e^{G_C}, 128 fp32
  static constexpr uint32_t TOTAL = EC + kPfD * 4;
};
static_assert(KdaLayout::STAGE % 16 == 0 && KdaLayout::AF % 16 == 0, "16-byte aligned tiles");
static_assert(kKdaCtas * (KdaLayout::TOTAL + 1024) <= 228 * 1024, "two CTAs per SM");

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

__global__ void __launch_bounds__(kPfThreads, kKdaCtas) prefill_kda_kernel(const PfArgs a) {
  using L_ = KdaLayout;
  extern __shared__ __align__(128) uint8_t sm[];
  const int head = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, q4 = lane & 3;
  const int L = a.L;
  const uint32_t base = smem_u32(sm);
  const float* ER = reinterpret_cast<const float*>(sm + L_::ER);
  const float* EC = reinterpret_cast<const float*>(sm + L_::EC);
  float* PART = reinterpret_cast<float*>(sm + L_::PART);

  // the state: warp w holds value rows 16w..16w+15, all 128 key columns, in accumulator layout
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

  if (L > 0) kda_load_chunk(sm, a, (size_t)head * L, min(kKc, L));
  cp_async_commit();
  for (int c0 = 0, ci = 0; c0 < L; c0 += kKc, ++ci) {
    const int n = min(kKc, L - c0);
    const size_t row0 = (size_t)head * L + c0;
    const uint32_t so = (ci & 1) * L_::STAGE;
    const uint8_t* st = sm + so;
    // the next chunk's inputs into the other stage (its last reader, the previous chunk's
    // phase b, is behind that chunk's last barrier)
    if (c0 + kKc < L) kda_load_chunk(sm + (L_::STAGE - so), a, row0 + kKc, min(kKc, L - c0 - kKc));
    cp_async_commit();
    cp_async_wait_one();
    __syncthreads();  // this chunk's inputs; every warp done with the previous chunk

    // ---- decayed operands: thread = (channels 2 jp, 2 jp + 1; tokens 4 tq..4 tq + 3) ----------
    // (cumulative log-gates in base 2, G log2(e), so each factor is one hardware exp2)
    {
      constexpr float kLog2e = 1.4426950408889634f;
      const int jp = tid & 63, tq = tid >> 6, j0 = 2 * jp;
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
        put_split2(sm + L_::KT, sm + L_::KT + L_::T128, idx, kk.x * tx, kk.y * ty);
        put_split2(sm + L_::QT, sm + L_::QT + L_::T128, idx, qq.x * tx, qq.y * ty);
        put_split2(sm + L_::KH, sm + L_::KH + L_::T128, idx, kk.x * hx, kk.y * hy);
        put_split2(sm + L_::KC, sm + L_::KC + L_::T128, idx, kk.x * cx, kk.y * cy);
      }
      if (tq == 0) {
        *reinterpret_cast<float2*>(sm + L_::ER + 4 * j0) = make_float2(fast_exp2(gr.x), fast_exp2(gr.y));
        *reinterpret_cast<float2*>(sm + L_::EC + 4 * j0) = make_float2(fast_exp2(gc.x), fast_exp2(gc.y));
      }
    }
    __syncthreads();

    // ---- phase a: V' = V - Kt S_r^T and O = Qt S_r^T on this warp's value slab; a partial of
    // A (warps 0-3) or P (warps 4-7) over key channels 32 (w & 3)..+31 ---------------------------
    float oacc[2][4], vacc[2][4];
    zero_acc(oacc);
    zero_acc(vacc);
    {
      const uint32_t kt = base + L_::KT, qt = base + L_::QT;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t bh[2][2], bl[2][2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const float2 e = *reinterpret_cast<const float2*>(ER + 16 * ks + 8 * half + 2 * q4);
#pragma unroll
          for (int nn = 0; nn < 2; ++nn)
            split2_bf16(sacc[2 * ks + half][2 * nn] * e.x, sacc[2 * ks + half][2 * nn + 1] * e.y,
                        bh[nn][half], bl[nn][half]);
        }
        const uint32_t off = 2u * ((lane & 15) * kLd128 + 16 * ks + 8 * (lane >> 4));
        uint32_t ah[4], al[4];
        ldsm_x4(kt + off, ah);
        ldsm_x4(kt + L_::T128 + off, al);
#pragma unroll
        for (int nn = 0; nn < 2; ++nn) {
          mma_bf16(vacc[nn], ah, bh[nn][0], bh[nn][1]);
          mma_bf16(vacc[nn], ah, bl[nn][0], bl[nn][1]);
          mma_bf16(vacc[nn], al, bh[nn][0], bh[nn][1]);
        }
        ldsm_x4(qt + off, ah);
        ldsm_x4(qt + L_::T128 + off, al);
#pragma unroll
        for (int nn = 0; nn < 2; ++nn) {
          mma_bf16(oacc[nn], ah, bh[nn][0], bh[nn][1]);
          mma_bf16(oacc[nn], ah, bl[nn][0], bl[nn][1]);
          mma_bf16(oacc[nn], al, bh[nn][0], bh[nn][1]);
        }
      }
      const __nv_bfloat16* Vr = reinterpret_cast<const __nv_bfloat16*>(st + L_::RV);
      store_split(vacc, reinterpret_cast<__nv_bfloat16*>(sm + L_::VP),
                  reinterpret_cast<__nv_bfloat16*>(sm + L_::VP + L_::T128), kLd128, 0, v0,
                  [&](int t, int vv, float x) { return __bfloat162float(Vr[t * kLd128 + vv]) - x; });

      const uint32_t ax = warp < 4 ? kt : qt, kh = base + L_::KH;
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

    // ---- phase b: warp 0 sums A and forms T = (I + A)^{-1} Diag(beta); warp 1 sums P ---------
    if (warp == 0) {
      const float* bet = reinterpret_cast<const float*>(st + L_::RB);
      float* Af = reinterpret_cast<float*>(sm + L_::AF);
#pragma unroll
      for (int e = lane; e < 256; e += 32) {
        const int t = e >> 4, s = e & 15;
        const float x = (PART[e] + PART[256 + e]) + (PART[512 + e] + PART[768 + e]);
        Af[t * 17 + s] = s < t ? bet[t] * x : 0.f;
      }
      __syncwarp();
      if (lane < kKc) {  // column c of (I + A)^{-1} by forward substitution
        const int c = lane;
        float rc[kKc];
#pragma unroll
        for (int t = 0; t < kKc; ++t) {
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int s = 0; s < t; ++s) {
            if (s & 1) s1 = fmaf(Af[t * 17 + s], rc[s], s1);
            else s0 = fmaf(Af[t * 17 + s], rc[s], s0);
          }
          rc[t] = t < c ? 0.f : (t == c ? 1.f : -(s0 + s1));
        }
        const float bc = bet[c];
        __nv_bfloat16* th = reinterpret_cast<__nv_bfloat16*>(sm + L_::TT);
        __nv_bfloat16* tl = reinterpret_cast<__nv_bfloat16*>(sm + L_::TT + L_::T16);
#pragma unroll
        for (int t = 0; t < kKc; ++t) split_bf16(rc[t] * bc, th[t * kLd16 + c], tl[t * kLd16 + c]);
      }
    } else if (warp == 1) {
      __nv_bfloat16* ph = reinterpret_cast<__nv_bfloat16*>(sm + L_::PP);
      __nv_bfloat16* pl = reinterpret_cast<__nv_bfloat16*>(sm + L_::PP + L_::T16);
#pragma unroll
      for (int e = lane; e < 256; e += 32) {
        const int t = e >> 4, s = e & 15;
        const float x = (PART[1024 + e] + PART[1280 + e]) + (PART[1536 + e] + PART[1792 + e]);
        split_bf16(s <= t ? x : 0.f, ph[t * kLd16 + s], pl[t * kLd16 + s]);
      }
    }
    __syncthreads();

    // ---- phase c (this warp's slab only): U = T V'; O += P U; S = S Diag(e^{G_C}) + U^T Kc ----
    {
      const uint32_t tt = base + L_::TT, pp = base + L_::PP, vp = base + L_::VP, u = base + L_::U;
      float uacc[2][4];
      zero_acc(uacc);
      warp_mma<2, 1, false, true>(uacc, tt, kLd16, 0, vp, kLd128, v0, 0);
      warp_mma<2, 1, false, true>(uacc, tt, kLd16, 0, vp + L_::T128, kLd128, v0, 0);
      warp_mma<2, 1, false, true>(uacc, tt + L_::T16, kLd16, 0, vp, kLd128, v0, 0);
      store_split(uacc, reinterpret_cast<__nv_bfloat16*>(sm + L_::U),
                  reinterpret_cast<__nv_bfloat16*>(sm + L_::U + L_::T128), kLd128, 0, v0,
                  [](int, int, float x) { return x; });
      __syncwarp();
      warp_mma<2, 1, false, true>(oacc, pp, kLd16, 0, u, kLd128, v0, 0);
      warp_mma<2, 1, false, true>(oacc, pp, kLd16, 0, u + L_::T128, kLd128, v0, 0);
      warp_mma<2, 1, false, true>(oacc, pp + L_::T16, kLd16, 0, u, kLd128, v0, 0);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int t = gid + 8 * hh;
          if (t < n) {
            __nv_bfloat162 ov;
            ov.x = __float2bfloat16_rn(oacc[nt][2 * hh]);
            ov.y = __float2bfloat16_rn(oacc[nt][2 * hh + 1]);
            *reinterpret_cast<__nv_bfloat162*>(a.o + (row0 + t) * kPfD + v0 + 8 * nt + 2 * q4) = ov;
          }
        }
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const float2 e = *reinterpret_cast<const float2*>(EC + 8 * nt + 2 * q4);
        sacc[nt][0] *= e.x; sacc[nt][1] *= e.y; sacc[nt][2] *= e.x; sacc[nt][3] *= e.y;
      }
      // A = U^T: stored [s][v] = [k][m]; B = Kc stored [s][j] = [k][n]
      const uint32_t kc = base + L_::KC;
      warp_mma<16, 1, true, true>(sacc, u, kLd128, v0, kc, kLd128, 0, 0);
      warp_mma<16, 1, true, true>(sacc, u, kLd128, v0, kc + L_::T128, kLd128, 0, 0);
      warp_mma<16, 1, true, true>(sacc, u + L_::T128, kLd128, v0, kc, kLd128, 0, 0);
    }
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
