// Tensor-core form of one windowed decode step (d = 128, bf16 activations and buffers), with the
// window flush's rank update on tensor cores too. Included by window_kernels.cuh.
//
// The products of a step, per head:
//   phase 1  F [x y] with F = diag(s) C, C the int8 (or int4) codes: an exact integer mma. Each
//            32-column chunk of x (and y) is written as X 2^(e-22) with X an integer of at most
//            22 bits, split into three signed 8-bit digits X = d1 2^16 + d2 2^8 + d3; the six
//            digit columns form the right-hand side of mma.m16n8k32.s8 (int32 accumulate, exact),
//            and the digits are recombined in fp32. Precision: 22 bits relative to the chunk's
//            largest entry.
//   phase 2  the pair coefficients <bk_i, k_t>, <bk_i, q_t> (scalar gate): mma.m16n8k16.bf16 with
//            the buffered keys and [k_t q_t] as exact bf16 operands, fp32 accumulate. The
//            diagonal gate needs a per-element decay and stays on FMA.
//   phase 3  the corrections sum_i a_i u_i, sum_i b_i u_i: U^T times the coefficients, each fp32
//            coefficient split into three bf16 (hi + mid + lo carries its 24 bits), fp32
//            accumulate.
//   flush    S_W = F Diag(e^{L_W}) + comps + U^T Kt, Kt_i = k_i e^{L_W - L_i}: mma.m16n8k16.bf16
//            with the fp32 operand (scaled U for the scalar gate, Kt for the diagonal gate) split
//            into three bf16 parts, fp32 accumulate; the epilogue adds the frozen state and the
//            compensators, picks compensator columns, takes row absmax and requantises.
// Warp w owns state rows 16w..16w+15 in every product; in a C fragment lane l holds rows
// 16w + l/4 and 16w + l/4 + 8, columns 2(l%4) and 2(l%4) + 1.
#pragma once

#include "mma_util.cuh"

namespace gdnq {


template <class C>
__device__ void flush_mma(const WinArgs& a, const WinLayout& L, uint8_t* sm, uint8_t* st, int head,
                          int P, float Ls, TcCtx& tc);

// Pair i's coefficients (a, b) as the three-way bf16 split rows of the phase-3 right-hand side.
__device__ __forceinline__ void put_coef(__nv_bfloat16* Bc, int bcs, int i, float av, float bv) {
  float h, m, l;
  split3(av, h, m, l);
  Bc[0 * bcs + i] = __float2bfloat16_rn(h);
  Bc[1 * bcs + i] = __float2bfloat16_rn(m);
  Bc[2 * bcs + i] = __float2bfloat16_rn(l);
  split3(bv, h, m, l);
  Bc[3 * bcs + i] = __float2bfloat16_rn(h);
  Bc[4 * bcs + i] = __float2bfloat16_rn(m);
  Bc[5 * bcs + i] = __float2bfloat16_rn(l);
}

template <class C>
__device__ __forceinline__ void step_head_mma(const WinArgs& a, const WinLayout& L, uint8_t* sm,
                                              uint8_t* st, int head, int P, float g_scalar,
                                              float beta, TcCtx& tc) {
  using bf = __nv_bfloat16;
  constexpr int D = 128;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, q4 = lane & 3;
  const int mi = lane >> 3, r8 = lane & 7;
  const int W = a.W, r = a.r, Wp = (W + 3) & ~3, Wr = (W + 15) & ~15, bcs = Wr + 8;
  // (with power tokens a full window is left to the window-end kernel: pos becomes W)
  const bool flush = (P + 1 == W) && a.comp_k == nullptr;
  const int Pp = (P + 15) & ~15;

  float* vec = reinterpret_cast<float*>(sm + L.vec);
  float* Lt = vec + 4 * D;     // the step's cumulative log-gate per column (the flush reads it)
  float* misc = vec + 7 * D;  // [0..3] k.q partials, [24] x block scale, [25] y block scale
  float* coef = reinterpret_cast<float*>(sm + L.coef);
  float *ca = coef, *cb = coef + (W + r);
  uint8_t* Bfrag = sm + L.tc;                                      // digits, fragment order
  bf* Bc = reinterpret_cast<bf*>(sm + L.tc + 8 * 144);  // [8][Wr + 8]

  const uint8_t* s_codes = st + L.codes;
  const float* s_scales = reinterpret_cast<const float*>(st + L.scales);
  bf* s_bk = reinterpret_cast<bf*>(st + L.bk);
  bf* s_bu = reinterpret_cast<bf*>(st + L.bu);
  float* s_bL = reinterpret_cast<float*>(st + L.bL);
  const int32_t* s_cidx = reinterpret_cast<const int32_t*>(st + L.cidx);
  const float* s_cu = reinterpret_cast<const float*>(st + L.cu);
  const bf* s_q = reinterpret_cast<const bf*>(st + L.q);
  const bf* s_k = reinterpret_cast<const bf*>(st + L.k);
  const bf* s_v = reinterpret_cast<const bf*>(st + L.v);
  const float* s_g = reinterpret_cast<const float*>(st + L.g);

  float Ls = 0.f;
  if constexpr (!C::DIAG) Ls = (P > 0 ? s_bL[P - 1] : 0.f) + g_scalar;

  // Warps 0-3 (group X) take the gates and the frozen-state products (phase 1) while warps 4-7
  // (group Y) take the pair coefficients (phase 2) and the buffer products (phase 3); both meet
  // before the per-row finish (phase 4).
  float* PR = vec;      // phase-1 results p = F x, r = F y by row
  float* RR = vec + D;
  float* WV = vec + 5 * D;  // phase-3 results U^T a, U^T b by row
  float* RV = vec + 6 * D;
  if (warp < 4) {
    // ---- gates, phase-1 digit columns, the step's key / log-gate appended ----------------
    // Warp w owns chunk w (lane l: column j = 32 w + l) of both x and y. Each vector gets one
    // block exponent, found by every warp from all 128 columns (no cross-warp step):
    // X = rint(v 2^(22-e)), |X| <= 2^22, three signed 8-bit digits X = d1 2^16 + d2 2^8 + d3.
    const int j = 32 * warp + lane;
    float mx = 0.f, my = 0.f, vx = 0.f, vy = 0.f, lj = Ls;
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      const int jj = lane + 32 * mm;
      float l = Ls, e = 1.f;
      if constexpr (C::DIAG) {
        l = (P > 0 ? s_bL[(P - 1) * D + jj] : 0.f) + s_g[jj];
        e = fast_exp(l);
      }
      float xv = e * __bfloat162float(s_k[jj]), yv = e * __bfloat162float(s_q[jj]);
      if constexpr (C::SMOOTH) {  // F = dequant Diag(2^e): the codes meet 2^e .* x
        const float f = pow2i(reinterpret_cast<const int8_t*>(st + L.sexp)[jj]);
        xv *= f;
        yv *= f;
      }
      mx = fmaxf(mx, fabsf(xv));
      my = fmaxf(my, fabsf(yv));
      if (mm == warp) {  // this lane's own column j
        vx = xv;
        vy = yv;
        lj = l;
      }
    }
    const float kj = __bfloat162float(s_k[j]), qj = __bfloat162float(s_q[j]);
    float kq = kj * qj;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, off));
      kq += __shfl_xor_sync(0xffffffffu, kq, off);
    }
    if (lane == 0) misc[warp] = kq;
    Lt[j] = lj;
    if (!flush) {
      static_cast<bf*>(a.buf_k)[(size_t)head * W * D + swz_el<bf, D>(P, j)] = s_k[j];
      if constexpr (C::DIAG) a.buf_L[((size_t)head * W + P) * D + j] = lj;
    } else {
      s_bk[swz_el<bf, D>(P, j)] = s_k[j];
      if constexpr (C::DIAG) s_bL[P * D + j] = lj;
    }
    if constexpr (!C::DIAG) {
      if (tid == 0) {
        if (!flush) a.buf_L[(size_t)head * Wp + P] = Ls;
        else s_bL[P] = Ls;
      }
    }
    const int k = digit_pos<C::INT4>(j);
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      const float m = side ? my : mx, val = side ? vy : vx;
      float mul = 0.f, scale = 0.f;
      if (m >= 0x1p-100f) {  // smaller vectors contribute nothing measurable
        // m = f 2^e2 with 0.5 <= f < 1 (m is normal); powers of two from exponent bits
        const int e2 = ((__float_as_int(m) >> 23) & 0xFF) - 126;
        mul = __int_as_float((22 - e2 + 127) << 23);
        scale = __int_as_float((e2 - 22 + 127) << 23);
      }
      const int X = __float2int_rn(val * mul);
      const int d3 = (int)(int8_t)(X & 0xFF);
      const int X1 = (X - d3) >> 8;  // exact: X - d3 is a multiple of 256
      const int d2 = (int)(int8_t)(X1 & 0xFF);
      const int d1 = (X1 - d2) >> 8;
      Bfrag[digit_off(3 * side + 0, k)] = (uint8_t)d1;
      Bfrag[digit_off(3 * side + 1, k)] = (uint8_t)d2;
      Bfrag[digit_off(3 * side + 2, k)] = (uint8_t)d3;
      if (tid == 0) misc[24 + side] = scale;
    }
    xsync();

    // ---- phase 1: p = F x, r = F y for rows 32w + 16mt + gid (+8) --------------------------
    // digit weights of this lane's columns 2q4, 2q4+1: x = columns 0..2, y = columns 3..5
    const float wx0 = q4 == 0 ? 65536.f : (q4 == 1 ? 1.f : 0.f);
    const float wx1 = q4 == 0 ? 256.f : 0.f;
    const float wy0 = q4 == 2 ? 256.f : 0.f;
    const float wy1 = q4 == 1 ? 65536.f : (q4 == 2 ? 1.f : 0.f);
    const uint4 bw0 = *reinterpret_cast<const uint4*>(Bfrag + (gid * 4 + q4) * 32);
    const uint4 bw1 = *reinterpret_cast<const uint4*>(Bfrag + (gid * 4 + q4) * 32 + 16);
    const uint32_t bw[8] = {bw0.x, bw0.y, bw0.z, bw0.w, bw1.x, bw1.y, bw1.z, bw1.w};
    const uint32_t cb0 = smem_u32(s_codes);
    const float gam = C::DIAG ? 1.f : fast_exp(Ls);
    const float sx = misc[24] * gam * (C::INT4 ? 0.0625f : 1.f);  // int4 codes entered as 16 c
    const float sy = misc[25] * gam * (C::INT4 ? 0.0625f : 1.f);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int row0 = 32 * warp + 16 * mt;
      float PX[2], PY[2];
      if constexpr (C::INT4) {
        PX[0] = PX[1] = PY[0] = PY[1] = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // each 32-column chunk is one scale group
          uint32_t A[4], w0, w1;
          ldsm_x2(cb0 + swz<64>(row0 + r8 + 8 * (mi & 1), 16 * c), w0, w1);
          i4x8_to_s8x16(w0, A[0], A[2]);
          i4x8_to_s8x16(w1, A[1], A[3]);
          int Cc[4] = {0, 0, 0, 0};
          mma_s8(Cc, A, bw[2 * c], bw[2 * c + 1]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float sg = s_scales[(row0 + gid + 8 * h) * C::NG + c];
            const float c0 = (float)Cc[2 * h], c1 = (float)Cc[2 * h + 1];
            PX[h] = fmaf(sg, wx0 * c0 + wx1 * c1, PX[h]);
            PY[h] = fmaf(sg, wy0 * c0 + wy1 * c1, PY[h]);
          }
        }
      } else {
        int Cc[4] = {0, 0, 0, 0};  // one exponent per vector: chunks accumulate exactly in int32
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t A[4];
          ldsm_x4(cb0 + swz<128>(row0 + r8 + 8 * (mi & 1), 32 * c + 16 * (mi >> 1)), A);
          mma_s8(Cc, A, bw[2 * c], bw[2 * c + 1]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float c0 = (float)Cc[2 * h], c1 = (float)Cc[2 * h + 1];
          PX[h] = wx0 * c0 + wx1 * c1;
          PY[h] = wy0 * c0 + wy1 * c1;
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        PX[h] += __shfl_xor_sync(0xffffffffu, PX[h], 1);
        PX[h] += __shfl_xor_sync(0xffffffffu, PX[h], 2);
        PY[h] += __shfl_xor_sync(0xffffffffu, PY[h], 1);
        PY[h] += __shfl_xor_sync(0xffffffffu, PY[h], 2);
      }
      if (q4 < 2) {  // lane q4 of the quad stores row row0 + gid + 8 q4
        const int v = row0 + gid + 8 * q4;
        const float srow = C::INT4 ? 1.f : s_scales[v];
        PR[v] = (q4 ? PX[1] : PX[0]) * sx * srow;
        RR[v] = (q4 ? PY[1] : PY[0]) * sy * srow;
      }
    }
  } else {
    const int ty = tid - 128, wy = warp - 4;
    // padding of the phase-3 product to a multiple of 16 pairs: zero coefficients for the rows
    // past the P pairs, whose write-vector rows hold zeros or an earlier head's finite values
    if (ty < 96) {
      const int i = P + (ty & 15);
      if (i < Pp) Bc[(ty >> 4) * bcs + i] = __float2bfloat16_rn(0.f);
    }
    if (a.comp_k) {
      // power tokens, entered at L = 0: coefficients <ck_c, x>, <ck_c, y>, one warp a token
      const float* s_ck = reinterpret_cast<const float*>(st + L.ck);
      for (int c = wy; c < r; c += 4) {
        float ax = 0.f, ay = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int jj = lane + 32 * m;
          float kd = s_ck[c * D + jj];
          if constexpr (C::DIAG) kd *= fast_exp((P > 0 ? s_bL[(P - 1) * D + jj] : 0.f) + s_g[jj]);
          ax = fmaf(kd, __bfloat162float(s_k[jj]), ax);
          ay = fmaf(kd, __bfloat162float(s_q[jj]), ay);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          ax += __shfl_xor_sync(0xffffffffu, ax, off);
          ay += __shfl_xor_sync(0xffffffffu, ay, off);
        }
        if (lane == 0) {
          const float e = C::DIAG ? 1.f : fast_exp(Ls);
          ca[W + c] = e * ax;
          cb[W + c] = e * ay;
        }
      }
    } else if (ty < r) {  // compensator pairs: key e_j entered at L = 0, coefficient x[j]
      const int j = s_cidx[ty] & (D - 1);
      float e;
      if constexpr (C::DIAG) e = fast_exp((P > 0 ? s_bL[(P - 1) * D + j] : 0.f) + s_g[j]);
      else e = fast_exp(Ls);
      ca[W + ty] = e * __bfloat162float(s_k[j]);
      cb[W + ty] = e * __bfloat162float(s_q[j]);
    }

    // ---- phase 2: pair coefficients, written as the split phase-3 right-hand side ------
    if constexpr (!C::DIAG) {
      const int tiles = Pp >> 4;
      const bf* bsrc = gid == 0 ? s_k : s_q;  // right-hand side columns: 0 = k_t, 1 = q_t
      for (int tile = wy; tile < tiles; tile += 4) {
        float Ce[4] = {0.f, 0.f, 0.f, 0.f}, Co[4] = {0.f, 0.f, 0.f, 0.f};  // even / odd k-steps
        const uint32_t kb = smem_u32(s_bk);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          uint32_t A[4];
          ldsm_x4(kb + swz<256>(16 * tile + r8 + 8 * (mi & 1), 2 * (16 * s + 8 * (mi >> 1))), A);
          uint32_t b0 = 0u, b1 = 0u;
          if (gid < 2) {
            b0 = *reinterpret_cast<const uint32_t*>(bsrc + 16 * s + 2 * q4);
            b1 = *reinterpret_cast<const uint32_t*>(bsrc + 16 * s + 8 + 2 * q4);
          }
          if (s & 1) mma_bf16(Co, A, b0, b1);
          else mma_bf16(Ce, A, b0, b1);
        }
        // the quad leader holds (a, b) of rows gid and gid+8; lane q4 splits one of the four
        const int ld = lane & ~3;
        const float a0 = __shfl_sync(0xffffffffu, Ce[0] + Co[0], ld);
        const float b0 = __shfl_sync(0xffffffffu, Ce[1] + Co[1], ld);
        const float a1 = __shfl_sync(0xffffffffu, Ce[2] + Co[2], ld);
        const float b1 = __shfl_sync(0xffffffffu, Ce[3] + Co[3], ld);
        const float vq = q4 == 0 ? a0 : (q4 == 1 ? b0 : (q4 == 2 ? a1 : b1));
        const int i = 16 * tile + gid + 8 * (q4 >> 1);
        if (i < P) {
          float h, m, l;
          split3(vq * fast_exp(Ls - s_bL[i]), h, m, l);
          const int row = (q4 & 1) ? 3 : 0;
          Bc[(row + 0) * bcs + i] = __float2bfloat16_rn(h);
          Bc[(row + 1) * bcs + i] = __float2bfloat16_rn(m);
          Bc[(row + 2) * bcs + i] = __float2bfloat16_rn(l);
        }
      }
    } else {
      // per-element decay e^{L_t[j] - L_i[j]}: FMA, 8 threads per pair; thread c takes columns
      // 8c..8c+7 and 64+8c..64+8c+7 (distinct banks across the 8 threads of a pair), as
      // adjacent column pairs in packed fp32 arithmetic
      const int c = ty & 7;
      F2 kr[8], qr[8], lr[8];
#pragma unroll
      for (int e2 = 0; e2 < 8; ++e2) {
        const int j = (e2 < 4 ? 8 * c : 64 + 8 * c) + 2 * (e2 & 3);
        kr[e2] = f2(__bfloat162float(s_k[j]), __bfloat162float(s_k[j + 1]));
        qr[e2] = f2(__bfloat162float(s_q[j]), __bfloat162float(s_q[j + 1]));
        lr[e2] = f2((P > 0 ? s_bL[(P - 1) * D + j] : 0.f) + s_g[j],
                    (P > 0 ? s_bL[(P - 1) * D + j + 1] : 0.f) + s_g[j + 1]);
      }
      const F2 neg1 = f2(-1.f, -1.f), log2e = f2(1.4426950408889634f, 1.4426950408889634f);
      const int npass = (P + 15) >> 4;
      for (int ps = 0; ps < npass; ++ps) {
        const int i = ps * 16 + (ty >> 3);
        F2 pa2 = f2(0.f, 0.f), pb2 = f2(0.f, 0.f);
        if (i < P) {
          float kk[16], ll[16];
          load_sw<bf, D, 8>(s_bk, i, 8 * c, kk);
          load_sw<bf, D, 8>(s_bk, i, 64 + 8 * c, kk + 8);
          Num<float>::load<8>(s_bL + i * D + 8 * c, ll);
          Num<float>::load<8>(s_bL + i * D + 64 + 8 * c, ll + 8);
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) {
            // (l_t - l_i) log2(e), then 2^x: the arithmetic of fast_exp, two columns at once
            const F2 d = f2_mul(f2_fma(f2(ll[2 * e2], ll[2 * e2 + 1]), neg1, lr[e2]), log2e);
            float d0, d1;
            f2_get(d, d0, d1);
            const F2 k2 = f2_mul(f2(kk[2 * e2], kk[2 * e2 + 1]), f2(exp2_hw(d0), exp2_hw(d1)));
            pa2 = f2_fma(k2, kr[e2], pa2);
            pb2 = f2_fma(k2, qr[e2], pb2);
          }
        }
        float pa, pb;
        {
          float a0, a1, b0, b1;
          f2_get(pa2, a0, a1);
          f2_get(pb2, b0, b1);
          pa = a0 + a1;
          pb = b0 + b1;
        }
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) {
          pa += __shfl_xor_sync(0xffffffffu, pa, off);
          pb += __shfl_xor_sync(0xffffffffu, pb, off);
        }
        if (c == 0 && i < P) put_coef(Bc, bcs, i, pa, pb);
      }
    }
    ysync();

    // ---- phase 3: U^T (a, b) for rows 32 wy + 16 mt + gid (+8) ----------------------------
    float C0[4] = {0.f, 0.f, 0.f, 0.f}, C1[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t ub = smem_u32(s_bu);
    for (int s = 0; s < Pp / 16; ++s) {
      uint32_t A0[4], A1[4];
      ldsm_x4_t(ub + swz<256>(16 * s + r8 + 8 * (mi >> 1), 2 * (32 * wy + 8 * (mi & 1))), A0);
      ldsm_x4_t(ub + swz<256>(16 * s + r8 + 8 * (mi >> 1), 2 * (32 * wy + 16 + 8 * (mi & 1))), A1);
      const uint32_t b0 = *reinterpret_cast<const uint32_t*>(Bc + gid * bcs + 16 * s + 2 * q4);
      const uint32_t b1 = *reinterpret_cast<const uint32_t*>(Bc + gid * bcs + 16 * s + 8 + 2 * q4);
      mma_bf16(C0, A0, b0, b1);
      mma_bf16(C1, A1, b0, b1);
    }
    // columns 0..2 belong to w, 3..5 to r
    const float wx0 = q4 <= 1 ? 1.f : 0.f, wx1 = q4 == 0 ? 1.f : 0.f;
    const float wy0 = q4 == 2 ? 1.f : 0.f, wy1 = (q4 == 1 || q4 == 2) ? 1.f : 0.f;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const float* Cc = mt ? C1 : C0;
      float Wv[2], Rv[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        Wv[h] = wx0 * Cc[2 * h] + wx1 * Cc[2 * h + 1];
        Rv[h] = wy0 * Cc[2 * h] + wy1 * Cc[2 * h + 1];
        Wv[h] += __shfl_xor_sync(0xffffffffu, Wv[h], 1);
        Wv[h] += __shfl_xor_sync(0xffffffffu, Wv[h], 2);
        Rv[h] += __shfl_xor_sync(0xffffffffu, Rv[h], 1);
        Rv[h] += __shfl_xor_sync(0xffffffffu, Rv[h], 2);
      }
      if (q4 < 2) {  // lane q4 of the quad stores row 32 wy + 16 mt + gid + 8 q4
        const int v = 32 * wy + 16 * mt + gid + 8 * q4;
        WV[v] = q4 ? Wv[1] : Wv[0];
        RV[v] = q4 ? Rv[1] : Rv[0];
      }
    }
  }
  csync();

  // ---- phase 4: u_t and o_t, one thread per row v (coalesced stores) ----------------------
  if (tid < D) {
    const int v = tid;
    float w = PR[v] + WV[v], rv = RR[v] + RV[v];
    for (int c = 0; c < r; ++c) {
      const float cu = s_cu[c * D + v];
      w = fmaf(ca[W + c], cu, w);
      rv = fmaf(cb[W + c], cu, rv);
    }
    const float u = beta * (__bfloat162float(s_v[v]) - w);
    const bf ubf = __float2bfloat16_rn(u);
    const float kq = misc[0] + misc[1] + misc[2] + misc[3];
    static_cast<bf*>(a.o)[(size_t)head * D + v] = __float2bfloat16_rn(rv + __bfloat162float(ubf) * kq);
    if (!flush) static_cast<bf*>(a.buf_u)[(size_t)head * W * D + swz_el<bf, D>(P, v)] = ubf;
    else s_bu[swz_el<bf, D>(P, v)] = ubf;
  }
  if (tid == 0) a.pos[head] = flush ? 0 : P + 1;
  if (!flush) return;
  csync();
  flush_mma<C>(a, L, sm, st, head, P, Ls, tc);
}

// ------------------------------------------------------------------------------------------
// Window end: materialise S_W = F Diag(e^{L_W}) + comps + U^T Kt on tensor cores, then
// compensators, absmax and requantisation, from the accumulators. npairs = P + 1 pairs (the
// step's pair included) sit in the stage; the gates end at L_W = Lt (per column) / Ls.
// ------------------------------------------------------------------------------------------
// 1 << k, hidden from the optimiser: a select over unrolled array elements keyed on it stays a
// select and is not turned back into a run-time index (which would move the array to local
// memory).
__device__ __forceinline__ uint32_t one_hot_opaque(int k) {
  uint32_t m = 1u << k;
  asm volatile("" : "+r"(m));
  return m;
}

template <class C>
__device__ void flush_mma(const WinArgs& a, const WinLayout& L, uint8_t* sm, uint8_t* st, int head,
                          int P, float Ls, TcCtx& tc) {
  using bf = __nv_bfloat16;
  constexpr int D = 128, QMAX = C::QMAX;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, q4 = lane & 3;
  const int mi = lane >> 3, r8 = lane & 7;
  const int W = a.W, r = a.r, Wr = (W + 15) & ~15;
  const int np = P + 1, Kp = (np + 15) & ~15;

  float* vec = reinterpret_cast<float*>(sm + L.vec);
  float *colexp = vec + 2 * D, *colmax = vec + 3 * D, *Lt = vec + 4 * D;
  int32_t* sel = reinterpret_cast<int32_t*>(vec + 7 * D + 4);
  float* fac = reinterpret_cast<float*>(sm + L.coef) + 2 * (W + r);
  uint8_t* s_codes = st + L.codes;
  const float* s_scales = reinterpret_cast<const float*>(st + L.scales);
  bf* s_bk = reinterpret_cast<bf*>(st + L.bk);
  bf* s_bu = reinterpret_cast<bf*>(st + L.bu);
  float* s_bL = reinterpret_cast<float*>(st + L.bL);
  bf* pl_mid = reinterpret_cast<bf*>(st + L.bL);  // diagonal gate: planes of Kt in bL's space
  bf* pl_lo = pl_mid + Wr * D;
  const int32_t* s_cidx = reinterpret_cast<const int32_t*>(st + L.cidx);
  const float* s_cu = reinterpret_cast<const float*>(st + L.cu);

  // ---- operands: colexp, per-pair factors or split Kt planes, zero padding rows ----------
  for (int j = tid; j < D; j += C::NT) {
    colexp[j] = fast_exp(C::DIAG ? Lt[j] : Ls);
    colmax[j] = 0.f;
  }
  for (int e = np * D + tid; e < Kp * D; e += C::NT) s_bu[e] = __float2bfloat16_rn(0.f);
  if constexpr (!C::DIAG) {
    for (int i = tid; i < Kp; i += C::NT) fac[i] = i < np ? fast_exp(Ls - s_bL[i]) : 0.f;
    for (int e = np * D + tid; e < Kp * D; e += C::NT) s_bk[e] = __float2bfloat16_rn(0.f);
  } else {
    // Kt[i][j] = k_i[j] e^{L_W[j] - L_i[j]} -> hi (over bk), mid and lo (over bL), pairs of
    // adjacent columns per thread; all of bL is read before any plane part is written there
    constexpr int kPairs = kMmaDiagMaxW * D / 2 / kThreads;  // column pairs per thread
    uint32_t mids[kPairs], los[kPairs];
#pragma unroll
    for (int t = 0; t < kPairs; ++t) {
      const int e = 2 * (tid + t * C::NT);
      mids[t] = los[t] = 0u;
      if (e < Kp * D) {
        float h0 = 0.f, m0 = 0.f, l0 = 0.f, h1 = 0.f, m1 = 0.f, l1 = 0.f;
        const int sw = swz_el<bf, D>(e / D, e % D);  // columns e, e+1 share a chunk
        if (e < np * D) {
          const int j = e % D;
          split3(__bfloat162float(s_bk[sw]) * fast_exp(Lt[j] - s_bL[e]), h0, m0, l0);
          split3(__bfloat162float(s_bk[sw + 1]) * fast_exp(Lt[j + 1] - s_bL[e + 1]), h1, m1, l1);
        }
        *reinterpret_cast<uint32_t*>(s_bk + sw) = pack_bf16(h0, h1);
        mids[t] = pack_bf16(m0, m1);
        los[t] = pack_bf16(l0, l1);
      }
    }
    csync();
#pragma unroll
    for (int t = 0; t < kPairs; ++t) {
      const int e = 2 * (tid + t * C::NT);
      if (e < Kp * D) {
        const int sw = swz_el<bf, D>(e / D, e % D);
        *reinterpret_cast<uint32_t*>(pl_mid + sw) = mids[t];
        *reinterpret_cast<uint32_t*>(pl_lo + sw) = los[t];
      }
    }
  }
  csync();

  // ---- the materialised state, all 16 n-tiles of this warp's 16 rows, computed once -------
  // acc[nt][0..3] = S_W at (v0, j), (v0, j+1), (v1, j), (v1, j+1), j = 8 nt + 2 q4. Warp w takes
  // rows rbase .. rbase + 15, inside the TMEM lanes it may access (32 (w % 4) ..).
  const int rbase = 32 * (warp & 3) + 16 * (warp >> 2);
  const int v0 = rbase + gid, v1 = v0 + 8;
  // scalar gate, at most 64 pairs: the rank update runs on tcgen05 with the accumulators in TMEM
  const bool use_tc = !C::DIAG && Kp <= 64;
  float acc[16][4];
  {
    const float s0 = C::INT4 ? 0.f : s_scales[v0], s1 = C::INT4 ? 0.f : s_scales[v1];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int j = 8 * nt + 2 * q4;
      float c00, c01, c10, c11, t0 = s0, t1 = s1;
      if constexpr (C::INT4) {
        // one byte = columns j (low nibble), j + 1 (high): bias to c + 8, 2^23 trick
        const uint32_t b0 = s_codes[swz<64>(v0, j / 2)] ^ 0x88u;
        const uint32_t b1 = s_codes[swz<64>(v1, j / 2)] ^ 0x88u;
        c00 = __uint_as_float(0x4B000000u | (b0 & 0xFu)) - 8388616.f;
        c01 = __uint_as_float(0x4B000000u | (b0 >> 4)) - 8388616.f;
        c10 = __uint_as_float(0x4B000000u | (b1 & 0xFu)) - 8388616.f;
        c11 = __uint_as_float(0x4B000000u | (b1 >> 4)) - 8388616.f;
        t0 = s_scales[v0 * C::NG + j / 32];
        t1 = s_scales[v1 * C::NG + j / 32];
      } else {
        const uint32_t h0 = *reinterpret_cast<const uint16_t*>(s_codes + swz<128>(v0, j)) ^ 0x8080u;
        const uint32_t h1 = *reinterpret_cast<const uint16_t*>(s_codes + swz<128>(v1, j)) ^ 0x8080u;
        c00 = __uint_as_float(__byte_perm(h0, 0x4B000000u, 0x7650)) - 8388736.f;
        c01 = __uint_as_float(__byte_perm(h0, 0x4B000000u, 0x7651)) - 8388736.f;
        c10 = __uint_as_float(__byte_perm(h1, 0x4B000000u, 0x7650)) - 8388736.f;
        c11 = __uint_as_float(__byte_perm(h1, 0x4B000000u, 0x7651)) - 8388736.f;
      }
      float e0 = colexp[j], e1 = colexp[j + 1];
      if constexpr (C::SMOOTH) {  // the frozen codes' factor 2^e (the old exponents)
        const int8_t* s_sexp = reinterpret_cast<const int8_t*>(st + L.sexp);
        e0 *= pow2i(s_sexp[j]);
        e1 *= pow2i(s_sexp[j + 1]);
      }
      acc[nt][0] = t0 * c00 * e0;
      acc[nt][1] = t0 * c01 * e1;
      acc[nt][2] = t1 * c10 * e0;
      acc[nt][3] = t1 * c11 * e1;
    }
    // compensator pairs (key e_jc at gate 0), added with selects so that no data-dependent
    // index reaches the accumulator array
    for (int c = 0; c < r; ++c) {
      const int jc = s_cidx[c] & (D - 1);
      const bool mine = ((jc & 7) >> 1) == q4, odd = jc & 1;
      const float ec = colexp[jc];
      const float u0 = mine ? s_cu[c * D + v0] * ec : 0.f;
      const float u1 = mine ? s_cu[c * D + v1] * ec : 0.f;
      const uint32_t hit = one_hot_opaque(jc >> 3);
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const bool h = (hit >> nt) & 1u;
        acc[nt][0] += (h && !odd) ? u0 : 0.f;
        acc[nt][1] += (h && odd) ? u0 : 0.f;
        acc[nt][2] += (h && !odd) ? u1 : 0.f;
        acc[nt][3] += (h && odd) ? u1 : 0.f;
      }
    }
    if (use_tc) {
      if constexpr (!C::DIAG) {
        // rank-Kp update on tcgen05: D (TMEM lanes = rows v, columns j) starts as the frozen part
        // above; A = (U Diag(fac))^T split into hi / mid / lo bf16, in TMEM (lane v, two pairs a
        // column); B = the keys, exact, permuted in place in the stage into 8 x 8 core matrices
        const uint32_t tl = tc.tmem + ((uint32_t)rbase << 16);
        tmem_st_frag8(tl, *reinterpret_cast<const float(*)[8][4]>(&acc[0]));
        tmem_st_frag8(tl + 64, *reinterpret_cast<const float(*)[8][4]>(&acc[8]));
        for (int n = 0; n < Kp / 16; ++n) {
          const int k0 = 16 * n + 4 * q4;
          uint32_t pk[3][4];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int v = hh ? v1 : v0;
            float h[4], m[4], l[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              split3(__bfloat162float(s_bu[swz_el<bf, D>(k0 + e, v)]) * fac[k0 + e], h[e], m[e], l[e]);
            pk[0][2 * hh] = pack_bf16(h[0], h[1]);
            pk[0][2 * hh + 1] = pack_bf16(h[2], h[3]);
            pk[1][2 * hh] = pack_bf16(m[0], m[1]);
            pk[1][2 * hh + 1] = pack_bf16(m[2], m[3]);
            pk[2][2 * hh] = pack_bf16(l[0], l[1]);
            pk[2][2 * hh + 1] = pack_bf16(l[2], l[3]);
          }
#pragma unroll
          for (int p = 0; p < 3; ++p)
            tmem_st_frag1(tl + 128 + 32 * p + 8 * n, pk[p][0], pk[p][1], pk[p][2], pk[p][3]);
        }
        // key rows [0, Kp): 16-byte chunk (i, c) to core matrix (c, i / 8), row i % 8
        uint8_t* kbytes = reinterpret_cast<uint8_t*>(s_bk);
        uint4 tmp[4];
        int dst[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int e = tid + C::NT * t, i = e >> 4, c = e & 15;
          dst[t] = -1;
          if (i < Kp) {
            tmp[t] = *reinterpret_cast<const uint4*>(kbytes + swz<256>(i, 16 * c));
            dst[t] = (c * (Kp >> 3) + (i >> 3)) * 128 + (i & 7) * 16;
          }
        }
        csync();
#pragma unroll
        for (int t = 0; t < 4; ++t)
          if (dst[t] >= 0) *reinterpret_cast<uint4*>(kbytes + dst[t]) = tmp[t];
        fence_async_smem();
        tc_wait_st();
        tc_fence_before();
        csync();
        if (tid == 0) {
          tc_fence_after();
          constexpr uint32_t kIdesc = idesc_bf16(128, 128, false, true);
          const uint32_t kb = smem_u32(kbytes);
          for (int kk = 0; kk < Kp / 16; ++kk)
#pragma unroll
            for (int p = 0; p < 3; ++p)
              umma_bf16_ts(tc.tmem, tc.tmem + 128 + 32 * p + 8 * kk,
                           interleave_desc(kb + 256u * kk, 128u, 16u * (uint32_t)Kp), kIdesc, 1u);
          umma_commit(tc.bar);
        }
        if (!mbar_wait_bounded(tc.bar, tc.phase)) report(a.status, GDN_DEVICE_WAIT_TIMEOUT);
        tc.phase ^= 1u;
        tc_fence_after();
        tmem_ld_frag8(tl, *reinterpret_cast<float(*)[8][4]>(&acc[0]));
        tmem_ld_frag8(tl + 64, *reinterpret_cast<float(*)[8][4]>(&acc[8]));
      }
    } else {
    // rank-Kp update U^T (v rows, pair k) times Kt (pair k, column j); the split left-hand
    // side of a k-step serves all 16 n-tiles
    const uint32_t ub = smem_u32(s_bu), kb = smem_u32(s_bk);
    const uint32_t mb = smem_u32(pl_mid), lb = smem_u32(pl_lo);
    for (int s = 0; s < Kp / 16; ++s) {
      uint32_t A[4];
      ldsm_x4_t(ub + swz<256>(16 * s + r8 + 8 * (mi >> 1), 2 * (rbase + 8 * (mi & 1))), A);
      uint32_t Ah[4], Am[4], Al[4];
      if constexpr (!C::DIAG) {
        const int i0 = 16 * s + 2 * q4;
        const float f0 = fac[i0], f1 = fac[i0 + 1], f2 = fac[i0 + 8], f3 = fac[i0 + 9];
        split3_pair(A[0], f0, f1, Ah[0], Am[0], Al[0]);
        split3_pair(A[1], f0, f1, Ah[1], Am[1], Al[1]);
        split3_pair(A[2], f2, f3, Ah[2], Am[2], Al[2]);
        split3_pair(A[3], f2, f3, Ah[3], Am[3], Al[3]);
      }
#pragma unroll
      for (int n2 = 0; n2 < 8; ++n2) {
        const uint32_t off = swz<256>(16 * s + r8 + 8 * (mi & 1), 2 * (16 * n2 + 8 * (mi >> 1)));
        uint32_t B[4];
        ldsm_x4_t(kb + off, B);
        if constexpr (!C::DIAG) {
          mma_bf16(acc[2 * n2], Ah, B[0], B[1]);
          mma_bf16(acc[2 * n2], Am, B[0], B[1]);
          mma_bf16(acc[2 * n2], Al, B[0], B[1]);
          mma_bf16(acc[2 * n2 + 1], Ah, B[2], B[3]);
          mma_bf16(acc[2 * n2 + 1], Am, B[2], B[3]);
          mma_bf16(acc[2 * n2 + 1], Al, B[2], B[3]);
        } else {
          mma_bf16(acc[2 * n2], A, B[0], B[1]);
          mma_bf16(acc[2 * n2 + 1], A, B[2], B[3]);
          ldsm_x4_t(mb + off, B);
          mma_bf16(acc[2 * n2], A, B[0], B[1]);
          mma_bf16(acc[2 * n2 + 1], A, B[2], B[3]);
          ldsm_x4_t(lb + off, B);
          mma_bf16(acc[2 * n2], A, B[0], B[1]);
          mma_bf16(acc[2 * n2 + 1], A, B[2], B[3]);
        }
      }
    }
    }
  }

  // ---- compensators: column max-abs, the top r (ties: lower index), taken out exactly -----
  if (r > 0 || C::SMOOTH) {
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      float m0 = fmaxf(fabsf(acc[nt][0]), fabsf(acc[nt][2]));
      float m1 = fmaxf(fabsf(acc[nt][1]), fabsf(acc[nt][3]));
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
      }
      if (gid == 0) {
        unsigned int* cm = reinterpret_cast<unsigned int*>(colmax) + 8 * nt + 2 * q4;
        atomicMax(cm, __float_as_uint(m0));
        atomicMax(cm + 1, __float_as_uint(m1));
      }
    }
    csync();
    if (warp == 0) {
      for (int c = 0; c < r; ++c) {
        float bv = -1.f;
        int bj = D;
        for (int j = lane; j < D; j += 32) {
          const float v = colmax[j];
          if (v > bv) { bv = v; bj = j; }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
          if (ov > bv || (ov == bv && oj < bj)) { bv = ov; bj = oj; }
        }
        if (lane == 0) {
          sel[c] = bj;
          colmax[bj] = -2.f;  // taken
        }
        __syncwarp();
      }
    }
    csync();
    if (tid < r) a.comp_idx[(size_t)head * ((r + 3) & ~3) + tid] = sel[tid];
    float* g_cu = a.comp_u + (size_t)head * r * D;
    for (int c = 0; c < r; ++c) {
      const int jc = sel[c];
      const bool mine = ((jc & 7) >> 1) == q4, odd = jc & 1;
      float x0 = 0.f, x1 = 0.f;
      bool here = false;
      const uint32_t hit = mine ? one_hot_opaque(jc >> 3) : 0u;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const bool h = (hit >> nt) & 1u;
        const bool he = h && !odd, ho = h && odd;
        here = here || h;
        x0 = he ? acc[nt][0] : (ho ? acc[nt][1] : x0);
        x1 = he ? acc[nt][2] : (ho ? acc[nt][3] : x1);
        acc[nt][0] = he ? 0.f : acc[nt][0];
        acc[nt][1] = ho ? 0.f : acc[nt][1];
        acc[nt][2] = he ? 0.f : acc[nt][2];
        acc[nt][3] = ho ? 0.f : acc[nt][3];
      }
      if (here) {
        g_cu[c * D + v0] = x0;
        g_cu[c * D + v1] = x1;
      }
    }
    // residual smoothing: column j's exponent from the residual's max-abs (a taken column has
    // colmax -2: exponent 0), the residual times 2^-e_j before the row absmax
    if constexpr (C::SMOOTH) {
      for (int j = tid; j < D; j += C::NT) {
        const int e = smooth_exponent(colmax[j]);
        a.smooth_exp[(size_t)head * D + j] = (int8_t)e;
        colexp[j] = pow2i(-e);  // colexp is dead once the tile is materialised
      }
      csync();
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const float f0 = colexp[8 * nt + 2 * q4], f1 = colexp[8 * nt + 2 * q4 + 1];
        acc[nt][0] *= f0;
        acc[nt][1] *= f1;
        acc[nt][2] *= f0;
        acc[nt][3] *= f1;
      }
    }
  }

  // ---- scales and codes into this warp's rows of the stage's code tile ---------------------
  // (the warp read its old code rows above and no other warp reads them)
  float* g_scales = a.scales + (size_t)head * a.scale_stride;
  __syncwarp();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int v = h ? v1 : v0;
#pragma unroll
    for (int gq = 0; gq < (C::INT4 ? 4 : 1); ++gq) {  // int4: groups of 4 n-tiles
      constexpr int NPG = C::INT4 ? 4 : 16;
      float m = 0.f;
#pragma unroll
      for (int nt = NPG * gq; nt < NPG * gq + NPG; ++nt)
        m = fmaxf(m, fmaxf(fabsf(acc[nt][2 * h]), fabsf(acc[nt][2 * h + 1])));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      const float sc = __fdiv_rn(m, (float)QMAX);
      const float inv = sc > 0.f ? __frcp_rn(sc) : 0.f;
      if (q4 == 0) g_scales[v * C::NG + gq] = sc;
#pragma unroll
      for (int nt = NPG * gq; nt < NPG * gq + NPG; ++nt) {
        int qv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float t = sc > 0.f ? rint_quotient(acc[nt][2 * h + e], sc, inv) : 0.f;
          qv[e] = (int)fminf(fmaxf(t, (float)-QMAX), (float)QMAX);
        }
        if constexpr (C::INT4)
          s_codes[swz<64>(v, 4 * nt + q4)] = (uint8_t)((qv[0] & 0xF) | ((qv[1] & 0xF) << 4));
        else
          *reinterpret_cast<uint16_t*>(s_codes + swz<128>(v, 8 * nt + 2 * q4)) =
              (uint16_t)((qv[0] & 0xFF) | ((qv[1] & 0xFF) << 8));
      }
    }
  }
  __syncwarp();
  // ---- this warp's 16 code rows to HBM, 16 bytes per lane per store -----------------------
  {
    constexpr int RB = C::ROW_BYTES, CH = 16 * RB / 16;  // 16-byte chunks of the warp's rows
    uint8_t* g_codes = a.codes + (size_t)head * a.code_stride + rbase * RB;
    const uint8_t* src = s_codes + rbase * RB;
#pragma unroll
    for (int ch = lane; ch < CH; ch += 32)
      *reinterpret_cast<uint4*>(g_codes + 16 * ch) = *reinterpret_cast<const uint4*>(src + 16 * ch);
  }
}

}  // namespace gdnq
