// Windowed low-bit state kernels: decode step with the fused window flush, forced flush,
// materialisation and initial quantization. One CTA of 256 threads per (sequence, head).
//
// Method: "LeapQuant: Efficient Linear Attention with Accurate Recurrent State Quantization",
// Abstract -- the state is frozen in low bits for a window of tokens; each step reads the frozen
// state plus buffered high-precision write pairs; the state is materialised and requantised once,
// at the window's end, with its largest-outlier key columns kept aside as compensator pairs.
//
// Per step, with P pairs in the window and L_t = L_{t-1} + g_t the cumulative log-gate:
//   x = e^{L_t} k_t, y = e^{L_t} q_t
//   w = F x + sum_c cu_c x[j_c] + sum_{i<P} bu_i <bk_i e^{L_t - bL_i}, k_t>   (= S_{t-1} Diag(a_t) k_t)
//   r = F y + sum_c cu_c y[j_c] + sum_{i<P} bu_i <bk_i e^{L_t - bL_i}, q_t>
//   u_t = beta_t (v_t - w), o_t = r + u_t <k_t, q_t>
// because S_{t-1} Diag(a)(I - beta k k^T) + beta v k^T = S_{t-1} Diag(a) + beta (v - S_{t-1} Diag(a) k) k^T.
//
// Data path of a CTA: one thread issues bulk async copies (TMA, 1-D) of the head's codes,
// scales, the P buffered pairs and the compensators into shared memory, all completing on one
// mbarrier; meanwhile the CTA loads the step's q, k and gate. Then
//   phase 1  dual mat-vec over the codes (dequantised in registers, fp32 accumulate, shuffles);
//   phase 2  per-pair coefficients <bk_i e^{..}, k_t>, <.., q_t>;
//   phase 3  w, r corrections from the buffered write vectors and compensators;
//   phase 4  u_t, o_t, append the pair (to HBM, or to shared memory when the window ends);
//   phase 5  (window end only) materialise the state tile by tile in registers, pick
//            compensator columns, absmax, requantise, store codes / scales / compensators.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "device_util.cuh"
#include "gdnq.h"
#include "tc_util.cuh"

namespace gdnq {

constexpr int kThreads = 256;

// Tensor memory of a persistent step CTA whose window flush runs its rank update on tcgen05
// (scalar gate): the CTA's TMEM columns (128 for the materialised state, 3 x 32 for the split
// write-vector operand), the mbarrier the products commit to, and that barrier's next phase.
struct TcCtx {
  uint32_t tmem;
  uint64_t* bar;
  uint32_t phase;
};
constexpr uint32_t kFlushTmemCols = 256;

template <int D_, bool DIAG_, bool INT4_, typename Act_, typename Buf_, bool SMOOTH_ = false>
struct WinCfg {
  static constexpr int D = D_;
  static constexpr bool DIAG = DIAG_;
  static constexpr bool INT4 = INT4_;
  // residual smoothing: frozen state dequant(codes, scales) Diag(2^e), e per key column
  static constexpr bool SMOOTH = SMOOTH_;
  using Act = Act_;
  using Buf = Buf_;
  static constexpr int NT = kThreads;
  static constexpr int QMAX = INT4 ? 7 : 127;
  static constexpr int GS = INT4 ? 32 : D;  // columns per scale
  static constexpr int NG = D / GS;         // scales per row
  static constexpr int ROW_BYTES = INT4 ? D / 2 : D;
  static constexpr int CODE_BYTES = D * ROW_BYTES;
  static constexpr int NSCALES = D * NG;
  // mat-vec mapping: 16 columns per thread chunk, CPR chunks per row, RPP rows per pass
  static constexpr int CPR = D / 16;
  static constexpr int RPP = NT / CPR;
  // tile mapping (flush / materialise / quantize): CG column groups of TC columns, RG row
  // groups, TR rows per thread per pass
  static constexpr int CG = 16;
  static constexpr int RG = NT / CG;
  static constexpr int TC = D / CG;
  static constexpr int TR = (D / RG) >= 2 ? 2 : 1;
  static constexpr int RPASS = RG * TR;
  static constexpr int NPASS = D / RPASS;
  // phase-3 mapping: one value channel per thread, G groups over the pairs
  static constexpr int G = NT / D;
  static_assert(D % 16 == 0 && D <= 128, "head size");
  static_assert(!INT4 || D % 32 == 0, "int4 needs whole groups of 32");
  static_assert(NPASS * RPASS == D, "tile passes");
  static_assert(TC <= GS, "a thread's columns share one scale");
  // Tensor-core (mma.sync) path: d = 128 with bf16 activations and bf16 buffers.
  static constexpr bool MMA = D == 128 && sizeof(Act) == 2 && sizeof(Buf) == 2;
};

__host__ __device__ constexpr uint32_t align128(uint32_t x) { return (x + 127u) & ~127u; }

// Shared-memory layout of a window kernel (byte offsets). A stage holds one head's staged data
// (frozen codes and scales, buffered pairs, compensators, and the step's q, k, v and, for the
// diagonal gate, g); the CTA keeps `nstages` stages plus per-head scratch (vectors,
// coefficients, reduction space) and, for the persistent step kernel, the pos / gate / beta of
// its whole head range.
struct WinLayout {
  uint32_t codes, scales, bk, bu, bL, cidx, cu, ck, q, k, v, g, sexp, stage_bytes;  // within a stage
  uint32_t bars, stage0, vec, coef, red, tc, harr, total;                 // within the CTA
};

// Tensor-core scratch: int8 digit matrix of the phase-1 right-hand side [8][144 B] and the bf16
// [8][Wr + 8] split coefficients of the correction products (row strides padded against bank
// conflicts).
__host__ __device__ constexpr uint32_t tc_scratch_bytes(int Wr) {
  return 8u * 144 + 8u * (Wr + 8) * 2 + 64;
}

// Per-CTA scratch first (barriers, vectors, coefficients, reduction space unless `red` is false,
// tensor-core scratch, the pos / gate / beta of the CTA's heads), then `nstages` stages whose
// buffered-pair regions hold `cap` rows (a multiple of 16, at most W rounded up to 16; -1 means
// that maximum). The kernels only ever read or write pair rows below the stage's cap. With
// `smooth` a stage also holds the head's D smoothing exponents; with `power` the r compensator
// token keys.
__host__ __device__ inline WinLayout win_layout(int D, int code_bytes, int nscales, int act_size,
                                                int buf_size, bool diag, int W, int r,
                                                int nstages, int per_cta, int cap = -1,
                                                bool red = true, bool smooth = false,
                                                bool power = false) {
  // buffer rows rounded up to 16: the mma k-steps read (zero-filled) rows past the window
  const int Wp = (W + 3) & ~3, rp = (r + 3) & ~3, Wr = (W + 15) & ~15;
  if (cap < 0) cap = Wr;
  WinLayout L;
  L.bars = 0;
  L.vec = 128;
  L.coef = align128(L.vec + 4u * (7 * D + 64));
  L.red = align128(L.coef + 4u * (2 * (W + r) + Wr + 4));  // a[W+r], b[W+r], fac[Wr]
  L.tc = align128(L.red + (red ? 4u * 2 * kThreads : 0u));
  L.harr = align128(L.tc + tc_scratch_bytes(Wr));
  L.stage0 = align128(L.harr + 12u * per_cta);
  L.codes = 0;
  L.scales = align128(L.codes + code_bytes);
  L.bk = align128(L.scales + 4u * nscales);
  L.bu = align128(L.bk + (uint32_t)cap * D * act_size);
  L.bL = align128(L.bu + (uint32_t)cap * D * buf_size);
  L.cidx = align128(L.bL + 4u * (diag ? (uint32_t)cap * D : (uint32_t)Wp));
  L.cu = align128(L.cidx + 4u * rp);
  L.ck = align128(L.cu + 4u * r * D);
  L.q = align128(L.ck + (power ? 4u * r * D : 0u));
  L.k = align128(L.q + (uint32_t)D * act_size);
  L.v = align128(L.k + (uint32_t)D * act_size);
  L.g = align128(L.v + (uint32_t)D * act_size);
  L.sexp = align128(L.g + (diag ? 4u * D : 0u));
  L.stage_bytes = align128(L.sexp + (smooth ? (uint32_t)D : 0u));
  L.total = L.stage0 + (uint32_t)nstages * L.stage_bytes;
  return L;
}

template <class C>
__host__ __device__ inline WinLayout win_layout(int W, int r, int nstages, int per_cta,
                                                int cap = -1, bool red = true,
                                                bool power = false) {
  return win_layout(C::D, C::CODE_BYTES, C::NSCALES, (int)sizeof(typename C::Act),
                    (int)sizeof(typename C::Buf), C::DIAG, W, r, nstages, per_cta, cap, red,
                    C::SMOOTH, power);
}

// The int4 (group 32) configuration that shares C's head size, gate and dtypes, and the shared-
// memory layout that holds a head of either format (codes of the int8 size, scales of the int4
// size) when MIX is set.
template <class C>
using Int4Of = WinCfg<C::D, C::DIAG, true, typename C::Act, typename C::Buf>;

template <class C, bool MIX>
__host__ __device__ inline WinLayout win_layout_mix(int W, int r, int nstages, int per_cta,
                                                    int cap = -1, bool red = true,
                                                    bool power = false) {
  if constexpr (!MIX) {
    return win_layout<C>(W, r, nstages, per_cta, cap, red, power);
  } else {
    return win_layout(C::D, C::CODE_BYTES, Int4Of<C>::NSCALES, (int)sizeof(typename C::Act),
                      (int)sizeof(typename C::Buf), C::DIAG, W, r, nstages, per_cta, cap, red);
  }
}

// Longest window whose diagonal-gate flush builds its split key planes in registers here.
constexpr int kMmaDiagMaxW = 128;

// Whether a configuration's decode step takes the tensor-core path (which needs no reduction
// space and whose pair regions may be sized to the furthest window position).
template <class C>
__host__ __device__ inline bool step_uses_mma(int W) {
  return C::MMA && (!C::DIAG || W <= kMmaDiagMaxW);
}

// Kernel arguments: the state's device pointers and the step's inputs (unused ones null).
struct WinArgs {
  uint8_t* codes;
  float* scales;
  void* buf_k;
  void* buf_u;
  float* buf_L;
  int32_t* comp_idx;
  float* comp_u;
  int32_t* pos;
  int32_t* status;
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  void* o;
  const float* S_in;       // quantize: fp32 states
  float* S_out;            // materialise: fp32 states
  const int32_t* seq_mask; // forced flush: [B] or null
  const int8_t* head_fmt;  // mixed formats: gdn_state_format of each head, else null
  uint32_t code_stride;    // bytes of codes per head
  uint32_t scale_stride;   // scales (floats) per head
  int H, W, r;
  int8_t* smooth_exp;      // residual smoothing: [heads][D] column exponents, else null
  float* comp_k;           // power compensator tokens: [heads][r][D] keys, else null
};

// 2^e for an integer e in [-126, 127], from the exponent bits (exact).
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

// Residual smoothing exponent of a column whose max-abs is m: floor(floor(log2 m) / 2) clamped
// to [-63, 63] (a subnormal m counts as 2^-127); 0 for m <= 0 (a zero or a taken column).
__device__ __forceinline__ int smooth_exponent(float m) {
  if (!(m > 0.f)) return 0;
  const int E = (int)(__float_as_uint(m) >> 23) - 127;
  return max(-63, min(63, E >> 1));  // arithmetic shift: floor(E / 2)
}

// Whether a head of a mixed-format state is held as int4 (group 32).
__device__ __forceinline__ bool head_is_int4(const WinArgs& a, int head) {
  return a.head_fmt != nullptr && a.head_fmt[head] == GDN_FMT_INT4_G32;
}

// N consecutive logical elements (from column col0) of row `row` of a swizzled [rows][D] tile
// of T, as fp32.
template <typename T, int D, int N>
__device__ __forceinline__ void load_sw(const T* base, int row, int col0, float* out) {
  constexpr int EPC = 16 / (int)sizeof(T);  // elements per 16-byte chunk
  if constexpr (N % EPC == 0) {
#pragma unroll
    for (int q = 0; q < N / EPC; ++q)
      Num<T>::template load<EPC>(base + swz_el<T, D>(row, col0 + q * EPC), out + q * EPC);
  } else {
#pragma unroll
    for (int e = 0; e < N; ++e) out[e] = Num<T>::to_f(base[swz_el<T, D>(row, col0 + e)]);
  }
}

__device__ __forceinline__ void report(int32_t* status, int bit) {
  if (status) atomicOr(status, bit);
}

// ------------------------------------------------------------------------------------------
// Staging: one head's frozen state, its first P buffered pairs, its compensators and (with_io)
// the step's q, k, v (and diagonal g), copied into a stage with bulk async copies completing on
// the stage's mbarrier. Issued by one thread. An out-of-range P arms the barrier with no copies.
// ------------------------------------------------------------------------------------------
// Zero rows for the stages' write-vector regions (read by bulk copies; never written).
constexpr int kZeroRowBytes = 4096;
static __device__ __align__(128) uint8_t g_zero_rows[kZeroRowBytes];

template <class C>
__device__ __forceinline__ void stage_issue(const WinArgs& a, const WinLayout& L, uint8_t* st,
                                            uint64_t* bar, int head, int P, bool with_io,
                                            int part = -1, int zrows = 0, bool full = false) {
  // part -1: every copy; part 0: codes, scales, q, k; part 1: the rest (two issuers, each
  // arriving once on a barrier that expects two arrivals). zrows > 0 (with part != 0) also
  // copies zeros over the write-vector rows P .. P + zrows - 1 of the stage.
  using Act = typename C::Act;
  using Buf = typename C::Buf;
  constexpr int D = C::D;
  const int W = a.W, r = a.r, Wp = (W + 3) & ~3, rp = (r + 3) & ~3;
  if (P < 0 || P > W || (P == W && !full)) {  // full: a window end of all W pairs
    mbar_arrive_expect_tx(bar, 0);
    return;
  }
  const bool p0 = part <= 0, p1 = part != 0;
  const uint32_t lbytes = C::DIAG ? 4u * P * D : 4u * ((P + 3) & ~3);
  uint32_t bytes = 0;
  if (p0) bytes += C::CODE_BYTES + 4u * C::NSCALES + (with_io ? 2u * D * sizeof(Act) : 0u);
  if constexpr (C::SMOOTH) {
    if (p0) bytes += (uint32_t)D;
  }
  if (p1) {
    if (P > 0) bytes += (uint32_t)P * D * (sizeof(Act) + sizeof(Buf)) + lbytes;
    if (r > 0) bytes += 4u * rp + 4u * r * D;
    if (r > 0 && a.comp_k) bytes += 4u * r * D;
    if (with_io) bytes += D * sizeof(Act) + (C::DIAG ? 4u * D : 0u);
    bytes += (uint32_t)zrows * D * sizeof(Buf);
  }
  mbar_arrive_expect_tx(bar, bytes);
  if (p0) {
    bulk_g2s(st + L.codes, a.codes + (size_t)head * a.code_stride, C::CODE_BYTES, bar);
    bulk_g2s(st + L.scales, a.scales + (size_t)head * a.scale_stride, 4u * C::NSCALES, bar);
    if constexpr (C::SMOOTH) bulk_g2s(st + L.sexp, a.smooth_exp + (size_t)head * D, (uint32_t)D, bar);
    if (with_io) {
      bulk_g2s(st + L.q, static_cast<const Act*>(a.q) + (size_t)head * D, D * sizeof(Act), bar);
      bulk_g2s(st + L.k, static_cast<const Act*>(a.k) + (size_t)head * D, D * sizeof(Act), bar);
    }
  }
  if (p1) {
    if (P > 0) {
      bulk_g2s(st + L.bk, static_cast<const Act*>(a.buf_k) + (size_t)head * W * D,
               (uint32_t)P * D * sizeof(Act), bar);
      bulk_g2s(st + L.bu, static_cast<const Buf*>(a.buf_u) + (size_t)head * W * D,
               (uint32_t)P * D * sizeof(Buf), bar);
      bulk_g2s(st + L.bL, a.buf_L + (size_t)head * (C::DIAG ? (size_t)W * D : (size_t)Wp), lbytes,
               bar);
    }
    if (r > 0) {
      bulk_g2s(st + L.cidx, a.comp_idx + (size_t)head * rp, 4u * rp, bar);
      bulk_g2s(st + L.cu, a.comp_u + (size_t)head * r * D, 4u * r * D, bar);
      if (a.comp_k) bulk_g2s(st + L.ck, a.comp_k + (size_t)head * r * D, 4u * r * D, bar);
    }
    if (with_io) {
      bulk_g2s(st + L.v, static_cast<const Act*>(a.v) + (size_t)head * D, D * sizeof(Act), bar);
      if constexpr (C::DIAG) bulk_g2s(st + L.g, a.g + (size_t)head * D, 4u * D, bar);
    }
    if (zrows > 0)
      bulk_g2s(st + L.bu + (uint32_t)P * D * sizeof(Buf), g_zero_rows,
               (uint32_t)zrows * D * sizeof(Buf), bar);
  }
}

// Bounded wait on a stage barrier by all threads; false (after reporting) when it ran out, in
// which case every thread returns.
__device__ __forceinline__ bool stage_wait(const WinArgs& a, uint64_t* bar, uint32_t parity) {
  const int timed_out = mbar_wait_bounded(bar, parity) ? 0 : 1;
  if (csync_or(timed_out)) {
    if (threadIdx.x == 0) report(a.status, GDN_DEVICE_WAIT_TIMEOUT);
    return false;
  }
  return true;
}

// ------------------------------------------------------------------------------------------
// Tile makers: fill acc[TR][TC] with the fp32 logical state at rows of pass `ps` and the
// thread's columns. Thread (rg, cg) = (tid / CG, tid % CG) owns rows ps*RPASS + rg*TR + a and
// columns cg*TC + b.
// ------------------------------------------------------------------------------------------

// Logical state from the staged window: frozen codes scaled by e^{L_end} (per column), plus
// compensators, plus `npairs` buffered pairs. Before use, `colexp` holds e^{L_end[j]} for all
// columns; for the scalar gate `fac[i]` holds e^{L_end - bL_i}; for the diagonal gate the bL
// region holds kt_i[j] = bk_i[j] e^{L_end[j] - bL_i[j]} in fp32.
template <class C>
struct WindowTile {
  const uint8_t* codes;
  const float* scales;
  const typename C::Act* bk;
  const typename C::Buf* bu;
  const float* ktil;
  const float* fac;
  const int32_t* cidx;
  const float* cu;
  const float* ck;     // power tokens: keys [r][D] (null: column tokens, keys e_{cidx})
  const float* colexp;
  const int8_t* sexp;  // smoothing exponents of the frozen codes (SMOOTH only)
  int npairs, r;

  __device__ __forceinline__ void operator()(int ps, float (&acc)[C::TR][C::TC]) const {
    constexpr int D = C::D, TC = C::TC, TR = C::TR;
    const int tid = threadIdx.x, cg = tid % C::CG, rg = tid / C::CG;
    const int c0 = cg * TC;
    float ce[TC], cf[TC];  // column decay; the frozen codes' factor (decay times 2^e)
#pragma unroll
    for (int b = 0; b < TC; ++b) {
      ce[b] = colexp[c0 + b];
      cf[b] = ce[b];
      if constexpr (C::SMOOTH) cf[b] *= pow2i(sexp[c0 + b]);
    }
#pragma unroll
    for (int a = 0; a < TR; ++a) {
      const int row = ps * C::RPASS + rg * TR + a;
      float cv[TC];
      if constexpr (C::INT4) {
        static_assert(TC == 8, "int4 tile is 8 columns per thread");
        const uint32_t w = *reinterpret_cast<const uint32_t*>(codes + swz<C::ROW_BYTES>(row, c0 / 2));
        i4x8_to_f32(w, cv);
      } else if constexpr (TC == 8) {
        const uint2 w = *reinterpret_cast<const uint2*>(codes + swz<C::ROW_BYTES>(row, c0));
        i8x4_to_f32(w.x, cv);
        i8x4_to_f32(w.y, cv + 4);
      } else {
#pragma unroll
        for (int b = 0; b < TC; ++b)
          cv[b] = (float)(int)reinterpret_cast<const int8_t*>(codes)[swz<C::ROW_BYTES>(row, c0 + b)];
      }
      const float s = scales[row * C::NG + c0 / C::GS];
#pragma unroll
      for (int b = 0; b < TC; ++b) acc[a][b] = s * cv[b] * cf[b];
    }
    for (int c = 0; c < r; ++c) {
      if (ck) {  // token cu_c (ck_c * e^{L_end})^T
#pragma unroll
        for (int b = 0; b < TC; ++b) {
          const float kd = ck[c * D + c0 + b] * ce[b];
#pragma unroll
          for (int a = 0; a < TR; ++a)
            acc[a][b] = fmaf(cu[c * D + ps * C::RPASS + rg * TR + a], kd, acc[a][b]);
        }
        continue;
      }
      const int j = cidx[c];
      if (j / TC == cg) {
#pragma unroll
        for (int b = 0; b < TC; ++b)
          if (c0 + b == j) {
#pragma unroll
            for (int a = 0; a < TR; ++a)
              acc[a][b] += cu[c * D + ps * C::RPASS + rg * TR + a] * ce[b];
          }
      }
    }
    for (int i = 0; i < npairs; ++i) {
      float uu[TR], kk[TC];
#pragma unroll
      for (int a = 0; a < TR; ++a)
        uu[a] = Num<typename C::Buf>::to_f(
            bu[swz_el<typename C::Buf, D>(i, ps * C::RPASS + rg * TR + a)]);
      if constexpr (C::DIAG) {
#pragma unroll
        for (int b = 0; b < TC; ++b) kk[b] = ktil[i * D + c0 + b];
      } else {
        load_sw<typename C::Act, D, TC>(bk, i, c0, kk);
        const float f = fac[i];
#pragma unroll
        for (int a = 0; a < TR; ++a) uu[a] *= f;
      }
#pragma unroll
      for (int a = 0; a < TR; ++a)
#pragma unroll
        for (int b = 0; b < TC; ++b) acc[a][b] = fmaf(uu[a], kk[b], acc[a][b]);
    }
  }
};

// fp32 states straight from HBM (initial quantization).
template <class C>
struct DenseTile {
  const float* S;  // this head's [D][D]
  __device__ __forceinline__ void operator()(int ps, float (&acc)[C::TR][C::TC]) const {
    const int tid = threadIdx.x, cg = tid % C::CG, rg = tid / C::CG;
#pragma unroll
    for (int a = 0; a < C::TR; ++a) {
      const int row = ps * C::RPASS + rg * C::TR + a;
      if constexpr (C::TC % 4 == 0) {
        Num<float>::load<C::TC>(S + (size_t)row * C::D + cg * C::TC, acc[a]);
      } else {
#pragma unroll
        for (int b = 0; b < C::TC; ++b) acc[a][b] = S[(size_t)row * C::D + cg * C::TC + b];
      }
    }
  }
};

// ------------------------------------------------------------------------------------------
// Requantisation of the state that `make` produces: compensator columns (top r by max-abs,
// ties to the lower index) go to comp_u / comp_idx in fp32 and are zeroed; each row (int4: each
// 32-column group) gets s = absmax / QMAX and codes rint(x / s) clamped to [-QMAX, QMAX], both
// quotients correctly rounded as IEEE single division rounds them. Codes, scales and compensators are written straight to HBM; the
// tile maker may still read the staged old state because rows of later passes are untouched
// and the old compensators live in shared memory. `colmax` (D floats) and `sel` (r ints) are
// shared scratch. Called by all threads. With residual smoothing (C::SMOOTH) the columns' max-abs
// are always taken; after the compensator choice column j gets e_j = smooth_exponent(max-abs of
// the residual column) (0 for a taken column), written to g_sexp, and the residual is quantized
// times 2^-e_j.
// ------------------------------------------------------------------------------------------
template <class C, class Maker>
__device__ void requantize_store(const Maker& make, int r, uint8_t* g_codes, float* g_scales,
                                 int32_t* g_cidx, float* g_cu, float* colmax, int32_t* sel,
                                 int8_t* g_sexp = nullptr) {
  constexpr int D = C::D, TR = C::TR, TC = C::TC, QMAX = C::QMAX;
  const int tid = threadIdx.x, cg = tid % C::CG, rg = tid / C::CG;
  const int lane = tid & 31, warp = tid >> 5;
  float acc[TR][TC];

  if (r > 0 || C::SMOOTH) {
    for (int j = tid; j < D; j += C::NT) colmax[j] = 0.f;
    csync();
    for (int ps = 0; ps < C::NPASS; ++ps) {
      make(ps, acc);
#pragma unroll
      for (int b = 0; b < TC; ++b) {
        float m = 0.f;
#pragma unroll
        for (int a = 0; a < TR; ++a) m = fmaxf(m, fabsf(acc[a][b]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (lane < 16)
          atomicMax(reinterpret_cast<unsigned int*>(colmax) + cg * TC + b, __float_as_uint(m));
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
    if constexpr (C::SMOOTH) {  // colmax[j] becomes the column's factor 2^-e_j
      for (int j = tid; j < D; j += C::NT) {
        const int e = smooth_exponent(colmax[j]);
        g_sexp[j] = (int8_t)e;
        colmax[j] = pow2i(-e);
      }
      csync();
    }
  }

  for (int ps = 0; ps < C::NPASS; ++ps) {
    make(ps, acc);
    for (int c = 0; c < r; ++c) {
      const int j = sel[c];
      if (j / TC == cg) {
#pragma unroll
        for (int b = 0; b < TC; ++b)
          if (cg * TC + b == j) {
#pragma unroll
            for (int a = 0; a < TR; ++a) {
              g_cu[c * D + ps * C::RPASS + rg * TR + a] = acc[a][b];
              acc[a][b] = 0.f;
            }
          }
      }
    }
    if constexpr (C::SMOOTH) {
#pragma unroll
      for (int b = 0; b < TC; ++b) {
        const float f = colmax[cg * TC + b];
#pragma unroll
        for (int a = 0; a < TR; ++a) acc[a][b] *= f;
      }
    }
#pragma unroll
    for (int a = 0; a < TR; ++a) {
      const int row = ps * C::RPASS + rg * TR + a;
      float m = 0.f;
#pragma unroll
      for (int b = 0; b < TC; ++b) m = fmaxf(m, fabsf(acc[a][b]));
      // lanes sharing a scale: 16 column groups per row (int8), 4 per 32-column group (int4)
      constexpr int span = C::GS / TC;
#pragma unroll
      for (int off = span / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      // s = fp32(m / QMAX) and the codes' quotients, correctly rounded from a reciprocal with
      // one fma correction (IEEE division only for tiny or zero scales)
      const float s = m >= 0x1p-100f ? quot_const(m, (float)QMAX, 1.f / (float)QMAX)
                                     : __fdiv_rn(m, (float)QMAX);
      const bool fast = s >= 0x1p-125f;
      const float inv = fast ? __frcp_rn(s) : 0.f;
      int q[TC];
#pragma unroll
      for (int b = 0; b < TC; ++b) {
        float t = fast ? rintf(quot_const(acc[a][b], s, inv))
                       : (s > 0.f ? rintf(__fdiv_rn(acc[a][b], s)) : 0.f);
        t = fminf(fmaxf(t, (float)-QMAX), (float)QMAX);
        q[b] = (int)t;
      }
      if constexpr (C::INT4) {
        uint32_t wv = 0;
#pragma unroll
        for (int m2 = 0; m2 < TC / 2; ++m2)
          wv |= (((uint32_t)q[2 * m2] & 0xFu) | (((uint32_t)q[2 * m2 + 1] & 0xFu) << 4)) << (8 * m2);
        *reinterpret_cast<uint32_t*>(g_codes + swz<C::ROW_BYTES>(row, cg * TC / 2)) = wv;
        if (cg % span == 0) g_scales[row * C::NG + (cg * TC) / C::GS] = s;
      } else {
        if constexpr (TC == 8) {
          uint2 wv;
          wv.x = ((uint32_t)q[0] & 0xFFu) | (((uint32_t)q[1] & 0xFFu) << 8) |
                 (((uint32_t)q[2] & 0xFFu) << 16) | (((uint32_t)q[3] & 0xFFu) << 24);
          wv.y = ((uint32_t)q[4] & 0xFFu) | (((uint32_t)q[5] & 0xFFu) << 8) |
                 (((uint32_t)q[6] & 0xFFu) << 16) | (((uint32_t)q[7] & 0xFFu) << 24);
          *reinterpret_cast<uint2*>(g_codes + swz<C::ROW_BYTES>(row, cg * TC)) = wv;
        } else {
#pragma unroll
          for (int b = 0; b < TC; ++b)
            reinterpret_cast<int8_t*>(g_codes)[swz<C::ROW_BYTES>(row, cg * TC + b)] = (int8_t)q[b];
        }
        if (cg == 0) g_scales[row] = s;
      }
    }
  }
  if (tid < r) g_cidx[tid] = sel[tid];
}

// Window-end preparation in shared memory for the logical state at cumulative gate `Lend`
// (per column in `Lvec` for the diagonal gate, scalar `Ls` otherwise) over `npairs` staged
// pairs of stage `st`: colexp[j] = e^{Lend[j]}; scalar gate: fac[i] = e^{Lend - bL_i}; diagonal
// gate: the stage's bL region becomes bk_i[j] e^{Lend[j] - bL_i[j]} (fp32, in place).
template <class C>
__device__ __forceinline__ void prepare_window_end(uint8_t* st, const WinLayout& L, int npairs,
                                                   const float* Lvec, float Ls, float* colexp,
                                                   float* fac) {
  constexpr int D = C::D;
  float* bL = reinterpret_cast<float*>(st + L.bL);
  const typename C::Act* bk = reinterpret_cast<const typename C::Act*>(st + L.bk);
  for (int j = threadIdx.x; j < D; j += C::NT) colexp[j] = fast_exp(C::DIAG ? Lvec[j] : Ls);
  if constexpr (C::DIAG) {
    for (int e = threadIdx.x; e < npairs * D; e += C::NT) {
      const int j = e % D;
      bL[e] = Num<typename C::Act>::to_f(bk[swz_el<typename C::Act, D>(e / D, j)]) *
              fast_exp(Lvec[j] - bL[e]);
    }
  } else {
    for (int i = threadIdx.x; i < npairs; i += C::NT) fac[i] = fast_exp(Ls - bL[i]);
  }
}

template <class C>
__device__ __forceinline__ WindowTile<C> window_tile(const uint8_t* st, const WinLayout& L,
                                                     int npairs, int r, const float* colexp,
                                                     const float* fac, bool power = false) {
  WindowTile<C> t;
  t.codes = st + L.codes;
  t.scales = reinterpret_cast<const float*>(st + L.scales);
  t.bk = reinterpret_cast<const typename C::Act*>(st + L.bk);
  t.bu = reinterpret_cast<const typename C::Buf*>(st + L.bu);
  t.ktil = reinterpret_cast<const float*>(st + L.bL);
  t.fac = fac;
  t.cidx = reinterpret_cast<const int32_t*>(st + L.cidx);
  t.cu = reinterpret_cast<const float*>(st + L.cu);
  t.ck = power ? reinterpret_cast<const float*>(st + L.ck) : nullptr;
  t.colexp = colexp;
  t.sexp = reinterpret_cast<const int8_t*>(st + L.sexp);
  t.npairs = npairs;
  t.r = r;
  return t;
}

}  // namespace gdnq
#include "window_mma.cuh"
namespace gdnq {

// ------------------------------------------------------------------------------------------
// One decode step (+ fused window flush) of one head whose data sit in stage `st`.
// Called by all threads; ends with every thread done reading the stage's inputs.
// ------------------------------------------------------------------------------------------
template <class C>
__device__ __forceinline__ void step_head(const WinArgs& a, const WinLayout& L, uint8_t* sm,
                                          uint8_t* st, int head, int P, float g_scalar,
                                          float beta, TcCtx& tc) {
  using Act = typename C::Act;
  using Buf = typename C::Buf;
  constexpr int D = C::D, CPR = C::CPR, RPP = C::RPP;
  if constexpr (C::MMA) {
    if (!C::DIAG || a.W <= kMmaDiagMaxW) {
      step_head_mma<C>(a, L, sm, st, head, P, g_scalar, beta, tc);
      return;
    }
  }
  const int tid = threadIdx.x, lane = tid & 31;
  const int W = a.W, r = a.r, Wp = (W + 3) & ~3;
  const bool flush = (P + 1 == W);

  float* vec = reinterpret_cast<float*>(sm + L.vec);
  float *kt = vec, *qt = vec + D, *xs = vec + 2 * D, *ys = vec + 3 * D, *Lt = vec + 4 * D;
  float *pv = vec + 5 * D, *rv = vec + 6 * D, *misc = vec + 7 * D;  // misc: kq, sel (as int)
  float* coef = reinterpret_cast<float*>(sm + L.coef);
  float *ca = coef, *cb = coef + (W + r), *fac = coef + 2 * (W + r);
  float* red = reinterpret_cast<float*>(sm + L.red);

  const uint8_t* s_codes = st + L.codes;
  const float* s_scales = reinterpret_cast<const float*>(st + L.scales);
  Act* s_bk = reinterpret_cast<Act*>(st + L.bk);
  Buf* s_bu = reinterpret_cast<Buf*>(st + L.bu);
  float* s_bL = reinterpret_cast<float*>(st + L.bL);
  const int32_t* s_cidx = reinterpret_cast<const int32_t*>(st + L.cidx);
  const float* s_cu = reinterpret_cast<const float*>(st + L.cu);
  const Act* s_q = reinterpret_cast<const Act*>(st + L.q);
  const Act* s_k = reinterpret_cast<const Act*>(st + L.k);
  const Act* s_v = reinterpret_cast<const Act*>(st + L.v);
  const float* s_g = reinterpret_cast<const float*>(st + L.g);

  // ---- gates and the scaled key / query -------------------------------------------------
  float Ls = 0.f;  // scalar-gate L_t
  if constexpr (!C::DIAG) Ls = (P > 0 ? s_bL[P - 1] : 0.f) + g_scalar;
  if (tid < D) {
    const float kj = Num<Act>::to_f(s_k[tid]), qj = Num<Act>::to_f(s_q[tid]);
    kt[tid] = kj;
    qt[tid] = qj;
    float l;
    if constexpr (C::DIAG) l = (P > 0 ? s_bL[(P - 1) * D + tid] : 0.f) + s_g[tid];
    else l = Ls;
    Lt[tid] = l;
    const float e = fast_exp(l);
    xs[tid] = e * kj;
    ys[tid] = e * qj;
  }
  csync();

  // ---- phase 1: p = F x, r = F y ---------------------------------------------------------
  {
    const int c = tid % CPR;
    float xr[16], yr[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      xr[e] = xs[c * 16 + e];
      yr[e] = ys[c * 16 + e];
      if constexpr (C::SMOOTH) {  // F = dequant Diag(2^e): the codes meet 2^e .* x
        const float f = pow2i(reinterpret_cast<const int8_t*>(st + L.sexp)[c * 16 + e]);
        xr[e] *= f;
        yr[e] *= f;
      }
    }
    for (int row = tid / CPR; row < D; row += RPP) {
      float cv[16];
      if constexpr (C::INT4) {
        const uint2 w = *reinterpret_cast<const uint2*>(s_codes + swz<C::ROW_BYTES>(row, c * 8));
        i4x8_to_f32(w.x, cv);
        i4x8_to_f32(w.y, cv + 8);
      } else {
        const uint4 w = *reinterpret_cast<const uint4*>(s_codes + swz<C::ROW_BYTES>(row, c * 16));
        i8x4_to_f32(w.x, cv);
        i8x4_to_f32(w.y, cv + 4);
        i8x4_to_f32(w.z, cv + 8);
        i8x4_to_f32(w.w, cv + 12);
      }
      float pa = 0.f, pb = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        pa = fmaf(cv[e], xr[e], pa);
        pb = fmaf(cv[e], yr[e], pb);
      }
      if constexpr (C::INT4) {
        const float s = s_scales[row * C::NG + (c * 16) / C::GS];
        pa *= s;
        pb *= s;
      }
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1) {
        pa += __shfl_xor_sync(0xffffffffu, pa, off);
        pb += __shfl_xor_sync(0xffffffffu, pb, off);
      }
      if (c == 0) {
        if constexpr (C::INT4) {
          pv[row] = pa;
          rv[row] = pb;
        } else {
          const float s = s_scales[row];
          pv[row] = pa * s;
          rv[row] = pb * s;
        }
      }
    }
  }

  // ---- phase 2: pair coefficients -------------------------------------------------------
  {
    const int c = tid % CPR;
    float kr[16], qr[16], lr[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      kr[e] = kt[c * 16 + e];
      qr[e] = qt[c * 16 + e];
      if constexpr (C::DIAG) lr[e] = Lt[c * 16 + e];
    }
    const int npass = (P + RPP - 1) / RPP;
    for (int ps = 0; ps < npass; ++ps) {
      const int i = ps * RPP + tid / CPR;
      float pa = 0.f, pb = 0.f;
      if (i < P) {
        float kk[16];
        load_sw<Act, D, 16>(s_bk, i, c * 16, kk);
        if constexpr (C::DIAG) {
          float ll[16];
          Num<float>::load<16>(s_bL + i * D + c * 16, ll);
#pragma unroll
          for (int e = 0; e < 16; ++e) kk[e] *= fast_exp(lr[e] - ll[e]);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pa = fmaf(kk[e], kr[e], pa);
          pb = fmaf(kk[e], qr[e], pb);
        }
      }
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1) {
        pa += __shfl_xor_sync(0xffffffffu, pa, off);
        pb += __shfl_xor_sync(0xffffffffu, pb, off);
      }
      if (c == 0 && i < P) {
        if constexpr (!C::DIAG) {
          const float f = fast_exp(Ls - s_bL[i]);
          pa *= f;
          pb *= f;
        }
        ca[i] = pa;
        cb[i] = pb;
      }
    }
    if (tid < r) {  // compensator pairs: key e_j entered at L = 0
      const int j = s_cidx[tid] & (D - 1);  // in range even for a never-quantized state
      ca[W + tid] = xs[j];
      cb[W + tid] = ys[j];
    }
    if (tid < 32) {
      float s = 0.f;
      for (int j = lane; j < D; j += 32) s = fmaf(kt[j], qt[j], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (lane == 0) misc[0] = s;
    }
  }
  csync();

  // ---- phase 3: corrections from the buffered write vectors and compensators -------------
  {
    const int v = tid % D, grp = tid / D;
    float aw = 0.f, ar = 0.f;
    for (int i = grp; i < P; i += C::G) {
      const float u = Num<Buf>::to_f(s_bu[swz_el<Buf, D>(i, v)]);
      aw = fmaf(ca[i], u, aw);
      ar = fmaf(cb[i], u, ar);
    }
    for (int cc = grp; cc < r; cc += C::G) {
      const float u = s_cu[cc * D + v];
      aw = fmaf(ca[W + cc], u, aw);
      ar = fmaf(cb[W + cc], u, ar);
    }
    red[grp * 2 * D + v] = aw;
    red[grp * 2 * D + D + v] = ar;
  }
  csync();

  // ---- phase 4: write vector, output, append -------------------------------------------
  if (tid < D) {
    const int v = tid;
    float w = pv[v], rr = rv[v];
#pragma unroll
    for (int gi = 0; gi < C::G; ++gi) {
      w += red[gi * 2 * D + v];
      rr += red[gi * 2 * D + D + v];
    }
    const float u = beta * (Num<Act>::to_f(s_v[v]) - w);
    const Buf ub = Num<Buf>::from_f(u);
    const float ur = Num<Buf>::to_f(ub);
    static_cast<Act*>(a.o)[(size_t)head * D + v] = Num<Act>::from_f(rr + ur * misc[0]);
    if (!flush) {
      static_cast<Buf*>(a.buf_u)[(size_t)head * W * D + swz_el<Buf, D>(P, v)] = ub;
      static_cast<Act*>(a.buf_k)[(size_t)head * W * D + swz_el<Act, D>(P, v)] = s_k[v];
      if constexpr (C::DIAG) a.buf_L[((size_t)head * W + P) * D + v] = Lt[v];
    } else {
      s_bu[swz_el<Buf, D>(P, v)] = ub;
      s_bk[swz_el<Act, D>(P, v)] = s_k[v];
      if constexpr (C::DIAG) s_bL[P * D + v] = Lt[v];
    }
  }
  if (tid == 0) {
    if constexpr (!C::DIAG) {
      if (!flush) a.buf_L[(size_t)head * Wp + P] = Ls;
      else s_bL[P] = Ls;
    }
    a.pos[head] = flush ? 0 : P + 1;
  }
  if (!flush) return;

  // ---- phase 5: window end -------------------------------------------------------------
  csync();
  float* colexp = xs;  // x, y are dead
  prepare_window_end<C>(st, L, P + 1, Lt, Ls, colexp, fac);
  csync();
  const WindowTile<C> tile = window_tile<C>(st, L, P + 1, r, colexp, fac);
  requantize_store<C>(tile, r, a.codes + (size_t)head * a.code_stride,
                      a.scales + (size_t)head * a.scale_stride,
                      a.comp_idx + (size_t)head * ((r + 3) & ~3), a.comp_u + (size_t)head * r * D,
                      ys, reinterpret_cast<int32_t*>(misc + 4),
                      C::SMOOTH ? a.smooth_exp + (size_t)head * D : nullptr);
}

// ------------------------------------------------------------------------------------------
// Decode step, persistent: CTA b owns heads [b * per_cta, (b + 1) * per_cta) and walks them in
// order while up to nstages - 1 later heads are already being copied into their stages.
// ------------------------------------------------------------------------------------------
constexpr int kStepThreads = kThreads;
constexpr int kMaxStages = 4;  // stage barriers in the first 64 bytes of shared memory
constexpr int kStepIssuer = kStepThreads - 32;  // lane 0 of the last warp issues stage copies

template <class C, bool MIX>
__global__ void __launch_bounds__(kStepThreads, 2)
    window_step_kernel(const WinArgs a, const int heads, const int per_cta, const int smem) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int tid = threadIdx.x;
  const int h0 = blockIdx.x * per_cta;
  const int nh = min(per_cta, heads - h0);
  if (nh <= 0) return;
  // the scalar-gate tensor-core path flushes windows on tcgen05: TMEM for the whole launch
  constexpr bool kTc = C::MMA && !C::DIAG;
  if constexpr (kTc) {
    if (tid < 32) {
      tmem_alloc(reinterpret_cast<uint32_t*>(sm + 104), kFlushTmemCols);
      tmem_relinquish();
    }
  }
  const bool mma = step_uses_mma<C>(a.W);
  const int Wr = (a.W + 15) & ~15;
  const bool power = a.comp_k != nullptr;  // power tokens: their keys ride in each stage
  const WinLayout L0 = win_layout_mix<C, MIX>(a.W, a.r, 0, per_cta, Wr, !mma, power);  // scratch
  int32_t* hpos = reinterpret_cast<int32_t*>(sm + L0.harr);
  float* hg = reinterpret_cast<float*>(hpos + per_cta);
  float* hb = hg + per_cta;
  int* pmax = reinterpret_cast<int*>(sm + L0.bars + 64);  // after the stage barriers (<= 4)
  // per stage: the furthest window position among the heads staged there so far (rows below it
  // may hold another head's write vectors)
  if (tid == 0) *pmax = 0;
  if (tid < kMaxStages) pmax[1 + tid] = 0;  // the stages' high-water marks (below)
  csync();
  int mp = 0;
  for (int i = tid; i < nh; i += C::NT) {
    const int P = a.pos[h0 + i];
    hpos[i] = P;
    if (P >= 0 && P < a.W) mp = max(mp, P);
    if constexpr (!C::DIAG) hg[i] = a.g[h0 + i];
    hb[i] = a.beta[h0 + i];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mp = max(mp, __shfl_xor_sync(0xffffffffu, mp, off));
  if ((tid & 31) == 0) atomicMax(pmax, mp);
  for (uint32_t e = tid; e < tc_scratch_bytes(Wr) / 4; e += C::NT)
    reinterpret_cast<uint32_t*>(sm + L0.tc)[e] = 0u;  // unused rows of the mma operands stay 0
  csync();
  // on the tensor-core path the stages are sized for the furthest window position among this
  // CTA's heads (row P may be written, the products read up to the next multiple of 16), so a
  // launch early in its windows keeps more heads' copies in flight
  const int cap = mma ? min(Wr, (*pmax + 16) & ~15) : Wr;
  const int nstages =
      min(kMaxStages, (smem - (int)L0.stage0) /
                          (int)win_layout_mix<C, MIX>(a.W, a.r, 1, per_cta, cap, !mma, power)
                              .stage_bytes);
  const WinLayout L = win_layout_mix<C, MIX>(a.W, a.r, nstages, per_cta, cap, !mma, power);
  // a head's stage copies and step in its own format (both fit the mixed layout)
  auto issue = [&](uint8_t* st, uint64_t* bar, int head, int P, int zrows) {
    if constexpr (MIX) {
      if (head_is_int4(a, head)) {
        stage_issue<Int4Of<C>>(a, L, st, bar, head, P, true, -1, zrows);
        return;
      }
    }
    stage_issue<C>(a, L, st, bar, head, P, true, -1, zrows);
  };
  // Every stage's write-vector rows start at zero (tensor-core path). The buffer product reads a
  // head's rows up to its position rounded up to 16, and the rows past its pairs meet zero
  // coefficients, so they must hold finite values: zeros, or -- when an earlier head staged
  // there had a further position (ragged windows) -- that head's write vectors, which
  // `restage` zeroes first, so that one head's non-finite values never reach another head's
  // results. The zeros are ordered before the stage copies by the proxy fence.
  if (mma) {
    const int n16 = cap * C::D * (int)sizeof(typename C::Buf) / 16;
    for (int s = 0; s < nstages; ++s) {
      uint4* bu = reinterpret_cast<uint4*>(sm + L.stage0 + s * L.stage_bytes + L.bu);
      for (int e = tid; e < n16; e += C::NT) bu[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.bars);
  // after the stage barriers: the row high-water marks (64..83), the flush products' barrier
  // (96) and the TMEM address (104)
  TcCtx tc{0u, reinterpret_cast<uint64_t*>(sm + 96), 0u};
  if (tid == 0) {
    for (int s = 0; s < nstages; ++s) mbar_init(&bars[s], 1);
    if constexpr (kTc) mbar_init(tc.bar, 1);
    fence_barrier_init();
  }
  tc_fence_before();
  csync();
  if constexpr (kTc) {
    tc_fence_after();
    tc.tmem = *reinterpret_cast<const uint32_t*>(sm + 104);
  }
  // Restage stage s with head index `hn` (one thread, once the stage is free). With ragged
  // windows the stage may hold another head's write vectors in [P, P rounded up to 16): the
  // copies then also bring zeros over them.
  auto restage = [&](int s, int hn) {
    int* hwm = reinterpret_cast<int*>(sm + 68) + s;  // after *pmax
    const int P = hpos[hn];
    int zrows = 0;
    if (P >= 0 && P < a.W) {
      const int m = *hwm;
      zrows = max(0, min((P + 15) & ~15, m) - P);
      *hwm = max(m, P + (P + 1 == a.W));  // a flush writes row P into the stage
    }
    issue(sm + L.stage0 + s * L.stage_bytes, &bars[s], h0 + hn, P, mma ? zrows : 0);
  };
  if (tid == 0)
    for (int s = 0; s < nstages && s < nh; ++s) restage(s, s);
  const bool first_ok = stage_wait(a, &bars[0], 0u);
  for (int n = 0; first_ok && n < nh; ++n) {
    // refill the stage head n - 1 left; the issuer is the last warp, which has the least work
    // early in a head (the pair-coefficient tiles go to warps 4, 5, ... in order)
    if (nstages > 1 && tid == kStepIssuer && n > 0 && n - 1 + nstages < nh)
      restage((n - 1) % nstages, n - 1 + nstages);
    uint8_t* st = sm + L.stage0 + (n % nstages) * L.stage_bytes;
    const int P = hpos[n];
    if (P >= 0 && P < a.W) {
      bool done = false;
      if constexpr (MIX) {
        if (head_is_int4(a, h0 + n)) {
          step_head<Int4Of<C>>(a, L, sm, st, h0 + n, P, C::DIAG ? 0.f : hg[n], hb[n], tc);
          done = true;
        }
      }
      if (!done) step_head<C>(a, L, sm, st, h0 + n, P, C::DIAG ? 0.f : hg[n], hb[n], tc);
    } else if (tid == 0) {
      report(a.status, GDN_DEVICE_BAD_POS);
    }
    // the stage's generic-proxy writes are ordered before the async copies that refill it
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    if (nstages == 1) {  // a single stage is refilled only once this head is done with it
      csync();
      if (tid == kStepIssuer && n + 1 < nh) restage(0, n + 1);
    }
    // one barrier ends the head (stage and scratch free) and agrees on the next head's copies
    int timed_out = 0;
    if (n + 1 < nh)
      timed_out = mbar_wait_bounded(&bars[(n + 1) % nstages], (uint32_t)((n + 1) / nstages) & 1u)
                      ? 0 : 1;
    if (csync_or(timed_out)) {
      if (tid == 0) report(a.status, GDN_DEVICE_WAIT_TIMEOUT);
      break;
    }
  }
  if constexpr (kTc) {  // every path ends here: the TMEM goes back
    tc_fence_before();
    csync();
    if (tid < 32) {
      tc_fence_after();
      tmem_dealloc(tc.tmem, kFlushTmemCols);
    }
  }
}

// ------------------------------------------------------------------------------------------
// Forced flush (mode 0) and materialisation (mode 1) of the logical state at the current pos.
// One CTA per head, one stage.
// ------------------------------------------------------------------------------------------
template <class C, int MODE>
__device__ __forceinline__ void window_state_body(const WinArgs& a, uint8_t* sm, int head) {
  constexpr int D = C::D;
  const bool power = a.comp_k != nullptr;
  const WinLayout L = win_layout<C>(a.W, a.r, 1, 0, -1, true, power);
  const int tid = threadIdx.x;
  const int W = a.W, r = a.r;
  const int P = a.pos[head];
  if (P < 0 || P >= W) {
    if (tid == 0) report(a.status, GDN_DEVICE_BAD_POS);
    return;
  }
  if (MODE == 0) {
    if (P == 0) return;
    if (a.seq_mask && a.seq_mask[head / a.H] == 0) return;
  }
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint8_t* st = sm + L.stage0;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    stage_issue<C>(a, L, st, bar, head, P, false);
  }
  csync();
  if (!stage_wait(a, bar, 0)) return;

  float* vec = reinterpret_cast<float*>(sm + L.vec);
  float *Lend = vec, *colexp = vec + D, *colmax = vec + 2 * D;
  int32_t* sel = reinterpret_cast<int32_t*>(vec + 7 * D);
  float* fac = reinterpret_cast<float*>(sm + L.coef);
  const float* s_bL = reinterpret_cast<const float*>(st + L.bL);
  float Ls = 0.f;
  if constexpr (C::DIAG) {
    for (int j = tid; j < D; j += C::NT) Lend[j] = P > 0 ? s_bL[(P - 1) * D + j] : 0.f;
  } else {
    Ls = P > 0 ? s_bL[P - 1] : 0.f;
  }
  csync();
  prepare_window_end<C>(st, L, P, Lend, Ls, colexp, fac);
  csync();
  const WindowTile<C> tile = window_tile<C>(st, L, P, r, colexp, fac, power);
  if constexpr (MODE == 0) {
    requantize_store<C>(tile, r, a.codes + (size_t)head * a.code_stride,
                        a.scales + (size_t)head * a.scale_stride,
                        a.comp_idx + (size_t)head * ((r + 3) & ~3),
                        a.comp_u + (size_t)head * r * D, colmax, sel,
                        C::SMOOTH ? a.smooth_exp + (size_t)head * D : nullptr);
    if (tid == 0) a.pos[head] = 0;
  } else {
    const int cg = tid % C::CG, rg = tid / C::CG;
    float acc[C::TR][C::TC];
    float* out = a.S_out + (size_t)head * D * D;
    for (int ps = 0; ps < C::NPASS; ++ps) {
      tile(ps, acc);
#pragma unroll
      for (int aa = 0; aa < C::TR; ++aa) {
        const int row = ps * C::RPASS + rg * C::TR + aa;
#pragma unroll
        for (int b = 0; b < C::TC; ++b) out[(size_t)row * D + cg * C::TC + b] = acc[aa][b];
      }
    }
  }
}

// One CTA per head. With MIX, a head whose head_fmt is INT4_G32 takes the int4 configuration.
template <class C, int MODE, bool MIX>
__global__ void __launch_bounds__(kThreads) window_state_kernel(const WinArgs a) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int head = blockIdx.x;
  if constexpr (MIX) {
    if (head_is_int4(a, head)) {
      window_state_body<Int4Of<C>, MODE>(a, sm, head);
      return;
    }
  }
  window_state_body<C, MODE>(a, sm, head);
}

// ------------------------------------------------------------------------------------------
// Power compensator tokens: the window end (MODE 0: forced flush of the selected heads with
// pos > 0; MODE 2: heads a decode step left full, pos == W) and the initial quantization
// (MODE 3, from S_in). One CTA per head: the state materialised in shared memory as fp32
// [D][D + 1], the tokens found by subspace iteration on it (as the header states: start from
// the r key columns of largest L2 norm, ties to the lower index; six times X <- orth(S^T S X),
// modified Gram-Schmidt in column order; keys x_c, values S x_c), the residual S (I - X X^T)
// quantized like any other state.
// ------------------------------------------------------------------------------------------
constexpr int kPowerIters = 6;

// Reads a [D][ld] fp32 tile of shared memory in the requantiser's tile mapping.
template <class C>
struct SmemTile {
  const float* S;
  int ld;
  __device__ __forceinline__ void operator()(int ps, float (&acc)[C::TR][C::TC]) const {
    const int tid = threadIdx.x, cg = tid % C::CG, rg = tid / C::CG;
#pragma unroll
    for (int a = 0; a < C::TR; ++a) {
      const int row = ps * C::RPASS + rg * C::TR + a;
#pragma unroll
      for (int b = 0; b < C::TC; ++b) acc[a][b] = S[row * ld + cg * C::TC + b];
    }
  }
};

// Shared memory of power_end_kernel: a region holding (window ends) a one-stage window layout
// and, once the state is materialised, the fp32 state tile [D][D + 1] from byte 128 on (the
// stage barrier keeps the first 128 bytes); then keys X, products Y and the second half's
// partial products ([D][xs] each, token-minor, xs = r rounded up to 4) and 512 floats of
// scratch. About 105 KB for W = 64, r = 4: two CTAs per SM.
template <class C>
__host__ __device__ inline uint32_t power_region_bytes(int W, int r, bool window) {
  const uint32_t tile = align128(128u + 4u * C::D * (C::D + 1));
  const uint32_t win = window ? win_layout<C>(W, r, 1, 0, -1, true, true).total : 0u;
  return tile > win ? tile : win;
}
template <class C>
__host__ __device__ inline uint32_t power_end_smem(int W, int r, bool window) {
  const uint32_t xs = (uint32_t)(r + 3) & ~3u;
  return power_region_bytes<C>(W, r, window) + align128(4u * (3u * C::D * xs + 512u));
}

// Warp sum of a value.
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// out = S in (TRANS: S^T in) for the token vectors in, both [D][xs] token-minor (xs a multiple
// of 4, r <= xs). Thread t takes index n = t % D of the product and one half of the summation
// index (t / D), four tokens at a time (one 16-byte load of the vectors per summation index,
// a broadcast); the second half's partial sums meet the first's through `part`.
template <class C, bool TRANS>
__device__ __forceinline__ void power_matvec(const float* Sm, int ld, int r, int xs,
                                             const float* in, float* out, float* part) {
  constexpr int D = C::D;
  static_assert(C::NT == 2 * D, "two threads per row or column");
  const int tid = threadIdx.x, n = tid % D, h = tid / D;
  const int m0 = h * (D / 2);
  float acc[GDN_MAX_COMPENSATORS];
#pragma unroll
  for (int c = 0; c < GDN_MAX_COMPENSATORS; ++c) acc[c] = 0.f;
#pragma unroll
  for (int c0 = 0; c0 < GDN_MAX_COMPENSATORS; c0 += 4) {
    if (c0 < r) {
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
      for (int m = m0; m < m0 + D / 2; ++m) {
        const float sv = TRANS ? Sm[m * ld + n] : Sm[n * ld + m];
        const float4 v = *reinterpret_cast<const float4*>(in + m * xs + c0);
        a0 = fmaf(sv, v.x, a0);
        a1 = fmaf(sv, v.y, a1);
        a2 = fmaf(sv, v.z, a2);
        a3 = fmaf(sv, v.w, a3);
      }
      acc[c0] = a0;
      acc[c0 + 1] = a1;
      acc[c0 + 2] = a2;
      acc[c0 + 3] = a3;
      if (h == 1) *reinterpret_cast<float4*>(part + n * xs + c0) = make_float4(a0, a1, a2, a3);
    }
  }
  csync();
  if (h == 0) {
#pragma unroll
    for (int c0 = 0; c0 < GDN_MAX_COMPENSATORS; c0 += 4) {
      if (c0 < r) {
        const float4 q = *reinterpret_cast<const float4*>(part + n * xs + c0);
        *reinterpret_cast<float4*>(out + n * xs + c0) =
            make_float4(acc[c0] + q.x, acc[c0 + 1] + q.y, acc[c0 + 2] + q.z, acc[c0 + 3] + q.w);
      }
    }
  }
  csync();
}

// The tokens of the state Sm ([D][ld] in shared memory): writes keys and values to HBM and
// leaves the residual in Sm. Called by all threads; r >= 1. X, Y and part are [D][xs].
template <class C>
__device__ void power_tokens(float* Sm, int ld, int r, float* X, float* Y, float* part,
                             float* scr, float* g_ck, float* g_cu) {
  constexpr int D = C::D;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int xs = (r + 3) & ~3;
  int* sel = reinterpret_cast<int*>(scr + D);
  if (tid < D) {  // squared column norms
    float s2 = 0.f;
    for (int i = 0; i < D; ++i) s2 = fmaf(Sm[i * ld + tid], Sm[i * ld + tid], s2);
    scr[tid] = s2;
  }
  csync();
  if (warp == 0) {  // start columns: largest norm first, ties to the lower index
    for (int c = 0; c < r; ++c) {
      float bv = -2.f;
      int bj = D;
      for (int j = lane; j < D; j += 32)
        if (scr[j] > bv) { bv = scr[j]; bj = j; }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
        if (ov > bv || (ov == bv && oj < bj)) { bv = ov; bj = oj; }
      }
      if (lane == 0) {
        sel[c] = bj;
        scr[bj] = -1.f;  // taken (norms are >= 0)
      }
      __syncwarp();
    }
  }
  csync();
  for (int e = tid; e < D * xs; e += C::NT) {
    const int j = e / xs, c = e % xs;
    X[e] = (c < r && j == sel[c]) ? 1.f : 0.f;  // (padding tokens stay 0)
  }
  csync();
  for (int it = 0; it < kPowerIters; ++it) {
    power_matvec<C, false>(Sm, ld, r, xs, X, Y, part);  // Y = S X
    power_matvec<C, true>(Sm, ld, r, xs, Y, X, part);   // X = S^T Y
    // modified Gram-Schmidt over the columns in order, run twice: S^T S X has columns that all
    // lean towards the dominant direction, and one pass in single precision leaves them
    // orthogonal only to about eps (sigma_1 / sigma_c)^2; the second pass restores
    // orthonormality (in exact arithmetic it changes nothing)
    if (warp == 0) {
      for (int pass = 0; pass < 2; ++pass)
      for (int c = 0; c < r; ++c) {
        float xc[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) xc[m] = X[(lane + 32 * m) * xs + c];
        for (int p = 0; p < c; ++p) {
          float d = 0.f;
#pragma unroll
          for (int m = 0; m < 4; ++m) d = fmaf(xc[m], X[(lane + 32 * m) * xs + p], d);
          d = warp_sum(d);
#pragma unroll
          for (int m = 0; m < 4; ++m) xc[m] = fmaf(-d, X[(lane + 32 * m) * xs + p], xc[m]);
        }
        float n2 = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) n2 = fmaf(xc[m], xc[m], n2);
        const float nrm = __fsqrt_rn(warp_sum(n2));
#pragma unroll
        for (int m = 0; m < 4; ++m)
          X[(lane + 32 * m) * xs + c] = nrm > 0.f ? __fdiv_rn(xc[m], nrm) : 0.f;
        __syncwarp();
      }
    }
    csync();
  }
  power_matvec<C, false>(Sm, ld, r, xs, X, Y, part);  // the values S x_c
  for (int e = tid; e < r * D; e += C::NT) {
    const int c = e / D, j = e % D;
    g_ck[e] = X[j * xs + c];
    g_cu[e] = Y[j * xs + c];
  }
  for (int e = tid; e < D * D; e += C::NT) {  // residual S - sum_c u_c x_c^T
    const int i = e / D, j = e % D;
    float acc = Sm[i * ld + j];
    for (int c = 0; c < r; ++c) acc = fmaf(-Y[i * xs + c], X[j * xs + c], acc);
    Sm[i * ld + j] = acc;
  }
  csync();
}

// One head of power_end_kernel; false when a stage wait ran out (reported; the CTA stops).
// `phase` is the stage barrier's parity, flipped by every completed wait.
template <class C, int MODE>
__device__ __forceinline__ bool power_end_head(const WinArgs& a, uint8_t* sm, uint64_t* bar,
                                               int head, uint32_t& phase) {
  constexpr int D = C::D, LD = D + 1;
  const int tid = threadIdx.x;
  const int W = a.W, r = a.r, xs = (r + 3) & ~3;
  float* Sm = reinterpret_cast<float*>(sm + 128);
  float* X = reinterpret_cast<float*>(sm + power_region_bytes<C>(W, r, MODE != 3));
  float* Y = X + D * xs;
  float* part = Y + D * xs;
  float* scr = part + D * xs;
  float* g_ck = a.comp_k + (size_t)head * r * D;
  float* g_cu = a.comp_u + (size_t)head * r * D;
  if constexpr (MODE == 3) {
    const float4* src = reinterpret_cast<const float4*>(a.S_in + (size_t)head * D * D);
    constexpr int kPer = D * D / 4 / C::NT;  // 16-byte loads per thread, all issued first
    float4 f[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) f[u] = src[tid + u * C::NT];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + u * C::NT, i = (4 * e) / D, j = (4 * e) % D;
      Sm[i * LD + j] = f[u].x;
      Sm[i * LD + j + 1] = f[u].y;
      Sm[i * LD + j + 2] = f[u].z;
      Sm[i * LD + j + 3] = f[u].w;
    }
    csync();
  } else {
    const int P = a.pos[head];
    if (MODE == 2) {
      if (P != W) return true;  // this head's window is not full
    } else {
      if (P < 0 || P >= W) {
        if (tid == 0) report(a.status, GDN_DEVICE_BAD_POS);
        return true;
      }
      if (P == 0) return true;
      if (a.seq_mask && a.seq_mask[head / a.H] == 0) return true;
    }
    const WinLayout L = win_layout<C>(W, r, 1, 0, -1, true, true);
    uint8_t* st = sm + L.stage0;
    if (tid == 0) stage_issue<C>(a, L, st, bar, head, P, false, -1, 0, true);
    if (!stage_wait(a, bar, phase)) return false;
    phase ^= 1u;
    float* vec = reinterpret_cast<float*>(sm + L.vec);
    float *Lend = vec, *colexp = vec + D;
    float* fac = reinterpret_cast<float*>(sm + L.coef);
    const float* s_bL = reinterpret_cast<const float*>(st + L.bL);
    float Ls = 0.f;
    if constexpr (C::DIAG) {
      for (int j = tid; j < D; j += C::NT) Lend[j] = P > 0 ? s_bL[(P - 1) * D + j] : 0.f;
    } else {
      Ls = P > 0 ? s_bL[P - 1] : 0.f;
    }
    csync();
    prepare_window_end<C>(st, L, P, Lend, Ls, colexp, fac);
    csync();
    const WindowTile<C> tile = window_tile<C>(st, L, P, r, colexp, fac, true);
    const int cg = tid % C::CG, rg = tid / C::CG;
    float acc[C::NPASS][C::TR][C::TC];  // the whole state first: the tile overwrites the stage
#pragma unroll
    for (int ps = 0; ps < C::NPASS; ++ps) tile(ps, acc[ps]);
    csync();  // (the stage's old tokens are read out before the new ones go to HBM)
#pragma unroll
    for (int ps = 0; ps < C::NPASS; ++ps)
#pragma unroll
      for (int aa = 0; aa < C::TR; ++aa)
#pragma unroll
        for (int b = 0; b < C::TC; ++b)
          Sm[(ps * C::RPASS + rg * C::TR + aa) * LD + cg * C::TC + b] = acc[ps][aa][b];
    csync();
  }
  if (r > 0) power_tokens<C>(Sm, LD, r, X, Y, part, scr, g_ck, g_cu);
  SmemTile<C> tile{Sm, LD};
  requantize_store<C>(tile, 0, a.codes + (size_t)head * a.code_stride,
                      a.scales + (size_t)head * a.scale_stride, nullptr, nullptr, scr,
                      reinterpret_cast<int32_t*>(scr + 256), nullptr);
  if (tid < r) a.comp_idx[(size_t)head * ((r + 3) & ~3) + tid] = -1;  // (no key columns)
  if (tid == 0) a.pos[head] = 0;
  // the tile's generic writes are ordered before the next head's stage copies over them
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  csync();
  return true;
}

// Persistent: CTA b takes heads b, b + grid, ... (two CTAs per SM); a launch after a decode step
// (MODE 2) passes over the heads whose windows are not full at the cost of one load each.
template <class C, int MODE>
__global__ void __launch_bounds__(kThreads, 2) power_end_kernel(const WinArgs a, const int heads) {
  extern __shared__ __align__(128) uint8_t sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm);  // the window layout's stage barrier
  if constexpr (MODE != 3) {
    if (threadIdx.x == 0) {
      mbar_init(bar, 1);
      fence_barrier_init();
    }
    csync();
  }
  uint32_t phase = 0u;
  for (int head = blockIdx.x; head < heads; head += gridDim.x)
    if (!power_end_head<C, MODE>(a, sm, bar, head, phase)) return;
}

// ------------------------------------------------------------------------------------------
// Initial quantization of fp32 states.
// ------------------------------------------------------------------------------------------
template <class C>
__device__ __forceinline__ void quantize_body(const WinArgs& a, int head) {
  constexpr int D = C::D;
  __shared__ float colmax[D];
  __shared__ int32_t sel[GDN_MAX_COMPENSATORS];
  DenseTile<C> tile;
  tile.S = a.S_in + (size_t)head * D * D;
  requantize_store<C>(tile, a.r, a.codes + (size_t)head * a.code_stride,
                      a.scales + (size_t)head * a.scale_stride,
                      a.comp_idx + (size_t)head * ((a.r + 3) & ~3),
                      a.comp_u + (size_t)head * a.r * D, colmax, sel,
                      C::SMOOTH ? a.smooth_exp + (size_t)head * D : nullptr);
  if (threadIdx.x == 0) a.pos[head] = 0;
}

template <class C, bool MIX>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const WinArgs a) {
  const int head = blockIdx.x;
  if constexpr (MIX) {
    if (head_is_int4(a, head)) {
      quantize_body<Int4Of<C>>(a, head);
      return;
    }
  }
  quantize_body<C>(a, head);
}

}  // namespace gdnq
