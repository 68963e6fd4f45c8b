/*
 * gdn_oracle.c -- plain, slow fp64 CPU oracle for gated delta-rule (GDN / KDA) decode over a
 * windowed low-bit recurrent state.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load this library. It shares no code, header, table or helper with the CUDA
 * library; both sides only see the same seeded inputs.
 *
 * What it restates (page title, part of the page):
 *   [LQ] "LeapQuant: Efficient Linear Attention with Accurate Recurrent State Quantization"
 *        (weekinpapers summary page), Abstract:
 *          - GDN and KDA keep a fixed-size recurrent state that every decode step reads and
 *            updates;
 *          - per-window quantization: the state stays frozen in low bits for a window of
 *            tokens and is quantized once, at the window's end;
 *          - inside a window, outputs come from the frozen low-bit state plus buffered
 *            high-precision updates;
 *          - a few high-precision "compensator tokens" keep the state's largest outliers and
 *            take the same update path as real tokens;
 *          - the residual is smoothed before quantization. The page gives no mechanism; the
 *            reading restated here (window_end's smooth option) is a per-key-column power-of-
 *            two rescaling before the per-row quantizer, the factor about the square root of
 *            the column's max-abs. Parity unpinned against the pages (they give no rule and no
 *            numbers for it); its arithmetic is pinned by a hand-worked fixture, the exponent's
 *            closed form, exactness without quantization and O1 = O2.
 *   [PW] "Low-Bit GDN Recurrent-State Quantization: Global Gradient-aware Allocation and
 *        Pure-Write Sliding Windows", Abstract: quantized write-back errors feed into later
 *        steps (why quantize-every-step, the window length 1 case, degrades); recent pure
 *        writes are kept as FP8 vector pairs, carried through the full transition, and merged
 *        into the low-bit history only once they leave the window.
 *
 * The recurrence, for one (sequence, head), state S in R^{d_v x d_k} (row i = value channel,
 * column j = key channel), gate a_t in R^{d_k} (GDN: all entries equal; KDA: per key channel):
 *
 *     S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,      o_t = S_t q_t.
 *
 * The gate enters as its logarithm g_t = log a_t, so products of gates over a window are sums.
 *
 * Four formulations live here; none calls another's step code:
 *   plain  -- the recurrence in fp64, optionally rounding the stored state to fp32 / bf16 after
 *             each step (the high-precision-state baselines and the fp32 warm-up);
 *   O1     -- the recurrence applied literally as matrix products (D x D transition matrix),
 *             with the state replaced by dequant(quant(S - C)) + C after every W-th step;
 *   O2     -- the buffered form: frozen low-bit state + buffered pairs (k_i, u_i, L_i) +
 *             compensator pairs, flushed (materialised, requantised) when the window fills.
 *             Optional storage roundings mirror what a GPU stores between steps.
 *   PW     -- the pure-write sliding window [PW]: a low-bit history requantised every step plus
 *             the last Wp pure writes as FP8 pairs (its readings are stated where it starts).
 *
 * Readings of the pages where they are silent (each one is listed in the design notes):
 *   - quantizer: symmetric absmax, s = absmax / 127 (int8, one scale per row) or absmax / 7
 *     (int4, one scale per group of 32 key channels); c = clamp(round-half-even(x / s)); a zero
 *     group has s = 0 and codes 0.
 *   - windows are [0, W), [W, 2W), ... from the start of decode; the output of a window's last
 *     step comes from the buffered form, before requantisation.
 *   - compensators: at every quantization, the r key columns with the largest max-abs (ties to
 *     the lower index) are taken out exactly as pairs (key e_j, value S[:, j]) and re-enter the
 *     next window at cumulative gate 0. PARITY UNPINNED against the pages: they give no rule.
 *     Only the exact decomposition S = residual + sum of pairs is pinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_FMT_NONE = 0, ORC_FMT_INT8 = 1, ORC_FMT_INT4 = 2 };
enum { ORC_ROUND_NONE = 0, ORC_ROUND_F32 = 1, ORC_ROUND_BF16 = 2 };

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------------------------
 * Storage roundings.
 * bfloat16: 8 significant bits, the exponent range of IEEE single; round to nearest, ties to
 * even. Written from that definition: find the quantum of x's binade (2^(e-8) where
 * 2^(e-1) <= |x| < 2^e), clamp it at the subnormal quantum 2^-133, and round x / quantum
 * to an integer with rint (ties to even in the default rounding mode).
 * ---------------------------------------------------------------------------------------- */
double orc_round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);                      /* x = m * 2^e, 0.5 <= |m| < 1 */
    int qexp = e - 8;
    if (qexp < -133) qexp = -133;
    double quantum = ldexp(1.0, qexp);
    double r = rint(x / quantum) * quantum;
    if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, x); /* beyond the largest bf16 */
    return r;
}

double orc_round_f32(double x) { return (double)(float)x; }

static double round_to(int mode, double x) {
    if (mode == ORC_ROUND_F32) return orc_round_f32(x);
    if (mode == ORC_ROUND_BF16) return orc_round_bf16(x);
    return x;
}

/* The storage value on the other side of x from round_to(mode, x): the two values of the
 * format that bracket x are lo = floor(x / q) q and lo + q, q the quantum of x's binade
 * (2^(e-8) for bfloat16, 2^(e-24) for single, never finer than the subnormal quantum); the
 * nearest one is the rounding, the other one is returned. When x is itself representable there
 * is no other side and x is returned. Used for the alternative result of a value that lies
 * within rounding noise of a midpoint (another correct implementation may round it the other
 * way). */
double orc_round_other(int mode, double x) {
    if (mode == ORC_ROUND_NONE || x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);
    const int bits = mode == ORC_ROUND_BF16 ? 8 : 24;
    int qexp = e - bits;
    const int qmin = mode == ORC_ROUND_BF16 ? -133 : -149;
    if (qexp < qmin) qexp = qmin;
    const double quantum = ldexp(1.0, qexp);
    const double lo = floor(x / quantum) * quantum, hi = lo + quantum;
    if (lo == x) return x;
    return round_to(mode, x) == lo ? hi : lo;
}

/* ------------------------------------------------------------------------------------------
 * Quantizer. codes are one int8 per entry (int4 codes lie in [-7, 7]); scales are [D][groups].
 * prec32 = 1 takes every decision in single precision, as a GPU does: the caller passes
 * fp32-representable values, s = fp32(absmax / qmax) and x / s is rounded to fp32 before rint.
 * (Rounding an fp64 quotient of two fp32 values to fp32 gives the correctly rounded fp32
 * quotient, so this is IEEE single division.)
 * ---------------------------------------------------------------------------------------- */
static int fmt_qmax(int fmt) { return fmt == ORC_FMT_INT4 ? 7 : 127; }
static int fmt_group(int fmt, int D) { return fmt == ORC_FMT_INT4 ? 32 : D; }

int orc_num_groups(int fmt, int D) { return D / fmt_group(fmt, D); }

static void quantize_group(const double* x, int n, int qmax, int prec32, int8_t* c, double* s_out) {
    double m = 0.0;
    for (int j = 0; j < n; ++j) m = fmax(m, fabs(x[j]));
    double s = m / (double)qmax;
    if (prec32) s = orc_round_f32(s);
    *s_out = s;
    for (int j = 0; j < n; ++j) {
        if (s == 0.0) { c[j] = 0; continue; }
        double t = x[j] / s;
        if (prec32) t = orc_round_f32(t);
        double r = rint(t);
        if (r > qmax) r = qmax;
        if (r < -qmax) r = -qmax;
        c[j] = (int8_t)r;
    }
}

/* S [D][D] -> codes [D][D], scales [D][groups]. Returns 0, or -1 for a bad format. */
int orc_quantize(int D, int fmt, int prec32, const double* S, int8_t* codes, double* scales) {
    if (fmt != ORC_FMT_INT8 && fmt != ORC_FMT_INT4) return -1;
    int gs = fmt_group(fmt, D), ng = D / gs, qmax = fmt_qmax(fmt);
    for (int i = 0; i < D; ++i)
        for (int g = 0; g < ng; ++g)
            quantize_group(S + (size_t)i * D + g * gs, gs, qmax, prec32,
                           codes + (size_t)i * D + g * gs, scales + (size_t)i * ng + g);
    return 0;
}

/* codes, scales -> S[i][j] = s_{i, group(j)} * c_ij */
void orc_dequantize(int D, int fmt, const int8_t* codes, const double* scales, double* S) {
    int gs = fmt_group(fmt, D), ng = D / gs;
    for (int i = 0; i < D; ++i)
        for (int j = 0; j < D; ++j)
            S[(size_t)i * D + j] = scales[(size_t)i * ng + j / gs] * (double)codes[(size_t)i * D + j];
}

/* int4 packing: byte m of a row holds column 2m in its low nibble and 2m+1 in its high nibble,
 * each a 4-bit two's complement number. */
void orc_pack_int4(int D, const int8_t* codes, uint8_t* packed) {
    for (int i = 0; i < D; ++i)
        for (int m = 0; m < D / 2; ++m) {
            unsigned lo = (unsigned)codes[(size_t)i * D + 2 * m] & 0xFu;
            unsigned hi = (unsigned)codes[(size_t)i * D + 2 * m + 1] & 0xFu;
            packed[(size_t)i * (D / 2) + m] = (uint8_t)(lo | (hi << 4));
        }
}

void orc_unpack_int4(int D, const uint8_t* packed, int8_t* codes) {
    for (int i = 0; i < D; ++i)
        for (int m = 0; m < D / 2; ++m) {
            unsigned b = packed[(size_t)i * (D / 2) + m];
            int lo = (int)(b & 0xFu), hi = (int)(b >> 4);
            codes[(size_t)i * D + 2 * m] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            codes[(size_t)i * D + 2 * m + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
        }
}

/* ------------------------------------------------------------------------------------------
 * Compensator selection: the r columns with the largest max-abs over the rows, ties to the
 * lower column index. Returns 1 when the r-th pick and the best column left out are within
 * 1e-6 relative (a near tie: another correct implementation may pick differently).
 * ---------------------------------------------------------------------------------------- */
int orc_select_columns(int D, int r, const double* S, int* idx) {
    double* colmax = (double*)calloc((size_t)D, sizeof(double));
    char* taken = (char*)calloc((size_t)D, 1);
    for (int j = 0; j < D; ++j)
        for (int i = 0; i < D; ++i) colmax[j] = fmax(colmax[j], fabs(S[(size_t)i * D + j]));
    double last = 0.0;
    for (int c = 0; c < r; ++c) {
        int best = -1;
        for (int j = 0; j < D; ++j)
            if (!taken[j] && (best < 0 || colmax[j] > colmax[best])) best = j;
        taken[best] = 1;
        idx[c] = best;
        last = colmax[best];
    }
    int near = 0;
    if (r > 0 && r < D) {
        double rest = -1.0;
        for (int j = 0; j < D; ++j)
            if (!taken[j] && colmax[j] > rest) rest = colmax[j];
        if (last - rest <= 1e-6 * fmax(last, rest)) near = 1;
    }
    free(colmax);
    free(taken);
    return near;
}

/* ------------------------------------------------------------------------------------------
 * Residual smoothing ("LeapQuant: Efficient Linear Attention with Accurate Recurrent State
 * Quantization", Abstract: the residual left after the compensators is smoothed before it is
 * quantized). The page names the step and no mechanism; the reading taken here is a per-key-
 * column rescaling of the residual R before the per-row quantizer, R = R' Diag(m), with
 * m_j = 2^{e_j} and e_j = floor(E_j / 2), E_j the binary exponent of column j's max-abs
 * (m_j ~ sqrt(colmax_j): the usual half-way migration of a column's range), e_j = 0 for a zero
 * column, e_j clamped to [-63, 63]. Powers of two make the rescaling exact, so the only rounding
 * left is the quantizer's; the frozen state is dequant(codes, scales) Diag(m), and a step's
 * products with it take m .* x.
 * ---------------------------------------------------------------------------------------- */
int orc_smooth_exponent(double colmax) {
    if (!(colmax > 0.0)) return 0;
    int x;
    frexp(colmax, &x);           /* colmax = f 2^x, f in [1/2, 1) */
    int E = x - 1;               /* floor(log2 colmax) */
    int e = E >= 0 ? E / 2 : -((1 - E) / 2);  /* floor(E / 2) */
    if (e < -63) e = -63;
    if (e > 63) e = 63;
    return e;
}

/* Window-end operation on a full state S (overwritten by the residual): take out r compensator
 * columns exactly, then (smooth) rescale the residual's columns by 2^{-e_j} into sexp, then
 * quantize the residual. fmt == NONE keeps the (rescaled) residual unquantized in S. Returns 1
 * on a near tie (of the column choice, or of a smoothing exponent). sexp may be NULL when smooth
 * is 0. */
/* ------------------------------------------------------------------------------------------
 * Compensator rule "power" (the pages name compensator tokens that keep the state's largest
 * outliers and share the update path of real tokens, and give no rule; this is the reading of
 * the tokens as the state's dominant rank-one parts): the r keys are an orthonormal basis X of
 * the state's dominant r-dimensional key (right singular) subspace, found by subspace
 * iteration, and the values are S x_c, so the tokens carry S X X^T and the residual is
 * S (I - X X^T).
 *   start:   x_c = e_{j_c}, j_1.. j_r the key columns of largest L2 norm (ties: lower index);
 *   iterate: ORC_POWER_ITERS times X <- orth(S^T (S X)), where orth is modified Gram-Schmidt
 *            over the columns in order (x_c minus its projections on x_1 .. x_{c-1}, then
 *            divided by its length; a column of length 0 stays 0);
 *   tokens:  key x_c, value u_c = S x_c.
 * prec32 stores keys and values in single precision, as a GPU does.
 * PARITY UNPINNED against the pages (no rule, no numbers): the start, the iteration count and
 * the orthogonalisation are this reading's choices. Pinned to the mathematics: an exactly
 * rank-r state is taken out whole, a planted dominant direction is found, the tokens' energy
 * matches the truncated SVD's, and the start and its ties follow the stated rule.
 * ---------------------------------------------------------------------------------------- */
#define ORC_POWER_ITERS 6

static void power_keys(int D, int r, const double* S, double* X) {
    double* nrm = (double*)calloc((size_t)D, sizeof(double));
    char* taken = (char*)calloc((size_t)D, 1);
    double* Y = (double*)malloc(sizeof(double) * (size_t)D * (r > 0 ? r : 1));
    for (int j = 0; j < D; ++j)
        for (int i = 0; i < D; ++i) nrm[j] += S[(size_t)i * D + j] * S[(size_t)i * D + j];
    for (int c = 0; c < r; ++c) {
        int best = -1;
        for (int j = 0; j < D; ++j)
            if (!taken[j] && (best < 0 || nrm[j] > nrm[best])) best = j;
        if (best >= 0) taken[best] = 1;  /* (r <= D: always a column left) */
        for (int j = 0; j < D; ++j) X[(size_t)c * D + j] = j == best ? 1.0 : 0.0;
    }
    for (int it = 0; it < ORC_POWER_ITERS; ++it) {
        for (int c = 0; c < r; ++c)           /* Y = S X */
            for (int i = 0; i < D; ++i) {
                double acc = 0.0;
                for (int j = 0; j < D; ++j) acc += S[(size_t)i * D + j] * X[(size_t)c * D + j];
                Y[(size_t)c * D + i] = acc;
            }
        for (int c = 0; c < r; ++c)           /* X = S^T Y */
            for (int j = 0; j < D; ++j) {
                double acc = 0.0;
                for (int i = 0; i < D; ++i) acc += S[(size_t)i * D + j] * Y[(size_t)c * D + i];
                X[(size_t)c * D + j] = acc;
            }
        for (int c = 0; c < r; ++c) {         /* modified Gram-Schmidt */
            double* xc = X + (size_t)c * D;
            for (int p = 0; p < c; ++p) {
                const double* xp = X + (size_t)p * D;
                double dot = 0.0;
                for (int j = 0; j < D; ++j) dot += xc[j] * xp[j];
                for (int j = 0; j < D; ++j) xc[j] -= dot * xp[j];
            }
            double n2 = 0.0;
            for (int j = 0; j < D; ++j) n2 += xc[j] * xc[j];
            const double n = sqrt(n2);
            for (int j = 0; j < D; ++j) xc[j] = n > 0.0 ? xc[j] / n : 0.0;
        }
    }
    free(nrm);
    free(taken);
    free(Y);
}

/* Window-end operation on a full state S (overwritten by the residual). The r compensator
 * tokens (keys ck [r][D], values cu [r][D]) are taken out exactly: rule 0 (columns) picks the r
 * key columns of largest max-abs (orc_select_columns), keys e_j, values the columns, zeroed in
 * S; rule 1 (power) as power_keys above, S <- S - sum_c cu_c ck_c^T. Then (smooth) the
 * residual's columns are rescaled by 2^{-e_j} into sexp and the residual is quantized.
 * fmt == NONE keeps the (rescaled) residual unquantized in S. Returns 1 on a near tie (of the
 * column choice, or of a smoothing exponent). sexp may be NULL when smooth is 0; cidx is the
 * column choice of rule 0 (the power rule leaves it as its start columns are not kept). */
static int window_end(int D, int fmt, int r, int prec32, int smooth, int rule, double* S,
                      int8_t* codes, double* scales, int* cidx, double* cu, double* ck,
                      int8_t* sexp) {
    int near = 0;
    if (rule == 1) {
        power_keys(D, r, S, ck);
        for (int c = 0; c < r; ++c) {
            double* kc = ck + (size_t)c * D;
            if (prec32)
                for (int j = 0; j < D; ++j) kc[j] = orc_round_f32(kc[j]);
            for (int i = 0; i < D; ++i) {
                double acc = 0.0;
                for (int j = 0; j < D; ++j) acc += S[(size_t)i * D + j] * kc[j];
                cu[(size_t)c * D + i] = prec32 ? orc_round_f32(acc) : acc;
            }
            cidx[c] = -1;
        }
        for (int c = 0; c < r; ++c)
            for (int i = 0; i < D; ++i)
                for (int j = 0; j < D; ++j)
                    S[(size_t)i * D + j] -= cu[(size_t)c * D + i] * ck[(size_t)c * D + j];
        if (prec32)
            for (size_t e = 0; e < (size_t)D * D; ++e) S[e] = orc_round_f32(S[e]);
    } else {
        near = orc_select_columns(D, r, S, cidx);
        for (int c = 0; c < r; ++c) {
            for (int i = 0; i < D; ++i) {
                cu[(size_t)c * D + i] = S[(size_t)i * D + cidx[c]];
                S[(size_t)i * D + cidx[c]] = 0.0;
            }
            for (int j = 0; j < D; ++j) ck[(size_t)c * D + j] = j == cidx[c] ? 1.0 : 0.0;
        }
    }
    if (smooth) {
        for (int j = 0; j < D; ++j) {
            double m = 0.0;
            for (int i = 0; i < D; ++i) m = fmax(m, fabs(S[(size_t)i * D + j]));
            sexp[j] = (int8_t)orc_smooth_exponent(m);
            /* the exponent steps where the max-abs crosses a power of 4: within 1e-6 relative
             * of one, another correct implementation may round it to the other side */
            if (m > 0.0) {
                double p4 = ldexp(1.0, 2 * (int)floor(log2(m) / 2.0 + 0.5));
                if (fabs(m - p4) <= 1e-6 * p4) near = 1;
            }
            for (int i = 0; i < D; ++i) S[(size_t)i * D + j] = ldexp(S[(size_t)i * D + j], -sexp[j]);
        }
    }
    if (fmt != ORC_FMT_NONE) orc_quantize(D, fmt, prec32, S, codes, scales);
    return near;
}

/* Columns j of S [D][D] times 2^{sexp[j]} (undoes the smoothing; exact). */
static void unsmooth(int D, const int8_t* sexp, double* S) {
    for (int i = 0; i < D; ++i)
        for (int j = 0; j < D; ++j) S[(size_t)i * D + j] = ldexp(S[(size_t)i * D + j], sexp[j]);
}

/* The window-end operation on its own (pins): S is overwritten by the (rescaled) residual. */
int orc_window_end(int D, int fmt, int r, int prec32, int smooth, int rule, double* S,
                   int8_t* codes, double* scales, int* cidx, double* cu, double* ck,
                   int8_t* sexp) {
    return window_end(D, fmt, r, prec32, smooth, rule, S, codes, scales, cidx, cu, ck, sexp);
}

static double gate_log(const double* g, int Dg, int j) { return Dg == 1 ? g[0] : g[j]; }

/* ------------------------------------------------------------------------------------------
 * plain: the recurrence in fp64. The product S Diag(a)(I - beta k k^T) is expanded by
 * distributivity, S' - beta (S' k) k^T with S' = S Diag(a). state_round rounds the stored
 * state after each step (fp32 / bf16 state baselines); o_t is taken from the new state before
 * that rounding. S0 may be NULL (zero state). o and S_out may be NULL.
 * Layouts: S [nh][D][D]; q, k, v [T][nh][D]; g [T][nh][Dg] (Dg = 1 or D); beta [T][nh].
 * ---------------------------------------------------------------------------------------- */
void orc_plain_run(int D, int T, int nh, int Dg, int state_round, const double* S0,
                   const double* q, const double* k, const double* v, const double* g,
                   const double* beta, double* o, double* S_out) {
#pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < nh; ++h) {
        double* S = (double*)malloc(sizeof(double) * (size_t)D * D);
        double* w = (double*)malloc(sizeof(double) * (size_t)D);
        double* a = (double*)malloc(sizeof(double) * (size_t)D);
        if (S0) memcpy(S, S0 + (size_t)h * D * D, sizeof(double) * (size_t)D * D);
        else memset(S, 0, sizeof(double) * (size_t)D * D);
        for (int t = 0; t < T; ++t) {
            const double* kt = k + ((size_t)t * nh + h) * D;
            const double* qt = q + ((size_t)t * nh + h) * D;
            const double* vt = v + ((size_t)t * nh + h) * D;
            const double* gt = g + ((size_t)t * nh + h) * Dg;
            double bt = beta[(size_t)t * nh + h];
            for (int j = 0; j < D; ++j) a[j] = exp(gate_log(gt, Dg, j));
            for (int i = 0; i < D; ++i)          /* S' = S Diag(a) */
                for (int j = 0; j < D; ++j) S[(size_t)i * D + j] *= a[j];
            for (int i = 0; i < D; ++i) {        /* w = S' k */
                double acc = 0.0;
                for (int j = 0; j < D; ++j) acc += S[(size_t)i * D + j] * kt[j];
                w[i] = acc;
            }
            for (int i = 0; i < D; ++i)          /* S' - beta w k^T + beta v k^T */
                for (int j = 0; j < D; ++j)
                    S[(size_t)i * D + j] += -bt * w[i] * kt[j] + bt * vt[i] * kt[j];
            if (o) {
                double* ot = o + ((size_t)t * nh + h) * D;
                for (int i = 0; i < D; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < D; ++j) acc += S[(size_t)i * D + j] * qt[j];
                    ot[i] = acc;
                }
            }
            if (state_round != ORC_ROUND_NONE)
                for (size_t e = 0; e < (size_t)D * D; ++e) S[e] = round_to(state_round, S[e]);
        }
        if (S_out) memcpy(S_out + (size_t)h * D * D, S, sizeof(double) * (size_t)D * D);
        free(S);
        free(w);
        free(a);
    }
}

/* ------------------------------------------------------------------------------------------
 * O1: the recurrence applied literally. Each step forms the D x D transition
 *     M = Diag(a_t) (I - beta_t k_t k_t^T),   M[j][l] = a_t[j] (delta_jl - beta_t k_t[j] k_t[l])
 * and sets S <- S M + beta_t v_t k_t^T, o_t = S q_t. Before the first step and after every
 * W-th step, S <- dequant(quant(S - C)) + C, where C holds the r compensator columns of S
 * (fmt NONE: S is left as it is). All decisions in fp64. Returns the number of near ties.
 * ---------------------------------------------------------------------------------------- */
static int dense_window_end(int D, int fmt, int r, int smooth, int rule, double* S) {
    if (fmt == ORC_FMT_NONE && r == 0 && !smooth) return 0;
    int ng = orc_num_groups(fmt == ORC_FMT_NONE ? ORC_FMT_INT8 : fmt, D);
    int8_t* codes = (int8_t*)malloc((size_t)D * D);
    double* scales = (double*)malloc(sizeof(double) * (size_t)D * ng);
    int* cidx = (int*)malloc(sizeof(int) * (size_t)(r > 0 ? r : 1));
    double* cu = (double*)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1) * D);
    double* ck = (double*)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1) * D);
    int8_t* sexp = (int8_t*)calloc((size_t)D, 1);
    int near = window_end(D, fmt, r, 0, smooth, rule, S, codes, scales, cidx, cu, ck, sexp);
    if (fmt != ORC_FMT_NONE) orc_dequantize(D, fmt, codes, scales, S);
    if (smooth) unsmooth(D, sexp, S);
    free(sexp);
    for (int c = 0; c < r; ++c)            /* the tokens back: S += cu_c ck_c^T */
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j)
                S[(size_t)i * D + j] += cu[(size_t)c * D + i] * ck[(size_t)c * D + j];
    free(codes);
    free(scales);
    free(cidx);
    free(cu);
    free(ck);
    return near;
}

int orc_o1_run(int D, int T, int W, int r, int fmt, int nh, int Dg, int smooth, int rule,
               const double* S0,
               const double* q, const double* k, const double* v, const double* g,
               const double* beta, double* o, double* S_out) {
    int ties = 0;
#pragma omp parallel for schedule(dynamic) reduction(+ : ties)
    for (int h = 0; h < nh; ++h) {
        size_t DD = (size_t)D * D;
        double* S = (double*)malloc(sizeof(double) * DD);
        double* M = (double*)malloc(sizeof(double) * DD);
        double* N = (double*)malloc(sizeof(double) * DD);
        if (S0) memcpy(S, S0 + (size_t)h * DD, sizeof(double) * DD);
        else memset(S, 0, sizeof(double) * DD);
        ties += dense_window_end(D, fmt, r, smooth, rule, S);
        for (int t = 0; t < T; ++t) {
            const double* kt = k + ((size_t)t * nh + h) * D;
            const double* qt = q + ((size_t)t * nh + h) * D;
            const double* vt = v + ((size_t)t * nh + h) * D;
            const double* gt = g + ((size_t)t * nh + h) * Dg;
            double bt = beta[(size_t)t * nh + h];
            for (int j = 0; j < D; ++j)
                for (int l = 0; l < D; ++l)
                    M[(size_t)j * D + l] =
                        exp(gate_log(gt, Dg, j)) * ((j == l ? 1.0 : 0.0) - bt * kt[j] * kt[l]);
            for (int i = 0; i < D; ++i)
                for (int l = 0; l < D; ++l) {
                    double acc = 0.0;
                    for (int j = 0; j < D; ++j) acc += S[(size_t)i * D + j] * M[(size_t)j * D + l];
                    N[(size_t)i * D + l] = acc + bt * vt[i] * kt[l];
                }
            memcpy(S, N, sizeof(double) * DD);
            if (o) {
                double* ot = o + ((size_t)t * nh + h) * D;
                for (int i = 0; i < D; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < D; ++j) acc += S[(size_t)i * D + j] * qt[j];
                    ot[i] = acc;
                }
            }
            if ((t + 1) % W == 0) ties += dense_window_end(D, fmt, r, smooth, rule, S);
        }
        if (S_out) memcpy(S_out + (size_t)h * DD, S, sizeof(double) * DD);
        free(S);
        free(M);
        free(N);
    }
    return ties;
}

/* ------------------------------------------------------------------------------------------
 * O2: the buffered form. Per head the state is
 *   F          the frozen state: dequant(codes, scales) (fmt NONE: an unquantized matrix);
 *   (ck, cu)   r compensator tokens, key ck[c], value cu[c], entered at cumulative gate 0 (the
 *              column rule's keys are e_{cidx[c]}; the power rule's are dense unit vectors);
 *   (bk, bu, bL)[0..P) buffered write pairs: key, write vector, cumulative log-gate vector;
 *   P          pairs in the window so far.
 * The logical state after the window's P steps, with L = bL[P-1] (0 if P == 0), is
 *   S = F Diag(e^L) + sum_c cu_c (ck_c * e^{L})^T + sum_i bu_i (bk_i * e^{L - bL_i})^T.
 * A step at position P:
 *   L_t = L + g_t;  x = e^{L_t} * k_t;  y = e^{L_t} * q_t
 *   w  = F x + sum_c cu_c <ck_c, x> + sum_i bu_i <bk_i * e^{L_t - bL_i}, k_t>   (= S Diag(a_t) k_t)
 *   r  = F y + sum_c cu_c <ck_c, y> + sum_i bu_i <bk_i * e^{L_t - bL_i}, q_t>   (= S Diag(a_t) q_t)
 *   u_t = beta_t (v_t - w);  o_t = r + u_t <k_t, q_t>;  append (k_t, u_t, L_t)
 * which is the recurrence through S Diag(a)(I - beta k k^T) + beta v k^T
 *   = S Diag(a) + beta (v - S Diag(a) k) k^T.
 * When P reaches W (or a flush is forced after the step) the logical state is materialised and
 * the window-end operation (compensators out, residual quantized) makes the next F.
 * smooth = 1 adds the residual smoothing of window_end: F = dequant(codes, scales) Diag(2^e),
 * so every product with F (steps, materialisation) sees the smoothing undone exactly.
 *
 * round_storage = 1 mirrors what a GPU keeps between steps: the initial state and the
 * materialised state are fp32, L is fp32, u_t is rounded to buf_round (bf16 / fp32), and the
 * quantizer decides in fp32. round_storage = 0 keeps everything in fp64.
 *
 * rule selects the compensator rule of window_end (0 columns, 1 power).
 * Outputs (any may be NULL): o [T][nh][D]; codes [nh][D][D]; scales [nh][D][groups];
 * cidx [nh][r] (column rule); cu, ck [nh][r][D]; pos [nh]; bk, bu, bL [nh][W][D]; S_out [nh][D][D] (the logical
 * state at the end); ties_out [nh] (near ties met per head); sexp_out [nh][D] (the smoothing
 * exponents of the last quantization); flush_mask [T][nh] forces a flush
 * after step t of head h when nonzero; u_raw [T][nh][D] receives every write vector before its
 * storage rounding; u_flip [T][nh][D], when nonzero at an entry, stores that write-vector entry
 * rounded to the other neighbour of its storage format (orc_round_other: the alternative result
 * of an entry that lies within rounding noise of a midpoint). Returns the number of near ties
 * met in compensator choices.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
    int D, W, r, fmt, Dg, round_storage, buf_round, smooth, rule;
} o2_cfg;

typedef struct {
    double *F, *scales, *cu, *ck, *bk, *bu, *bL;
    int8_t *codes, *sexp;
    int* cidx;
    int P;
} o2_head;

static void o2_current_L(const o2_cfg* c, const o2_head* s, double* L) {
    for (int j = 0; j < c->D; ++j) L[j] = s->P > 0 ? s->bL[(size_t)(s->P - 1) * c->D + j] : 0.0;
}

/* Logical state at cumulative gate L (the window's current end), written into S. */
static void o2_materialize(const o2_cfg* c, const o2_head* s, const double* L, double* S) {
    int D = c->D;
    for (int i = 0; i < D; ++i)
        for (int j = 0; j < D; ++j) S[(size_t)i * D + j] = s->F[(size_t)i * D + j] * exp(L[j]);
    for (int cc = 0; cc < c->r; ++cc)  /* token cu_c ck_c^T entered at gate 0 */
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j)
                S[(size_t)i * D + j] += s->cu[(size_t)cc * D + i] * s->ck[(size_t)cc * D + j] * exp(L[j]);
    for (int p = 0; p < s->P; ++p)
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j)
                S[(size_t)i * D + j] += s->bu[(size_t)p * D + i] * s->bk[(size_t)p * D + j] *
                                        exp(L[j] - s->bL[(size_t)p * D + j]);
}

/* Quantize a full state S (destroyed) into the head's frozen part and compensators. */
static int o2_set_frozen(const o2_cfg* c, o2_head* s, double* S) {
    int D = c->D;
    if (c->round_storage)
        for (size_t e = 0; e < (size_t)D * D; ++e) S[e] = orc_round_f32(S[e]);
    int near = window_end(D, c->fmt, c->r, c->round_storage, c->smooth, c->rule, S, s->codes,
                          s->scales, s->cidx, s->cu, s->ck, s->sexp);
    if (c->fmt != ORC_FMT_NONE) orc_dequantize(D, c->fmt, s->codes, s->scales, s->F);
    else memcpy(s->F, S, sizeof(double) * (size_t)D * D);
    if (c->smooth) unsmooth(D, s->sexp, s->F);
    s->P = 0;
    return near;
}

static int o2_flush(const o2_cfg* c, o2_head* s, double* scratch_S, double* scratch_L) {
    o2_current_L(c, s, scratch_L);
    o2_materialize(c, s, scratch_L, scratch_S);
    return o2_set_frozen(c, s, scratch_S);
}

static void o2_step(const o2_cfg* c, o2_head* s, const double* qt, const double* kt, const double* vt,
                    const double* gt, double bt, double* ot, double* Lt, double* x, double* y,
                    double* w, double* rr, double* u_raw, const uint8_t* u_flip) {
    int D = c->D;
    o2_current_L(c, s, Lt);
    for (int j = 0; j < D; ++j) {
        Lt[j] = Lt[j] + gate_log(gt, c->Dg, j);
        if (c->round_storage) Lt[j] = orc_round_f32(Lt[j]);
        x[j] = exp(Lt[j]) * kt[j];
        y[j] = exp(Lt[j]) * qt[j];
    }
    for (int i = 0; i < D; ++i) {
        double a = 0.0, b = 0.0;
        for (int j = 0; j < D; ++j) {
            a += s->F[(size_t)i * D + j] * x[j];
            b += s->F[(size_t)i * D + j] * y[j];
        }
        w[i] = a;
        rr[i] = b;
    }
    for (int cc = 0; cc < c->r; ++cc) {  /* tokens: coefficients <ck_c, x>, <ck_c, y> */
        double ax = 0.0, ay = 0.0;
        for (int j = 0; j < D; ++j) {
            ax += s->ck[(size_t)cc * D + j] * x[j];
            ay += s->ck[(size_t)cc * D + j] * y[j];
        }
        for (int i = 0; i < D; ++i) {
            w[i] += s->cu[(size_t)cc * D + i] * ax;
            rr[i] += s->cu[(size_t)cc * D + i] * ay;
        }
    }
    for (int p = 0; p < s->P; ++p) {
        double a = 0.0, b = 0.0;
        for (int j = 0; j < D; ++j) {
            double f = exp(Lt[j] - s->bL[(size_t)p * D + j]);
            a += s->bk[(size_t)p * D + j] * f * kt[j];
            b += s->bk[(size_t)p * D + j] * f * qt[j];
        }
        for (int i = 0; i < D; ++i) {
            w[i] += s->bu[(size_t)p * D + i] * a;
            rr[i] += s->bu[(size_t)p * D + i] * b;
        }
    }
    double kq = 0.0;
    for (int j = 0; j < D; ++j) kq += kt[j] * qt[j];
    double* un = s->bu + (size_t)s->P * D;
    for (int i = 0; i < D; ++i) {
        double u = bt * (vt[i] - w[i]);
        if (u_raw) u_raw[i] = u;
        if (c->round_storage)
            u = (u_flip && u_flip[i]) ? orc_round_other(c->buf_round, u) : round_to(c->buf_round, u);
        un[i] = u;
        if (ot) ot[i] = rr[i] + u * kq;
    }
    memcpy(s->bk + (size_t)s->P * D, kt, sizeof(double) * (size_t)D);
    memcpy(s->bL + (size_t)s->P * D, Lt, sizeof(double) * (size_t)D);
    s->P += 1;
}

int orc_o2_run(int D, int T, int W, int r, int fmt, int nh, int Dg, int round_storage,
               int buf_round, int smooth, int rule, const double* S0, const double* q, const double* k,
               const double* v, const double* g, const double* beta, const uint8_t* flush_mask,
               double* o, int8_t* codes_out, double* scales_out, int* cidx_out, double* cu_out,
               double* ck_out, int* pos_out,
               double* bk_out, double* bu_out, double* bL_out, double* S_out, int* ties_out,
               int8_t* sexp_out, double* u_raw, const uint8_t* u_flip) {
    o2_cfg c = {D, W, r, fmt, Dg, round_storage, buf_round, smooth, rule};
    int ng = orc_num_groups(fmt == ORC_FMT_NONE ? ORC_FMT_INT8 : fmt, D);
    int ties = 0;
#pragma omp parallel for schedule(dynamic) reduction(+ : ties)
    for (int h = 0; h < nh; ++h) {
        size_t DD = (size_t)D * D;
        o2_head s;
        s.F = (double*)calloc(DD, sizeof(double));
        s.scales = (double*)calloc((size_t)D * ng, sizeof(double));
        s.codes = (int8_t*)calloc(DD, 1);
        s.sexp = (int8_t*)calloc((size_t)D, 1);
        s.cidx = (int*)calloc((size_t)(r > 0 ? r : 1), sizeof(int));
        s.cu = (double*)calloc((size_t)(r > 0 ? r : 1) * D, sizeof(double));
        s.ck = (double*)calloc((size_t)(r > 0 ? r : 1) * D, sizeof(double));
        s.bk = (double*)calloc((size_t)W * D, sizeof(double));
        s.bu = (double*)calloc((size_t)W * D, sizeof(double));
        s.bL = (double*)calloc((size_t)W * D, sizeof(double));
        double* Sx = (double*)malloc(sizeof(double) * DD);
        double* vec = (double*)malloc(sizeof(double) * (size_t)D * 5);
        double *Lt = vec, *x = vec + D, *y = vec + 2 * D, *w = vec + 3 * D, *rr = vec + 4 * D;

        if (S0) memcpy(Sx, S0 + (size_t)h * DD, sizeof(double) * DD);
        else memset(Sx, 0, sizeof(double) * DD);
        int hties = o2_set_frozen(&c, &s, Sx);
        for (int t = 0; t < T; ++t) {
            size_t th = (size_t)t * nh + h;
            o2_step(&c, &s, q + th * D, k + th * D, v + th * D, g + th * Dg, beta[th],
                    o ? o + th * D : NULL, Lt, x, y, w, rr, u_raw ? u_raw + th * D : NULL,
                    u_flip ? u_flip + th * D : NULL);
            int forced = flush_mask && flush_mask[th];
            if (s.P == W || forced) hties += o2_flush(&c, &s, Sx, Lt);
        }
        ties += hties;
        if (ties_out) ties_out[h] = hties;
        if (codes_out) memcpy(codes_out + h * DD, s.codes, DD);
        if (scales_out) memcpy(scales_out + (size_t)h * D * ng, s.scales, sizeof(double) * (size_t)D * ng);
        if (cidx_out && r > 0) memcpy(cidx_out + (size_t)h * r, s.cidx, sizeof(int) * (size_t)r);
        if (cu_out && r > 0) memcpy(cu_out + (size_t)h * r * D, s.cu, sizeof(double) * (size_t)r * D);
        if (ck_out && r > 0) memcpy(ck_out + (size_t)h * r * D, s.ck, sizeof(double) * (size_t)r * D);
        if (pos_out) pos_out[h] = s.P;
        if (sexp_out) memcpy(sexp_out + (size_t)h * D, s.sexp, (size_t)D);
        if (bk_out) memcpy(bk_out + (size_t)h * W * D, s.bk, sizeof(double) * (size_t)W * D);
        if (bu_out) memcpy(bu_out + (size_t)h * W * D, s.bu, sizeof(double) * (size_t)W * D);
        if (bL_out) memcpy(bL_out + (size_t)h * W * D, s.bL, sizeof(double) * (size_t)W * D);
        if (S_out) {
            o2_current_L(&c, &s, Lt);
            o2_materialize(&c, &s, Lt, S_out + h * DD);
        }
        free(s.F); free(s.scales); free(s.codes); free(s.sexp); free(s.cidx); free(s.cu); free(s.ck);
        free(s.bk); free(s.bu); free(s.bL); free(Sx); free(vec);
    }
    return ties;
}


/* ------------------------------------------------------------------------------------------
 * PW: the pure-write sliding window ("Low-Bit GDN Recurrent-State Quantization: Global
 * Gradient-aware Allocation and Pure-Write Sliding Windows", Abstract). The state is a low-bit
 * history H plus the pure writes of the last Wp steps, each kept apart as a pair of FP8 vectors
 * (x, y) standing for the rank-one matrix x y^T. The pure write of step t is its state-free term
 * beta_t v_t k_t^T, so a pair starts as x = beta_t v_t, y = k_t. The full transition
 * Z -> Z Diag(a) (I - beta k k^T) applied to x y^T only changes the key side,
 *     y -> (I - beta k k^T) Diag(a) y = a.y - beta <k, a.y> k,
 * so a pair stays a pair while it is carried through later steps. A pair leaves the window Wp
 * steps after its write and is then added to the history, which is requantised. Since the
 * history also takes the transition every step, it is requantised every step (the low-bit
 * write-back that the window keeps recent writes out of).
 *
 * Readings (the page gives no more than the sentence above; each is listed in the design notes):
 *   - FP8 is e4m3 (the finite variant: 4 exponent bits, bias 7, 3 mantissa bits, largest 448)
 *     with one fp32 scale per vector, s = absmax / 448; stored t = e4m3(x / s), value s * t.
 *   - Step t: the pair written at t - Wp (if any) is added to the history first; the history
 *     then takes step t's transition; the pairs still in the window take it on their key side;
 *     the new pair (beta v, k) enters. Wp = 0: the write joins the history at once (this is
 *     quantize-every-step write-back).
 *   - o_t = S_t q_t from the step's results before they are stored (the history before its
 *     requantisation, the carried keys and the new pair before FP8 rounding): the rounding at
 *     the write reaches the output from the next step on, as in the window form.
 * quant = 0 keeps the history exact; fp8 = 0 keeps pairs exact. prec32 rounds what a GPU stores
 * (the write vector beta v, carried keys, merged history entries) to fp32 and takes the
 * quantizer's and the FP8 decisions in single precision.
 * ---------------------------------------------------------------------------------------- */

/* Nearest e4m3 value, ties to even, saturating at +-448. From the format's definition: normal
 * values 2^(E-7) (1 + m/8) for E = 1..15 (E = 15, m = 7 is NaN, so 448 = 2^8 * 1.75 is the
 * largest), subnormals 2^-6 (m/8); the spacing in x's binade [2^(e-1), 2^e) is 2^(e-4), never
 * finer than the subnormal spacing 2^-9. */
double orc_round_e4m3(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    double m = fabs(x);
    if (m >= 448.0) return copysign(448.0, x);
    int e;
    frexp(m, &e);                          /* m = f 2^e, 0.5 <= f < 1 */
    int qexp = e - 4;
    if (qexp < -9) qexp = -9;
    double quantum = ldexp(1.0, qexp);
    double r = rint(m / quantum) * quantum; /* 448 < r only for m in (448, 464): excluded above */
    return copysign(r, x);
}

/* FP8 round trip of an n-vector with one scale: s = absmax / 448, out = s * e4m3(x / s).
 * Returns the scale. prec32: x is first rounded to fp32 and each decision is taken in fp32. */
double orc_fp8_vector(int n, int prec32, const double* x, double* out) {
    double m = 0.0;
    for (int j = 0; j < n; ++j) m = fmax(m, fabs(prec32 ? orc_round_f32(x[j]) : x[j]));
    double s = m / 448.0;
    if (prec32) s = orc_round_f32(s);
    for (int j = 0; j < n; ++j) {
        if (s == 0.0) { out[j] = 0.0; continue; }
        double t = (prec32 ? orc_round_f32(x[j]) : x[j]) / s;
        if (prec32) t = orc_round_f32(t);
        double y = s * orc_round_e4m3(t);
        out[j] = prec32 ? orc_round_f32(y) : y;
    }
    return s;
}

int orc_pw_run(int D, int T, int Wp, int fmt, int nh, int Dg, int quant, int fp8, int prec32,
               const double* S0, const double* q, const double* k, const double* v,
               const double* g, const double* beta, double* o, int8_t* codes_out,
               double* scales_out, double* px_out, double* py_out, double* S_out) {
    if (Wp < 0 || (quant && fmt != ORC_FMT_INT8 && fmt != ORC_FMT_INT4)) return -1;
    const int qfmt = fmt == ORC_FMT_INT4 ? ORC_FMT_INT4 : ORC_FMT_INT8;
    const int ng = orc_num_groups(qfmt, D);
#pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < nh; ++h) {
        const size_t DD = (size_t)D * D;
        const int ns = Wp > 0 ? Wp : 1;
        double* H = (double*)malloc(sizeof(double) * DD);   /* history as stored (dequantised) */
        int8_t* codes = (int8_t*)calloc(DD, 1);
        double* scales = (double*)calloc((size_t)D * ng, sizeof(double));
        double* px = (double*)calloc((size_t)ns * D, sizeof(double)); /* pair x, by ring slot */
        double* py = (double*)calloc((size_t)ns * D, sizeof(double)); /* pair y, by ring slot */
        double* pyn = (double*)malloc(sizeof(double) * (size_t)ns * D);  /* carried keys */
        double* a = (double*)malloc(sizeof(double) * D);
        double* w = (double*)malloc(sizeof(double) * D);
        double* x = (double*)malloc(sizeof(double) * D);
        if (S0) memcpy(H, S0 + h * DD, sizeof(double) * DD);
        else memset(H, 0, sizeof(double) * DD);
        if (quant) {
            orc_quantize(D, qfmt, prec32, H, codes, scales);
            orc_dequantize(D, qfmt, codes, scales, H);
        }
        for (int t = 0; t < T; ++t) {
            const size_t th = (size_t)t * nh + h;
            const double* kt = k + th * D;
            const double* qt = q + th * D;
            const double* vt = v + th * D;
            const double* gt = g + th * Dg;
            const double bt = beta[th];
            for (int j = 0; j < D; ++j) a[j] = exp(gate_log(gt, Dg, j));
            const int slot = Wp > 0 ? t % Wp : 0;
            /* the pair written Wp steps ago leaves the window: into the history */
            if (Wp > 0 && t >= Wp)
                for (int i = 0; i < D; ++i)
                    for (int j = 0; j < D; ++j)
                        H[(size_t)i * D + j] += px[(size_t)slot * D + i] * py[(size_t)slot * D + j];
            /* history: H <- H Diag(a) (I - beta k k^T) */
            for (int i = 0; i < D; ++i) {
                double acc = 0.0;
                for (int j = 0; j < D; ++j) {
                    H[(size_t)i * D + j] *= a[j];
                    acc += H[(size_t)i * D + j] * kt[j];
                }
                w[i] = acc;
            }
            for (int i = 0; i < D; ++i)
                for (int j = 0; j < D; ++j) H[(size_t)i * D + j] -= bt * w[i] * kt[j];
            /* pairs still in the window (written at t-Wp+1 .. t-1): key side of the transition */
            const int carried = Wp > 0 ? (t < Wp - 1 ? t : Wp - 1) : 0;
            for (int p = 1; p <= carried; ++p) {
                const int sl = (t - p) % Wp;
                const double* y = py + (size_t)sl * D;
                double* yn = pyn + (size_t)sl * D;
                double ky = 0.0;
                for (int j = 0; j < D; ++j) ky += kt[j] * a[j] * y[j];
                for (int j = 0; j < D; ++j) yn[j] = a[j] * y[j] - bt * ky * kt[j];
            }
            /* the pure write of this step */
            for (int i = 0; i < D; ++i) {
                x[i] = bt * vt[i];
                if (prec32) x[i] = orc_round_f32(x[i]);
            }
            if (Wp == 0)
                for (int i = 0; i < D; ++i)
                    for (int j = 0; j < D; ++j) H[(size_t)i * D + j] += x[i] * kt[j];
            /* o_t = S_t q_t, before storage rounding */
            if (o) {
                double* ot = o + th * D;
                for (int i = 0; i < D; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < D; ++j) acc += H[(size_t)i * D + j] * qt[j];
                    ot[i] = acc;
                }
                for (int p = 1; p <= carried; ++p) {
                    const int sl = (t - p) % Wp;
                    double yq = 0.0;
                    for (int j = 0; j < D; ++j) yq += pyn[(size_t)sl * D + j] * qt[j];
                    for (int i = 0; i < D; ++i) ot[i] += px[(size_t)sl * D + i] * yq;
                }
                if (Wp > 0) {
                    double kq = 0.0;
                    for (int j = 0; j < D; ++j) kq += kt[j] * qt[j];
                    for (int i = 0; i < D; ++i) ot[i] += x[i] * kq;
                }
            }
            /* storage: history requantised (or fp32), carried keys and the new pair rounded */
            if (quant) {
                if (prec32)
                    for (size_t e = 0; e < DD; ++e) H[e] = orc_round_f32(H[e]);
                orc_quantize(D, qfmt, prec32, H, codes, scales);
                orc_dequantize(D, qfmt, codes, scales, H);
            } else if (prec32) {
                for (size_t e = 0; e < DD; ++e) H[e] = orc_round_f32(H[e]);
            }
            for (int p = 1; p <= carried; ++p) {
                const int sl = (t - p) % Wp;
                double* y = py + (size_t)sl * D;
                const double* yn = pyn + (size_t)sl * D;
                if (fp8) orc_fp8_vector(D, prec32, yn, y);
                else
                    for (int j = 0; j < D; ++j) y[j] = prec32 ? orc_round_f32(yn[j]) : yn[j];
            }
            if (Wp > 0) {
                double* xs = px + (size_t)slot * D;
                double* ys = py + (size_t)slot * D;
                if (fp8) {
                    orc_fp8_vector(D, prec32, x, xs);
                    orc_fp8_vector(D, prec32, kt, ys);
                } else {
                    memcpy(xs, x, sizeof(double) * D);
                    for (int j = 0; j < D; ++j) ys[j] = prec32 ? orc_round_f32(kt[j]) : kt[j];
                }
            }
        }
        if (codes_out) memcpy(codes_out + h * DD, codes, DD);
        if (scales_out) memcpy(scales_out + (size_t)h * D * ng, scales, sizeof(double) * (size_t)D * ng);
        if (px_out && Wp > 0) memcpy(px_out + (size_t)h * Wp * D, px, sizeof(double) * (size_t)Wp * D);
        if (py_out && Wp > 0) memcpy(py_out + (size_t)h * Wp * D, py, sizeof(double) * (size_t)Wp * D);
        if (S_out) {
            double* S = S_out + h * DD;
            memcpy(S, H, sizeof(double) * DD);
            const int live = T < Wp ? T : Wp;  /* pairs written at T-live .. T-1 */
            for (int p = 1; p <= live; ++p) {
                const int sl = (T - p) % Wp;
                for (int i = 0; i < D; ++i)
                    for (int j = 0; j < D; ++j)
                        S[(size_t)i * D + j] += px[(size_t)sl * D + i] * py[(size_t)sl * D + j];
            }
        }
        free(H); free(codes); free(scales); free(px); free(py); free(pyn);
        free(a); free(w); free(x);
    }
    return 0;
}
