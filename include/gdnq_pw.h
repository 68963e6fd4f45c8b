/*
 * gdnq_pw.h -- C ABI of libgdnq, part 2: the pure-write sliding window over a low-bit
 * recurrent state, for NVIDIA B200 (sm_100a).
 *
 * The method ("Low-Bit GDN Recurrent-State Quantization: Global Gradient-aware Allocation and
 * Pure-Write Sliding Windows", Abstract): the most recent pure writes are kept apart from the
 * low-bit history as FP8 vector pairs; while they are in the window they are carried through the
 * full GDN transition, and a pair is merged into the low-bit history only once it has left the
 * window. The paper's "PW-S8" keeps 8 such pairs.
 *
 * Per (sequence, head), with D = d (head size), the logical state is
 *     S = dequant(codes, scales) + sum over the pairs p in the window of x_p y_p^T,
 * x_p = sx_p * e4m3(pair_x_p), y_p = sy_p * e4m3(pair_y_p). One decode step with inputs
 * q, k, v, g (a = e^g), beta:
 *   1. if the window is full, its oldest pair (x_o, y_o) leaves: M = dequant(H) + x_o y_o^T,
 *      else M = dequant(H);
 *   2. the history takes the transition: H' = M Diag(a) (I - beta k k^T)  (with Wp = 0 the
 *      write joins at once: H' += beta v k^T);
 *   3. every other pair in the window takes it on its key side:
 *      y_p' = a.y_p - beta <k, a.y_p> k  (x_p is unchanged);
 *   4. the step's pure write enters as a new pair x = beta v, y = k (Wp > 0);
 *   5. o = S' q, from H', the y_p' and the new pair before they are rounded for storage;
 *   6. storage: H' is requantised (every step: the transition changes it), each y_p' and the
 *      new pair are rounded to FP8 with a fresh scale.
 * FP8 is e4m3 (largest finite value 448) with one fp32 scale per vector, s = absmax / 448 (IEEE
 * single division), stored code e4m3(x / s) rounded to nearest even with saturation (a zero
 * vector has s = 0 and codes 0). The history quantizer is the one of gdn_state_quantize.
 *
 * Conventions are those of gdnq.h: device pointers, caller-owned buffers, asynchronous work on
 * `stream`, checks before anything is enqueued, B * H == 0 a valid empty batch, status bits in
 * the optional status word (GDN_DEVICE_BAD_POS: a head's count was out of range and the head was
 * skipped; GDN_DEVICE_WAIT_TIMEOUT: a bounded wait for a staging copy ran out).
 */
#ifndef GDNQ_PW_H
#define GDNQ_PW_H

#include "gdnq.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Largest number of pure-write pairs per head. */
#define GDN_PW_MAX_WINDOW 16

typedef struct {
    int32_t B, H;      /* sequences, heads per sequence (>= 0) */
    int32_t d;         /* head size, d_k = d_v; this build: 128 */
    int32_t Wp;        /* pure-write pairs kept per head, 0..GDN_PW_MAX_WINDOW */
    int32_t gate;      /* gdn_gate_kind */
    int32_t fmt;       /* history: GDN_FMT_INT8 or GDN_FMT_INT4_G32 */
    int32_t act_dtype; /* gdn_dtype of q, k, v, o */
} gdn_pw_config;

/*
 * Caller-owned device buffers of a batch (Wr = Wp rounded up to a multiple of 4):
 *   codes    the history's codes: layout, packing and tile swizzle of gdn_state.codes for fmt
 *   scales   the history's scales, as gdn_state.scales
 *   pairs    uint8 [B][H][2][Wp][D]   e4m3 codes: [0][slot] the value side x of the pair in that
 *                                     ring slot, [1][slot] its key side y
 *   pscales  fp32  [B][H][2][Wr]      their scales: [0][slot] of x, [1][slot] of y
 *   count    int32 [B][H]             writes n since the window was last emptied, stored as n
 *                                     while n < Wp and as Wp + (n mod Wp) after (0 when Wp = 0);
 *                                     the write made m writes before the next one lives in slot
 *                                     (count - m) mod Wp, the next write goes to count mod Wp
 *   status   int32 [1], optional
 * Entries of pairs / pscales in slots not holding a pair are scratch and never read.
 */
typedef struct {
    void* codes;
    float* scales;
    uint8_t* pairs;
    float* pscales;
    int32_t* count;
    int32_t* status;
} gdn_pw_state;

typedef struct {
    size_t codes, scales, pairs, pscales, count;
} gdn_pw_sizes;

/* Checks cfg and fills *out (bytes of each buffer for the batch). Host-only. */
gdn_status gdn_pw_state_sizes(const gdn_pw_config* cfg, gdn_pw_sizes* out);

/*
 * History <- quantize(S) exactly as gdn_state_quantize does (no compensators), count <- 0 (an
 * empty window). S device fp32 [B][H][D][D], read only. Draining a window into the history is
 * gdn_pw_materialize followed by this call.
 */
gdn_status gdn_pw_quantize(const gdn_pw_config* cfg, const float* S, const gdn_pw_state* state,
                           gdn_stream_t stream);

/*
 * One decode step for every (sequence, head), as described at the top of this file.
 *   q, k, v  device act [B][H][D] (16-byte aligned); g device fp32 [B][H] (scalar gate) or
 *   [B][H][D] (diagonal gate, 16-byte aligned), the log of the gate; beta device fp32 [B][H];
 *   o device act [B][H][D].
 * A head whose count is out of range is skipped and reported through state->status.
 */
gdn_status gdn_pw_decode_step(const gdn_pw_config* cfg, const gdn_pw_state* state, const void* q,
                              const void* k, const void* v, const float* g, const float* beta,
                              void* o, gdn_stream_t stream);

/* T consecutive steps, one launch each, inputs stacked along a leading time axis as for
 * gdn_decode_window_steps. */
gdn_status gdn_pw_decode_steps(const gdn_pw_config* cfg, const gdn_pw_state* state, int32_t T,
                               const void* q, const void* k, const void* v, const float* g,
                               const float* beta, void* o, gdn_stream_t stream);

/* Writes the logical state (history plus the pairs in the window) of every head as fp32
 * [B][H][D][D] to S, without changing the state. */
gdn_status gdn_pw_materialize(const gdn_pw_config* cfg, const gdn_pw_state* state, float* S,
                              gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDNQ_PW_H */
