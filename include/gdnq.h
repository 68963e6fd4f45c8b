/*
 * gdnq.h -- C ABI of libgdnq: gated delta-rule (GDN / KDA) decode over a low-bit recurrent
 * state with per-window quantization, for NVIDIA B200 (sm_100a).
 *
 * The method ("LeapQuant: Efficient Linear Attention with Accurate Recurrent State
 * Quantization", Abstract): every decode step of a GDN / KDA layer reads and updates a fixed-size
 * recurrent state per (sequence, head). Here that state is kept in HBM as int8 codes with one
 * fp32 absmax scale per row (or packed int4 codes with one scale per 32 key channels) and is
 * frozen for a window of W tokens. Inside the window each step reads the frozen state plus the
 * window's buffered high-precision write pairs; when the window fills, the state is
 * materialised, its r largest-outlier key columns are kept aside in fp32 as compensator pairs,
 * and the rest is requantised, in the same kernel.
 *
 * Recurrence, per (sequence, head), S in R^{d_v x d_k} (row = value channel, column = key
 * channel), gate a_t = exp(g_t) (GDN: one scalar per head; KDA: one per key channel):
 *     S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,      o_t = S_t q_t
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers unless the name says host; the caller owns and
 *     allocates every buffer (sizes from gdn_state_sizes). The library allocates no device
 *     memory and keeps no state between calls except a thread-local last-error message.
 *   - State buffers, fp32 state arrays (S), the staging buffer and, for the window step, q, k, v
 *     and a per-channel g must be 16-byte aligned (they are moved with bulk async copies); o,
 *     beta, a scalar g, the status word, seq_mask and the baseline step's inputs need only their
 *     element alignment (GDN_ERR_INVALID_ARG otherwise).
 *   - Work is enqueued on `stream` and runs asynchronously; a GDN_OK return means the launch
 *     was accepted. Arguments are checked before anything is enqueued; on any error nothing is
 *     enqueued, except GDN_ERR_CUDA from a launch, after which outputs are undefined.
 *   - B * H == 0 is a valid empty batch: the call checks its arguments and returns GDN_OK.
 *   - Layouts are dense, row-major, batch-major: [B][H][...].
 */
#ifndef GDNQ_H
#define GDNQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (same handle type); NULL is the legacy default stream. */
typedef struct CUstream_st* gdn_stream_t;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size or enum value */
    GDN_ERR_UNSUPPORTED = 2,  /* valid but not built: head size, format, window too large */
    GDN_ERR_CUDA = 3,         /* a CUDA call failed; gdn_last_error() has the CUDA message */
    GDN_ERR_TIMEOUT = 4       /* reserved: a bounded device wait ran out (see status word) */
} gdn_status;

/* Bits a kernel ORs into gdn_state.status (when it is not NULL). */
#define GDN_DEVICE_WAIT_TIMEOUT 0x1 /* a bounded wait for a staging copy ran out */
#define GDN_DEVICE_BAD_POS 0x2      /* a head's pos was outside [0, W): the head was skipped */

typedef enum { GDN_GATE_SCALAR = 0, GDN_GATE_DIAG = 1 } gdn_gate_kind;

typedef enum {
    GDN_FMT_INT8 = 0,     /* int8 codes, one fp32 scale per state row */
    GDN_FMT_INT4_G32 = 1, /* packed int4 codes, one fp32 scale per row and 32 key channels */
    GDN_FMT_BF16 = 2,     /* plain bf16 state (baseline step only) */
    GDN_FMT_FP32 = 3,     /* plain fp32 state (baseline step only) */
    GDN_FMT_MIXED = 4     /* INT8 or INT4_G32 per head, as gdn_state.head_fmt says (d = 128) */
} gdn_state_format;

typedef enum { GDN_DTYPE_F32 = 0, GDN_DTYPE_BF16 = 1 } gdn_dtype;

/* Largest compensator count per head. */
#define GDN_MAX_COMPENSATORS 16

/*
 * How the r compensator tokens are chosen at every quantization ("LeapQuant ..." Abstract: the
 * state's largest outliers are kept as a few high-precision compensator tokens that share the
 * update path of real tokens; the page gives no rule -- both rules are readings):
 *   GDN_COMP_COLUMNS  the r key columns of largest max-abs (ties: lower index); token c has key
 *                     e_{comp_idx[c]} and value that column.
 *   GDN_COMP_POWER    the state's dominant r-dimensional key subspace, by subspace iteration:
 *                     start from the r key columns of largest L2 norm (ties: lower index), six
 *                     times X <- orth(S^T S X) (modified Gram-Schmidt over the columns in order,
 *                     run twice in single precision, which is the same in exact arithmetic;
 *                     a column of length 0 stays 0); token c has key x_c (comp_k[c], unit
 *                     length) and value S x_c, and the residual S (I - X X^T) is quantized.
 *                     Built for d = 128, bf16 activations and buffers, INT8 / INT4_G32 states
 *                     without smoothing, W <= 64 (GDN_ERR_UNSUPPORTED elsewhere). A decode step
 *                     whose window fills leaves it full (pos = W inside the call) and a second
 *                     kernel of the same call runs the window end, so pos is back to 0 when the
 *                     call's work is done.
 */
typedef enum { GDN_COMP_COLUMNS = 0, GDN_COMP_POWER = 1 } gdn_comp_rule;

typedef struct {
    int32_t B, H;      /* sequences, heads per sequence (>= 0) */
    int32_t d_k, d_v;  /* head sizes; this build: d_k == d_v in {16, 128} */
    int32_t W;         /* window length in tokens (>= 1) */
    int32_t r;         /* compensator pairs per head, 0..GDN_MAX_COMPENSATORS */
    int32_t gate;      /* gdn_gate_kind */
    int32_t fmt;       /* gdn_state_format */
    int32_t act_dtype; /* gdn_dtype of q, k, v, o and of the buffered keys */
    int32_t buf_dtype; /* gdn_dtype of the buffered write vectors u */
    int32_t smooth;    /* gdn_smoothing: residual smoothing at every quantization (INT8 and
                          INT4_G32 states; 0 elsewhere) */
    int32_t comp_rule; /* gdn_comp_rule of the compensator tokens (0: columns) */
} gdn_config;

/*
 * Residual smoothing ("LeapQuant ..." Abstract: the residual left after the compensators is
 * smoothed before quantization; the page gives no mechanism, this is the reading built here).
 * At every quantization (gdn_state_quantize, each window end, gdn_window_flush), after the
 * compensator columns are taken out, key column j of the residual R gets an exponent
 *     e_j = floor(E_j / 2) clamped to [-63, 63],  E_j = floor(log2 max_i |R_ij|)  (e_j = 0 for a
 *                                                    zero column),
 * and the residual is quantized as R Diag(2^-e) (per-row or per-group scales as usual), so the
 * frozen state is dequant(codes, scales) Diag(2^e): a column's factor is the power of two at or
 * below the square root of its max-abs, which halves (in log scale) the spread of column ranges
 * a row's scale must cover. Powers of two make the rescaling exact (fp32, away from the
 * subnormal range); the exponents live in gdn_state.smooth_exp.
 */
typedef enum { GDN_SMOOTH_NONE = 0, GDN_SMOOTH_POW2_COLUMNS = 1 } gdn_smoothing;

/*
 * The windowed low-bit state of a batch: caller-owned device buffers, per head (D = d_k = d_v,
 * Wp = W rounded up to a multiple of 4, rp = r rounded up to a multiple of 4):
 *   codes    int8  [B][H][D][D]        (GDN_FMT_INT8)
 *            uint8 [B][H][D][D/2]      (GDN_FMT_INT4_G32; byte m of a row holds column 2m in
 *                                       its low nibble, 2m+1 in its high nibble, 4-bit two's
 *                                       complement codes in [-7, 7])
 *   scales   fp32  [B][H][D]           (int8: row i dequantises as scales[i] * code)
 *            fp32  [B][H][D][D/32]     (int4: group g of row i covers columns 32g..32g+31)
 *   buf_k    act   [B][H][W][D]        buffered keys (the step's k, stored as given)
 *   buf_u    buf   [B][H][W][D]        buffered write vectors u_i = beta_i (v_i - w_i)
 *   buf_L    fp32  [B][H][Wp]          (scalar gate) cumulative log-gate of each pair
 *            fp32  [B][H][W][D]        (diagonal gate) the same per key channel
 *   comp_idx int32 [B][H][rp]          key column of each compensator pair (r > 0, columns rule)
 *   comp_u   fp32  [B][H][r][D]        value of each compensator token (r > 0 only)
 *   comp_k   fp32  [B][H][r][D]        key of each compensator token (r > 0, power rule only;
 *                                       16-byte aligned)
 *   pos      int32 [B][H]              pairs already in the window, 0 <= pos < W
 *   status   int32 [1], optional       device word the kernels OR GDN_DEVICE_* bits into
 *   head_fmt int8  [B][H]              (GDN_FMT_MIXED only) GDN_FMT_INT8 or GDN_FMT_INT4_G32 for
 *                                       each head; read by every call, written by none
 *   smooth_exp int8 [B][H][D]          (smooth != 0 only, 16-byte aligned) the smoothing exponent
 *                                       e_j of each key column of the frozen codes
 * With GDN_FMT_MIXED ("Low-Bit GDN Recurrent-State Quantization ...", Abstract: bit widths
 * allocated per head under a model-wide budget) every head has the slot of the larger format:
 *   codes    uint8 [B][H][D][D]        an INT8 head fills its slot as above; an INT4_G32 head
 *                                       uses its first D*D/2 bytes, laid out as for INT4_G32
 *   scales   fp32  [B][H][D][D/32]     an INT4_G32 head fills its slot; an INT8 head uses its
 *                                       first D floats
 * and every entry point treats each head exactly as a call with that head's format would.
 * Tiles are stored swizzled: in each per-head [rows][RB-byte] tile of codes, buf_k and buf_u,
 * the 16-byte chunk c of row i is stored at chunk c ^ x(i), x(i) = i & 7 when RB >= 128, else
 * (i * RB / 128) & (RB / 16 - 1) (identity for 16-byte rows). A row's bytes keep their order
 * within a chunk. This lets the kernels copy a head's tiles into shared memory with one bulk
 * copy each and read eight consecutive rows at one column without bank conflicts.
 * gdn_state_materialize returns the logical state in plain row-major order.
 * The logical state of a head with P = pos pairs and L = buf_L[P-1] (0 when P == 0) is
 *   S = dequant(codes, scales) Diag(2^e) Diag(e^L) + sum_c comp_u[c] (ck_c * e^{L})^T
 *       + sum_{i<P} buf_u[i] (buf_k[i] * e^{L - buf_L[i]})^T,
 * ck_c = e_{comp_idx[c]} (columns rule) or comp_k[c] (power rule).
 * (Diag(2^e) only with smoothing.) Entries of buf_k / buf_u / buf_L at index >= pos are scratch
 * and never read.
 */
typedef struct {
    void* codes;
    float* scales;
    void* buf_k;
    void* buf_u;
    float* buf_L;
    int32_t* comp_idx;
    float* comp_u;
    int32_t* pos;
    int32_t* status;
    const int8_t* head_fmt;
    int8_t* smooth_exp;
    float* comp_k;
} gdn_state;

/* Byte sizes of each buffer of gdn_state for the whole batch (0 where unused), and the dynamic
 * shared memory one decode-step CTA needs. */
typedef struct {
    size_t codes, scales, buf_k, buf_u, buf_L, comp_idx, comp_u, pos;
    size_t smem_step;
    size_t head_fmt;
    size_t smooth_exp;
    size_t comp_k;
} gdn_sizes;

/* Checks cfg and fills *out. Host-only: touches no device. The buffers are the parts of the
 * windowed state that "LeapQuant ..." (Abstract) names: the low-bit state frozen for the window
 * (codes, scales), the window's high-precision buffered updates (buf_k, buf_u, buf_L) and the
 * compensator tokens (comp_idx, comp_u). Errors: GDN_ERR_INVALID_ARG for a null argument or bad
 * field, GDN_ERR_UNSUPPORTED for a configuration this build lacks. */
gdn_status gdn_state_sizes(const gdn_config* cfg, gdn_sizes* out);

/*
 * Initial quantization of a batch of fp32 states ("LeapQuant ..." Abstract: the state held in
 * low bits; compensator tokens keep the largest outliers). For every head: the r key columns of
 * S with the largest max-abs (ties to the lower index) are copied to comp_u / comp_idx and
 * zeroed, then each row (int4: each 32-column group) gets s = absmax / qmax (qmax 127 or 7,
 * IEEE single division) and codes c = clamp(rint(x / s), -qmax, qmax); a zero row gets s = 0
 * and codes 0 (with smoothing, the rows are those of the rescaled residual and smooth_exp is
 * written). pos is set to 0; the window buffer is left as it is.
 *   S   device fp32 [B][H][D][D], read only.
 */
gdn_status gdn_state_quantize(const gdn_config* cfg, const float* S, const gdn_state* state,
                              gdn_stream_t stream);

/*
 * One decode step for every (sequence, head) ("LeapQuant ..." Abstract: within a window,
 * outputs come from the fixed low-bit state together with high-precision buffered updates; the
 * state is quantized once, at the window's end). With P = pos, L = buf_L[P-1] (0 if P == 0):
 *   L_t = L + g_t;  x = e^{L_t} k_t;  y = e^{L_t} q_t   (scalar gate: e^{L_t} is a scalar)
 *   w = F x + sum_c comp_u[c] x[comp_idx[c]] + sum_{i<P} buf_u[i] <buf_k[i] e^{L_t - buf_L[i]}, k_t>
 *   r = the same with y and q_t                         (F = dequantised codes, times
 *                                                        Diag(2^smooth_exp) with smoothing)
 *   u_t = round_buf(beta_t (v_t - w));  o_t = round_act(r + u_t <k_t, q_t>)
 * then (k_t, u_t, L_t) is appended at index P. When P + 1 == W the window is flushed in the same
 * kernel: the logical state (with the new pair) is materialised in fp32, compensators, codes (and
 * with smoothing the exponents) are rebuilt exactly as in gdn_state_quantize, and pos becomes 0;
 * otherwise pos becomes P + 1.
 * The step's output is taken before that requantisation.
 *   q, k, v  device act [B][H][D];  g device fp32 [B][H] (scalar) or [B][H][D] (diagonal), the
 *   log of the gate (<= 0 for a decaying gate);  beta device fp32 [B][H];  o device act [B][H][D].
 * A head whose pos is outside [0, W) is skipped and reported through state->status.
 */
gdn_status gdn_decode_window_step(const gdn_config* cfg, const gdn_state* state, const void* q,
                                  const void* k, const void* v, const float* g,
                                  const float* beta, void* o, gdn_stream_t stream);

/*
 * T consecutive decode steps, one kernel launch per step, inputs stacked along a leading time
 * axis: q, k, v, o [T][B][H][D]; g [T][B][H](/[D]); beta [T][B][H]. Same as T calls of
 * gdn_decode_window_step. T >= 0.
 */
gdn_status gdn_decode_window_steps(const gdn_config* cfg, const gdn_state* state, int32_t T,
                                   const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, void* o, gdn_stream_t stream);

/*
 * End-to-end variant of gdn_decode_window_steps whose per-step inputs and outputs live in HOST
 * memory (pinned memory is needed for the copies to overlap; pageable memory works but
 * serialises). Each step's inputs are copied into a device staging slot, the step kernel runs,
 * and its output is copied back, pipelined over two slots and three streams: `stream` runs the
 * kernels, two internal streams (created and destroyed by this call) run the copies. Returns
 * after everything is enqueued; the host output is complete once `stream` has finished.
 *   host_q, host_k, host_v, host_o  host act [T][B][H][D]; host_g host fp32 [T][B][H](/[D]);
 *   host_beta host fp32 [T][B][H];
 *   staging        device buffer of staging_bytes >= gdn_host_staging_bytes(cfg) bytes.
 */
size_t gdn_host_staging_bytes(const gdn_config* cfg);
gdn_status gdn_decode_window_steps_host(const gdn_config* cfg, const gdn_state* state, int32_t T,
                                        const void* host_q, const void* host_k,
                                        const void* host_v, const float* host_g,
                                        const float* host_beta, void* host_o, void* staging,
                                        size_t staging_bytes, gdn_stream_t stream);

/*
 * The same T decode steps from host buffers as gdn_decode_window_steps_host, for callers that
 * may not allocate device memory themselves -- for instance a process whose device memory is
 * owned by another framework's allocator and fixed at start-up -- and so cannot provide the
 * staging buffer. (The method's pages describe no such entry point; it is an interface
 * convenience of this library only.)
 *   - Staging lives in one fixed device array inside the library, GDN_FIXED_STAGING_BYTES
 *     (16 MiB) per device, reserved when the library is loaded. The call allocates nothing:
 *     no device or host memory, no streams, no events.
 *   - Needs one staging slot, gdn_host_staging_bytes(cfg) / 2 bytes, to fit in
 *     GDN_FIXED_STAGING_BYTES: about 1 KiB per (sequence, head) pair for bf16 and d = 128, so up
 *     to roughly 16,000 pairs per call; a larger batch gets GDN_ERR_UNSUPPORTED with the sizes
 *     in gdn_last_error() and nothing is enqueued.
 *   - Nothing in the array needs to start at zero: every step overwrites the inputs it uses.
 *   - Runs serially on `stream` (per step: copy in, the step kernel, copy out), with no overlap
 *     of copies and kernels; returns after everything is enqueued. host_o is complete once
 *     `stream` has finished. Pinned host memory is needed for the copies to be asynchronous.
 *   - All calls on one device share the array: two calls whose work overlaps in time (on
 *     different streams, or from different host threads) race on it. Serialise them.
 *   - Every call looks up the array's address in the current device's context
 *     (cudaGetSymbolAddress; GDN_ERR_CUDA if that fails), so a call after cudaDeviceReset uses
 *     the array of the new context.
 * Arguments, layouts and errors otherwise as gdn_decode_window_steps_host.
 */
#define GDN_FIXED_STAGING_BYTES ((size_t)16 << 20)
gdn_status gdn_decode_window_steps_host_fixed(const gdn_config* cfg, const gdn_state* state,
                                              int32_t T, const void* host_q, const void* host_k,
                                              const void* host_v, const float* host_g,
                                              const float* host_beta, void* host_o,
                                              gdn_stream_t stream);

/*
 * Forced window flush ("LeapQuant ..." Abstract: the state is quantized once, at its window's
 * end; this runs that window-end operation early): for every head whose sequence is selected
 * (seq_mask == NULL selects all;
 * otherwise device int32 [B], nonzero = selected) and whose pos > 0, materialise the logical
 * state, rebuild compensators and codes as gdn_state_quantize does, and set pos = 0. Heads with
 * pos == 0 are left untouched (their logical state is already the frozen one). Used to hand a
 * compact state (empty buffer) to a checkpoint, or to end a sequence's window early.
 */
gdn_status gdn_window_flush(const gdn_config* cfg, const gdn_state* state,
                            const int32_t* seq_mask, gdn_stream_t stream);

/*
 * Writes the logical state of every head (formula above) as fp32 [B][H][D][D] to S, without
 * changing the state: the materialisation that "LeapQuant ..." (Abstract) performs at a
 * window's end, before the requantisation, i.e. the frozen low-bit state carried through the
 * window plus the buffered updates and the compensator tokens.
 */
gdn_status gdn_state_materialize(const gdn_config* cfg, const gdn_state* state, float* S,
                                 gdn_stream_t stream);

/*
 * Baseline ("LeapQuant ..." Abstract: its kernel speedups are measured against decode over an
 * FP32 recurrent state; the bf16 state is the usual half-precision alternative): one plain
 * decode step over a high-precision state (cfg->fmt GDN_FMT_FP32 or
 * GDN_FMT_BF16; W, r and buf_dtype are ignored). The state S [B][H][D][D] is read once and
 * written once, in place:
 *   w = S (a_t * k_t);  u = beta_t (v_t - w);  S <- S Diag(a_t) + u k_t^T (rounded to nearest
 *   even for bf16);  o_t = S Diag(a_t) q_t + u <k_t, q_t>   (taken before the state rounding)
 * q, k, v, o, g, beta as for gdn_decode_window_step.
 */
gdn_status gdn_baseline_step(const gdn_config* cfg, void* S, const void* q, const void* k,
                             const void* v, const float* g, const float* beta, void* o,
                             gdn_stream_t stream);

/* Name of a status code (static string). */
const char* gdn_status_string(gdn_status status);

/* Detail of the last error returned on the calling thread (static per-thread buffer, "" if none). */
const char* gdn_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* GDNQ_H */
