/*
 * gdnq_prefill.h -- C ABI of libgdnq, part 3: chunkwise-parallel GDN prefill, the step that
 * produces the recurrent state decode starts from, for NVIDIA B200 (sm_100a).
 *
 * The method ("LinQuant: Functional Invariances for Low-Precision Linear Recurrences",
 * Abstract: a linear recurrence's prefill evaluated chunk by chunk as dense matrix products):
 * the L tokens of a prompt run through the gated delta rule of gdnq.h,
 *     S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,     o_t = S_t q_t,
 * for every (sequence, head), with a scalar gate (GDN: a_t = e^{g_t} on every key channel) or a
 * per-key-channel gate (KDA: a_t = e^{g_t}, one log-gate per key channel), in chunks whose
 * intra-chunk part is a handful of dense products (the UT / WY form of the delta rule); only the
 * state passes from one chunk to the next. Scalar gate: 64-token chunks. Per-channel gate:
 * 16-token chunks, the pairwise decays e^{G_t - G_s} taken through the chunk's eighth token. The
 * final state can then be quantized for decode with gdn_state_quantize.
 *
 * Conventions are those of gdnq.h (device pointers, caller-owned buffers, asynchronous work on
 * `stream`, argument checks before anything is enqueued, B * H == 0 a valid empty batch).
 */
#ifndef GDNQ_PREFILL_H
#define GDNQ_PREFILL_H

#include "gdnq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * L prompt tokens of every head, in place on S.
 *   cfg     B, H, d_k = d_v = 128, gate GDN_GATE_SCALAR or GDN_GATE_DIAG, act_dtype
 *           GDN_DTYPE_BF16 (this build); W, r, fmt and buf_dtype are ignored.
 *   L       tokens per sequence, >= 0 (any length: a last partial chunk is padded inside the
 *           kernel with tokens that change nothing).
 *   q, k, v device bf16 [B][H][L][D] (head-major: each head's tokens contiguous), 16-byte
 *           aligned; k and q as the decode step takes them (the layer's normalisation applied).
 *   g       device fp32, the log of the gate, finite: [B][H][L] for the scalar gate (4-byte
 *           aligned); [B][H][L][D] for the per-channel gate (16-byte aligned), where every
 *           channel's log-gate summed over any 8 consecutive tokens must stay above -80 (for
 *           example g >= -10 everywhere) so that the chunk's decay factors e^{+-(G_t - G_r)} stay
 *           finite in fp32; beyond that the results are undefined.
 *   beta    device fp32 [B][H][L].
 *   o       device bf16 [B][H][L][D], written for every token.
 *   S       device fp32 [B][H][D][D], 16-byte aligned: the state before the prompt on entry, after
 *           it on return (row = value channel, column = key channel).
 *   workspace, workspace_bytes  device scratch the caller provides, 16-byte aligned, at least
 *           gdn_prefill_workspace_bytes(cfg, L) bytes (none for the per-channel gate, where the
 *           pointer may be NULL). The scalar gate keeps there, for every 64-token chunk, what
 *           does not depend on the state (the chunk's T = (I + A)^{-1} Diag(beta) and decayed
 *           scores P as split operand tiles, and its gates: 33,792 bytes), computed by a first
 *           kernel over all chunks at once; the second kernel carries the state through the
 *           chunks. Contents on entry are ignored; on return they are scratch.
 * Arithmetic: products on tensor cores (tcgen05 for the scalar gate, the state in tensor memory;
 * mma.sync for the per-channel gate's 16-token chunks, the state in registers) with fp32
 * accumulation; q, k, v enter exactly, every
 * fp32 operand (the state, the chunk's triangular inverse, the corrected values, the decayed
 * scores, keys and queries, the write vectors) as the sum of two bf16 parts; the triangular
 * inverse in fp32.
 * Errors: GDN_ERR_INVALID_ARG for a null or misaligned pointer (when B * H > 0 and L > 0), L < 0
 * or a malformed cfg; GDN_ERR_UNSUPPORTED for d_k or d_v other than 128 or activations other
 * than bf16 (nothing is enqueued on either); a failed launch as GDN_ERR_CUDA.
 */
gdn_status gdn_prefill(const gdn_config* cfg, int32_t L, const void* q, const void* k,
                       const void* v, const float* g, const float* beta, void* o, float* S,
                       void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/* Bytes of workspace gdn_prefill needs for cfg and a prompt of L tokens (0 for the per-channel
 * gate, for an empty batch or prompt, or for a cfg gdn_prefill rejects). Host-only. */
size_t gdn_prefill_workspace_bytes(const gdn_config* cfg, int32_t L);

#ifdef __cplusplus
}
#endif

#endif /* GDNQ_PREFILL_H */
