// Internal launch interface between the C ABI (api.cu) and the kernel translation units.
#pragma once

#include <cuda_runtime.h>

#include "gdnq.h"
#include "gdnq_pw.h"

namespace gdnq {

struct WinArgs;
struct BaseArgs;
struct PwArgs;
struct PfArgs;

enum class WinOp { Step, Flush, Materialize, Quantize };

// Largest dynamic shared memory per CTA on sm_100 (bytes).
constexpr int kMaxSmemPerCta = 227 * 1024;

// Most heads one persistent step CTA walks (its per-head pos / gate / beta live in shared memory).
constexpr int kMaxHeadsPerCta = 1024;

// Dynamic shared memory a window kernel needs for this configuration at the least (one stage,
// the largest per-CTA head range).
size_t window_smem_bytes(const gdn_config& cfg);

// Launch one window kernel over `heads` CTAs. Returns cudaErrorNotSupported for a configuration
// that is not instantiated (the C ABI rejects those earlier).
cudaError_t launch_window_int8(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                               cudaStream_t stream);
cudaError_t launch_window_int4(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                               cudaStream_t stream);
cudaError_t launch_window_mixed(WinOp op, const gdn_config& cfg, const WinArgs& a, int heads,
                                cudaStream_t stream);
// The same with residual smoothing (cfg.smooth != GDN_SMOOTH_NONE).
cudaError_t launch_window_int8_smooth(WinOp op, const gdn_config& cfg, const WinArgs& a,
                                      int heads, cudaStream_t stream);
cudaError_t launch_window_int4_smooth(WinOp op, const gdn_config& cfg, const WinArgs& a,
                                      int heads, cudaStream_t stream);
// Pure-write sliding window: the persistent decode step, or the materialisation (one CTA per
// head), over `heads` heads.
enum class PwOp { Step, Materialize };
cudaError_t launch_pw(PwOp op, const gdn_pw_config& cfg, const PwArgs& a, int heads,
                      cudaStream_t stream);
// Chunkwise prefill: one CTA per head; diag selects the per-key-channel gate (g [heads][L][128]).
cudaError_t launch_prefill(const PfArgs& a, int heads, bool diag, cudaStream_t stream);
size_t prefill_smem_bytes(bool diag);
size_t prefill_workspace_bytes(bool diag, int64_t heads, int L);
cudaError_t launch_baseline(const gdn_config& cfg, const BaseArgs& a, int heads,
                            cudaStream_t stream);

}  // namespace gdnq
