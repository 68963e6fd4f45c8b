// C ABI of libgdnq: argument checks, buffer sizes, dispatch to the kernels, and the pipelined
// host-buffer decode loop. See include/gdnq.h for the contract of every entry point.
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "baseline_kernels.cuh"
#include "gdnq.h"
#include "gdnq_prefill.h"
#include "gdnq_pw.h"
#include "launch.h"
#include "prefill_args.h"
#include "pw_kernels.cuh"
#include "window_kernels.cuh"

// Staging of gdn_decode_window_steps_host_fixed: one fixed array per device, reserved when the
// module loads (no allocation at call time).
static __device__ __align__(256) uint8_t g_fixed_staging[GDN_FIXED_STAGING_BYTES];

namespace {

thread_local char g_last_error[512] = "";

gdn_status fail(gdn_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return st;
}

gdn_status cuda_fail(cudaError_t e, const char* where) {
  return fail(GDN_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}


gdn_status need_ptr(const void* p, const char* name, unsigned align = 16) {
  if (!p) return fail(GDN_ERR_INVALID_ARG, "%s is null", name);
  if ((reinterpret_cast<uintptr_t>(p) & (align - 1)) != 0)
    return fail(GDN_ERR_INVALID_ARG, "%s is not %u-byte aligned", name, align);
  return GDN_OK;
}

int64_t heads_of(const gdn_config* c) { return (int64_t)c->B * (int64_t)c->H; }
size_t act_size(const gdn_config* c) { return c->act_dtype == GDN_DTYPE_F32 ? 4 : 2; }
size_t buf_size(const gdn_config* c) { return c->buf_dtype == GDN_DTYPE_F32 ? 4 : 2; }
int round4(int x) { return (x + 3) & ~3; }

enum class Use { Window, Baseline };

// Checks every field of cfg for `use`; host-only.
gdn_status check_config(const gdn_config* c, Use use) {
  if (!c) return fail(GDN_ERR_INVALID_ARG, "cfg is null");
  if (c->B < 0 || c->H < 0) return fail(GDN_ERR_INVALID_ARG, "B=%d, H=%d must be >= 0", c->B, c->H);
  if (heads_of(c) > INT32_MAX) return fail(GDN_ERR_INVALID_ARG, "B*H exceeds 2^31-1");
  if (c->gate != GDN_GATE_SCALAR && c->gate != GDN_GATE_DIAG)
    return fail(GDN_ERR_INVALID_ARG, "gate=%d is not a gdn_gate_kind", c->gate);
  if (c->fmt < GDN_FMT_INT8 || c->fmt > GDN_FMT_MIXED)
    return fail(GDN_ERR_INVALID_ARG, "fmt=%d is not a gdn_state_format", c->fmt);
  if (c->act_dtype != GDN_DTYPE_F32 && c->act_dtype != GDN_DTYPE_BF16)
    return fail(GDN_ERR_INVALID_ARG, "act_dtype=%d is not a gdn_dtype", c->act_dtype);
  if (c->d_k < 1 || c->d_v < 1) return fail(GDN_ERR_INVALID_ARG, "d_k=%d, d_v=%d", c->d_k, c->d_v);
  if (c->d_k != c->d_v) return fail(GDN_ERR_UNSUPPORTED, "d_k != d_v is not built");
  if (c->d_k != 16 && c->d_k != 128)
    return fail(GDN_ERR_UNSUPPORTED, "head size %d is not built (16, 128)", c->d_k);
  if (use == Use::Baseline) {
    if (c->fmt != GDN_FMT_FP32 && c->fmt != GDN_FMT_BF16)
      return fail(GDN_ERR_INVALID_ARG, "baseline step needs fmt FP32 or BF16");
    return GDN_OK;
  }
  if (c->fmt != GDN_FMT_INT8 && c->fmt != GDN_FMT_INT4_G32 && c->fmt != GDN_FMT_MIXED)
    return fail(GDN_ERR_INVALID_ARG, "windowed state needs fmt INT8, INT4_G32 or MIXED");
  if (c->buf_dtype != GDN_DTYPE_F32 && c->buf_dtype != GDN_DTYPE_BF16)
    return fail(GDN_ERR_INVALID_ARG, "buf_dtype=%d is not a gdn_dtype", c->buf_dtype);
  if (c->W < 1) return fail(GDN_ERR_INVALID_ARG, "W=%d must be >= 1", c->W);
  if (c->r < 0 || c->r > c->d_k)
    return fail(GDN_ERR_INVALID_ARG, "r=%d must lie in [0, d_k]", c->r);
  if (c->r > GDN_MAX_COMPENSATORS)
    return fail(GDN_ERR_UNSUPPORTED, "r=%d exceeds %d", c->r, GDN_MAX_COMPENSATORS);
  if (c->smooth != GDN_SMOOTH_NONE && c->smooth != GDN_SMOOTH_POW2_COLUMNS)
    return fail(GDN_ERR_INVALID_ARG, "smooth=%d is not a gdn_smoothing", c->smooth);
  if (c->smooth != GDN_SMOOTH_NONE && c->fmt == GDN_FMT_MIXED)
    return fail(GDN_ERR_UNSUPPORTED, "residual smoothing is built for INT8 and INT4_G32 states");
  if (c->fmt == GDN_FMT_INT4_G32 && c->d_k % 32 != 0)
    return fail(GDN_ERR_UNSUPPORTED, "int4 with group 32 needs d_k %% 32 == 0");
  if ((c->fmt == GDN_FMT_INT4_G32 || c->fmt == GDN_FMT_MIXED) && c->d_k != 128)
    return fail(GDN_ERR_UNSUPPORTED, "int4 and mixed states are built for d_k = 128");
  if (c->W > (1 << 20)) return fail(GDN_ERR_UNSUPPORTED, "W=%d is too large", c->W);
  if (c->comp_rule != GDN_COMP_COLUMNS && c->comp_rule != GDN_COMP_POWER)
    return fail(GDN_ERR_INVALID_ARG, "comp_rule=%d is not a gdn_comp_rule", c->comp_rule);
  if (c->comp_rule == GDN_COMP_POWER &&
      (c->d_k != 128 || c->act_dtype != GDN_DTYPE_BF16 || c->buf_dtype != GDN_DTYPE_BF16 ||
       c->fmt == GDN_FMT_MIXED || c->smooth != GDN_SMOOTH_NONE || c->W > 64))
    return fail(GDN_ERR_UNSUPPORTED,
                "power compensator tokens are built for d = 128, bf16 activations and buffers, "
                "INT8 / INT4_G32 states without smoothing and W <= 64");
  const size_t smem = gdnq::window_smem_bytes(*c);
  if (smem > (size_t)gdnq::kMaxSmemPerCta)
    return fail(GDN_ERR_UNSUPPORTED, "W=%d, r=%d need %zu bytes of shared memory per CTA (max %d)",
                c->W, c->r, smem, gdnq::kMaxSmemPerCta);
  return GDN_OK;
}

struct PerHead {
  size_t codes, scales, buf_k, buf_u, buf_L, comp_idx, comp_u, comp_k;
};

bool power_rule(const gdn_config* c) { return c->comp_rule == GDN_COMP_POWER && c->r > 0; }

PerHead per_head_bytes(const gdn_config* c) {
  const size_t D = (size_t)c->d_k;
  const bool int4 = c->fmt == GDN_FMT_INT4_G32, mixed = c->fmt == GDN_FMT_MIXED;
  PerHead p;  // a mixed state gives every head the larger slot of each buffer
  p.codes = int4 ? D * D / 2 : D * D;
  p.scales = 4 * (int4 || mixed ? D * (D / 32) : D);
  p.buf_k = (size_t)c->W * D * act_size(c);
  p.buf_u = (size_t)c->W * D * buf_size(c);
  p.buf_L = 4 * (c->gate == GDN_GATE_DIAG ? (size_t)c->W * D : (size_t)round4(c->W));
  p.comp_idx = 4 * (size_t)round4(c->r);
  p.comp_u = 4 * (size_t)c->r * D;
  p.comp_k = power_rule(c) ? 4 * (size_t)c->r * D : 0;
  return p;
}

gdn_status check_state(const gdn_config* c, const gdn_state* s) {
  if (!s) return fail(GDN_ERR_INVALID_ARG, "state is null");
  gdn_status st;
  if ((st = need_ptr(s->codes, "state.codes")) != GDN_OK) return st;
  if ((st = need_ptr(s->scales, "state.scales")) != GDN_OK) return st;
  if ((st = need_ptr(s->buf_k, "state.buf_k")) != GDN_OK) return st;
  if ((st = need_ptr(s->buf_u, "state.buf_u")) != GDN_OK) return st;
  if ((st = need_ptr(s->buf_L, "state.buf_L")) != GDN_OK) return st;
  if ((st = need_ptr(s->pos, "state.pos")) != GDN_OK) return st;
  if (c->r > 0) {
    if ((st = need_ptr(s->comp_idx, "state.comp_idx")) != GDN_OK) return st;
    if ((st = need_ptr(s->comp_u, "state.comp_u")) != GDN_OK) return st;
  }
  if (power_rule(c) && (st = need_ptr(s->comp_k, "state.comp_k")) != GDN_OK) return st;
  if (s->status && (reinterpret_cast<uintptr_t>(s->status) & 3u) != 0)
    return fail(GDN_ERR_INVALID_ARG, "state.status is not 4-byte aligned");
  if (c->fmt == GDN_FMT_MIXED && !s->head_fmt)
    return fail(GDN_ERR_INVALID_ARG, "state.head_fmt is null for a mixed-format state");
  if (c->smooth != GDN_SMOOTH_NONE && (st = need_ptr(s->smooth_exp, "state.smooth_exp")) != GDN_OK)
    return st;
  return GDN_OK;
}

// Per-step inputs. The baseline step reads them element by element (element alignment is
// enough); the window step copies q, k, v and a per-channel g with bulk async copies, which
// need 16-byte aligned sources.
gdn_status check_inputs(const gdn_config* c, const void* q, const void* k, const void* v,
                        const float* g, const float* beta, const void* o, bool bulk) {
  const unsigned ea = (unsigned)act_size(c);
  const unsigned qa = bulk ? 16u : ea;
  const unsigned ga = bulk && c->gate == GDN_GATE_DIAG ? 16u : 4u;
  gdn_status st;
  if ((st = need_ptr(q, "q", qa)) != GDN_OK) return st;
  if ((st = need_ptr(k, "k", qa)) != GDN_OK) return st;
  if ((st = need_ptr(v, "v", qa)) != GDN_OK) return st;
  if ((st = need_ptr(g, "g", ga)) != GDN_OK) return st;
  if ((st = need_ptr(beta, "beta", 4)) != GDN_OK) return st;
  if ((st = need_ptr(o, "o", ea)) != GDN_OK) return st;
  return GDN_OK;
}

gdnq::WinArgs make_args(const gdn_config* c, const gdn_state* s) {
  gdnq::WinArgs a;
  std::memset(&a, 0, sizeof a);
  a.codes = static_cast<uint8_t*>(s->codes);
  a.scales = s->scales;
  a.buf_k = s->buf_k;
  a.buf_u = s->buf_u;
  a.buf_L = s->buf_L;
  a.comp_idx = s->comp_idx;
  a.comp_u = s->comp_u;
  a.pos = s->pos;
  a.status = s->status;
  const PerHead ph = per_head_bytes(c);
  a.code_stride = (uint32_t)ph.codes;
  a.scale_stride = (uint32_t)(ph.scales / 4);
  a.head_fmt = c->fmt == GDN_FMT_MIXED ? s->head_fmt : nullptr;
  a.smooth_exp = c->smooth != GDN_SMOOTH_NONE ? s->smooth_exp : nullptr;
  a.comp_k = power_rule(c) ? s->comp_k : nullptr;
  a.H = c->H;
  a.W = c->W;
  a.r = c->r;
  return a;
}

gdn_status launch(gdnq::WinOp op, const gdn_config* c, const gdnq::WinArgs& a,
                  gdn_stream_t stream, const char* where) {
  const int heads = (int)heads_of(c);
  const bool sm = c->smooth != GDN_SMOOTH_NONE;
  const cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = c->fmt == GDN_FMT_INT4_G32
                      ? (sm ? gdnq::launch_window_int4_smooth(op, *c, a, heads, st)
                            : gdnq::launch_window_int4(op, *c, a, heads, st))
                  : c->fmt == GDN_FMT_MIXED
                      ? gdnq::launch_window_mixed(op, *c, a, heads, st)
                      : (sm ? gdnq::launch_window_int8_smooth(op, *c, a, heads, st)
                            : gdnq::launch_window_int8(op, *c, a, heads, st));
  if (e != cudaSuccess) return cuda_fail(e, where);
  return GDN_OK;
}

// Byte offsets of one staging slot of the host-buffer loop (each region 256-byte aligned).
struct Slot {
  size_t q, k, v, g, beta, o, bytes;
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

Slot slot_layout(const gdn_config* c) {
  const size_t H = (size_t)heads_of(c), D = (size_t)c->d_k;
  const size_t act = H * D * act_size(c);
  const size_t gb = 4 * H * (c->gate == GDN_GATE_DIAG ? D : 1);
  Slot s;
  s.q = 0;
  s.k = up256(s.q + act);
  s.v = up256(s.k + act);
  s.g = up256(s.v + act);
  s.beta = up256(s.g + gb);
  s.o = up256(s.beta + 4 * H);
  s.bytes = up256(s.o + act);
  return s;
}

}  // namespace

namespace gdnq {

size_t window_smem_bytes(const gdn_config& c) {
  const int D = c.d_k;
  const bool int4 = c.fmt == GDN_FMT_INT4_G32, mixed = c.fmt == GDN_FMT_MIXED;
  const int code_bytes = int4 ? D * D / 2 : D * D;
  const int nscales = int4 || mixed ? D * (D / 32) : D;
  return win_layout(D, code_bytes, nscales, (int)act_size(&c), (int)buf_size(&c),
                    c.gate == GDN_GATE_DIAG, c.W, c.r, 1, kMaxHeadsPerCta, -1, true,
                    c.smooth != GDN_SMOOTH_NONE, c.comp_rule == GDN_COMP_POWER)
      .total;
}

}  // namespace gdnq


// ---- pure-write sliding window ----------------------------------------------------------------
namespace {

int64_t pw_heads(const gdn_pw_config* c) { return (int64_t)c->B * (int64_t)c->H; }
size_t pw_act_size(const gdn_pw_config* c) { return c->act_dtype == GDN_DTYPE_F32 ? 4 : 2; }

gdn_status check_pw_config(const gdn_pw_config* c) {
  if (!c) return fail(GDN_ERR_INVALID_ARG, "cfg is null");
  if (c->B < 0 || c->H < 0) return fail(GDN_ERR_INVALID_ARG, "B=%d, H=%d must be >= 0", c->B, c->H);
  if (pw_heads(c) > INT32_MAX) return fail(GDN_ERR_INVALID_ARG, "B*H exceeds 2^31-1");
  if (c->gate != GDN_GATE_SCALAR && c->gate != GDN_GATE_DIAG)
    return fail(GDN_ERR_INVALID_ARG, "gate=%d is not a gdn_gate_kind", c->gate);
  if (c->fmt != GDN_FMT_INT8 && c->fmt != GDN_FMT_INT4_G32)
    return fail(GDN_ERR_INVALID_ARG, "the history needs fmt INT8 or INT4_G32 (got %d)", c->fmt);
  if (c->act_dtype != GDN_DTYPE_F32 && c->act_dtype != GDN_DTYPE_BF16)
    return fail(GDN_ERR_INVALID_ARG, "act_dtype=%d is not a gdn_dtype", c->act_dtype);
  if (c->d < 1) return fail(GDN_ERR_INVALID_ARG, "d=%d", c->d);
  if (c->d != 128) return fail(GDN_ERR_UNSUPPORTED, "head size %d is not built (128)", c->d);
  if (c->Wp < 0) return fail(GDN_ERR_INVALID_ARG, "Wp=%d must be >= 0", c->Wp);
  if (c->Wp > GDN_PW_MAX_WINDOW)
    return fail(GDN_ERR_UNSUPPORTED, "Wp=%d exceeds %d", c->Wp, GDN_PW_MAX_WINDOW);
  return GDN_OK;
}

struct PwPerHead {
  size_t codes, scales, pairs, pscales;
};

PwPerHead pw_per_head(const gdn_pw_config* c) {
  const size_t D = (size_t)c->d;
  const bool int4 = c->fmt == GDN_FMT_INT4_G32;
  PwPerHead p;
  p.codes = int4 ? D * D / 2 : D * D;
  p.scales = 4 * (int4 ? D * (D / 32) : D);
  p.pairs = 2 * (size_t)c->Wp * D;
  p.pscales = 8 * (size_t)round4(c->Wp);
  return p;
}

gdn_status check_pw_state(const gdn_pw_config* c, const gdn_pw_state* s) {
  if (!s) return fail(GDN_ERR_INVALID_ARG, "state is null");
  gdn_status st;
  if ((st = need_ptr(s->codes, "state.codes")) != GDN_OK) return st;
  if ((st = need_ptr(s->scales, "state.scales")) != GDN_OK) return st;
  if ((st = need_ptr(s->count, "state.count", 4)) != GDN_OK) return st;
  if (c->Wp > 0) {
    if ((st = need_ptr(s->pairs, "state.pairs")) != GDN_OK) return st;
    if ((st = need_ptr(s->pscales, "state.pscales")) != GDN_OK) return st;
  }
  if (s->status && (reinterpret_cast<uintptr_t>(s->status) & 3u) != 0)
    return fail(GDN_ERR_INVALID_ARG, "state.status is not 4-byte aligned");
  return GDN_OK;
}

gdnq::PwArgs make_pw_args(const gdn_pw_config* c, const gdn_pw_state* s) {
  gdnq::PwArgs a;
  std::memset(&a, 0, sizeof a);
  a.codes = static_cast<uint8_t*>(s->codes);
  a.scales = s->scales;
  a.pairs = s->pairs;
  a.pscales = s->pscales;
  a.count = s->count;
  a.status = s->status;
  a.Wp = c->Wp;
  return a;
}

// The window configuration whose quantize kernel writes the same history layout.
gdn_config pw_as_window(const gdn_pw_config* c) {
  gdn_config w;
  std::memset(&w, 0, sizeof w);
  w.B = c->B;
  w.H = c->H;
  w.d_k = w.d_v = c->d;
  w.W = 1;
  w.r = 0;
  w.gate = c->gate;
  w.fmt = c->fmt;
  w.act_dtype = w.buf_dtype = c->act_dtype;
  return w;
}

}  // namespace

extern "C" {

const char* gdn_status_string(gdn_status st) {
  switch (st) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
  }
  return "GDN_UNKNOWN_STATUS";
}

const char* gdn_last_error(void) { return g_last_error; }

gdn_status gdn_state_sizes(const gdn_config* cfg, gdn_sizes* out) {
  g_last_error[0] = 0;
  if (!out) return fail(GDN_ERR_INVALID_ARG, "out is null");
  gdn_status st = check_config(cfg, Use::Window);
  if (st != GDN_OK) return st;
  const PerHead p = per_head_bytes(cfg);
  const size_t n = (size_t)heads_of(cfg);
  out->codes = n * p.codes;
  out->scales = n * p.scales;
  out->buf_k = n * p.buf_k;
  out->buf_u = n * p.buf_u;
  out->buf_L = n * p.buf_L;
  out->comp_idx = cfg->r > 0 ? n * p.comp_idx : 0;
  out->comp_u = cfg->r > 0 ? n * p.comp_u : 0;
  out->pos = n * 4;
  out->smem_step = gdnq::window_smem_bytes(*cfg);
  out->head_fmt = cfg->fmt == GDN_FMT_MIXED ? n : 0;
  out->smooth_exp = cfg->smooth != GDN_SMOOTH_NONE ? n * (size_t)cfg->d_k : 0;
  out->comp_k = n * p.comp_k;
  return GDN_OK;
}

gdn_status gdn_state_quantize(const gdn_config* cfg, const float* S, const gdn_state* state,
                              gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_config(cfg, Use::Window);
  if (st != GDN_OK) return st;
  if (heads_of(cfg) == 0) return GDN_OK;
  if ((st = check_state(cfg, state)) != GDN_OK) return st;
  if ((st = need_ptr(S, "S")) != GDN_OK) return st;
  gdnq::WinArgs a = make_args(cfg, state);
  a.S_in = S;
  return launch(gdnq::WinOp::Quantize, cfg, a, stream, "gdn_state_quantize");
}

gdn_status gdn_decode_window_step(const gdn_config* cfg, const gdn_state* state, const void* q,
                                  const void* k, const void* v, const float* g,
                                  const float* beta, void* o, gdn_stream_t stream) {
  return gdn_decode_window_steps(cfg, state, 1, q, k, v, g, beta, o, stream);
}

gdn_status gdn_decode_window_steps(const gdn_config* cfg, const gdn_state* state, int32_t T,
                                   const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, void* o, gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_config(cfg, Use::Window);
  if (st != GDN_OK) return st;
  if (T < 0) return fail(GDN_ERR_INVALID_ARG, "T=%d must be >= 0", T);
  if (heads_of(cfg) == 0 || T == 0) return GDN_OK;
  if ((st = check_state(cfg, state)) != GDN_OK) return st;
  if ((st = check_inputs(cfg, q, k, v, g, beta, o, true)) != GDN_OK) return st;
  const size_t H = (size_t)heads_of(cfg), D = (size_t)cfg->d_k;
  const size_t act_step = H * D * act_size(cfg);
  const size_t g_step = H * (cfg->gate == GDN_GATE_DIAG ? D : 1);
  gdnq::WinArgs a = make_args(cfg, state);
  for (int32_t t = 0; t < T; ++t) {
    a.q = static_cast<const uint8_t*>(q) + t * act_step;
    a.k = static_cast<const uint8_t*>(k) + t * act_step;
    a.v = static_cast<const uint8_t*>(v) + t * act_step;
    a.g = g + t * g_step;
    a.beta = beta + t * H;
    a.o = static_cast<uint8_t*>(o) + t * act_step;
    if ((st = launch(gdnq::WinOp::Step, cfg, a, stream, "gdn_decode_window_step")) != GDN_OK)
      return st;
  }
  return GDN_OK;
}

size_t gdn_host_staging_bytes(const gdn_config* cfg) {
  if (check_config(cfg, Use::Window) != GDN_OK) return 0;
  return 2 * slot_layout(cfg).bytes;
}

gdn_status gdn_decode_window_steps_host(const gdn_config* cfg, const gdn_state* state, int32_t T,
                                        const void* host_q, const void* host_k,
                                        const void* host_v, const float* host_g,
                                        const float* host_beta, void* host_o, void* staging,
                                        size_t staging_bytes, gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_config(cfg, Use::Window);
  if (st != GDN_OK) return st;
  if (T < 0) return fail(GDN_ERR_INVALID_ARG, "T=%d must be >= 0", T);
  if (heads_of(cfg) == 0 || T == 0) return GDN_OK;
  if ((st = check_state(cfg, state)) != GDN_OK) return st;
  if (!host_q || !host_k || !host_v || !host_g || !host_beta || !host_o)
    return fail(GDN_ERR_INVALID_ARG, "a host input / output pointer is null");
  if ((st = need_ptr(staging, "staging")) != GDN_OK) return st;
  const Slot sl = slot_layout(cfg);
  if (staging_bytes < 2 * sl.bytes)
    return fail(GDN_ERR_INVALID_ARG, "staging holds %zu bytes, needs %zu", staging_bytes,
                2 * sl.bytes);
  const size_t H = (size_t)heads_of(cfg), D = (size_t)cfg->d_k;
  const size_t act_step = H * D * act_size(cfg);
  const size_t g_step = 4 * H * (cfg->gate == GDN_GATE_DIAG ? D : 1);
  const cudaStream_t cs = (cudaStream_t)stream;

  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev[7] = {};  // start, in[2], comp[2], out[2]
  cudaError_t e = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking);
  for (int i = 0; i < 7 && e == cudaSuccess; ++i)
    e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
  cudaEvent_t ev_start = ev[0], *ev_in = ev + 1, *ev_comp = ev + 3, *ev_out = ev + 5;
  if (e == cudaSuccess) e = cudaEventRecord(ev_start, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h2d, ev_start, 0);
  gdnq::WinArgs a = make_args(cfg, state);
  for (int32_t t = 0; t < T && e == cudaSuccess; ++t) {
    const int s = t & 1;
    uint8_t* base = static_cast<uint8_t*>(staging) + s * sl.bytes;
    if (t >= 2) e = cudaStreamWaitEvent(h2d, ev_comp[s], 0);  // slot's inputs consumed
    const uint8_t* hq = static_cast<const uint8_t*>(host_q) + t * act_step;
    const uint8_t* hk = static_cast<const uint8_t*>(host_k) + t * act_step;
    const uint8_t* hv = static_cast<const uint8_t*>(host_v) + t * act_step;
    const uint8_t* hg = reinterpret_cast<const uint8_t*>(host_g) + t * g_step;
    const uint8_t* hb = reinterpret_cast<const uint8_t*>(host_beta) + t * 4 * H;
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.q, hq, act_step, cudaMemcpyHostToDevice, h2d);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.k, hk, act_step, cudaMemcpyHostToDevice, h2d);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.v, hv, act_step, cudaMemcpyHostToDevice, h2d);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.g, hg, g_step, cudaMemcpyHostToDevice, h2d);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.beta, hb, 4 * H, cudaMemcpyHostToDevice, h2d);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[s], h2d);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_in[s], 0);
    if (e == cudaSuccess && t >= 2) e = cudaStreamWaitEvent(cs, ev_out[s], 0);  // slot's o read
    if (e != cudaSuccess) break;
    a.q = base + sl.q;
    a.k = base + sl.k;
    a.v = base + sl.v;
    a.g = reinterpret_cast<const float*>(base + sl.g);
    a.beta = reinterpret_cast<const float*>(base + sl.beta);
    a.o = base + sl.o;
    st = launch(gdnq::WinOp::Step, cfg, a, stream, "gdn_decode_window_steps_host");
    if (st != GDN_OK) break;
    e = cudaEventRecord(ev_comp[s], cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(d2h, ev_comp[s], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<uint8_t*>(host_o) + t * act_step, base + sl.o, act_step,
                          cudaMemcpyDeviceToHost, d2h);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out[s], d2h);
  }
  // completion of `stream` implies the host outputs are written
  for (int s = 0; s < 2 && e == cudaSuccess && st == GDN_OK && s < T; ++s)
    e = cudaStreamWaitEvent(cs, ev_out[(T - 1 - s) & 1], 0);
  for (int i = 0; i < 7; ++i)
    if (ev[i]) cudaEventDestroy(ev[i]);
  if (h2d) cudaStreamDestroy(h2d);
  if (d2h) cudaStreamDestroy(d2h);
  if (st != GDN_OK) return st;
  if (e != cudaSuccess) return cuda_fail(e, "gdn_decode_window_steps_host");
  return GDN_OK;
}

gdn_status gdn_decode_window_steps_host_fixed(const gdn_config* cfg, const gdn_state* state,
                                              int32_t T, const void* host_q, const void* host_k,
                                              const void* host_v, const float* host_g,
                                              const float* host_beta, void* host_o,
                                              gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_config(cfg, Use::Window);
  if (st != GDN_OK) return st;
  if (T < 0) return fail(GDN_ERR_INVALID_ARG, "T=%d must be >= 0", T);
  if (heads_of(cfg) == 0 || T == 0) return GDN_OK;
  if ((st = check_state(cfg, state)) != GDN_OK) return st;
  if (!host_q || !host_k || !host_v || !host_g || !host_beta || !host_o)
    return fail(GDN_ERR_INVALID_ARG, "a host input / output pointer is null");
  const Slot sl = slot_layout(cfg);
  if (sl.bytes > GDN_FIXED_STAGING_BYTES)
    return fail(GDN_ERR_UNSUPPORTED,
                "gdn_decode_window_steps_host_fixed: one staging slot needs %zu bytes for %lld "
                "heads, the fixed staging array holds %zu; use gdn_decode_window_steps_host",
                sl.bytes, (long long)heads_of(cfg), (size_t)GDN_FIXED_STAGING_BYTES);
  // The array's device address in the current device's context, looked up on every call (a
  // host-side use of the symbol itself is not a device address). Not cached: after a
  // cudaDeviceReset the context and the module are created anew and the array may move.
  void* base_v = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&base_v, g_fixed_staging);
  if (e != cudaSuccess)
    return cuda_fail(e, "gdn_decode_window_steps_host_fixed: cudaGetSymbolAddress");
  uint8_t* base = static_cast<uint8_t*>(base_v);
  const size_t H = (size_t)heads_of(cfg), D = (size_t)cfg->d_k;
  const size_t act_step = H * D * act_size(cfg);
  const size_t g_step = 4 * H * (cfg->gate == GDN_GATE_DIAG ? D : 1);
  const cudaStream_t cs = (cudaStream_t)stream;
  gdnq::WinArgs a = make_args(cfg, state);
  a.q = base + sl.q;
  a.k = base + sl.k;
  a.v = base + sl.v;
  a.g = reinterpret_cast<const float*>(base + sl.g);
  a.beta = reinterpret_cast<const float*>(base + sl.beta);
  a.o = base + sl.o;
  // one slot: on a single stream the copies of step t + 1 follow the step-t kernel and its copy
  // of o, so nothing is overwritten early
  for (int32_t t = 0; t < T; ++t) {
    const uint8_t* hq = static_cast<const uint8_t*>(host_q) + t * act_step;
    const uint8_t* hk = static_cast<const uint8_t*>(host_k) + t * act_step;
    const uint8_t* hv = static_cast<const uint8_t*>(host_v) + t * act_step;
    const uint8_t* hg = reinterpret_cast<const uint8_t*>(host_g) + t * g_step;
    const uint8_t* hb = reinterpret_cast<const uint8_t*>(host_beta) + t * 4 * H;
    e = cudaMemcpyAsync(base + sl.q, hq, act_step, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.k, hk, act_step, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.v, hv, act_step, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.g, hg, g_step, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + sl.beta, hb, 4 * H, cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_decode_window_steps_host_fixed: copy in");
    st = launch(gdnq::WinOp::Step, cfg, a, stream, "gdn_decode_window_steps_host_fixed");
    if (st != GDN_OK) return st;
    e = cudaMemcpyAsync(static_cast<uint8_t*>(host_o) + t * act_step, base + sl.o, act_step,
                        cudaMemcpyDeviceToHost, cs);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_decode_window_steps_host_fixed: copy out");
  }
  return GDN_OK;
}

gdn_status gdn_window_flush(const gdn_config* cfg, const gdn_state* state,
                            const int32_t* seq_mask, gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_config(cfg, Use::Window);
  if (st != GDN_OK) return st;
  if (heads_of(cfg) == 0) return GDN_OK;
  if ((st = check_state(cfg, state)) != GDN_OK) return st;
  if (seq_mask && (reinterpret_cast<uintptr_t>(seq_mask) & 3u) != 0)
    return fail(GDN_ERR_INVALID_ARG, "seq_mask is not 4-byte aligned");
  gdnq::WinArgs a = make_args(cfg, state);
  a.seq_mask = seq_mask;
  return launch(gdnq::WinOp::Flush, cfg, a, stream, "gdn_window_flush");
}

gdn_status gdn_state_materialize(const gdn_config* cfg, const gdn_state* state, float* S,
                                 gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_config(cfg, Use::Window);
  if (st != GDN_OK) return st;
  if (heads_of(cfg) == 0) return GDN_OK;
  if ((st = check_state(cfg, state)) != GDN_OK) return st;
  if ((st = need_ptr(S, "S")) != GDN_OK) return st;
  gdnq::WinArgs a = make_args(cfg, state);
  a.S_out = S;
  return launch(gdnq::WinOp::Materialize, cfg, a, stream, "gdn_state_materialize");
}

gdn_status gdn_baseline_step(const gdn_config* cfg, void* S, const void* q, const void* k,
                             const void* v, const float* g, const float* beta, void* o,
                             gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_config(cfg, Use::Baseline);
  if (st != GDN_OK) return st;
  if (heads_of(cfg) == 0) return GDN_OK;
  if ((st = need_ptr(S, "S")) != GDN_OK) return st;
  if ((st = check_inputs(cfg, q, k, v, g, beta, o, false)) != GDN_OK) return st;
  gdnq::BaseArgs a{S, q, k, v, g, beta, o};
  cudaError_t e = gdnq::launch_baseline(*cfg, a, (int)heads_of(cfg), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "gdn_baseline_step");
  return GDN_OK;
}

gdn_status gdn_pw_state_sizes(const gdn_pw_config* cfg, gdn_pw_sizes* out) {
  g_last_error[0] = 0;
  if (!out) return fail(GDN_ERR_INVALID_ARG, "out is null");
  gdn_status st = check_pw_config(cfg);
  if (st != GDN_OK) return st;
  const PwPerHead p = pw_per_head(cfg);
  const size_t n = (size_t)pw_heads(cfg);
  out->codes = n * p.codes;
  out->scales = n * p.scales;
  out->pairs = n * p.pairs;
  out->pscales = cfg->Wp > 0 ? n * p.pscales : 0;
  out->count = n * 4;
  return GDN_OK;
}

gdn_status gdn_pw_quantize(const gdn_pw_config* cfg, const float* S, const gdn_pw_state* state,
                           gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_pw_config(cfg);
  if (st != GDN_OK) return st;
  if (pw_heads(cfg) == 0) return GDN_OK;
  if ((st = check_pw_state(cfg, state)) != GDN_OK) return st;
  if ((st = need_ptr(S, "S")) != GDN_OK) return st;
  const gdn_config w = pw_as_window(cfg);
  gdnq::WinArgs a;
  std::memset(&a, 0, sizeof a);
  a.codes = static_cast<uint8_t*>(state->codes);
  a.scales = state->scales;
  a.pos = state->count;  // the quantize kernel empties the window: count = 0
  a.status = state->status;
  a.S_in = S;
  const PwPerHead ph = pw_per_head(cfg);
  a.code_stride = (uint32_t)ph.codes;
  a.scale_stride = (uint32_t)(ph.scales / 4);
  a.H = cfg->H;
  a.W = 1;
  a.r = 0;
  return launch(gdnq::WinOp::Quantize, &w, a, stream, "gdn_pw_quantize");
}

gdn_status gdn_pw_decode_step(const gdn_pw_config* cfg, const gdn_pw_state* state, const void* q,
                              const void* k, const void* v, const float* g, const float* beta,
                              void* o, gdn_stream_t stream) {
  return gdn_pw_decode_steps(cfg, state, 1, q, k, v, g, beta, o, stream);
}

gdn_status gdn_pw_decode_steps(const gdn_pw_config* cfg, const gdn_pw_state* state, int32_t T,
                               const void* q, const void* k, const void* v, const float* g,
                               const float* beta, void* o, gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_pw_config(cfg);
  if (st != GDN_OK) return st;
  if (T < 0) return fail(GDN_ERR_INVALID_ARG, "T=%d must be >= 0", T);
  if (pw_heads(cfg) == 0 || T == 0) return GDN_OK;
  if ((st = check_pw_state(cfg, state)) != GDN_OK) return st;
  const gdn_config w = pw_as_window(cfg);
  if ((st = check_inputs(&w, q, k, v, g, beta, o, true)) != GDN_OK) return st;
  const size_t H = (size_t)pw_heads(cfg), D = (size_t)cfg->d;
  const size_t act_step = H * D * pw_act_size(cfg);
  const size_t g_step = H * (cfg->gate == GDN_GATE_DIAG ? D : 1);
  gdnq::PwArgs a = make_pw_args(cfg, state);
  for (int32_t t = 0; t < T; ++t) {
    a.q = static_cast<const uint8_t*>(q) + t * act_step;
    a.k = static_cast<const uint8_t*>(k) + t * act_step;
    a.v = static_cast<const uint8_t*>(v) + t * act_step;
    a.g = g + t * g_step;
    a.beta = beta + t * H;
    a.o = static_cast<uint8_t*>(o) + t * act_step;
    const cudaError_t e =
        gdnq::launch_pw(gdnq::PwOp::Step, *cfg, a, (int)H, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_pw_decode_step");
  }
  return GDN_OK;
}

gdn_status gdn_pw_materialize(const gdn_pw_config* cfg, const gdn_pw_state* state, float* S,
                              gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st = check_pw_config(cfg);
  if (st != GDN_OK) return st;
  if (pw_heads(cfg) == 0) return GDN_OK;
  if ((st = check_pw_state(cfg, state)) != GDN_OK) return st;
  if ((st = need_ptr(S, "S")) != GDN_OK) return st;
  gdnq::PwArgs a = make_pw_args(cfg, state);
  a.S_out = S;
  const cudaError_t e = gdnq::launch_pw(gdnq::PwOp::Materialize, *cfg, a, (int)pw_heads(cfg),
                                        (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "gdn_pw_materialize");
  return GDN_OK;
}

namespace {
gdn_status check_prefill_config(const gdn_config* cfg) {
  if (!cfg) return fail(GDN_ERR_INVALID_ARG, "cfg is null");
  if (cfg->B < 0 || cfg->H < 0)
    return fail(GDN_ERR_INVALID_ARG, "B=%d, H=%d must be >= 0", cfg->B, cfg->H);
  if (heads_of(cfg) > INT32_MAX) return fail(GDN_ERR_INVALID_ARG, "B*H exceeds 2^31-1");
  if (cfg->gate != GDN_GATE_SCALAR && cfg->gate != GDN_GATE_DIAG)
    return fail(GDN_ERR_INVALID_ARG, "gate=%d is not a gdn_gate_kind", cfg->gate);
  if (cfg->act_dtype != GDN_DTYPE_F32 && cfg->act_dtype != GDN_DTYPE_BF16)
    return fail(GDN_ERR_INVALID_ARG, "act_dtype=%d is not a gdn_dtype", cfg->act_dtype);
  if (cfg->d_k < 1 || cfg->d_v < 1)
    return fail(GDN_ERR_INVALID_ARG, "d_k=%d, d_v=%d", cfg->d_k, cfg->d_v);
  if (cfg->d_k != 128 || cfg->d_v != 128)
    return fail(GDN_ERR_UNSUPPORTED, "prefill is built for d_k = d_v = 128");
  if (cfg->act_dtype != GDN_DTYPE_BF16)
    return fail(GDN_ERR_UNSUPPORTED, "prefill is built for bf16 activations");
  return GDN_OK;
}
}  // namespace

size_t gdn_prefill_workspace_bytes(const gdn_config* cfg, int32_t L) {
  g_last_error[0] = 0;
  if (check_prefill_config(cfg) != GDN_OK || L < 0) return 0;
  return gdnq::prefill_workspace_bytes(cfg->gate == GDN_GATE_DIAG, heads_of(cfg), L);
}

gdn_status gdn_prefill(const gdn_config* cfg, int32_t L, const void* q, const void* k,
                       const void* v, const float* g, const float* beta, void* o, float* S,
                       void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
  g_last_error[0] = 0;
  gdn_status st0 = check_prefill_config(cfg);
  if (st0 != GDN_OK) return st0;
  if (L < 0) return fail(GDN_ERR_INVALID_ARG, "L=%d must be >= 0", L);
  if (heads_of(cfg) == 0) return GDN_OK;
  if ((size_t)heads_of(cfg) * (size_t)L * 128 > (size_t)INT64_MAX / 4)
    return fail(GDN_ERR_INVALID_ARG, "B*H*L is too large");
  gdn_status st;
  if ((st = need_ptr(S, "S")) != GDN_OK) return st;
  if (L > 0) {
    if ((st = need_ptr(q, "q")) != GDN_OK) return st;
    if ((st = need_ptr(k, "k")) != GDN_OK) return st;
    if ((st = need_ptr(v, "v")) != GDN_OK) return st;
    if ((st = need_ptr(g, "g", cfg->gate == GDN_GATE_DIAG ? 16 : 4)) != GDN_OK) return st;
    if ((st = need_ptr(beta, "beta", 4)) != GDN_OK) return st;
    if ((st = need_ptr(o, "o", 4)) != GDN_OK) return st;
    const size_t need = gdnq::prefill_workspace_bytes(cfg->gate == GDN_GATE_DIAG, heads_of(cfg), L);
    if (need > 0) {
      if ((st = need_ptr(workspace, "workspace")) != GDN_OK) return st;
      if (workspace_bytes < need)
        return fail(GDN_ERR_INVALID_ARG, "workspace holds %zu bytes, the prompt needs %zu",
                    workspace_bytes, need);
    }
  }
  gdnq::PfArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.g = g;
  a.beta = beta;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.S = S;
  a.ws = static_cast<uint8_t*>(workspace);
  a.L = L;
  const cudaError_t e = gdnq::launch_prefill(a, (int)heads_of(cfg), cfg->gate == GDN_GATE_DIAG,
                                             (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "gdn_prefill");
  return GDN_OK;
}

}  // extern "C"
