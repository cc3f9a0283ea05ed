// C ABI of the MoE layer forward: validation, workspace carving, launch
// sequencing and host-side statistics.  Declarations and contracts are in
// include/moe.h.
#include "common.cuh"

#include <atomic>
#include <math.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

using namespace moe;

namespace {

thread_local char g_last_error[512] = "";
thread_local cudaEvent_t g_events[MOE_PHASE_COUNT] = {};
thread_local int g_nevents = 0;

cudaError_t mark(int phase, cudaStream_t s) {
  return g_nevents ? cudaEventRecord(g_events[phase], s) : cudaSuccess;
}

void set_error(const char *fmt, const char *a, const char *b = "") {
  snprintf(g_last_error, sizeof(g_last_error), fmt, a, b);
}

moe_status cuda_fail(cudaError_t err, const char *where) {
  set_error("%s: %s", where, cudaGetErrorString(err));
  return MOE_ERR_CUDA;
}

bool aligned16(const void *p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }
bool aligned16_or_null(const void *p) { return ((uintptr_t)p & 15u) == 0; }

int64_t capacity_of(const moe_config &c) {
  return moe_capacity(c.num_tokens, c.top_k, c.num_experts, c.capacity_factor);
}

bool fused_gate_up(const moe_config &c) { return c.weight_layout == MOE_LAYOUT_FUSED_GATE_UP; }

// Dense weights need both SwiGLU projections; ReLU uses w1 / w3 only.  The
// fused gate/up layout carries both in w1 and leaves the w2 slots empty.
moe_status check_weights(const moe_config &c, const moe_weights *w) {
  if (!w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w1) || !aligned16(w->w3)) return MOE_ERR_INVALID_ARG;
  const bool fused = fused_gate_up(c);
  if (fused && (w->w2 || w->scale2 || w->bias2)) return MOE_ERR_INVALID_ARG;
  if (c.act == MOE_ACT_SWIGLU && !fused && !aligned16(w->w2)) return MOE_ERR_INVALID_ARG;
  if (c.weight_dtype == MOE_Q4_AFFINE_G64) {
    if (!aligned16(w->scale1) || !aligned16(w->scale3) || !aligned16(w->bias1) || !aligned16(w->bias3))
      return MOE_ERR_INVALID_ARG;
    if (!fused && (!aligned16(w->scale2) || !aligned16(w->bias2))) return MOE_ERR_INVALID_ARG;
  }
  if (c.shared_intermediate > 0) {
    if (!aligned16(w->shared1) || !aligned16(w->shared2) || !aligned16(w->shared3)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe_status check_ws(const moe_config &c, const void *ws, size_t ws_bytes) {
  if (!aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < ws_layout(c).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status clear_status(void *ws, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(ws, 0, 256, s);
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "status clear");
}

FfnArgs ffn_args(const moe_config &c, const WsLayout &L, void *ws) {
  FfnArgs a{};
  a.kind = c.weight_dtype == MOE_F32 ? 0 : (c.weight_dtype == MOE_BF16 ? 1 : 2);
  a.act = c.act;
  a.E = c.num_experts;
  a.rows_cap = c.num_tokens * c.top_k;
  a.rows = 0;
  a.d = c.hidden;
  a.F = c.intermediate;
  a.h = ws_ptr<char>(ws, L.h);
  a.status = ws_ptr<int>(ws, L.status);
  return a;
}

// The bf16 grouped GEMM runs on one SM per tile unless MOE_TC_PAIR=1 is set
// in the environment, which selects the kernel on pairs of SMs (same
// results bit for bit; measured slower on the dense workloads, so it is not
// the default).  The fused gather always runs on one SM.
bool pair_env() {
  const char *env = getenv("MOE_TC_PAIR");
  return env && env[0] == '1';
}

bool use_pair_gemm(const FfnArgs &a) {
  if (a.gather || a.shared_rows > 0) return false;
  return pair_env();
}

// moe_forward runs the shared expert as one more group of the bf16 grouped
// GEMM (both phases) when it has the experts' width, unless the routed
// experts are to run on pairs of SMs (that kernel has no shared group).
bool shared_in_grouped_gemm(const moe_config &c) {
  return c.shared_intermediate > 0 && c.shared_intermediate == c.intermediate && c.weight_dtype == MOE_BF16 &&
         c.act_dtype == MOE_BF16 && !(pair_env() && !c.fused_gather);
}

// 4-bit weights: decode-sized groups (a few token rows per expert) go to the
// warp-level kernel, whose 8-token MMA blocks fit them; larger groups to the
// tcgen05 kernel.  MOE_Q4_KERNEL=mma / tc in the environment forces one.
bool use_q4_mma(const FfnArgs &a) {
  if (!q4_mma_supported(a.d, a.F)) return false;
  const char *env = getenv("MOE_Q4_KERNEL");
  if (env && strcmp(env, "mma") == 0) return true;
  if (env && strcmp(env, "tc") == 0) return !q4_tc_supported(a.d, a.F);
  return (long long)a.rows_cap <= 16LL * a.E;
}

cudaError_t run_q4(const FfnArgs &a, cudaStream_t s) {
  if (use_q4_mma(a)) return launch_ffn_q4_mma(a, s);
  return q4_tc_supported(a.d, a.F) ? launch_ffn_q4_tc(a, s) : launch_ffn_q4(a, s);
}

cudaError_t run_ffn(const FfnArgs &a, cudaStream_t s) {
  switch (a.kind) {
    case 0: return launch_ffn_simt_f32(a, s);
    case 1: return use_pair_gemm(a) ? launch_ffn_tc2_bf16(a, s) : launch_ffn_tc_bf16(a, s);
    default: return run_q4(a, s);
  }
}

moe_status do_route(const moe_config &c, const void *x, const float *w_router, const float *bias,
                    int32_t *ids, float *wts, float *prob_sum, void *ws, cudaStream_t s,
                    const int32_t *forced = nullptr) {
  const WsLayout L = ws_layout(c);
  cudaError_t err = launch_route(c, x, w_router, bias, ids, wts, ws_ptr<double>(ws, L.route_part), prob_sum, s,
                                 L.route_logits != L.total && route_logits_bytes(c) ? ws_ptr<double>(ws, L.route_logits)
                                                                                   : nullptr,
                                 forced, ws_ptr<int>(ws, L.status));
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, forced ? "moe_route_forced" : "moe_route");
}

moe_status do_permute(const moe_config &c, const void *x, const int32_t *ids, const float *wts, int32_t *off,
                      int32_t *perm_token, float *perm_w, int32_t *slot_row, void *x_perm, int32_t *raw,
                      int32_t *kept, int32_t *dropped, void *ws, cudaStream_t s) {
  const WsLayout L = ws_layout(c);
  cudaError_t err = launch_permute(c, x, ids, wts, capacity_of(c), off, perm_token, perm_w, slot_row, x_perm,
                                   raw, kept, dropped, ws_ptr<int32_t>(ws, L.blk_counts),
                                   ws_ptr<int32_t>(ws, L.blk_base), ws_ptr<int32_t>(ws, L.local_rank),
                                   ws_ptr<int>(ws, L.status), s);
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_permute");
}

// gather (nullable): x_perm is the token matrix itself and row r of the
// expert-sorted order is token gather[r] (bf16 tensor-core path only).
// shared_x / shared_out (nullable): the shared expert's tokens and output,
// computed as one more group of the same two launches.
moe_status do_ffn(const moe_config &c, const void *x_perm, const int32_t *off, const moe_weights *w, void *y,
                  void *ws, cudaStream_t s, cudaEvent_t mid = nullptr, const int32_t *gather = nullptr,
                  const void *shared_x = nullptr, void *shared_out = nullptr) {
  const WsLayout L = ws_layout(c);
  FfnArgs a = ffn_args(c, L, ws);
  if (shared_x) {
    a.shared_rows = c.num_tokens;
    a.shared_x = shared_x;
    a.shared_w1 = w->shared1;
    a.shared_w2 = w->shared2;
    a.shared_w3 = w->shared3;
    a.shared_h = ws_ptr<char>(ws, L.shared_h);
    a.shared_y = shared_out;
  }
  a.mid_event = mid;
  a.offsets = off;
  a.x = x_perm;
  a.gather = gather;
  a.x_rows = c.num_tokens;
  a.w1 = w->w1;
  a.w2 = w->w2;
  a.w3 = w->w3;
  a.s1 = w->scale1;
  a.s2 = w->scale2;
  a.s3 = w->scale3;
  a.b1 = w->bias1;
  a.b2 = w->bias2;
  a.b3 = w->bias3;
  a.w_stride = c.intermediate;
  if (fused_gate_up(c)) {
    // expert e's up rows follow its F gate rows: the up view starts F rows in
    // and both views step 2F rows per expert
    const size_t F = (size_t)c.intermediate, d = (size_t)c.hidden;
    a.w_stride = 2 * c.intermediate;
    if (c.weight_dtype == MOE_Q4_AFFINE_G64) {
      a.w2 = static_cast<const char *>(w->w1) + F * (d / 2);
      a.s2 = static_cast<const char *>(w->scale1) + F * (d / 64) * 2;
      a.b2 = static_cast<const char *>(w->bias1) + F * (d / 64) * 2;
    } else {
      a.w2 = static_cast<const char *>(w->w1) + F * d * (c.weight_dtype == MOE_F32 ? 4 : 2);
    }
  }
  a.y = y;
  cudaError_t err = run_ffn(a, s);
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_grouped_ffn");
}

moe_status do_shared(const moe_config &c, const void *x, const moe_weights *w, void *out, void *ws,
                     cudaStream_t s) {
  const WsLayout L = ws_layout(c);
  FfnArgs a = ffn_args(c, L, ws);
  a.kind = c.act_dtype == MOE_F32 ? 0 : 1;
  a.act = MOE_ACT_SWIGLU;
  a.E = 1;
  a.offsets = nullptr;
  a.rows = c.num_tokens;
  a.rows_cap = c.num_tokens;
  a.F = c.shared_intermediate;
  a.x = x;
  a.w1 = w->shared1;
  a.w2 = w->shared2;
  a.w3 = w->shared3;
  a.w_stride = c.shared_intermediate;
  a.h = ws_ptr<char>(ws, L.shared_h);
  a.y = out;
  cudaError_t err = run_ffn(a, s);
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_shared_expert");
}

}  // namespace

void moe::set_last_error_text(const char *text) { set_error("%s%s", text); }

static std::atomic<long long> g_launches{0};
void moe::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static constexpr uint64_t kDefaultWaitNs = 2000000000ull;
static std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
uint64_t moe::wait_timeout_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

extern "C" {

int64_t moe_capacity(int32_t num_tokens, int32_t top_k, int32_t num_experts, float capacity_factor) {
  if (num_tokens < 1 || top_k < 1 || num_experts < 1 || !(capacity_factor >= 0.0f) || isinf(capacity_factor))
    return -2;
  if (capacity_factor == 0.0f) return -1;
  const double exact = (double)num_tokens * (double)top_k / (double)num_experts * (double)capacity_factor;
  const int64_t c = (int64_t)exact;   // truncation, as int() of a positive float
  return c < 1 ? 1 : c;
}

moe_status moe_validate(const moe_config *cfg) {
  if (!cfg) return MOE_ERR_INVALID_ARG;
  const moe_config &c = *cfg;
  if (c.num_experts < 2) return MOE_ERR_INVALID_ARG;
  if (c.top_k < 1 || c.top_k > c.num_experts) return MOE_ERR_INVALID_TOPK;
  if (!(c.capacity_factor >= 0.0f) || isinf(c.capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (c.capacity_factor > 0.0f && c.capacity_factor < 1.0f) return MOE_ERR_CAPACITY_TOO_TIGHT;
  if (!(c.aux_alpha >= 0.0f)) return MOE_ERR_INVALID_ARG;
  if (c.num_tokens < 1 || c.hidden < 1 || c.intermediate < 1) return MOE_ERR_INVALID_ARG;
  if (c.act != MOE_ACT_RELU && c.act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (c.weight_layout != MOE_LAYOUT_SEPARATE && c.weight_layout != MOE_LAYOUT_FUSED_GATE_UP)
    return MOE_ERR_INVALID_ARG;
  if (c.weight_layout == MOE_LAYOUT_FUSED_GATE_UP && c.act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (c.fused_gather != 0 && c.fused_gather != 1) return MOE_ERR_INVALID_ARG;
  if (c.act_dtype != MOE_F32 && c.act_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c.weight_dtype != MOE_F32 && c.weight_dtype != MOE_BF16 && c.weight_dtype != MOE_Q4_AFFINE_G64)
    return MOE_ERR_INVALID_ARG;
  if (c.shared_intermediate < 0) return MOE_ERR_INVALID_ARG;
  if (c.router == MOE_ROUTER_SOFTMAX_TOPK) {
    if (c.routed_scaling != 1.0f) return MOE_ERR_INVALID_ARG;
  } else if (c.router == MOE_ROUTER_SIGMOID_GROUP) {
    if (!(c.routed_scaling > 0.0f) || isinf(c.routed_scaling)) return MOE_ERR_INVALID_ARG;
    if (c.n_group < 1 || c.num_experts % c.n_group != 0) return MOE_ERR_INVALID_ARG;
    if (c.num_experts / c.n_group < 2) return MOE_ERR_INVALID_ARG;
    if (c.topk_group < 1 || c.topk_group > c.n_group) return MOE_ERR_INVALID_ARG;
    if (c.top_k > c.topk_group * (c.num_experts / c.n_group)) return MOE_ERR_INVALID_TOPK;
    if (c.n_group > kMaxGroups) return MOE_ERR_UNSUPPORTED;
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  // what the kernels cover
  if (c.num_experts > kMaxExperts || c.top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)c.num_tokens * c.top_k > (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
  const bool f32 = c.act_dtype == MOE_F32 && c.weight_dtype == MOE_F32;
  const bool bf16 = c.act_dtype == MOE_BF16 && c.weight_dtype == MOE_BF16;
  const bool q4 = c.act_dtype == MOE_BF16 && c.weight_dtype == MOE_Q4_AFFINE_G64;
  if (!f32 && !bf16 && !q4) return MOE_ERR_UNSUPPORTED;
  if (c.act_dtype == MOE_BF16 && (c.hidden % 8 != 0 || c.intermediate % 8 != 0)) return MOE_ERR_UNSUPPORTED;
  if (bf16 && (int64_t)c.num_experts * (c.intermediate > c.hidden ? c.intermediate : c.hidden) > INT32_MAX / 2)
    return MOE_ERR_UNSUPPORTED;
  if (q4 && (c.hidden % 64 != 0 || c.intermediate % 64 != 0 || c.act != MOE_ACT_SWIGLU))
    return MOE_ERR_UNSUPPORTED;
  if (c.shared_intermediate > 0) {
    if (q4) return MOE_ERR_UNSUPPORTED;
    if (c.act_dtype == MOE_BF16 && c.shared_intermediate % 8 != 0) return MOE_ERR_UNSUPPORTED;
  }
  if (f32 && (int64_t)c.num_tokens * c.top_k > 65535LL * 8) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

size_t moe_workspace_size(const moe_config *cfg) {
  if (moe_validate(cfg) != MOE_OK) return 0;
  return ws_layout(*cfg).total;
}

moe_status moe_aux_loss(const moe_config *cfg, const int32_t *kept_counts_host, const float *prob_sum_host,
                        double *aux_raw, double *aux_scaled) {
  if (!cfg || !kept_counts_host || !prob_sum_host || !aux_raw || !aux_scaled) return MOE_ERR_INVALID_ARG;
  const moe_config &c = *cfg;
  if (c.num_tokens < 1 || c.num_experts < 1) return MOE_ERR_INVALID_ARG;
  double s = 0.0;
  for (int e = 0; e < c.num_experts; ++e)
    s += ((double)kept_counts_host[e] / c.num_tokens) * ((double)prob_sum_host[e] / c.num_tokens);
  *aux_raw = (double)c.num_experts * s;
  *aux_scaled = (double)c.aux_alpha * *aux_raw;
  return MOE_OK;
}

moe_status moe_routing_health(const moe_config *cfg, const int32_t *kept_counts_host, int32_t dropped,
                              double *entropy_ratio, double *max_share, double *dropped_fraction,
                              int32_t *collapsed) {
  if (!cfg || !kept_counts_host) return MOE_ERR_INVALID_ARG;
  const moe_config &c = *cfg;
  if (c.num_tokens < 1 || c.num_experts < 1 || c.top_k < 1) return MOE_ERR_INVALID_ARG;
  double total = 0.0;
  for (int e = 0; e < c.num_experts; ++e) total += kept_counts_host[e];
  double ratio = 0.0, mx = 0.0;
  const double df = (double)dropped / (double)((int64_t)c.num_tokens * c.top_k);
  if (total > 0.0) {
    double ent = 0.0;
    for (int e = 0; e < c.num_experts; ++e) {
      const double sh = kept_counts_host[e] / total;
      if (sh > 0.0) ent -= sh * log(sh);
      if (sh > mx) mx = sh;
    }
    const double me = log((double)c.num_experts);
    ratio = me > 0.0 ? ent / me : 0.0;
  }
  if (entropy_ratio) *entropy_ratio = ratio;
  if (max_share) *max_share = mx;
  if (dropped_fraction) *dropped_fraction = total > 0.0 ? df : 1.0;
  if (collapsed) *collapsed = ratio < 0.5 ? 1 : 0;
  return MOE_OK;
}

const char *moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_INVALID_TOPK: return "top_k outside [1, num_experts]";
    case MOE_ERR_CAPACITY_TOO_TIGHT: return "capacity_factor below 1.0 drops tokens under perfectly uniform routing";
    case MOE_ERR_UNSUPPORTED: return "configuration not supported by this library";
    case MOE_ERR_WORKSPACE: return "workspace missing or smaller than moe_workspace_size()";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE: return "device-side failure recorded in the workspace";
  }
  return "unknown status";
}

const char *moe_last_error(void) { return g_last_error; }

int64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

moe_status moe_set_wait_timeout_ns(uint64_t ns) {
  g_wait_ns.store(ns == 0 ? kDefaultWaitNs : ns, std::memory_order_relaxed);
  return MOE_OK;
}

moe_status moe_workspace_status(const void *ws, moe_stream_t stream) {
  if (!aligned16(ws)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err = cudaStreamSynchronize(s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_workspace_status");
  int code = 0;
  err = cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (err != cudaSuccess) return cuda_fail(err, "moe_workspace_status");
  if (code == 0) return MOE_OK;
  const char *what = "unknown";
  switch (code) {
    case kDevBadExpertId: what = "dispatch: expert id outside [0, E)"; break;
    case kDevDuplicateId: what = "dispatch: a token names the same expert twice"; break;
    case kDevTimeoutProducer: what = "tensor-core kernel: TMA producer wait timed out"; break;
    case kDevTimeoutMma: what = "tensor-core kernel: MMA issuer wait timed out"; break;
    case kDevTimeoutEpilogue: what = "tensor-core kernel: epilogue / converter wait timed out"; break;
    case kDevTimeoutDrain: what = "tensor-core kernel: in-flight work did not drain after an abort"; break;
    case kDevBadOffsets: what = "grouped FFN: expert_offsets not 0-based, non-decreasing and within T*k"; break;
  }
  char num[32];
  snprintf(num, sizeof(num), "%d", code);
  set_error("device status %s: %s", num, what);
  return MOE_ERR_DEVICE;
}

moe_status moe_workspace_region(const moe_config *cfg, int32_t region, size_t *offset, size_t *bytes) {
  if (!offset || !bytes) return MOE_ERR_INVALID_ARG;
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = ws_layout(*cfg);
  size_t begin = 0, end = 0;
  switch (region) {
    case MOE_WS_OFFSETS: begin = L.offsets; end = L.perm_token; break;
    case MOE_WS_PERM_TOKEN: begin = L.perm_token; end = L.perm_w; break;
    case MOE_WS_PERM_W: begin = L.perm_w; end = L.slot_row; break;
    case MOE_WS_SLOT_ROW: begin = L.slot_row; end = L.topk_ids; break;
    case MOE_WS_X_PERM: begin = L.x_perm; end = L.h; break;
    case MOE_WS_H: begin = L.h; end = L.y_perm; break;
    case MOE_WS_Y_PERM: begin = L.y_perm; end = L.shared_h; break;
    case MOE_WS_SHARED_H: begin = L.shared_h; end = L.shared_out; break;
    case MOE_WS_SHARED_OUT: begin = L.shared_out; end = L.x_stage; break;
    case MOE_WS_ROUTER_LOGITS: begin = L.route_logits; end = L.blk_counts; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  *offset = begin;
  *bytes = L.region_bytes[region];
  if (begin + *bytes > end) return MOE_ERR_INVALID_ARG;   // layout and sizes disagree: a library bug
  return MOE_OK;
}

moe_status moe_set_phase_events(void *const *events, int32_t count) {
  if (count == 0) {
    g_nevents = 0;
    return MOE_OK;
  }
  if (count != MOE_PHASE_COUNT || !events) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < MOE_PHASE_COUNT; ++i) {
    if (!events[i]) return MOE_ERR_INVALID_ARG;
    g_events[i] = reinterpret_cast<cudaEvent_t>(events[i]);
  }
  g_nevents = count;
  return MOE_OK;
}

moe_status moe_route(const moe_config *cfg, const void *x, const float *w_router, const float *router_bias,
                     int32_t *topk_ids, float *topk_w, float *prob_sum, void *ws, size_t ws_bytes,
                     moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16_or_null(router_bias) || !aligned16(topk_ids) ||
      !aligned16(topk_w) || !aligned16(prob_sum))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  return do_route(c, x, w_router, router_bias, topk_ids, topk_w, prob_sum, ws, s);
}

moe_status moe_route_forced(const moe_config *cfg, const void *x, const float *w_router, const float *router_bias,
                            const int32_t *forced_ids, int32_t *topk_ids, float *topk_w, float *prob_sum, void *ws,
                            size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16_or_null(router_bias) || !aligned16(forced_ids) ||
      !aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(prob_sum))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  return do_route(c, x, w_router, router_bias, topk_ids, topk_w, prob_sum, ws, s, forced_ids);
}

moe_status moe_update_bias(const moe_config *cfg, const int32_t *counts, float *expert_bias, float coeff,
                           moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  if (!aligned16(counts) || !aligned16(expert_bias)) return MOE_ERR_INVALID_ARG;
  if (!(coeff >= 0.0f) || isinf(coeff)) return MOE_ERR_INVALID_ARG;
  cudaError_t err = launch_bias_update(cfg->num_experts, counts, expert_bias, coeff,
                                       reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_update_bias");
}

moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *topk_ids, const float *topk_w,
                       int32_t *expert_offsets, int32_t *perm_token, float *perm_w, int32_t *slot_row,
                       void *x_perm, const moe_stats *stats, void *ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(expert_offsets) || !aligned16(perm_token) ||
      !aligned16(perm_w) || !aligned16(slot_row) || !aligned16_or_null(x) || !aligned16_or_null(x_perm))
    return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!stats || !aligned16(stats->raw_counts) || !aligned16(stats->kept_counts) || !aligned16(stats->dropped))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  return do_permute(c, x, topk_ids, topk_w, expert_offsets, perm_token, perm_w, slot_row, x_perm,
                    stats->raw_counts, stats->kept_counts, stats->dropped, ws, s);
}

moe_status moe_expert_counts(const moe_config *cfg, const int32_t *topk_ids, int32_t *raw_counts, void *ws,
                             size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!aligned16(topk_ids) || !aligned16(raw_counts)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  const WsLayout L = ws_layout(c);
  // the dispatch's own histogram and scan, without a capacity and without the gather
  cudaError_t err = launch_permute(c, nullptr, topk_ids, nullptr, -1, ws_ptr<int32_t>(ws, L.offsets),
                                   ws_ptr<int32_t>(ws, L.perm_token), ws_ptr<float>(ws, L.perm_w),
                                   ws_ptr<int32_t>(ws, L.slot_row), nullptr, raw_counts,
                                   ws_ptr<int32_t>(ws, L.kept_counts), ws_ptr<int32_t>(ws, L.dropped),
                                   ws_ptr<int32_t>(ws, L.blk_counts), ws_ptr<int32_t>(ws, L.blk_base),
                                   ws_ptr<int32_t>(ws, L.local_rank), ws_ptr<int>(ws, L.status), s);
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_expert_counts");
}

moe_status moe_permute_shard(const moe_config *cfg, const void *x, const int32_t *topk_ids, const float *topk_w,
                             const int32_t *counts_by_rank, int32_t world, int32_t rank, int64_t capacity,
                             int32_t *expert_offsets, int32_t *perm_token, float *perm_w, int32_t *slot_row,
                             void *x_perm, const moe_stats *stats, void *ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (capacity < -1 || world < 1 || rank < 0 || rank >= world) return MOE_ERR_INVALID_ARG;
  if (world > 1 && !counts_by_rank) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(expert_offsets) || !aligned16(perm_token) ||
      !aligned16(perm_w) || !aligned16(slot_row) || !aligned16_or_null(x) || !aligned16_or_null(x_perm) ||
      !aligned16_or_null(counts_by_rank))
    return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!stats || !aligned16(stats->raw_counts) || !aligned16(stats->kept_counts) || !aligned16(stats->dropped))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  const WsLayout L = ws_layout(c);
  cudaError_t err = launch_permute(c, x, topk_ids, topk_w, capacity, expert_offsets, perm_token, perm_w, slot_row,
                                   x_perm, stats->raw_counts, stats->kept_counts, stats->dropped,
                                   ws_ptr<int32_t>(ws, L.blk_counts), ws_ptr<int32_t>(ws, L.blk_base),
                                   ws_ptr<int32_t>(ws, L.local_rank), ws_ptr<int>(ws, L.status), s,
                                   rank > 0 ? counts_by_rank : nullptr, rank);
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_permute_shard");
}

moe_status moe_ep_local_ids(const int32_t *recv_counts, int32_t world, int32_t experts_per_rank, int32_t rows,
                            int32_t *ids, moe_stream_t stream) {
  if (world < 1 || experts_per_rank < 1 || (int64_t)world * experts_per_rank > kMaxExperts || rows < 0)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(recv_counts) || (rows > 0 && !aligned16(ids))) return MOE_ERR_INVALID_ARG;
  cudaError_t err = launch_ep_local_ids(recv_counts, world, experts_per_rank, rows, ids,
                                        reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_ep_local_ids");
}

moe_status moe_grouped_ffn(const moe_config *cfg, const void *x_perm, const int32_t *expert_offsets,
                           const moe_weights *w, void *y_perm, void *ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!aligned16(x_perm) || !aligned16(expert_offsets) || !aligned16(y_perm)) return MOE_ERR_INVALID_ARG;
  if ((st = check_weights(c, w)) != MOE_OK) return st;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  return do_ffn(c, x_perm, expert_offsets, w, y_perm, ws, s);
}

moe_status moe_shared_expert(const moe_config *cfg, const void *x, const moe_weights *w, void *shared_out,
                             void *ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (c.shared_intermediate < 1) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(shared_out) || !w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->shared1) || !aligned16(w->shared2) || !aligned16(w->shared3)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  return do_shared(c, x, w, shared_out, ws, s);
}

moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *slot_row, const float *topk_w,
                       const void *shared_out, void *out, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!aligned16(y_perm) || !aligned16(slot_row) || !aligned16(topk_w) || !aligned16_or_null(shared_out) ||
      !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  cudaError_t err = launch_combine(c, y_perm, slot_row, topk_w, shared_out, out,
                                   reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_combine");
}

static moe_status forward_impl(const moe_config &c, const void *x, const float *w_router,
                               const float *router_bias, const moe_weights *w, void *out, int32_t *topk_ids,
                               float *topk_w, const moe_stats *stats, void *ws, cudaStream_t s) {
  const WsLayout L = ws_layout(c);
  int32_t *ids = topk_ids ? topk_ids : ws_ptr<int32_t>(ws, L.topk_ids);
  float *wts = topk_w ? topk_w : ws_ptr<float>(ws, L.topk_w);
  int32_t *raw = stats && stats->raw_counts ? stats->raw_counts : ws_ptr<int32_t>(ws, L.raw_counts);
  int32_t *kept = stats && stats->kept_counts ? stats->kept_counts : ws_ptr<int32_t>(ws, L.kept_counts);
  float *psum = stats && stats->prob_sum ? stats->prob_sum : ws_ptr<float>(ws, L.prob_sum);
  int32_t *dropped = stats && stats->dropped ? stats->dropped : ws_ptr<int32_t>(ws, L.dropped);
  int32_t *off = ws_ptr<int32_t>(ws, L.offsets);
  moe_status st;
  cudaError_t err;
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  if ((err = mark(MOE_PHASE_START, s)) != cudaSuccess) return cuda_fail(err, "phase event");
  if ((st = do_route(c, x, w_router, router_bias, ids, wts, psum, ws, s)) != MOE_OK) return st;
  if ((err = mark(MOE_PHASE_ROUTE, s)) != cudaSuccess) return cuda_fail(err, "phase event");
  // with the fused gather, bf16 tensor-core experts read their token rows
  // straight from x: the permutation is built but no row is copied
  const bool fused_gather = c.weight_dtype == MOE_BF16 && c.fused_gather;
  int32_t *perm_token = ws_ptr<int32_t>(ws, L.perm_token);
  void *x_perm = fused_gather ? nullptr : ws_ptr<char>(ws, L.x_perm);
  if ((st = do_permute(c, x, ids, wts, off, perm_token, ws_ptr<float>(ws, L.perm_w),
                       ws_ptr<int32_t>(ws, L.slot_row), x_perm, raw, kept, dropped, ws, s)) != MOE_OK)
    return st;
  if ((err = mark(MOE_PHASE_PERMUTE, s)) != cudaSuccess) return cuda_fail(err, "phase event");
  void *y_perm = ws_ptr<char>(ws, L.y_perm);
  void *shared = c.shared_intermediate > 0 ? ws_ptr<char>(ws, L.shared_out) : nullptr;
  const bool shared_fused = shared && shared_in_grouped_gemm(c);
  if ((st = do_ffn(c, fused_gather ? x : x_perm, off, w, y_perm, ws, s, g_nevents ? g_events[MOE_PHASE_FFN1] : nullptr,
                   fused_gather ? perm_token : nullptr, shared_fused ? x : nullptr,
                   shared_fused ? shared : nullptr)) != MOE_OK)
    return st;
  if ((err = mark(MOE_PHASE_FFN2, s)) != cudaSuccess) return cuda_fail(err, "phase event");
  if (shared && !shared_fused && (st = do_shared(c, x, w, shared, ws, s)) != MOE_OK) return st;
  if ((err = mark(MOE_PHASE_SHARED, s)) != cudaSuccess) return cuda_fail(err, "phase event");
  err = launch_combine(c, y_perm, ws_ptr<int32_t>(ws, L.slot_row), wts, shared, out, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_forward combine");
  if ((err = mark(MOE_PHASE_COMBINE, s)) != cudaSuccess) return cuda_fail(err, "phase event");
  return MOE_OK;
}

moe_status moe_forward(const moe_config *cfg, const void *x, const float *w_router, const float *router_bias,
                       const moe_weights *w, void *out, int32_t *topk_ids, float *topk_w, const moe_stats *stats,
                       void *ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16_or_null(router_bias) || !aligned16(out) ||
      !aligned16_or_null(topk_ids) || !aligned16_or_null(topk_w))
    return MOE_ERR_INVALID_ARG;
  if (stats && (!aligned16_or_null(stats->raw_counts) || !aligned16_or_null(stats->kept_counts) ||
                !aligned16_or_null(stats->prob_sum) || !aligned16_or_null(stats->dropped)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_weights(c, w)) != MOE_OK) return st;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  return forward_impl(c, x, w_router, router_bias, w, out, topk_ids, topk_w, stats, ws,
                      reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_forward_host(const moe_config *cfg, const void *x_host, const float *w_router,
                            const float *router_bias, const moe_weights *w, void *out_host,
                            int32_t *kept_counts_host, float *prob_sum_host, int32_t *dropped_host, void *ws,
                            size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!x_host || !out_host || !aligned16(w_router) || !aligned16_or_null(router_bias))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_weights(c, w)) != MOE_OK) return st;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(c);
  const size_t act_bytes = act_size(c) * (size_t)c.num_tokens * c.hidden;
  void *xd = ws_ptr<char>(ws, L.x_stage);
  void *od = ws_ptr<char>(ws, L.out_stage);
  cudaError_t err = cudaMemcpyAsync(xd, x_host, act_bytes, cudaMemcpyHostToDevice, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_forward_host h2d");
  if ((st = forward_impl(c, xd, w_router, router_bias, w, od, nullptr, nullptr, nullptr, ws, s)) != MOE_OK)
    return st;
  err = cudaMemcpyAsync(out_host, od, act_bytes, cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess && kept_counts_host)
    err = cudaMemcpyAsync(kept_counts_host, ws_ptr<char>(ws, L.kept_counts), sizeof(int32_t) * c.num_experts,
                          cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess && prob_sum_host)
    err = cudaMemcpyAsync(prob_sum_host, ws_ptr<char>(ws, L.prob_sum), sizeof(float) * c.num_experts,
                          cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess && dropped_host)
    err = cudaMemcpyAsync(dropped_host, ws_ptr<char>(ws, L.dropped), sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_forward_host d2h");
}

}  // extern "C"
