// Shared definitions of the MoE library: workspace layout, device status
// codes and small device helpers.  Internal to the library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------- tiling constants
constexpr int kRouteTokens = 32;      // tokens per router block
constexpr int kRouteThreads = 256;
constexpr int kPermTokens = 256;      // tokens per dispatch count block
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 32;
constexpr int kMaxGroups = 32;

// ---------------------------------------------------------------- device status
// The first word of the workspace holds 0 or the code of the first failure a
// kernel recorded (atomicCAS from 0).
enum DeviceStatus : int {
  kDevOk = 0,
  kDevBadExpertId = 1,       // dispatch: topk id outside [0, E)
  kDevDuplicateId = 2,       // dispatch: a token names the same expert twice
  kDevTimeoutProducer = 10,  // tensor-core kernel: TMA producer waited too long
  kDevTimeoutMma = 11,       // tensor-core kernel: MMA issuer waited too long
  kDevTimeoutEpilogue = 12,  // tensor-core kernel: epilogue / converter waited too long
  kDevTimeoutDrain = 13,     // tensor-core kernel: in-flight work did not drain after an abort
  kDevBadOffsets = 20,       // grouped FFN: expert_offsets not 0-based / non-decreasing / in range
};

__device__ __forceinline__ void record_status(int *status, int code) {
  atomicCAS(status, 0, code);
}

// Programmatic dependent launch.  Every kernel of this library starts with
// pdl_wait(): when it was launched with launch_pdl it waits there until the
// previous kernel on the stream has completed and its writes are visible
// (otherwise the wait is a no-op).  Short kernels then let the next kernel be
// scheduled at once (pdl_enter); the persistent grouped GEMMs do so only when
// their tile loops are done.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// short kernels: wait, then let the next kernel be scheduled at once
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_trigger();
}

// Counts every kernel this library launches (moe_kernel_launches).
void note_launch();
// Bound on every barrier wait of the tensor-core kernels, in ns of
// %globaltimer (moe_set_wait_timeout_ns; 2 s by default).
uint64_t wait_timeout_ns();

template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t s, Args &&...args) {
  note_launch();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}
// the short kernels: scheduled while the previous kernel finishes
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args &&...args) {
  return launch_kernel(true, kern, grid, block, smem, s, static_cast<Args &&>(args)...);
}
// the persistent grouped GEMMs: a plain stream dependency (with PDL edges
// into them the Mixtral-style layer step measured 2-9 % slower on B200)
template <typename... KArgs, typename... Args>
inline cudaError_t launch_plain(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                Args &&...args) {
  return launch_kernel(false, kern, grid, block, smem, s, static_cast<Args &&>(args)...);
}

// Grouped kernels' view of the group offsets, read by ONE full warp into
// shared memory: off[i] = min(max(0, src[0..i]), rows_cap) (the running
// maximum, so the copy is non-decreasing and in range) with off[0] = 0, and
// tile_start[e] = sum over e' < e of units(off[e'+1] - off[e']),
// tile_start[n] = the total.  src == nullptr stands for one group of `rows`
// rows ({0, rows}, n = 1).  Loads are coalesced and the scans are warp
// shuffles, so the cost does not grow with one memory round trip per group.
// Returns true (on every lane) when src needed any repair.
template <class Units>
__device__ __forceinline__ bool warp_group_offsets(const int32_t *src, int n, int rows, int rows_cap, int32_t *off,
                                                   int32_t *tile_start, Units units) {
  const unsigned full = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  int carry = 0;
  bool bad = false;
  for (int base = 0; base <= n; base += 32) {
    const int i = base + lane;
    const int v = i <= n ? (src ? src[i] : (i == 0 ? 0 : rows)) : 0;
    int m = i <= n ? v : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(full, m, o);
      if (lane >= o) m = max(m, t);
    }
    m = max(m, carry);
    const int val = min(m, rows_cap);
    if (i <= n) {
      off[i] = val;
      if (val != v || (i == 0 && v != 0)) bad = true;
    }
    carry = __shfl_sync(full, m, 31);
  }
  __syncwarp();
  if (lane == 0) off[0] = 0;
  __syncwarp();
  int total = 0;
  for (int base = 0; base < n; base += 32) {
    const int e = base + lane;
    const int u = e < n ? units(off[e + 1] - off[e]) : 0;
    int x = u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(full, x, o);
      if (lane >= o) x += t;
    }
    if (e < n) tile_start[e] = total + x - u;
    total += __shfl_sync(full, x, 31);
  }
  if (lane == 0) tile_start[n] = total;
  __syncwarp();
  return __any_sync(full, bad);
}

size_t route_logits_bytes(const moe_config &c);       // defined in router.cu
size_t route_logits_f64_bytes(const moe_config &c);   // its float64 logits partials [ks][T][E]

// ---------------------------------------------------------------- workspace
struct WsLayout {
  size_t status;       // int32[64]
  size_t route_part;   // double[nb_route][E]
  size_t route_logits; // double[ks][T][E] (split router pass only)
  size_t blk_counts;   // int32[nb_perm][E]
  size_t blk_base;     // int32[nb_perm][E]
  size_t local_rank;   // int32[T*k]
  size_t offsets;      // int32[E+1]
  size_t perm_token;   // int32[T*k]
  size_t perm_w;       // float[T*k]
  size_t slot_row;     // int32[T*k]
  size_t topk_ids;     // int32[T*k]
  size_t topk_w;       // float[T*k]
  size_t raw_counts;   // int32[E]
  size_t kept_counts;  // int32[E]
  size_t prob_sum;     // float[E]
  size_t dropped;      // int32[1]
  size_t x_perm;       // act[T*k][d]
  size_t h;            // act[T*k][F]   (grouped FFN intermediate)
  size_t y_perm;       // act[T*k][d]
  size_t shared_h;     // act[T][Fs]
  size_t shared_out;   // act[T][d]
  size_t x_stage;      // act[T][d]   (moe_forward_host)
  size_t out_stage;    // act[T][d]
  size_t total;
  size_t region_bytes[MOE_WS_REGION_COUNT];   // unpadded sizes of the moe_ws_region buffers
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline size_t act_size(const moe_config &c) { return c.act_dtype == MOE_F32 ? 4 : 2; }

inline int route_blocks(const moe_config &c) {
  return (c.num_tokens + kRouteTokens - 1) / kRouteTokens;
}
// tokens per block of the selection pass over logits partials: 8 when
// 32-token blocks would leave more than half of the 148 SMs idle
inline int select_tokens_per_block(int T) { return (T + kRouteTokens - 1) / kRouteTokens < 74 ? 8 : 32; }
// probability-sum rows any route plan writes (at most one per 8 tokens)
inline int route_part_rows(const moe_config &c) {
  const int sel = (c.num_tokens + select_tokens_per_block(c.num_tokens) - 1) / select_tokens_per_block(c.num_tokens);
  return sel > route_blocks(c) ? sel : route_blocks(c);
}
inline int perm_blocks(const moe_config &c) {
  return (c.num_tokens + kPermTokens - 1) / kPermTokens;
}

inline WsLayout ws_layout(const moe_config &c) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t here = off;
    off = align_up(off + bytes, 256);
    return here;
  };
  const size_t T = (size_t)c.num_tokens, E = (size_t)c.num_experts, K = (size_t)c.top_k;
  const size_t d = (size_t)c.hidden, F = (size_t)c.intermediate;
  const size_t Fs = (size_t)(c.shared_intermediate > 0 ? c.shared_intermediate : 0);
  const size_t es = act_size(c);
  const size_t slots = T * K;
  L.status = take(256);
  L.route_part = take(sizeof(double) * route_part_rows(c) * E);
  L.route_logits = take(route_logits_bytes(c));
  L.region_bytes[MOE_WS_ROUTER_LOGITS] = route_logits_f64_bytes(c);
  L.blk_counts = take(sizeof(int32_t) * perm_blocks(c) * E);
  L.blk_base = take(sizeof(int32_t) * perm_blocks(c) * E);
  L.local_rank = take(sizeof(int32_t) * slots);
  size_t *rb = L.region_bytes;
  L.offsets = take(rb[MOE_WS_OFFSETS] = sizeof(int32_t) * (E + 1));
  L.perm_token = take(rb[MOE_WS_PERM_TOKEN] = sizeof(int32_t) * slots);
  L.perm_w = take(rb[MOE_WS_PERM_W] = sizeof(float) * slots);
  L.slot_row = take(rb[MOE_WS_SLOT_ROW] = sizeof(int32_t) * slots);
  L.topk_ids = take(sizeof(int32_t) * slots);
  L.topk_w = take(sizeof(float) * slots);
  L.raw_counts = take(sizeof(int32_t) * E);
  L.kept_counts = take(sizeof(int32_t) * E);
  L.prob_sum = take(sizeof(float) * E);
  L.dropped = take(sizeof(int32_t));
  // bf16 experts with the fused gather read their rows from x directly: no copy buffer
  L.x_perm = take(rb[MOE_WS_X_PERM] = c.weight_dtype == MOE_BF16 && c.fused_gather ? 0 : es * slots * d);
  L.h = take(rb[MOE_WS_H] = es * slots * F);
  L.y_perm = take(rb[MOE_WS_Y_PERM] = es * slots * d);
  L.shared_h = take(rb[MOE_WS_SHARED_H] = es * T * Fs);
  L.shared_out = take(rb[MOE_WS_SHARED_OUT] = Fs ? es * T * d : 0);
  L.x_stage = take(es * T * d);
  L.out_stage = take(es * T * d);
  L.total = off;
  return L;
}

template <typename P>
inline P *ws_ptr(void *ws, size_t off) {
  return reinterpret_cast<P *>(static_cast<char *>(ws) + off);
}

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ---------------------------------------------------------------- launchers (one per kernel file)
// Router launch shape.  split: the logits are first computed in `ks` slices
// of the hidden dimension (float64 partials in the workspace) and summed by a
// selection pass -- for batches too small to fill the GPU with whole rows.
struct RoutePlan {
  bool split;
  bool tc;          // bf16 tokens: selection-grade logits on the bf16 tensor cores (router_tc.cu), exact re-weighting
  bool i8;          // bf16 tokens: bounded-error logits on the integer tensor cores (router_i8.cu)
  int ks, kchunk;
  int tpw;          // tokens per warp of the tiled kernel (4 or 8)
};
RoutePlan route_plan(const moe_config &c, bool allow_split);

// Tensor-core logits: expert tile width, padded expert count, hidden slices.
struct TcRoutePlan {
  int nte, e_pad, ks, kb_per_slice;
  size_t wsplit_bytes;   // the three bf16 slices of the router weight, [3][e_pad][d]
};
TcRoutePlan tc_route_plan(const moe_config &c);
// Splits w_router into wsplit and writes float64 logits partials [ks][T][E].
cudaError_t launch_route_tc_logits(const moe_config &c, const void *x, const float *w_router,
                                   __nv_bfloat16 *wsplit, double *logits, int *status, cudaStream_t s);

// Integer tensor-core logits: expert tile width, padded sizes, hidden slices.
struct I8RoutePlan {
  int n, e_pad, d_pad, ks, kb_per_slice;
};
// Its workspace: float64 logits partials [ks][T][E], the weight's digit planes
// [4][e_pad][d_pad], the scale exponents and the error-bound norms.
struct I8RouteBuffers {
  double *logits;
  int8_t *wdig;
  int *sx, *sw;
  double *xst;    // [T][4]: |dx|_1, |xhat|_2, |x2|_2, 0
  double *wst;    // [e_pad][4]: |w|_inf, |dw|_2, |w3|_2, 0
  int *xcnt;      // [T] elements each token row's digits round (dx != 0)
  int *xidx;      // [T][round_list] the first round_list of them: index
  double *xdx;    // [T][round_list] and dx (x - xhat)
  int round_list;
  int *flag_count; // tokens listed for the exact recomputation (zeroed by the preparation pass)
  int *flag_list;  // [T]
};
bool i8_route_supported(const moe_config &c);
I8RoutePlan i8_route_plan(const moe_config &c);
size_t i8_route_bytes(const moe_config &c, const I8RoutePlan &t);
I8RouteBuffers i8_route_buffers(const moe_config &c, const I8RoutePlan &t, void *base);
cudaError_t launch_route_i8_logits(const moe_config &c, const void *x, const float *w_router,
                                   const I8RoutePlan &t, const I8RouteBuffers &b, int *status, cudaStream_t s);

// logits == nullptr forbids the split pass (no workspace for it).
cudaError_t launch_route(const moe_config &c, const void *x, const float *w_router,
                         const float *router_bias, int32_t *topk_ids, float *topk_w,
                         double *route_part, float *prob_sum, cudaStream_t s,
                         double *logits = nullptr, const int32_t *forced_ids = nullptr,
                         int *status = nullptr);
// Aux-loss-free balancing: expert_bias[e] += coeff * sign(sum(counts) - E * counts[e]).
cudaError_t launch_bias_update(int E, const int32_t *counts, float *expert_bias, float coeff, cudaStream_t s);

cudaError_t launch_permute(const moe_config &c, const void *x, const int32_t *topk_ids,
                           const float *topk_w, int64_t capacity, int32_t *expert_offsets,
                           int32_t *perm_token, float *perm_w, int32_t *slot_row, void *x_perm,
                           int32_t *raw_counts, int32_t *kept_counts, int32_t *dropped,
                           int32_t *blk_counts, int32_t *blk_base, int32_t *local_rank,
                           int *status, cudaStream_t s, const int32_t *counts_by_rank = nullptr,
                           int rank = 0);
// Expert parallelism: local expert id of each received row ([world][e_local] counts, device).
cudaError_t launch_ep_local_ids(const int32_t *recv_counts, int world, int e_local, int rows, int32_t *ids,
                                cudaStream_t s);

// Two-phase expert FFN over groups.  `offsets` == nullptr means one group of
// `rows` rows (the shared expert).  Writes the intermediate to `h` and the
// result to `y`.
struct FfnArgs {
  int kind;                 // 0 = fp32 SIMT, 1 = bf16 tensor cores, 2 = q4 (bf16 act)
  int act;                  // moe_act
  int E;                    // groups
  int rows_cap;             // allocated rows of x / h / y
  int rows;                 // used when offsets == nullptr
  int d, F;
  const int32_t *offsets;   // [E+1] device or nullptr
  const void *x;            // [rows_cap, d]
  const void *w1, *w2, *w3; // [E,F,d], [E,F,d], [E,d,F] (q4: packed codes)
  const void *s1, *s2, *s3, *b1, *b2, *b3;  // q4 scale / bias
  int w_stride;             // rows from one expert's w1 (w2) block to the next: F, or 2F when
                            // gate and up rows are stacked per expert (w2 = w1 + F rows)
  const int32_t *gather;    // bf16 tensor-core path only: phase 1 reads row gather[r] of x ([x_rows, d])
  int x_rows;               // instead of row r of an expert-sorted copy (the fused dispatch gather)
  void *h;                  // [rows_cap, F]
  void *y;                  // [rows_cap, d]
  int *status;
  cudaEvent_t mid_event;    // recorded between the two phases when not null
  // bf16 tensor-core path only: the shared expert as one more group of both
  // phases (0 rows: none).  Its width must equal F.
  int shared_rows;
  const void *shared_x;     // [shared_rows, d]
  const void *shared_w1, *shared_w2, *shared_w3;   // [F, d], [F, d], [d, F]
  void *shared_h;           // [shared_rows, F]
  void *shared_y;           // [shared_rows, d]
};

cudaError_t launch_ffn_simt_f32(const FfnArgs &a, cudaStream_t s);
cudaError_t launch_ffn_tc_bf16(const FfnArgs &a, cudaStream_t s);
cudaError_t launch_ffn_tc2_bf16(const FfnArgs &a, cudaStream_t s);   // pairs of SMs (cta_group::2), no gather
cudaError_t launch_ffn_q4(const FfnArgs &a, cudaStream_t s);       // SIMT, any d, F multiple of 64
bool q4_tc_supported(int d, int F);                                 // the tensor-core 4-bit path's shapes
cudaError_t launch_ffn_q4_tc(const FfnArgs &a, cudaStream_t s);
bool q4_mma_supported(int d, int F);                                // the warp-level 4-bit path's shapes
cudaError_t launch_ffn_q4_mma(const FfnArgs &a, cudaStream_t s);

// Replaces the text moe_last_error() returns on this thread.
void set_last_error_text(const char *text);

cudaError_t launch_combine(const moe_config &c, const void *y_perm, const int32_t *slot_row,
                           const float *topk_w, const void *shared_out, void *out,
                           cudaStream_t s);

}  // namespace moe
