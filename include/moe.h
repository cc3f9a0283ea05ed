/*
 * moe.h -- C ABI of the B200 (sm_100a) Mixture-of-Experts layer forward.
 *
 * One MoE layer on one GPU, local dispatch, no expert parallelism:
 *
 *     route  ->  dispatch (permute)  ->  grouped expert FFN  ->  combine
 *
 * following the pipeline of the "Mixture-of-Experts" design doc (The pipeline:
 * router, local dispatcher, grouped GEMM over the ragged per-expert token
 * groups, weighted combine) and the layer defined in the "Mixture of Experts"
 * blog (route, moe_layer, route_and_sort / SortedRouting, moe_forward,
 * load_balancing_loss).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers are DEVICE pointers unless the parameter name ends in _host.
 *    The caller owns every buffer; the library never allocates device or host
 *    memory.  Scratch comes from the caller's workspace `ws` of at least
 *    moe_workspace_size(cfg) bytes (16-byte aligned, any contents).
 *  - Every device pointer must be 16-byte aligned, else MOE_ERR_INVALID_ARG.
 *  - Row-major layouts; "[A,B]" means A rows of B contiguous elements.
 *  - Activations (x, x_perm, h, y_perm, out) have the config's act_dtype
 *    (MOE_F32 or MOE_BF16).  Router weights, routing weights, probabilities
 *    and biases are float32 whatever the activation dtype (router in fp32:
 *    the blog's RouterPrecisionWarning; a reduced-precision router is not
 *    offered).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Argument errors are detected on the host, before any
 *    launch, and returned as a status.  A launch failure returns MOE_ERR_CUDA
 *    with the CUDA message in moe_last_error().  Kernels that wait on
 *    on-chip barriers give up after a bounded time and record the failure in
 *    the workspace; moe_workspace_status() reads it.
 *  - Calls that take `ws` clear its status word first, so two calls that use
 *    the same workspace must not overlap on the GPU.
 *  - Environment (read at every launch):
 *    MOE_TC_PAIR=1 runs the bf16 grouped FFN without the fused gather on
 *    pairs of SMs (256-row tiles, one tcgen05 cta_group::2 MMA per pair);
 *    the results are the same bits as the default one-SM kernel.
 *    MOE_Q4_KERNEL=mma | tc picks the 4-bit grouped FFN kernel: warp-level
 *    MMA fragments (the default when the groups average at most 16 rows) or
 *    tcgen05 with the weight operand in tensor memory (the default for
 *    larger groups).  Both need hidden and intermediate sizes that are
 *    multiples of 128 (else a CUDA-core kernel runs); their results agree
 *    within the bf16 output tolerance, not bit for bit.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* a cudaStream_t */

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* shape, null or misaligned pointer, bad enum */
  MOE_ERR_INVALID_TOPK = 2,        /* top_k outside [1, num_experts] (blog: InvalidTopK) */
  MOE_ERR_CAPACITY_TOO_TIGHT = 3,  /* 0 < capacity_factor < 1 (blog: CapacityTooTight) */
  MOE_ERR_UNSUPPORTED = 4,         /* valid MoE, but a shape/dtype this library has no kernel for */
  MOE_ERR_WORKSPACE = 5,           /* ws NULL or smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 6,                /* CUDA runtime error; text in moe_last_error() */
  MOE_ERR_DEVICE = 7               /* a kernel recorded a device-side failure (moe_workspace_status) */
} moe_status;

typedef enum moe_router_kind {
  MOE_ROUTER_SOFTMAX_TOPK = 0,   /* Edge0 RouterKind.SOFTMAX_TOPK */
  MOE_ROUTER_SIGMOID_GROUP = 1   /* Edge0 RouterKind.SIGMOID_GROUP */
} moe_router_kind;

typedef enum moe_act { MOE_ACT_RELU = 0, MOE_ACT_SWIGLU = 1 } moe_act;

typedef enum moe_dtype {
  MOE_F32 = 0,
  MOE_BF16 = 1,
  MOE_Q4_AFFINE_G64 = 2   /* weights only: Edge0 QuantSpec(bits=4, group_size=64, mode=affine) */
} moe_dtype;

/* How the gate and up projections are stored ("MoE Spec and Routing",
 * WeightLayout and "Bundle layout and the up-first order"). */
typedef enum moe_weight_layout {
  MOE_LAYOUT_SEPARATE = 0,        /* w1 = gate [E,F,d], w2 = up [E,F,d] */
  MOE_LAYOUT_FUSED_GATE_UP = 1    /* w1 = gate_up [E,2F,d]: per expert, F gate rows then F up rows; w2 = NULL */
} moe_weight_layout;

/*
 * Layer configuration (the blog's MoEConfig and Edge0's MoESpec, flattened
 * into plain fields).  Enum-valued fields are int32 so the layout is fixed.
 */
typedef struct moe_config {
  int32_t num_tokens;           /* T >= 1 */
  int32_t hidden;               /* d >= 1 */
  int32_t intermediate;         /* F >= 1, expert FFN width */
  int32_t num_experts;          /* E in [2, 256] (blog MoEConfig: at least 2) */
  int32_t top_k;                /* k in [1, min(E, 32)] */
  int32_t router;               /* moe_router_kind */
  int32_t norm_topk_prob;       /* 1: renormalise the selected weights */
  float routed_scaling;         /* sigmoid_group: weights multiplied by this; softmax: must be 1 */
  int32_t n_group;              /* sigmoid_group: groups of E/n_group consecutive experts (<= 32) */
  int32_t topk_group;           /* sigmoid_group: surviving groups, 1..n_group */
  float capacity_factor;        /* 0: no capacity limit; else >= 1 */
  int32_t act;                  /* moe_act */
  int32_t act_dtype;            /* MOE_F32 or MOE_BF16 */
  int32_t weight_dtype;         /* MOE_F32 (with F32 act), MOE_BF16 or MOE_Q4_AFFINE_G64 (with BF16 act) */
  int32_t shared_intermediate;  /* 0: no shared expert; else the shared SwiGLU expert's width */
  float aux_alpha;              /* balancing-loss coefficient >= 0 (blog default 0.01) */
  int32_t weight_layout;        /* moe_weight_layout; FUSED_GATE_UP needs SwiGLU */
  int32_t fused_gather;         /* 1: with bf16 experts, moe_forward gathers each expert's token rows
                                   inside the grouped GEMM (TMA gather of x rows) instead of copying them
                                   into an expert-sorted buffer; no such buffer is then part of the
                                   workspace.  Same results; on B200 the copy is faster for the bench
                                   shapes (the GEMM re-fetches its token tile for every output tile).
                                   0 (default): copy.  No effect with other weight types. */
} moe_config;

/*
 * Expert weights, stacked over experts on axis 0 (Edge0 WeightLayout.SEPARATE).
 *   w1: W_in (ReLU) or W_gate (SwiGLU)   [E, F, d]
 *   w2: W_up (SwiGLU only, else NULL)    [E, F, d]
 *   w3: W_out (ReLU) or W_down (SwiGLU)  [E, d, F]
 * dtype = weight_dtype.  For MOE_Q4_AFFINE_G64, w1..w3 hold packed codes as
 * int32 words, [E, N, K/8] (element j of a row is the unsigned nibble at bits
 * 4*(j%8) of word j/8), and scale_i / bias_i are bf16 [E, N, K/64]: the
 * weight is scale*q + bias, one scale/bias pair per 64 consecutive elements
 * of the reduction axis K (d for w1/w2, F for w3).
 * With weight_layout = MOE_LAYOUT_FUSED_GATE_UP the gate and up matrices
 * come as ONE tensor in w1, [E, 2F, d] (Q4: codes [E, 2F, d/8], scale1 /
 * bias1 [E, 2F, d/64]): expert e's F gate rows are followed by its F up rows,
 * so splitting one expert's projection into two halves along the output axis
 * gives (gate, up), and the experts' blocks are interleaved, not two stacked
 * tensors.  w2, scale2 and bias2 must then be NULL.  The shared expert always
 * uses the separate layout.
 *   shared1/2/3: the always-active shared expert (MoE competition docs:
 *   "Shared expert"; Edge0 MoESpec.shared_experts), SwiGLU,
 *   [Fs, d], [Fs, d], [d, Fs] in act_dtype; NULL when shared_intermediate = 0.
 */
typedef struct moe_weights {
  const void *w1, *w2, *w3;
  const void *scale1, *scale2, *scale3;
  const void *bias1, *bias2, *bias3;
  const void *shared1, *shared2, *shared3;
} moe_weights;

/* Per-call routing statistics (device, caller-owned, int32 / float32).
 *   raw_counts[E]  slots routed to each expert before the capacity cut;
 *   kept_counts[E] slots kept (the blog's len(assignments[e]));
 *   prob_sum[E]    sum over ALL tokens of the router probability of e (the
 *                  softmax probability; for sigmoid_group the raw sigmoid),
 *                  so P_e = prob_sum[e] / T;
 *   dropped[1]     slots dropped by the capacity cut. */
typedef struct moe_stats {
  int32_t *raw_counts;
  int32_t *kept_counts;
  float *prob_sum;
  int32_t *dropped;
} moe_stats;

/* ---------------------------------------------------------------- host-only */

/* Blog MoEConfig.capacity_for: max(1, int(T*k/E*cf)), evaluated in double left
 * to right with truncation.  Returns -1 for cf == 0 (no limit) and -2 for an
 * invalid argument (T < 1, k < 1, E < 1, cf < 0 or not finite). */
int64_t moe_capacity(int32_t num_tokens, int32_t top_k, int32_t num_experts, float capacity_factor);

/* Checks a configuration; no device work.  Rules: E >= 2; 1 <= k <= E
 * (MOE_ERR_INVALID_TOPK); 0 < cf < 1 -> MOE_ERR_CAPACITY_TOO_TIGHT; alpha >= 0;
 * T, d, F >= 1; sigmoid_group needs E % n_group == 0, E/n_group >= 2,
 * 1 <= topk_group <= n_group <= 32, k <= topk_group*E/n_group; softmax needs
 * routed_scaling == 1.  Then MOE_ERR_UNSUPPORTED for what no kernel covers:
 * E > 256, k > 32, dtype pairs other than F32/F32, BF16/BF16, BF16/Q4;
 * BF16 needs d % 8 == 0 and F % 8 == 0 (16-byte rows); Q4 needs d % 64 == 0,
 * F % 64 == 0 and SwiGLU; a shared expert is offered with F32 and BF16
 * weights. */
moe_status moe_validate(const moe_config *cfg);

/* Bytes of workspace any call below needs for this config (0 if invalid). */
size_t moe_workspace_size(const moe_config *cfg);

/* Balancing loss from host copies of the stats: aux_raw = E * sum_e f_e P_e
 * with f_e = kept_counts[e]/T and P_e = prob_sum[e]/T (blog
 * load_balancing_loss), aux_scaled = aux_alpha * aux_raw. */
moe_status moe_aux_loss(const moe_config *cfg, const int32_t *kept_counts_host,
                        const float *prob_sum_host, double *aux_raw, double *aux_scaled);

/* Routing health from host copies (blog routing_health): entropy of the kept
 * share histogram over log(E), the largest share, dropped / (T*k), and
 * collapsed = entropy_ratio < 0.5.  Any output pointer may be NULL. */
moe_status moe_routing_health(const moe_config *cfg, const int32_t *kept_counts_host,
                              int32_t dropped, double *entropy_ratio, double *max_share,
                              double *dropped_fraction, int32_t *collapsed);

const char *moe_status_string(moe_status s);
/* Text of the last MOE_ERR_CUDA / MOE_ERR_DEVICE seen by this thread. */
const char *moe_last_error(void);

/* Kernels this library has launched in this process so far (all threads,
 * every entry point, including launches captured into a CUDA graph, which a
 * graph replay then repeats without passing through here).  The difference
 * across one call is that call's launch count. */
int64_t moe_kernel_launches(void);

/* Bound on every on-chip barrier wait of the tensor-core kernels (grouped
 * GEMMs, the 4-bit tcgen05 FFN, the router's integer and bf16 tensor-core
 * logits and the integer plan's token-row streaming), in nanoseconds of the GPU's global
 * timer, for the launches that follow (process-wide, all threads).  When a
 * wait runs out, the kernel records where in the workspace status word
 * (moe_workspace_status: MOE_ERR_DEVICE, "... wait timed out"), lets the
 * copies and tensor-core work it already issued finish (waiting at most
 * 200 ms for them), frees its tensor memory and returns, leaving the CUDA
 * context usable; that call's outputs are then incomplete.  0 restores the
 * default of 2 s, far above any wait of a healthy launch.  A short limit
 * makes a launch fail on purpose, which is how the failure path is tested. */
moe_status moe_set_wait_timeout_ns(uint64_t ns);

/* Synchronises `stream` and reads the device status word a kernel leaves in
 * `ws` (MOE_OK, or MOE_ERR_DEVICE with the site in moe_last_error()). */
moe_status moe_workspace_status(const void *ws, moe_stream_t stream);

/* Where moe_forward keeps its intermediates inside `ws` (host only, no device
 * work), so a caller can read them after the stream is synchronised (for
 * example the permutation the dispatch built, or the expert-sorted rows the
 * grouped FFN consumed) and check that nothing is written outside them.
 * Regions, in moe_forward's terms:
 *   MOE_WS_OFFSETS     expert_offsets [E+1] int32
 *   MOE_WS_PERM_TOKEN  perm_token [T*k] int32 (first off[E] valid)
 *   MOE_WS_PERM_W      perm_w [T*k] f32
 *   MOE_WS_SLOT_ROW    slot_row [T,k] int32
 *   MOE_WS_X_PERM      x_perm [T*k, d] act_dtype (0 bytes with the fused gather)
 *   MOE_WS_H           the grouped FFN intermediate [T*k, F] act_dtype; also
 *                      the intermediate of moe_grouped_ffn
 *   MOE_WS_Y_PERM      y_perm [T*k, d] act_dtype
 *   MOE_WS_SHARED_H    the shared expert's intermediate [T, Fs] (0 bytes without one)
 *   MOE_WS_SHARED_OUT  the shared expert's output [T, d] (0 bytes without one)
 *   MOE_WS_ROUTER_LOGITS  the router's float64 logits partials [ks][T][E] when
 *                      its plan computes them in the workspace (bf16 batches of
 *                      512 tokens or more, or the split CUDA-core pass; the
 *                      logit of (t, e) is the sum over the ks slices), else 0
 *                      bytes.  On the integer tensor-core plan each logit is
 *                      within |dx_t|_1 |w_e|_inf + |xhat_t|_2 |dw_e|_2 +
 *                      |x2_t|_2 |w3_e|_2 of x_t . w_e (see moe_route).
 * Rows at or past off[E] (and, in x_perm / h / y_perm, every row when the
 * layer routes nothing) are never written.  *offset is a byte offset from the
 * start of ws (256-byte aligned) and *bytes the region's size; the layout is
 * a function of the configuration only.  Returns MOE_ERR_INVALID_ARG for an
 * unknown region or NULL output, or the moe_validate status. */
typedef enum moe_ws_region {
  MOE_WS_OFFSETS = 0,
  MOE_WS_PERM_TOKEN = 1,
  MOE_WS_PERM_W = 2,
  MOE_WS_SLOT_ROW = 3,
  MOE_WS_X_PERM = 4,
  MOE_WS_H = 5,
  MOE_WS_Y_PERM = 6,
  MOE_WS_SHARED_H = 7,
  MOE_WS_SHARED_OUT = 8,
  MOE_WS_ROUTER_LOGITS = 9,
  MOE_WS_REGION_COUNT = 10
} moe_ws_region;
moe_status moe_workspace_region(const moe_config *cfg, int32_t region, size_t *offset, size_t *bytes);

/* Optional phase timing.  Registers MOE_PHASE_COUNT CUDA events (cudaEvent_t
 * handles created by the caller, in moe_phase order) that the following
 * moe_forward / moe_forward_host calls made by this thread record on their
 * stream at the phase boundaries; count = 0 (events may be NULL) turns it
 * off.  The events only mark time: they add no synchronisation. */
typedef enum moe_phase {
  MOE_PHASE_START = 0,    /* before the router */
  MOE_PHASE_ROUTE = 1,    /* router done */
  MOE_PHASE_PERMUTE = 2,  /* dispatch done */
  MOE_PHASE_FFN1 = 3,     /* first expert GEMM (gate/up or in) done */
  MOE_PHASE_FFN2 = 4,     /* second expert GEMM (down or out) done */
  MOE_PHASE_SHARED = 5,   /* shared expert done (same as FFN2 without one) */
  MOE_PHASE_COMBINE = 6,  /* combine done */
  MOE_PHASE_COUNT = 7
} moe_phase;
moe_status moe_set_phase_events(void *const *events, int32_t count);

/* ---------------------------------------------------------------- device calls */

/* Router (blog route / Router.route; Edge0 select_from_logits and
 * group_select_from_logits).  logits = x W_r^T in fp32 products with float64
 * accumulation, then
 *   softmax_topk:  p = softmax(logits [+ router_bias]); the k largest p (ties
 *                  to the lower expert index) in rank order; weight p_j, or
 *                  p_j / max(sum_sel p, 1e-12) when norm_topk_prob;
 *   sigmoid_group: s = sigmoid(logits); selection = s [+ router_bias]; groups
 *                  ranked by the sum of their two largest selection scores,
 *                  the best topk_group kept; the k largest selection scores
 *                  among them; weight = s_j [/ (sum s + 1e-20)] * routed_scaling.
 * In:  x [T,d] act_dtype; w_router [E,d] f32; router_bias [E] f32 or NULL
 *      (softmax: added to the logits; sigmoid_group: selection only).
 * Out: topk_ids [T,k] int32 (slot j = j-th choice), topk_w [T,k] f32,
 *      prob_sum [E] f32 (see moe_stats).
 * Uses ws (partial sums). */
moe_status moe_route(const moe_config *cfg, const void *x, const float *w_router,
                     const float *router_bias, int32_t *topk_ids, float *topk_w,
                     float *prob_sum, void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_route without a workspace, for callers that cannot allocate device
 * memory (no page has a counterpart: this exists for library users only).
 * Callers hosted by a framework that owns every device allocation, or on a
 * path where an allocation and the synchronisation it can imply are not
 * allowed, have no `ws` to pass.  Same arguments as moe_route, minus ws: the
 * router's one scratch buffer (per-block partial probability sums) is a
 * fixed device array inside the library, 1 MiB on every GPU that loads it,
 * held until the process exits.
 * Results agree with moe_route's within the router tolerances (ids on tokens
 * whose selection margin exceeds 1e-4, weights 1e-6 and prob_sum 1e-5
 * relative): this call always uses the CUDA-core router with whole-row
 * blocks, never the split or tensor-core pass (their logits live in the
 * workspace), so large bf16 batches also route more slowly than moe_route.
 * Limit: ceil(T/32) * E <= 131072 (e.g. T = 16384 with E = 256); larger
 * problems return MOE_ERR_UNSUPPORTED with the reason in moe_last_error().
 * The first call in each CUDA context of a device looks up that context's
 * copy of the array (with the device current), so make it before any stream
 * capture.  All calls share the array: calls that overlap on the GPU race,
 * so serialise them.  Each call writes every entry it reads; nothing carries
 * over. */
moe_status moe_route_noalloc(const moe_config *cfg, const void *x, const float *w_router,
                             const float *router_bias, int32_t *topk_ids, float *topk_w,
                             float *prob_sum, moe_stream_t stream);

/* Router replay ("Mixture-of-Experts" design doc, Router replay (R3)): the
 * expert choice is forced to recorded ids while the weights still come from
 * this router's own gate.  Logits, scores and prob_sum are those of
 * moe_route; then token t's slots j = 0..k-1 take expert forced_ids[t, j] in
 * that order, weighted as moe_route weights its own choices:
 *   softmax_topk:  w_j = p[t, id_j], or p[t, id_j] / max(sum_j p[t, id_j], 1e-12)
 *                  when norm_topk_prob;
 *   sigmoid_group: w_j = s[t, id_j] [/ (sum_j s[t, id_j] + 1e-20)] * routed_scaling
 *                  (the selection bias and the group limit take no part).
 * In:  forced_ids [T,k] int32 device, k distinct ids in [0, E) per token.
 * Out: topk_ids [T,k] (a copy of forced_ids), topk_w [T,k], prob_sum [E].
 * A recorded id outside [0, E) (a missing-route sentinel) or one repeated in
 * its row is not replayed silently: its slot gets weight 0 and is left out of
 * the normalising sum, and the call records a device status, which
 * moe_workspace_status(ws) reports as MOE_ERR_DEVICE (moe_permute rejects
 * the same ids).  Uses ws. */
moe_status moe_route_forced(const moe_config *cfg, const void *x, const float *w_router,
                            const float *router_bias, const int32_t *forced_ids, int32_t *topk_ids,
                            float *topk_w, float *prob_sum, void *ws, size_t ws_bytes,
                            moe_stream_t stream);

/* Aux-loss-free balancing bias update ("Mixture-of-Experts" design doc,
 * Aux-loss-free load balancing): each expert's routing bias takes one step of
 * size coeff toward balanced use, up for an under-used expert and down for an
 * over-used one:
 *   mean = sum_e counts[e] / E;
 *   expert_bias[e] += coeff if counts[e] < mean; -= coeff if counts[e] > mean;
 *   unchanged if counts[e] == mean (compared exactly, as E*counts[e] vs the sum).
 * counts [E] int32 device: the step's assignments per expert, normally
 * moe_stats.raw_counts (before the capacity cut).  expert_bias [E] f32
 * device, updated in place by one fp32 add.  coeff: the step size
 * (load_balance_coeff), >= 0 and finite, else MOE_ERR_INVALID_ARG; 0 leaves
 * the bias as it is (the scheme off).  Only num_experts of cfg is used
 * beyond validation.  Stream-ordered, no workspace, one launch. */
moe_status moe_update_bias(const moe_config *cfg, const int32_t *counts, float *expert_bias, float coeff,
                           moe_stream_t stream);

/* Dispatch (blog moe_layer capacity loop; route_and_sort / SortedRouting).
 * A slot (t, j) with expert e is kept iff fewer than `capacity` slots of e
 * belong to earlier tokens (in-order dropping); capacity = moe_capacity(...),
 * unlimited when capacity_factor == 0.  Kept slots are laid out expert by
 * expert, ascending token within an expert.
 * In:  x [T,d] (may be NULL: indices only); topk_ids [T,k] (each token's ids
 *      distinct and in [0,E), else a device error is recorded); topk_w [T,k].
 * Out: expert_offsets [E+1] (expert e owns rows [off[e], off[e+1])),
 *      perm_token [T*k] (first off[E] entries valid), perm_w [T*k],
 *      slot_row [T,k] (row of the slot in x_perm, -1 if dropped),
 *      x_perm [T*k, d] act_dtype (row r = x[perm_token[r]]; rows >= off[E]
 *      untouched), stats->raw_counts, kept_counts, dropped (prob_sum unused).
 * Uses ws. */
moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *topk_ids,
                       const float *topk_w, int32_t *expert_offsets, int32_t *perm_token,
                       float *perm_w, int32_t *slot_row, void *x_perm, const moe_stats *stats,
                       void *ws, size_t ws_bytes, moe_stream_t stream);

/* Token-sharded dispatch with the in-order capacity rule of the whole batch
 * (blog moe_layer: capacity is "per BATCH"; its in-order cut then spans the
 * token shards held by different GPUs).  A batch split into contiguous token
 * shards, shard r on rank r, keeps on rank r a slot of expert e iff
 *   (slots of e on shards 0..r-1) + (its rank among this shard's slots of e) < capacity.
 * The slot counts of every shard are the one exchange the sharded layer
 * needs: each rank runs moe_expert_counts on its shard and the ranks
 * all-gather the results into counts_by_rank.
 *
 * moe_expert_counts: raw per-expert slot counts of this shard's topk_ids
 *   (the histogram of the dispatch, no capacity, no gather).  Out: raw_counts
 *   [E] int32 (device).  Uses ws.
 * moe_permute_shard: moe_permute with capacity = the WHOLE batch's capacity
 *   (moe_capacity(T_total, ...), -1 for none) and counts_by_rank [world, E]
 *   int32 (device; row q = the moe_expert_counts of shard q; may be NULL
 *   when world == 1 or rank == 0); 0 <= rank < world, else
 *   MOE_ERR_INVALID_ARG.  cfg->num_tokens is this shard's token count.  The
 *   library forms the prefix over the earlier ranks itself.  Same outputs
 *   as moe_permute.  Uses ws. */
moe_status moe_expert_counts(const moe_config *cfg, const int32_t *topk_ids, int32_t *raw_counts, void *ws,
                             size_t ws_bytes, moe_stream_t stream);
moe_status moe_permute_shard(const moe_config *cfg, const void *x, const int32_t *topk_ids, const float *topk_w,
                             const int32_t *counts_by_rank, int32_t world, int32_t rank, int64_t capacity,
                             int32_t *expert_offsets, int32_t *perm_token, float *perm_w, int32_t *slot_row,
                             void *x_perm, const moe_stats *stats, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Expert parallelism ("Mixture-of-Experts" design doc, The pipeline: the
 * expert-parallel dispatch): rank r of `world` holds experts
 * [r*experts_per_rank, (r+1)*experts_per_rank).  After the all-to-all of
 * rows, the received rows are grouped by source rank and, inside a source,
 * by local expert, with recv_counts[s][e] rows of local expert e from rank s
 * (recv_counts [world, experts_per_rank] int32, device).  This writes the
 * local expert id of each of the `rows` received rows into ids [rows] int32
 * (device), in arrival order, ready for moe_permute with top_k = 1; rows
 * past the sum of the counts get -1, which moe_permute rejects.
 * world * experts_per_rank <= 256.  Stream-ordered, no workspace. */
moe_status moe_ep_local_ids(const int32_t *recv_counts, int32_t world, int32_t experts_per_rank, int32_t rows,
                            int32_t *ids, moe_stream_t stream);

/* Grouped expert FFN over the ragged groups (design doc: one grouped matmul
 * over the per-expert token groups; blog moe_forward: two GEMMs per expert
 * over contiguous slices).  For every expert e and row r in
 * [off[e], off[e+1]):
 *   ReLU:   y[r] = W_out[e] relu(W_in[e] x[r])
 *   SwiGLU: y[r] = W_down[e] (silu(W_gate[e] x[r]) * (W_up[e] x[r]))
 * fp32 accumulation; with BF16 the intermediate is rounded to bf16 once.
 * In:  x_perm [T*k, d], expert_offsets [E+1] (off[0] = 0, non-decreasing,
 *      off[E] <= T*k), weights.  Out: y_perm [T*k, d] (rows >= off[E] untouched).
 * Uses ws (the intermediate). */
moe_status moe_grouped_ffn(const moe_config *cfg, const void *x_perm,
                           const int32_t *expert_offsets, const moe_weights *w, void *y_perm,
                           void *ws, size_t ws_bytes, moe_stream_t stream);

/* Shared expert on every token (MoE competition docs, "Shared expert"):
 * out[t] = W_s3 (silu(W_s1 x[t]) * (W_s2 x[t])), weight 1, no routed scaling.
 * In: x [T,d]; w->shared1..3.  Out: shared_out [T,d].  Uses ws. */
moe_status moe_shared_expert(const moe_config *cfg, const void *x, const moe_weights *w,
                             void *shared_out, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Combine (blog moe_layer accumulation / moe_forward weighted scatter-add),
 * as a deterministic gather: out[t] = sum_{j: slot_row[t,j] >= 0}
 * topk_w[t,j] * y_perm[slot_row[t,j]] (+ shared_out[t]), summed in fp32 in
 * slot order and rounded once to act_dtype.  Dropped slots add nothing; a
 * token with every slot dropped gets 0 (plus the shared output).
 * In: y_perm [T*k,d], slot_row [T,k], topk_w [T,k], shared_out [T,d] or NULL.
 * Out: out [T,d] (fully overwritten). */
moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *slot_row,
                       const float *topk_w, const void *shared_out, void *out,
                       moe_stream_t stream);

/* The whole layer: route, permute, grouped FFN, shared expert, combine.
 * With bf16 weights and a shared expert as wide as the routed ones
 * (shared_intermediate == intermediate), the shared expert runs as one more
 * group of the grouped FFN's two launches (the same results, bit for bit, as
 * moe_shared_expert); otherwise it is a launch of its own.
 * topk_ids / topk_w (outputs, [T,k]) and stats may be NULL (kept in ws).
 * Out: out [T,d] act_dtype.  Uses ws. */
moe_status moe_forward(const moe_config *cfg, const void *x, const float *w_router,
                       const float *router_bias, const moe_weights *w, void *out,
                       int32_t *topk_ids, float *topk_w, const moe_stats *stats, void *ws,
                       size_t ws_bytes, moe_stream_t stream);

/* moe_forward with the activations on the HOST: copies x_host [T,d] to the
 * device, runs the layer and copies back out_host [T,d] plus, when not NULL,
 * kept_counts_host [E], prob_sum_host [E] and dropped_host [1] (what the
 * balancing loss needs).  Weights and router stay device-resident.  Host
 * buffers should be pinned (cudaHostAlloc) for the copies to be
 * asynchronous; results are valid after `stream` is synchronised.  Uses ws
 * (device staging for x and out). */
moe_status moe_forward_host(const moe_config *cfg, const void *x_host, const float *w_router,
                            const float *router_bias, const moe_weights *w, void *out_host,
                            int32_t *kept_counts_host, float *prob_sum_host,
                            int32_t *dropped_host, void *ws, size_t ws_bytes,
                            moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
