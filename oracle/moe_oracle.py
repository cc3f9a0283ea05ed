"""CPU oracle for the MoE layer forward (route -> dispatch -> expert MLPs -> combine).

TEST INFRASTRUCTURE, NOT THE PRODUCT.  This module is the plain, slow,
obviously-correct statement of what the layer computes, used to check the
CUDA path.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm may import it.  It shares no code with the CUDA
library and imports nothing from the package: it reads plain numpy arrays
(bf16 inputs arrive as their uint16 bit patterns and are widened exactly).

All arithmetic is float64 on the exact stored input values.  Each function
names the passage it follows:

  [MoE blog]  "Mixture of Experts" (the three listings: the pure-Python layer,
              the NumPy class-based layer and the sorted/permuted layer);
  [Edge0]     "MoE Spec and Routing" (RouterKind, QuantSpec, WeightLayout,
              MoESpec, the two routing functions, the _swiglu argument order);
  [Skill]     "moe-architecture" skill page (Operating procedure);
  [Compdocs]  "Mixture-of-Experts Documentation" (Core Terms: shared expert);
  [dockyard]  "Mixture-of-Experts" design doc (The pipeline).

Readings where the pages are silent or disagree (kept identical in the design
notes): ties in top-k go to the lower index (the pure-Python listing's stable
sort); capacity = max(1, int(T*k/E*cf)) with k; dropped slots are not
renormalised; f_e counts kept slots / T; P_e for sigmoid routing is the mean
raw sigmoid score (parity unpinned: no page defines it); the 4-bit format
(w = scale*q + bias, q unsigned 0..15, 8 codes per little-endian 32-bit word)
is this project's own (parity of the format itself is by construction).
"""
from __future__ import annotations

import math
from typing import Callable, Mapping, Optional

import numpy as np

SAFE_MARGIN = 1e-4


# ----------------------------------------------------------------------------
# stored values -> float64

def widen(a) -> np.ndarray:
    """Exact widening of a stored array to float64.

    uint16 arrays are bf16 bit patterns: the bf16 value is the float32 whose
    upper 16 bits are those bits.
    """
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def dequant_q4(codes: np.ndarray, scales: np.ndarray, biases: np.ndarray) -> np.ndarray:
    """4-bit affine, group size 64 ([Edge0] QuantSpec bits=4, group_size=64, affine).

    codes  [N, K/8] int32/uint32: element j of a row is the 4-bit field at
           bits 4*(j % 8) of word j // 8 (unsigned 0..15);
    scales [N, K/64], biases [N, K/64]: bf16 bits (or floats);
    returns W [N, K] float64 with W[n, j] = scale[n, j//64] * q[n, j] + bias[n, j//64].
    """
    words = np.asarray(codes).astype(np.int64) & 0xFFFFFFFF
    n_rows, n_words = words.shape
    q = np.empty((n_rows, n_words * 8), dtype=np.float64)
    for j in range(8):
        q[:, j::8] = ((words >> (4 * j)) & 0xF).astype(np.float64)
    s = widen(scales)
    b = widen(biases)
    group = np.arange(q.shape[1]) // 64
    return s[:, group] * q + b[:, group]


# ----------------------------------------------------------------------------
# capacity

def capacity(n_tokens: int, top_k: int, n_experts: int, capacity_factor: float) -> Optional[int]:
    """Per-expert buffer size, max(1, int(T*k/E*cf)) ([MoE blog] moe_layer and
    MoEConfig.capacity_for).  Evaluated left to right in float64 with int()
    truncating.  cf <= 0 means "no capacity limit" and returns None."""
    if capacity_factor is None or capacity_factor <= 0.0:
        return None
    return max(1, int(n_tokens * top_k / n_experts * float(capacity_factor)))


# ----------------------------------------------------------------------------
# router

def router_logits(x, w_router, logit_bias=None) -> np.ndarray:
    """logits = x W_r^T in float64 ([MoE blog] route / Router.route; the gate is
    nn.Linear(hidden, E, bias=False) per [Skill] step 2).  ``logit_bias`` is an
    optional per-expert additive term on the logits (used only to skew the
    Switch-style workload)."""
    logits = widen(x) @ widen(w_router).T
    if logit_bias is not None:
        logits = logits + widen(logit_bias)[None, :]
    return logits


def softmax(logits: np.ndarray) -> np.ndarray:
    """Max-shifted softmax along the expert axis ([MoE blog] softmax)."""
    shifted = logits - logits.max(axis=-1, keepdims=True)
    e = np.exp(shifted)
    return e / e.sum(axis=-1, keepdims=True)


def rank_desc(scores: np.ndarray) -> np.ndarray:
    """Experts ordered by descending score, ties to the lower index (the stable
    sort in [MoE blog] route)."""
    return np.argsort(-scores, axis=-1, kind="stable")


def route_softmax_topk(logits: np.ndarray, top_k: int, norm: bool = True):
    """Softmax top-k with optional renormalisation ([MoE blog] route;
    [Edge0] select_from_logits, norm_topk_prob).

    Returns ids [T,k] (slot j = j-th best), weights [T,k], probabilities [T,E]
    and the selection margin p_(k) - p_(k+1) per token (inf when k == E).
    """
    p = softmax(logits)
    order = rank_desc(p)
    ids = order[:, :top_k]
    chosen = np.take_along_axis(p, ids, axis=-1)
    if norm:
        kept_mass = chosen.sum(axis=-1, keepdims=True)
        weights = chosen / np.maximum(kept_mass, 1e-12)
    else:
        weights = chosen.copy()
    if top_k < p.shape[1]:
        nxt = np.take_along_axis(p, order[:, top_k:top_k + 1], axis=-1)[:, 0]
        margin = chosen[:, -1] - nxt
    else:
        margin = np.full(p.shape[0], np.inf)
    return ids.astype(np.int32), weights, p, margin


def sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


def route_sigmoid_group(logits: np.ndarray, top_k: int, n_group: int, topk_group: int,
                        routed_scaling: float, norm: bool = True, expert_bias=None):
    """Sigmoid scores with group-limited top-k and routed scaling
    ([Edge0] group_select_from_logits).

    Steps, in the page's order:
      s = sigmoid(logits); selection score sel = s + bias (bias optional);
      each group of E/n_group consecutive experts is scored by the sum of its
      two largest sel; the best topk_group groups survive (ties to the lower
      group index) and the others' sel become -inf;
      the top_k experts by sel among the survivors are chosen (ties to the lower
      expert index);
      weights are the chosen experts' raw s (bias excluded), divided by
      (sum + 1e-20) when norm is set, then multiplied by routed_scaling.
    Returns ids [T,k], weights [T,k], s [T,E] and the margin per token: the
    smaller of the expert margin sel_(k) - sel_(k+1) among the survivors and
    the group margin g_(topk_group) - g_(topk_group+1).
    """
    n_tok, n_exp = logits.shape
    s = sigmoid(logits)
    sel = s + (widen(expert_bias)[None, :] if expert_bias is not None else 0.0)
    gsize = n_exp // n_group
    grouped = sel.reshape(n_tok, n_group, gsize)
    top2 = -np.sort(-grouped, axis=-1)[:, :, :2]
    gscore = top2.sum(axis=-1)                                   # [T, n_group]
    gorder = rank_desc(gscore)
    keep_groups = gorder[:, :topk_group]
    gmask = np.zeros((n_tok, n_group), dtype=bool)
    np.put_along_axis(gmask, keep_groups, True, axis=-1)
    emask = np.repeat(gmask, gsize, axis=1)
    masked = np.where(emask, sel, -np.inf)
    order = rank_desc(masked)
    ids = order[:, :top_k]
    weights = np.take_along_axis(s, ids, axis=-1)
    if norm:
        weights = weights / (weights.sum(axis=-1, keepdims=True) + 1e-20)
    weights = weights * routed_scaling
    chosen_sel = np.take_along_axis(masked, ids, axis=-1)
    if top_k < topk_group * gsize:
        nxt = np.take_along_axis(masked, order[:, top_k:top_k + 1], axis=-1)[:, 0]
        e_margin = chosen_sel[:, -1] - nxt
    else:
        e_margin = np.full(n_tok, np.inf)
    if topk_group < n_group:
        gs = np.take_along_axis(gscore, gorder, axis=-1)
        g_margin = gs[:, topk_group - 1] - gs[:, topk_group]
    else:
        g_margin = np.full(n_tok, np.inf)
    return ids.astype(np.int32), weights, s, np.minimum(e_margin, g_margin)


# ----------------------------------------------------------------------------
# dispatch

def dispatch(ids: np.ndarray, n_experts: int, cap: Optional[int], weights=None) -> dict:
    """In-order capacity cut and the expert-sorted permutation.

    Follows [MoE blog] moe_layer: visit tokens in order and each token's chosen
    experts in rank order; a slot joins expert e's list while the list is
    shorter than ``cap``, otherwise it is dropped (it passes through with no
    expert applied).  The lists laid end to end are the permutation of the
    sorted listing (SortedRouting.order / expert_offsets).

    Returns raw_counts[E], kept_counts[E], expert_offsets[E+1], perm_token[R],
    perm_w[R] (when weights are given), slot_row[T,k] (row of the permuted
    buffer, -1 for a dropped slot) and dropped (slot count).
    """
    n_tok, top_k = ids.shape
    lists = [[] for _ in range(n_experts)]
    raw = np.zeros(n_experts, dtype=np.int64)
    dropped = 0
    where = np.full((n_tok, top_k), -1, dtype=np.int64)   # index inside the expert list
    for t in range(n_tok):
        for j in range(top_k):
            e = int(ids[t, j])
            raw[e] += 1
            if cap is not None and len(lists[e]) >= cap:
                dropped += 1
                continue
            where[t, j] = len(lists[e])
            lists[e].append((t, j))
    kept = np.array([len(l) for l in lists], dtype=np.int64)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    perm_token = np.array([t for l in lists for (t, _) in l], dtype=np.int64)
    slot_row = np.full((n_tok, top_k), -1, dtype=np.int64)
    for t in range(n_tok):
        for j in range(top_k):
            if where[t, j] >= 0:
                slot_row[t, j] = offsets[int(ids[t, j])] + where[t, j]
    out = dict(raw_counts=raw, kept_counts=kept, expert_offsets=offsets,
               perm_token=perm_token, slot_row=slot_row, dropped=int(dropped))
    if weights is not None:
        w = np.asarray(weights)
        out["perm_w"] = np.array([w[t, j] for l in lists for (t, j) in l], dtype=np.float64)
    return out


# ----------------------------------------------------------------------------
# experts

def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def expert_mlp(x_rows: np.ndarray, w1: np.ndarray, w3: np.ndarray, act: str,
               w2: Optional[np.ndarray] = None) -> np.ndarray:
    """One expert applied to each row of ``x_rows`` (float64).

    relu:   y = W_out relu(W_in x)                 ([MoE blog] expert_forward)
    swiglu: y = W_down (silu(W_gate x) * (W_up x)) ([Skill] step 1, MistralMLP
            with silu; [Edge0] _swiglu(up, gate) = silu(gate) * up)
    w1 = W_in / W_gate [F, d], w2 = W_up [F, d], w3 = W_out / W_down [d, F].
    No biases.  The intermediate stays in float64.
    """
    if act == "relu":
        h = x_rows @ w1.T
        h = np.where(h > 0.0, h, 0.0)
    elif act == "swiglu":
        h = silu(x_rows @ w1.T) * (x_rows @ w2.T)
    else:
        raise ValueError(act)
    return h @ w3.T


def fuse_gate_up(gate, up) -> np.ndarray:
    """[Edge0] WeightLayout.FUSED_GATE_UP: ONE stacked tensor in which expert
    e's block is its gate rows followed by its up rows, built expert by expert
    ("interleaved expert by expert"), not by putting one whole stack after
    the other.  gate, up [E, F, ...] -> [E, 2F, ...]."""
    gate, up = np.asarray(gate), np.asarray(up)
    assert gate.shape == up.shape
    return np.stack([np.concatenate([gate[e], up[e]], axis=0) for e in range(gate.shape[0])])


def split_gate_up(block: np.ndarray):
    """One expert's fused block [2F, ...] -> (gate, up): the two halves along
    the output axis, gate first ([Edge0] one split(x_gu, 2) gives (gate, up))."""
    block = np.asarray(block)
    half = block.shape[0] // 2
    assert 2 * half == block.shape[0]
    return block[:half], block[half:]


def expert_weights_f64(raw: Mapping, act: str):
    """Widen (or dequantise) one expert's stored weights to float64.  A fused
    gate/up block (key w13, or q13/s13/b13 when 4-bit) is split first."""
    if "w13" in raw or "q13" in raw:
        raw = dict(raw)
        for fused, (a, b) in (("w13", ("w1", "w2")), ("q13", ("q1", "q2")), ("s13", ("s1", "s2")),
                              ("b13", ("b1", "b2"))):
            if fused in raw:
                raw[a], raw[b] = split_gate_up(raw.pop(fused))
    if "q1" in raw:
        w1 = dequant_q4(raw["q1"], raw["s1"], raw["b1"])
        w2 = dequant_q4(raw["q2"], raw["s2"], raw["b2"]) if act == "swiglu" else None
        w3 = dequant_q4(raw["q3"], raw["s3"], raw["b3"])
    else:
        w1 = widen(raw["w1"])
        w2 = widen(raw["w2"]) if act == "swiglu" else None
        w3 = widen(raw["w3"])
    return w1, w2, w3


def combine(n_tokens: int, width: int, ids: np.ndarray, weights: np.ndarray,
            slot_row: np.ndarray, expert_out: Callable[[int, np.ndarray], np.ndarray],
            tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """out[t] = sum over t's kept slots of w_{t,j} * y_{e_j}(x_t)
    ([MoE blog] moe_layer accumulation; the sorted listing's weight-then-
    scatter-add).  A dropped slot adds nothing.  ``expert_out(e, toks)``
    returns expert e's output rows for tokens ``toks``.  Only ``tokens`` (all
    when None) are evaluated; other rows stay 0."""
    toks = np.arange(n_tokens) if tokens is None else np.asarray(tokens)
    out = np.zeros((n_tokens, width), dtype=np.float64)
    by_expert: dict = {}
    for t in toks:
        for j in range(ids.shape[1]):
            if slot_row[t, j] >= 0:
                by_expert.setdefault(int(ids[t, j]), []).append((int(t), j))
    for e in sorted(by_expert):
        pairs = by_expert[e]
        y = expert_out(e, np.array([t for t, _ in pairs]))
        for row, (t, j) in enumerate(pairs):
            out[t] += weights[t, j] * y[row]
    return out


# ----------------------------------------------------------------------------
# balancing loss and health

def aux_loss(kept_counts: np.ndarray, prob_mean: np.ndarray, n_tokens: int,
             n_experts: int, alpha: float):
    """E * sum_e f_e * P_e with f_e = kept count / T (a hard count) and P_e the
    mean router probability over all tokens ([MoE blog] load_balancing_loss,
    _balancing_loss, balancing_loss).  Returns (raw, alpha * raw)."""
    f = np.asarray(kept_counts, dtype=np.float64) / n_tokens
    raw = float(n_experts * np.sum(f * np.asarray(prob_mean, dtype=np.float64)))
    return raw, alpha * raw


def routing_health(kept_counts: np.ndarray, dropped: int, n_tokens: int, top_k: int,
                   n_experts: int) -> dict:
    """Shares, entropy over the kept-slot histogram, entropy ratio against log E,
    max share, dropped fraction and the collapse flag (ratio < 0.5)
    ([MoE blog] routing_health / RoutingHealth)."""
    counts = np.asarray(kept_counts, dtype=np.float64)
    total = counts.sum()
    if total <= 0.0:
        return dict(entropy_ratio=0.0, max_share=0.0, dropped_fraction=1.0, collapsed=True)
    shares = counts / total
    nz = shares[shares > 0.0]
    entropy = float(-np.sum(nz * np.log(nz)))
    max_entropy = math.log(n_experts)
    ratio = entropy / max_entropy if max_entropy > 0.0 else 0.0
    return dict(entropy_ratio=ratio, max_share=float(shares.max()),
                dropped_fraction=dropped / max(1, n_tokens * top_k), collapsed=ratio < 0.5)


# ----------------------------------------------------------------------------
# the layer

def route(x, w_router, *, top_k: int, router: str = "softmax_topk", norm: bool = True,
          routed_scaling: float = 1.0, n_group: int = 1, topk_group: int = 1,
          expert_bias=None, logit_bias=None) -> dict:
    """The router step of [dockyard] The pipeline (1): logits, scores,
    selection and weights.  Returns ids, weights, probs (the router's
    per-expert probability used for P_e), margin and logits."""
    logits = router_logits(x, w_router, logit_bias)
    if router == "softmax_topk":
        ids, w, p, margin = route_softmax_topk(logits, top_k, norm)
    elif router == "sigmoid_group":
        ids, w, p, margin = route_sigmoid_group(logits, top_k, n_group, topk_group,
                                                routed_scaling, norm, expert_bias)
    else:
        raise ValueError(router)
    return dict(ids=ids, weights=w, probs=p, margin=margin, logits=logits,
                prob_sum=p.sum(axis=0))


def route_forced(x, w_router, forced_ids, *, top_k: int, router: str = "softmax_topk",
                 norm: bool = True, routed_scaling: float = 1.0, logit_bias=None) -> dict:
    """Router replay ([dockyard] Router replay (R3)): the expert ids are the
    recorded ones, the weights come from this router's own gate.

    The scores are those of ``route`` (softmax probabilities, or raw sigmoid
    scores); slot j of token t takes expert forced_ids[t, j] with the score
    of that expert, then the same renormalisation (and routed scaling) as the
    free router.  The selection bias and the group limit take no part: they
    only choose experts.  A recorded id outside [0, E), or one repeated in its
    row, is a bad route: the slot's weight is 0 and it is left out of the
    normalising sum; ``bad`` [T, k] marks such slots (the caller must reject
    them, never replay them silently).  Margins are +inf: nothing is chosen.
    """
    logits = router_logits(x, w_router, logit_bias)
    ids = np.asarray(forced_ids, dtype=np.int64)
    n_tok, n_exp = logits.shape
    assert ids.shape == (n_tok, top_k)
    scores = softmax(logits) if router == "softmax_topk" else sigmoid(logits)
    weights = np.zeros((n_tok, top_k), dtype=np.float64)
    bad = np.zeros((n_tok, top_k), dtype=bool)
    for t in range(n_tok):
        seen = set()
        for j in range(top_k):
            e = int(ids[t, j])
            if e < 0 or e >= n_exp or e in seen:
                bad[t, j] = True
                continue
            seen.add(e)
            weights[t, j] = scores[t, e]
    total = weights.sum(axis=-1, keepdims=True)
    if router == "softmax_topk":
        if norm:
            weights = weights / np.maximum(total, 1e-12)
    else:
        if norm:
            weights = weights / (total + 1e-20)
        weights = weights * routed_scaling
    return dict(ids=ids.astype(np.int32), weights=weights, probs=scores, bad=bad,
                margin=np.full(n_tok, np.inf), logits=logits, prob_sum=scores.sum(axis=0))


def update_bias(bias, counts, coeff: float) -> np.ndarray:
    """One step of the aux-loss-free balancing bias ([dockyard] Aux-loss-free
    load balancing): an expert that took fewer assignments than the mean
    count goes up by ``coeff``, one that took more goes down by ``coeff``, one
    exactly at the mean stays.  The mean is compared as an exact fraction.
    The bias is a float32 parameter: the new value is the float64 result
    rounded to float32 (a single rounding for the sizes used here)."""
    from fractions import Fraction
    counts = [int(c) for c in np.asarray(counts).ravel()]
    mean = Fraction(sum(counts), len(counts))
    b = np.asarray(bias, dtype=np.float32).astype(np.float64)
    out = np.empty(len(counts), dtype=np.float32)
    for e, c in enumerate(counts):
        step = 1.0 if c < mean else (-1.0 if c > mean else 0.0)
        out[e] = np.float32(b[e] + step * float(np.float32(coeff)))
    return out


def layer_forward(x, w_router, experts: Callable[[int], Mapping], *, top_k: int, act: str,
                  capacity_factor: float = 0.0, router: str = "softmax_topk",
                  norm: bool = True, routed_scaling: float = 1.0, n_group: int = 1,
                  topk_group: int = 1, expert_bias=None, logit_bias=None,
                  shared: Optional[Mapping] = None, aux_alpha: float = 0.01,
                  tokens: Optional[np.ndarray] = None, routing: Optional[dict] = None) -> dict:
    """route -> dispatch -> expert MLPs -> combine ([dockyard] The pipeline),
    plus the shared expert on every token with weight 1 ([Compdocs] shared
    expert) and the balancing loss.

    ``experts(e)`` returns expert e's stored weights (keys w1/w2/w3 or
    q1/s1/b1 ...); ``shared`` holds ws1/ws2/ws3 for a shared SwiGLU expert.
    ``tokens`` restricts the expert evaluation to a subset of rows (routing
    and dispatch always cover the whole batch, because capacity depends on
    it); ``routing`` replaces the oracle's own routing (ids, weights, probs) to
    check later stages on another router's decisions.
    """
    xf = widen(x)
    n_tok, width = xf.shape
    n_exp = np.asarray(w_router).shape[0]
    r = routing if routing is not None else route(
        x, w_router, top_k=top_k, router=router, norm=norm, routed_scaling=routed_scaling,
        n_group=n_group, topk_group=topk_group, expert_bias=expert_bias, logit_bias=logit_bias)
    cap = capacity(n_tok, top_k, n_exp, capacity_factor)
    disp = dispatch(np.asarray(r["ids"]), n_exp, cap, r["weights"])

    cache: dict = {}

    def expert_out(e: int, toks: np.ndarray) -> np.ndarray:
        if e not in cache:
            cache.clear()          # one expert's float64 weights at a time
            cache[e] = expert_weights_f64(experts(e), act)
        w1, w2, w3 = cache[e]
        return expert_mlp(xf[toks], w1, w3, act, w2)

    out = combine(n_tok, width, np.asarray(r["ids"]), np.asarray(r["weights"], dtype=np.float64),
                  disp["slot_row"], expert_out, tokens)
    if shared is not None:
        toks = np.arange(n_tok) if tokens is None else np.asarray(tokens)
        out[toks] += expert_mlp(xf[toks], widen(shared["ws1"]), widen(shared["ws3"]), "swiglu",
                                widen(shared["ws2"]))
    prob_mean = np.asarray(r["probs"], dtype=np.float64).mean(axis=0)
    aux_raw, aux = aux_loss(disp["kept_counts"], prob_mean, n_tok, n_exp, aux_alpha)
    health = routing_health(disp["kept_counts"], disp["dropped"], n_tok, top_k, n_exp)
    return dict(out=out, routing=r, dispatch=disp, capacity=cap, aux_raw=aux_raw, aux=aux,
                health=health)
