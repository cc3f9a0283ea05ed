"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` takes the oracle module and raises AssertionError on a
mismatch.  They are run on the real oracle (test_oracle_pins.py) and on
deliberately broken copies of it (test_oracle_mutants.py), which must each
fail at least one pin.

What pins what:
  * hand-worked fixtures under tests/golden/ (exact rationals derived from
    the pages' definitions, with citations);
  * independent library routines: scipy's softmax, torch's silu / linear;
  * brute force: best-subset enumeration for top-k and group-limited top-k,
    dense evaluation of every expert masked by the kept top-k weights;
  * closed forms: capacity at the pages' shapes, balanced and collapsed
    balancing losses, renormalised weights summing to 1 (or routed_scaling);
  * cross-agreement with the two other formulations of the drop rule on the
    pages (per-expert nonzero truncation; stable argsort with per-expert
    cursors).
"""
from __future__ import annotations

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _num(v) -> float:
    """Decode a fixture number: floats, 'a/b' rationals, 'lnN' / '-lnN'."""
    if isinstance(v, (int, float)):
        return float(v)
    s = str(v)
    neg = s.startswith("-")
    if neg:
        s = s[1:]
    if s.startswith("ln"):
        val = math.log(float(s[2:]))
    else:
        val = float(Fraction(s))
    return -val if neg else val


def _arr(v) -> np.ndarray:
    return np.vectorize(_num, otypes=[np.float64])(np.array(v, dtype=object))


def _load(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


def _rng(seed=0):
    return np.random.default_rng(seed)


def _tiny_layer(rng, T=24, d=6, F=5, E=4, k=2, act="relu"):
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d))
    w1 = rng.standard_normal((E, F, d)) * 0.5
    w2 = rng.standard_normal((E, F, d)) * 0.5
    w3 = rng.standard_normal((E, d, F)) * 0.5
    experts = lambda e: dict(w1=w1[e], w2=w2[e], w3=w3[e])
    return x, wr, w1, w2, w3, experts


# ---------------------------------------------------------------- fixtures

def pin_hand_softmax_top2_capacity(O):
    g = _load("hand_softmax_top2_capacity.json")
    inp, exp = g["inputs"], g["expected"]
    x = _arr(inp["x"])
    wr = _arr(inp["w_router"])
    scales = inp["w_in_scale_per_expert"]
    E = wr.shape[0]
    d = x.shape[1]
    experts = lambda e: dict(w1=np.eye(d) * scales[e], w3=np.eye(d))
    res = O.layer_forward(x, wr, experts, top_k=inp["top_k"], act=inp["act"],
                          capacity_factor=inp["capacity_factor"], aux_alpha=inp["alpha"])
    r, dsp = res["routing"], res["dispatch"]
    assert np.array_equal(r["ids"], np.array(exp["ids"])), r["ids"]
    assert np.allclose(r["weights"], _arr(exp["weights"]), rtol=0, atol=1e-12)
    assert res["capacity"] == exp["capacity"]
    assert dsp["dropped"] == exp["dropped"]
    assert np.array_equal(dsp["kept_counts"], exp["kept_counts"])
    assert np.array_equal(dsp["expert_offsets"], exp["expert_offsets"])
    assert np.array_equal(dsp["perm_token"], exp["perm_token"])
    assert np.array_equal(dsp["slot_row"], np.array(exp["slot_row"]))
    assert np.allclose(res["out"], _arr(exp["out"]), rtol=0, atol=1e-12), res["out"]
    assert abs(res["aux_raw"] - _num(exp["aux_raw"])) < 1e-12
    assert abs(res["aux"] - _num(exp["aux"])) < 1e-14
    assert E == 3


def pin_hand_sigmoid_group(O):
    g = _load("hand_sigmoid_group.json")
    inp, exp = g["inputs"], g["expected"]
    logits = _arr(inp["logits"])[None, :]
    for case, bias in (("no_bias", None), ("bias", np.array(exp["bias"]["bias"]))):
        ids, w, s, _ = O.route_sigmoid_group(logits, inp["top_k"], inp["n_group"],
                                             inp["topk_group"], inp["routed_scaling"], True, bias)
        assert list(ids[0]) == exp[case]["ids"], (case, ids)
        assert np.allclose(w[0], _arr(exp[case]["weights"]), rtol=0, atol=1e-12), (case, w)


# ---------------------------------------------------------------- router

def pin_softmax_textbook(O):
    from scipy.special import softmax as sp_softmax
    rng = _rng(1)
    logits = rng.standard_normal((50, 9)) * 4.0
    assert np.allclose(O.softmax(logits), sp_softmax(logits, axis=-1), rtol=1e-13, atol=0)
    # large logits must not overflow (the max shift)
    big = np.array([[1000.0, 999.0, 0.0]])
    p = O.softmax(big)
    assert np.all(np.isfinite(p)) and abs(p.sum() - 1.0) < 1e-15


def pin_softmax_topk_bruteforce(O):
    rng = _rng(2)
    for E, k in ((4, 1), (5, 2), (6, 3), (8, 2)):
        logits = rng.standard_normal((40, E)) * 2.0
        ids, w, p, margin = O.route_softmax_topk(logits, k, True)
        assert np.allclose(p.sum(axis=1), 1.0, atol=1e-14)
        for t in range(logits.shape[0]):
            best = max(itertools.combinations(range(E), k), key=lambda c: sum(p[t, list(c)]))
            assert set(ids[t]) == set(best)
            # slots in rank order
            assert all(p[t, ids[t, j]] >= p[t, ids[t, j + 1]] for j in range(k - 1))
            assert abs(w[t].sum() - 1.0) < 1e-14
            assert np.allclose(w[t], p[t, ids[t]] / p[t, ids[t]].sum(), rtol=1e-14)
            rest = [e for e in range(E) if e not in ids[t]]
            if rest:
                assert abs(margin[t] - (p[t, ids[t, -1]] - max(p[t, rest]))) < 1e-15


def pin_softmax_topk_special_cases(O):
    rng = _rng(3)
    logits = rng.standard_normal((20, 6))
    # k == E with renormalisation returns the full softmax in rank order
    ids, w, p, _ = O.route_softmax_topk(logits, 6, True)
    assert np.allclose(np.take_along_axis(p, ids, 1), w, rtol=1e-14)
    # k == 1 with renormalisation: weight 1
    ids, w, p, _ = O.route_softmax_topk(logits, 1, True)
    assert np.allclose(w, 1.0, atol=1e-15)
    assert np.array_equal(ids[:, 0], np.argmax(p, axis=1))
    # without renormalisation the weights are the raw probabilities
    ids, w, p, _ = O.route_softmax_topk(logits, 2, False)
    assert np.allclose(w, np.take_along_axis(p, ids, 1), rtol=0, atol=0)
    # ties go to the lower expert index
    tie = np.array([[0.5, 1.0, 1.0, 0.0]])
    ids, _, _, _ = O.route_softmax_topk(tie, 1, True)
    assert ids[0, 0] == 1


def _group_bruteforce(sel, s, k, n_group, topk_group, scaling):
    E = sel.shape[0]
    gsize = E // n_group
    gscore = []
    for g in range(n_group):
        vals = sorted(sel[g * gsize:(g + 1) * gsize], reverse=True)
        gscore.append(vals[0] + vals[1])
    best_groups = max(itertools.combinations(range(n_group), topk_group),
                      key=lambda c: sum(gscore[i] for i in c))
    pool = [e for g in best_groups for e in range(g * gsize, (g + 1) * gsize)]
    best = max(itertools.combinations(pool, k), key=lambda c: sum(sel[list(c)]))
    w = s[list(best)]
    w = w / (w.sum() + 1e-20) * scaling
    return set(best), dict(zip(best, w))


def pin_sigmoid_group_bruteforce(O):
    rng = _rng(4)
    for (E, n_group, topk_group, k) in ((8, 4, 2, 3), (12, 3, 2, 4), (16, 4, 1, 2), (8, 2, 2, 5)):
        logits = rng.standard_normal((30, E)) * 2.0
        bias = rng.uniform(-0.3, 0.3, E)
        ids, w, s, _ = O.route_sigmoid_group(logits, k, n_group, topk_group, 2.5, True, bias)
        assert np.allclose(s, 1.0 / (1.0 + np.exp(-logits)), rtol=1e-15)
        for t in range(logits.shape[0]):
            sel = s[t] + bias
            chosen, wmap = _group_bruteforce(sel, s[t], k, n_group, topk_group, 2.5)
            assert set(ids[t]) == chosen, (t, ids[t], chosen)
            for j in range(k):
                assert abs(w[t, j] - wmap[ids[t, j]]) < 1e-13
            assert abs(w[t].sum() - 2.5) < 1e-13
            assert all(sel[ids[t, j]] >= sel[ids[t, j + 1]] for j in range(k - 1))


def _group_margin_bruteforce(sel, k, n_group, topk_group):
    """The parity margin of one token, by enumeration: the smaller of the
    group margin (topk_group-th best group score minus the next best, over
    every group; +inf when every group survives) and the expert margin (k-th
    best selection score minus the (k+1)-th among the experts of the best
    groups; +inf when the survivors number exactly k)."""
    E = sel.shape[0]
    gsize = E // n_group
    gscore = []
    for g in range(n_group):
        vals = sorted(sel[g * gsize:(g + 1) * gsize], reverse=True)
        gscore.append(vals[0] + vals[1])
    best_groups = max(itertools.combinations(range(n_group), topk_group),
                      key=lambda c: sum(gscore[i] for i in c))
    ranked = sorted(gscore, reverse=True)
    g_margin = ranked[topk_group - 1] - ranked[topk_group] if topk_group < n_group else math.inf
    pool = sorted((sel[e] for g in best_groups for e in range(g * gsize, (g + 1) * gsize)), reverse=True)
    e_margin = pool[k - 1] - pool[k] if k < len(pool) else math.inf
    return min(g_margin, e_margin), g_margin, e_margin


def pin_sigmoid_group_margin(O):
    """The margin that decides which tokens' ids must match bit for bit
    ([Edge0] group_select_from_logits: the cut between kept and dropped groups
    and the cut between the k-th and (k+1)-th expert are both decisions), by
    brute force over the groups, on the selection score (bias included).
    Both kinds of cut must be the smaller one on some tokens, so that a margin
    that leaves one of them out, or is measured on the raw score, fails."""
    rng = _rng(24)
    group_decides = expert_decides = 0
    for (E, n_group, topk_group, k) in ((8, 4, 2, 3), (12, 3, 2, 4), (16, 4, 1, 2), (16, 8, 3, 5),
                                        (8, 2, 2, 5), (6, 3, 1, 2)):
        logits = rng.standard_normal((60, E)) * 1.5
        bias = rng.uniform(-0.4, 0.4, E)
        _, _, s, margin = O.route_sigmoid_group(logits, k, n_group, topk_group, 2.5, True, bias)
        for t in range(logits.shape[0]):
            ref, g_m, e_m = _group_margin_bruteforce(s[t] + bias, k, n_group, topk_group)
            assert abs(margin[t] - ref) < 1e-13 or (math.isinf(ref) and math.isinf(margin[t])), \
                (E, n_group, topk_group, k, t, margin[t], ref)
            group_decides += g_m < e_m
            expert_decides += e_m < g_m
    assert group_decides > 20 and expert_decides > 20, (group_decides, expert_decides)
    # every group kept and exactly k survivors: nothing can flip
    _, _, _, m = O.route_sigmoid_group(rng.standard_normal((5, 8)), 8, 4, 4, 1.0, True, None)
    assert np.all(np.isinf(m))


def pin_sigmoid_group_reductions(O):
    rng = _rng(5)
    logits = rng.standard_normal((25, 8))
    # every group kept (topk_group == n_group) or one group: plain sigmoid top-k
    for n_group, topk_group in ((4, 4), (1, 1), (2, 2)):
        ids, w, s, _ = O.route_sigmoid_group(logits, 3, n_group, topk_group, 1.0, False, None)
        plain = np.argsort(-s, axis=1, kind="stable")[:, :3]
        assert np.array_equal(ids, plain)
        assert np.allclose(w, np.take_along_axis(s, plain, 1), rtol=0, atol=0)
    # the bias moves selection but never the weights
    bias = np.zeros(8)
    bias[7] = 10.0
    ids, w, s, _ = O.route_sigmoid_group(logits, 2, 4, 2, 1.0, False, bias)
    assert np.all(ids[:, 0] == 7)
    assert np.allclose(w[:, 0], s[:, 7], rtol=0, atol=0)


# ---------------------------------------------------------------- capacity / dispatch

def pin_capacity_closed_forms(O):
    assert O.capacity(64, 2, 4, 1.25) == 40          # tiny workload
    assert O.capacity(8192, 1, 64, 1.0) == 128        # Switch-style workload
    assert O.capacity(3, 1, 4, 1.0) == 1              # max(1, int(0.75))
    assert O.capacity(10, 2, 4, 1.5) == 7             # int(7.5)
    assert O.capacity(4096, 2, 8, 0.0) is None        # no limit


def _drops_nonzero_style(ids, E, cap):
    """Per expert: slots in row-major nonzero order, the first ``cap`` kept
    (the class-based listing's truncation)."""
    kept = {}
    dropped = 0
    for e in range(E):
        pos, ranks = np.nonzero(ids == e)
        if cap is not None and pos.size > cap:
            dropped += pos.size - cap
            pos, ranks = pos[:cap], ranks[:cap]
        kept[e] = list(zip(pos.tolist(), ranks.tolist()))
    return kept, dropped


def _drops_argsort_style(ids, E, cap):
    """Stable argsort of the flat token-major slots by expert, then a cursor
    per expert (the sorted listing's route_and_sort)."""
    T, k = ids.shape
    flat = ids.reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    keep = np.ones(order.size, dtype=bool)
    cursor = 0
    dropped = 0
    for e in range(E):
        c = int(counts[e])
        if cap is not None and c > cap:
            keep[cursor + cap:cursor + c] = False
            dropped += c - cap
        cursor += c
    kept_order = order[keep]
    return [int(s // k) for s in kept_order], [int(s % k) for s in kept_order], dropped


def pin_dispatch_cross_agreement(O):
    rng = _rng(6)
    for T, E, k, cf in ((50, 4, 2, 1.0), (64, 8, 3, 1.25), (33, 5, 1, 1.0), (40, 6, 2, 0.0)):
        logits = rng.standard_normal((T, E)) + rng.standard_normal(E) * 2.0
        ids, w, _, _ = O.route_softmax_topk(logits, k, True)
        cap = O.capacity(T, k, E, cf)
        dsp = O.dispatch(ids, E, cap, w)
        kept_nz, dropped_nz = _drops_nonzero_style(ids, E, cap)
        toks, ranks, dropped_as = _drops_argsort_style(ids, E, cap)
        assert dsp["dropped"] == dropped_nz == dropped_as
        assert dsp["perm_token"].tolist() == toks
        assert dsp["perm_token"].tolist() == [t for e in range(E) for (t, _) in kept_nz[e]]
        assert np.allclose(dsp["perm_w"], [w[t, j] for t, j in zip(toks, ranks)], rtol=0, atol=0)
        for r, (t, j) in enumerate(zip(toks, ranks)):
            assert dsp["slot_row"][t, j] == r
        assert int((dsp["slot_row"] >= 0).sum()) == len(toks)


def pin_dispatch_invariants(O):
    rng = _rng(7)
    T, E, k = 60, 5, 2
    logits = rng.standard_normal((T, E)) + np.array([2.0, 1.0, 0.0, -1.0, -2.0])
    ids, w, _, _ = O.route_softmax_topk(logits, k, True)
    for cap in (1, 7, 20, None):
        dsp = O.dispatch(ids, E, cap, w)
        assert dsp["kept_counts"].sum() + dsp["dropped"] == T * k
        assert np.array_equal(dsp["raw_counts"], np.bincount(ids.reshape(-1), minlength=E))
        if cap is None:
            assert dsp["dropped"] == 0
        else:
            assert np.all(dsp["kept_counts"] <= cap)
        off = dsp["expert_offsets"]
        for e in range(E):
            toks = dsp["perm_token"][off[e]:off[e + 1]]
            users = sorted(set(np.nonzero(ids == e)[0].tolist()))
            # kept tokens are the earliest users of the expert, ascending
            assert toks.tolist() == users[:len(toks)]
        if cap == 1:
            for e in range(E):
                users = np.nonzero((ids == e).any(axis=1))[0]
                if users.size:
                    assert dsp["perm_token"][off[e]] == users[0] and off[e + 1] - off[e] == 1


# ---------------------------------------------------------------- experts / combine

def _dense_masked(x, wr_ids, weights, slot_row, w1, w2, w3, act):
    """Every expert on every token (torch, float64), masked by the kept top-k
    weights."""
    import torch
    import torch.nn.functional as Fn
    xt = torch.from_numpy(x)
    T, k = wr_ids.shape
    E = w1.shape[0]
    mask = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            if slot_row[t, j] >= 0:
                mask[t, wr_ids[t, j]] += weights[t, j]
    out = torch.zeros_like(xt)
    for e in range(E):
        a = Fn.linear(xt, torch.from_numpy(w1[e]))
        if act == "relu":
            h = Fn.relu(a)
        else:
            h = Fn.silu(a) * Fn.linear(xt, torch.from_numpy(w2[e]))
        y = Fn.linear(h, torch.from_numpy(w3[e]))
        out += torch.from_numpy(mask[:, e:e + 1]) * y
    return out.numpy()


def pin_dense_bruteforce(O):
    rng = _rng(8)
    for act, cf in (("relu", 1.0), ("swiglu", 1.25), ("relu", 0.0)):
        x, wr, w1, w2, w3, experts = _tiny_layer(rng, act=act)
        skew = np.array([1.5, 0.5, 0.0, -0.5])      # hot expert 0 overflows at cf = 1
        res = O.layer_forward(x, wr, experts, top_k=2, act=act, capacity_factor=cf,
                              logit_bias=skew)
        r, dsp = res["routing"], res["dispatch"]
        ref = _dense_masked(x, r["ids"], r["weights"], dsp["slot_row"], w1, w2, w3, act)
        assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-12)
        if cf == 1.0:
            assert dsp["dropped"] > 0
        # a token with every slot dropped outputs exactly zero
        for t in range(x.shape[0]):
            if np.all(dsp["slot_row"][t] < 0):
                assert np.all(res["out"][t] == 0.0)


def pin_single_expert_is_plain_mlp(O):
    import torch
    rng = _rng(9)
    T, d, F = 7, 5, 6
    x = rng.standard_normal((T, d))
    w1 = rng.standard_normal((F, d))
    w2 = rng.standard_normal((F, d))
    w3 = rng.standard_normal((d, F))
    wr = np.zeros((2, d))
    # expert 0 always wins: logit bias
    lb = np.array([50.0, 0.0])
    for act in ("relu", "swiglu"):
        experts = lambda e: dict(w1=w1, w2=w2, w3=w3)
        res = O.layer_forward(x, wr, experts, top_k=1, act=act, logit_bias=lb)
        mlp = torch.nn.Linear(d, F, bias=False).double()
        up = torch.nn.Linear(d, F, bias=False).double()
        down = torch.nn.Linear(F, d, bias=False).double()
        with torch.no_grad():
            mlp.weight.copy_(torch.from_numpy(w1))
            up.weight.copy_(torch.from_numpy(w2))
            down.weight.copy_(torch.from_numpy(w3))
            xt = torch.from_numpy(x)
            h = torch.relu(mlp(xt)) if act == "relu" else torch.nn.functional.silu(mlp(xt)) * up(xt)
            ref = down(h).numpy()
        assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-12)


def pin_swiglu_argument_order(O):
    """silu goes on the gate projection, not the up projection (Edge0 _swiglu(up, gate))."""
    import torch
    rng = _rng(10)
    x = rng.standard_normal((4, 3))
    wg = rng.standard_normal((5, 3))
    wu = rng.standard_normal((5, 3))
    wd = rng.standard_normal((3, 5))
    y = O.expert_mlp(x, wg, wd, "swiglu", wu)
    xt = torch.from_numpy(x)
    ref = (torch.nn.functional.silu(xt @ torch.from_numpy(wg).T) * (xt @ torch.from_numpy(wu).T)) @ torch.from_numpy(wd).T
    assert np.allclose(y, ref.numpy(), rtol=1e-13, atol=1e-13)
    swapped = (torch.nn.functional.silu(xt @ torch.from_numpy(wu).T) * (xt @ torch.from_numpy(wg).T)) @ torch.from_numpy(wd).T
    assert not np.allclose(y, swapped.numpy(), rtol=1e-3)


def pin_shared_expert_adds_everywhere(O):
    rng = _rng(11)
    x, wr, w1, w2, w3, experts = _tiny_layer(rng, act="swiglu")
    d = x.shape[1]
    shared = dict(ws1=rng.standard_normal((3, d)), ws2=rng.standard_normal((3, d)),
                  ws3=rng.standard_normal((d, 3)))
    a = O.layer_forward(x, wr, experts, top_k=2, act="swiglu")
    b = O.layer_forward(x, wr, experts, top_k=2, act="swiglu", shared=shared)
    import torch
    import torch.nn.functional as Fn
    xt = torch.from_numpy(x)
    sh = Fn.linear(Fn.silu(Fn.linear(xt, torch.from_numpy(shared["ws1"]))) *
                   Fn.linear(xt, torch.from_numpy(shared["ws2"])), torch.from_numpy(shared["ws3"]))
    assert np.allclose(b["out"] - a["out"], sh.numpy(), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- balancing loss

def pin_aux_closed_forms(O):
    E, k, T = 4, 2, 8
    # balanced: every expert gets T*k/E kept slots and p is uniform -> E * sum (k/E)(1/E) = k
    raw, scaled = O.aux_loss(np.full(E, T * k // E), np.full(E, 1.0 / E), T, E, 0.01)
    assert abs(raw - k) < 1e-15 and abs(scaled - 0.01 * k) < 1e-17
    # collapsed: every token to experts 0 and 1 with p = (1/2, 1/2, 0, 0) -> E * (1*1/2 + 1*1/2) = E
    raw, _ = O.aux_loss(np.array([T, T, 0, 0]), np.array([0.5, 0.5, 0.0, 0.0]), T, E, 0.01)
    assert abs(raw - E) < 1e-15
    # through the layer: f_e uses KEPT counts (after the capacity cut) and P_e all tokens
    rng = _rng(12)
    x, wr, w1, w2, w3, experts = _tiny_layer(rng, T=40)
    wr = wr + np.array([3.0, 0.0, 0.0, 0.0])[:, None]
    res = O.layer_forward(x, wr, experts, top_k=2, act="relu", capacity_factor=1.0, aux_alpha=0.02)
    dsp, r = res["dispatch"], res["routing"]
    assert dsp["dropped"] > 0
    f = dsp["kept_counts"] / 40.0
    P = r["probs"].mean(axis=0)
    assert abs(res["aux_raw"] - 4 * float(np.dot(f, P))) < 1e-14
    assert abs(res["aux"] - 0.02 * res["aux_raw"]) < 1e-16
    # without drops sum f = k
    res = O.layer_forward(x, wr, experts, top_k=2, act="relu")
    assert abs(res["dispatch"]["kept_counts"].sum() / 40.0 - 2.0) < 1e-15


def pin_health(O):
    h = O.routing_health(np.array([5, 5, 5, 5]), 0, 10, 2, 4)
    assert abs(h["entropy_ratio"] - 1.0) < 1e-15 and not h["collapsed"]
    h = O.routing_health(np.array([20, 0, 0, 0]), 0, 10, 2, 4)
    assert h["entropy_ratio"] == 0.0 and h["collapsed"] and h["max_share"] == 1.0
    h = O.routing_health(np.array([3, 3, 0, 0]), 14, 10, 2, 4)
    assert abs(h["dropped_fraction"] - 0.7) < 1e-15
    assert abs(h["entropy_ratio"] - math.log(2) / math.log(4)) < 1e-15


# ---------------------------------------------------------------- 4-bit weights

def _pack_py(q_row):
    words = []
    for w0 in range(0, len(q_row), 8):
        v = 0
        for j in range(8):
            v |= int(q_row[w0 + j]) << (4 * j)
        words.append(v - (1 << 32) if v >= (1 << 31) else v)
    return words


def pin_q4_roundtrip(O):
    rng = _rng(13)
    N, K = 3, 128
    q = rng.integers(0, 16, (N, K))
    # exactly representable scales / biases (bf16 bit patterns of 2^-6, -3*2^-5 ...)
    def bf16_bits(v):
        return np.array(v, dtype=np.float32).view(np.uint32).__rshift__(16).astype(np.uint16)
    scale = np.array([[2.0 ** -6, 2.0 ** -5], [0.75, 0.5], [1.0, 2.0 ** -8]], dtype=np.float32)
    bias = np.array([[-0.125, 0.25], [-6.0, 1.0], [0.0, -0.5]], dtype=np.float32)
    codes = np.array([_pack_py(row) for row in q], dtype=np.int64).astype(np.int32)
    W = O.dequant_q4(codes, bf16_bits(scale), bf16_bits(bias))
    g = np.arange(K) // 64
    expect = scale.astype(np.float64)[:, g] * q + bias.astype(np.float64)[:, g]
    assert np.array_equal(W, expect)
    # the affine grid round-trips: q = (W - bias) / scale exactly
    assert np.array_equal((W - bias.astype(np.float64)[:, g]) / scale.astype(np.float64)[:, g], q)


# ---------------------------------------------------------------- weight layout

def pin_fused_gate_up_split(O):
    """The fused layout's projection splits into (gate, up) per expert: checked
    by brute force with torch's linear on the separate stacks."""
    import torch
    rng = _rng(21)
    E, F, d = 3, 4, 5
    gate = rng.standard_normal((E, F, d))
    up = rng.standard_normal((E, F, d))
    fused = O.fuse_gate_up(gate, up)
    assert fused.shape == (E, 2 * F, d)
    x = rng.standard_normal((7, d))
    for e in range(E):
        xg = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(gate[e])).numpy()
        xu = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(up[e])).numpy()
        xgu = x @ fused[e].T
        assert np.allclose(xgu[:, :F], xg, rtol=0, atol=1e-12) and np.allclose(xgu[:, F:], xu, rtol=0, atol=1e-12)
        g2, u2 = O.split_gate_up(fused[e])
        assert np.array_equal(g2, gate[e]) and np.array_equal(u2, up[e])
        w3 = rng.standard_normal((d, F))
        a = O.expert_weights_f64(dict(w13=fused[e], w3=w3), "swiglu")
        b = O.expert_weights_f64(dict(w1=gate[e], w2=up[e], w3=w3), "swiglu")
        assert all(np.array_equal(p, q) for p, q in zip(a, b))


# ---------------------------------------------------------------- router replay

def pin_route_forced_replays_free_route(O):
    """Replaying the free router's own choices gives its weights back (the free
    router is pinned by brute force above); a permuted replay permutes them."""
    rng = _rng(22)
    x = rng.standard_normal((30, 6))
    wr = rng.standard_normal((8, 6))
    bias = rng.uniform(-0.3, 0.3, 8)
    for kw in (dict(router="softmax_topk", norm=True), dict(router="softmax_topk", norm=False),
               dict(router="sigmoid_group", norm=True, routed_scaling=2.5, n_group=4, topk_group=2,
                    expert_bias=bias)):
        free = O.route(x, wr, top_k=3, **kw)
        fkw = {k_: v for k_, v in kw.items() if k_ not in ("n_group", "topk_group", "expert_bias")}
        rep = O.route_forced(x, wr, free["ids"], top_k=3, **fkw)
        assert np.array_equal(rep["ids"], free["ids"]) and not rep["bad"].any()
        assert np.allclose(rep["weights"], free["weights"], rtol=1e-13, atol=0), kw
        assert np.allclose(rep["prob_sum"], free["prob_sum"], rtol=1e-13, atol=0)
        perm = free["ids"][:, ::-1].copy()
        rep2 = O.route_forced(x, wr, perm, top_k=3, **fkw)
        assert np.allclose(rep2["weights"], free["weights"][:, ::-1], rtol=1e-13, atol=0)


def pin_route_forced_bad_ids(O):
    """A sentinel or repeated recorded id is flagged, weighted 0 and left out of
    the renormalisation (closed form: the remaining weights sum to 1)."""
    rng = _rng(23)
    x = rng.standard_normal((3, 5))
    wr = rng.standard_normal((6, 5))
    ids = np.array([[0, 1, 2], [-1, 3, 4], [5, 5, 2]], dtype=np.int32)
    rep = O.route_forced(x, wr, ids, top_k=3, router="softmax_topk", norm=True)
    assert rep["bad"].tolist() == [[False] * 3, [True, False, False], [False, True, False]]
    assert rep["weights"][1, 0] == 0.0 and rep["weights"][2, 1] == 0.0
    assert np.allclose(rep["weights"].sum(axis=1), 1.0, rtol=0, atol=1e-15)
    p = np.exp(x @ wr.T - (x @ wr.T).max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert abs(rep["weights"][1, 1] - p[1, 3] / (p[1, 3] + p[1, 4])) < 1e-15


# ---------------------------------------------------------------- balancing bias

def pin_hand_bias_update(O):
    g = _load("hand_bias_update.json")
    for case in g["cases"]:
        bias = _arr(case["bias"]).astype(np.float32)
        out = O.update_bias(bias, np.array(case["counts"]), _num(case["coeff"]))
        assert out.dtype == np.float32
        assert np.array_equal(out.astype(np.float64), _arr(case["expected"])), (case, out)


PINS = [v for k_, v in sorted(globals().items()) if k_.startswith("pin_")]
