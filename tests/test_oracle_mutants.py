"""Plant plausible mistakes in a private copy of the oracle (CPU only) and check
that the pins catch every one of them."""
import importlib.util
import os

import numpy as np
import pytest

from oracle_pins import PINS

ORACLE_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "oracle", "moe_oracle.py")


def fresh_oracle():
    spec = importlib.util.spec_from_file_location("moe_oracle_mutant", ORACLE_PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def m_topk_ascending(O):
    O.rank_desc = lambda s: np.argsort(s, axis=-1, kind="stable")


def m_ties_to_higher_index(O):
    def rank(s):
        E = s.shape[-1]
        rev = np.argsort(-s[..., ::-1], axis=-1, kind="stable")
        return E - 1 - rev
    O.rank_desc = rank


def m_no_renorm(O):
    orig = O.route_softmax_topk
    O.route_softmax_topk = lambda l, k, norm=True: orig(l, k, False)


def m_softmax_no_exp(O):
    O.softmax = lambda l: (l - l.min(-1, keepdims=True)) / (l - l.min(-1, keepdims=True)).sum(-1, keepdims=True)


def m_sigmoid_weights_with_bias(O):
    orig = O.route_sigmoid_group

    def f(logits, top_k, n_group, topk_group, routed_scaling, norm=True, expert_bias=None):
        ids, w, s, m = orig(logits, top_k, n_group, topk_group, routed_scaling, norm, expert_bias)
        if expert_bias is not None:
            sel = s + np.asarray(expert_bias)[None, :]
            w = np.take_along_axis(sel, ids, -1)
            if norm:
                w = w / (w.sum(-1, keepdims=True) + 1e-20)
            w = w * routed_scaling
        return ids, w, s, m
    O.route_sigmoid_group = f


def m_group_score_top1(O):
    src = open(ORACLE_PATH).read().replace("[:, :, :2]", "[:, :, :1]")
    ns = {}
    exec(compile(src, ORACLE_PATH, "exec"), ns)
    O.route_sigmoid_group = ns["route_sigmoid_group"]


def m_margin_without_group_cut(O):
    src = open(ORACLE_PATH).read().replace("np.minimum(e_margin, g_margin)", "e_margin")
    ns = {}
    exec(compile(src, ORACLE_PATH, "exec"), ns)
    O.route_sigmoid_group = ns["route_sigmoid_group"]


def m_margin_on_raw_score(O):
    src = open(ORACLE_PATH).read().replace(
        "chosen_sel = np.take_along_axis(masked, ids, axis=-1)",
        "masked = np.where(emask, s, -np.inf)\n    chosen_sel = np.take_along_axis(masked, ids, axis=-1)")
    assert src != open(ORACLE_PATH).read()
    ns = {}
    exec(compile(src, ORACLE_PATH, "exec"), ns)
    O.route_sigmoid_group = ns["route_sigmoid_group"]


def m_no_routed_scaling(O):
    orig = O.route_sigmoid_group
    O.route_sigmoid_group = lambda l, k, g, tg, rs, norm=True, b=None: orig(l, k, g, tg, 1.0, norm, b)


def m_capacity_without_k(O):
    def cap(T, k, E, cf):
        if cf is None or cf <= 0.0:
            return None
        return max(1, int(T / E * cf))
    O.capacity = cap


def m_capacity_rounds_up(O):
    import math

    def cap(T, k, E, cf):
        if cf is None or cf <= 0.0:
            return None
        return max(1, math.ceil(T * k / E * cf))
    O.capacity = cap


def m_drop_keeps_latest(O):
    orig = O.dispatch

    def f(ids, E, cap, weights=None):
        T = ids.shape[0]
        out = orig(ids[::-1].copy(), E, cap, None if weights is None else np.asarray(weights)[::-1].copy())
        out["perm_token"] = T - 1 - out["perm_token"]
        out["slot_row"] = out["slot_row"][::-1].copy()
        return out
    O.dispatch = f


def m_relu_identity(O):
    orig = O.expert_mlp
    O.expert_mlp = lambda x, w1, w3, act, w2=None: (x @ w1.T) @ w3.T if act == "relu" else orig(x, w1, w3, act, w2)


def m_swiglu_swapped(O):
    orig = O.expert_mlp
    O.expert_mlp = lambda x, w1, w3, act, w2=None: orig(x, w2, w3, act, w1) if act == "swiglu" else orig(x, w1, w3, act, w2)


def m_combine_unweighted(O):
    orig = O.combine
    O.combine = lambda T, W, ids, w, sr, eo, tokens=None: orig(T, W, ids, np.ones_like(w), sr, eo, tokens)


def m_aux_raw_counts(O):
    orig = O.dispatch

    def f(ids, E, cap, weights=None):
        out = orig(ids, E, cap, weights)
        out["kept_counts"] = out["raw_counts"].copy()
        return out
    O.dispatch = f


def m_aux_wrong_mean(O):
    O.aux_loss = lambda kept, P, T, E, alpha: ((E * float(np.sum(kept / T * P)) / E),
                                              alpha * float(np.sum(kept / T * P)))


def m_q4_nibble_order(O):
    src = open(ORACLE_PATH).read().replace("(words >> (4 * j))", "(words >> (4 * (7 - j)))")
    ns = {}
    exec(compile(src, ORACLE_PATH, "exec"), ns)
    O.dequant_q4 = ns["dequant_q4"]


def m_q4_group_32(O):
    src = open(ORACLE_PATH).read().replace("np.arange(q.shape[1]) // 64", "np.arange(q.shape[1]) // 32 % s.shape[1]")
    ns = {}
    exec(compile(src, ORACLE_PATH, "exec"), ns)
    O.dequant_q4 = ns["dequant_q4"]


def m_bf16_widen_wrong(O):
    O.widen = lambda a: (np.asarray(a).astype(np.float64) if np.asarray(a).dtype != np.uint16
                         else np.asarray(a).astype(np.float64) / 65536.0)


def m_fused_wholesale(O):
    # both stacks one after the other, then cut into experts: rows misalign
    O.fuse_gate_up = lambda g, u: np.concatenate([np.asarray(g), np.asarray(u)], axis=0).reshape(
        (np.asarray(g).shape[0], 2 * np.asarray(g).shape[1]) + np.asarray(g).shape[2:])


def m_split_up_first(O):
    orig = O.split_gate_up
    O.split_gate_up = lambda b: orig(b)[::-1]


def m_forced_no_renorm(O):
    orig = O.route_forced
    O.route_forced = lambda *a, **kw: orig(*a, **{**kw, "norm": False})


def m_forced_keeps_repeats(O):
    orig = O.route_forced

    def forced(x, w, ids, **kw):
        ids = np.asarray(ids)
        r = orig(x, w, ids, **kw)
        # treat a repeated id as a good route: copy the first occurrence's score in
        for t in range(ids.shape[0]):
            for j in range(ids.shape[1]):
                if r["bad"][t, j] and 0 <= ids[t, j] < r["probs"].shape[1]:
                    r["bad"][t, j] = False
                    r["weights"][t, j] = r["probs"][t, ids[t, j]]
        return r
    O.route_forced = forced


def m_bias_sign_flipped(O):
    orig = O.update_bias
    O.update_bias = lambda b, c, coeff: orig(b, c, -coeff)


def m_bias_integer_mean(O):
    def upd(bias, counts, coeff):
        counts = np.asarray(counts)
        mean = counts.sum() // len(counts)
        step = np.where(counts < mean, 1.0, np.where(counts > mean, -1.0, 0.0))
        return (np.asarray(bias, dtype=np.float64) + step * coeff).astype(np.float32)
    O.update_bias = upd


MUTANTS = [v for k_, v in sorted(globals().items()) if k_.startswith("m_")]


@pytest.mark.parametrize("mutate", MUTANTS, ids=[m.__name__ for m in MUTANTS])
def test_mutant_is_caught(mutate):
    O = fresh_oracle()
    mutate(O)
    caught = []
    for pin in PINS:
        try:
            pin(O)
        except Exception as exc:  # noqa: BLE001  (any failure counts as caught)
            caught.append((pin.__name__, type(exc).__name__))
    assert caught, f"mutant {mutate.__name__} passed every pin"
