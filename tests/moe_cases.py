"""Shared helpers for the tests: workload -> library config / weights, and the
oracle run on host copies of the same inputs."""
from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_41_b200 import api
from mixture_experts_layer_41_b200.inputs import Workload, to_host
from oracle import moe_oracle as O


def cfg_of(w: Workload):
    wf = "q4_affine_g64" if w.weight_format == "q4_affine_g64" else w.dtype
    return api.make_config(num_tokens=w.T, hidden=w.d, intermediate=w.F, num_experts=w.E, top_k=w.k,
                           router=w.router, norm_topk_prob=w.norm_topk_prob,
                           routed_scaling=w.routed_scaling if w.router == "sigmoid_group" else 1.0,
                           n_group=w.n_group, topk_group=w.topk_group, capacity_factor=w.capacity_factor,
                           act=w.act, act_dtype=w.dtype, weight_dtype=wf, shared_intermediate=w.shared_F,
                           aux_alpha=w.aux_alpha)


def weights_of(inp: dict) -> dict:
    keys = ("w1", "w2", "w3", "q1", "q2", "q3", "s1", "s2", "s3", "b1", "b2", "b3", "ws1", "ws2", "ws3")
    out = {k: inp.get(k) for k in keys if inp.get(k) is not None}
    # the C struct names codes w1..w3 for both dense and 4-bit weights
    for i in "123":
        if "q" + i in out:
            out["w" + i] = out.pop("q" + i)
    return out


def router_bias_of(w: Workload, inp: dict):
    """The per-expert bias the router takes: logit bias (softmax) or
    selection bias (sigmoid_group)."""
    return inp["logit_bias"] if w.router == "softmax_topk" else inp["expert_bias"]


class HostExperts:
    """Lazy host copies of one expert's stored weights, for the oracle."""

    def __init__(self, inp: dict):
        self.inp = inp
        self.cache: dict = {}

    def __call__(self, e: int) -> dict:
        if e in self.cache:
            return self.cache[e]
        out = {}
        for key in ("w1", "w2", "w3", "q1", "q2", "q3", "s1", "s2", "s3", "b1", "b2", "b3"):
            t = self.inp.get(key)
            if t is not None:
                out[key] = to_host(t[e])
        self.cache = {e: out}
        return out


def oracle_forward(w: Workload, inp: dict, tokens=None, routing=None) -> dict:
    shared = None
    if w.shared_F:
        shared = {k: to_host(inp[k]) for k in ("ws1", "ws2", "ws3")}
    return O.layer_forward(
        to_host(inp["x"]), to_host(inp["w_router"]), HostExperts(inp), top_k=w.k, act=w.act,
        capacity_factor=w.capacity_factor, router=w.router, norm=w.norm_topk_prob,
        routed_scaling=w.routed_scaling, n_group=w.n_group, topk_group=w.topk_group,
        expert_bias=to_host(inp.get("expert_bias")), logit_bias=to_host(inp.get("logit_bias")),
        shared=shared, aux_alpha=w.aux_alpha, tokens=tokens, routing=routing)


def oracle_route(w: Workload, inp: dict) -> dict:
    return O.route(to_host(inp["x"]), to_host(inp["w_router"]), top_k=w.k, router=w.router,
                   norm=w.norm_topk_prob, routed_scaling=w.routed_scaling, n_group=w.n_group,
                   topk_group=w.topk_group, expert_bias=to_host(inp.get("expert_bias")),
                   logit_bias=to_host(inp.get("logit_bias")))


def rel_max_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / max |ref| (the layer-output parity measure)."""
    denom = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / (denom if denom > 0 else 1.0)


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
