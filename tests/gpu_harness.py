"""Runs the layer through the C ABI stage by stage and checks each stage
against the oracle on the same seeded inputs (GPU tests only)."""
from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_41_b200 import api
from mixture_experts_layer_41_b200.inputs import Workload, make_inputs, to_host
from moe_cases import (HostExperts, as_f64, cfg_of, oracle_route, rel_max_err, router_bias_of,
                       weights_of)
from oracle import moe_oracle as O

WEIGHT_RTOL = 1e-6      # routing weights, relative (spec bound)
PROB_RTOL = 1e-5        # prob_sum, relative
AUX_RTOL = 1e-5


def out_tol(w: Workload) -> float:
    return 1e-5 if w.dtype == "f32" else 2e-2


class Run:
    """Device buffers + one staged pass through the C ABI."""

    def __init__(self, w: Workload, seed: int = 0, inp=None):
        self.w = w
        self.cfg = cfg_of(w)
        self.dev = torch.device("cuda")
        self.inp = inp if inp is not None else make_inputs(w, seed=seed, device=self.dev)
        self.weights = weights_of(self.inp)
        self.bias = router_bias_of(w, self.inp)
        T, k, E, d = w.T, w.k, w.E, w.d
        dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        i32 = dict(dtype=torch.int32, device=self.dev)
        self.ws = torch.empty(api.moe_workspace_size(self.cfg), dtype=torch.uint8, device=self.dev)
        self.ids = torch.empty((T, k), **i32)
        self.wts = torch.empty((T, k), dtype=torch.float32, device=self.dev)
        self.prob_sum = torch.empty(E, dtype=torch.float32, device=self.dev)
        self.offsets = torch.empty(E + 1, **i32)
        self.perm_token = torch.empty(T * k, **i32)
        self.perm_w = torch.empty(T * k, dtype=torch.float32, device=self.dev)
        self.slot_row = torch.empty((T, k), **i32)
        self.x_perm = torch.empty((T * k, d), dtype=dt, device=self.dev)
        self.y_perm = torch.empty((T * k, d), dtype=dt, device=self.dev)
        self.shared = torch.empty((T, d), dtype=dt, device=self.dev) if w.shared_F else None
        self.out = torch.empty((T, d), dtype=dt, device=self.dev)
        self.stats = dict(raw_counts=torch.empty(E, **i32), kept_counts=torch.empty(E, **i32),
                          prob_sum=self.prob_sum, dropped=torch.empty(4, **i32))

    def staged(self):
        c = self.cfg
        api.moe_route(c, self.inp["x"], self.inp["w_router"], self.bias, self.ids, self.wts, self.prob_sum, self.ws)
        api.moe_permute(c, self.inp["x"], self.ids, self.wts, self.offsets, self.perm_token, self.perm_w,
                        self.slot_row, self.x_perm, self.stats, self.ws)
        api.moe_grouped_ffn(c, self.x_perm, self.offsets, self.weights, self.y_perm, self.ws)
        if self.shared is not None:
            api.moe_shared_expert(c, self.inp["x"], self.weights, self.shared, self.ws)
        api.moe_combine(c, self.y_perm, self.slot_row, self.wts, self.shared, self.out)
        torch.cuda.synchronize()
        return self

    def forward(self, out=None):
        out = self.out if out is None else out
        api.moe_forward(self.cfg, self.inp["x"], self.inp["w_router"], self.bias, self.weights, out, self.ids,
                        self.wts, self.stats, self.ws)
        torch.cuda.synchronize()
        return out

    def status(self) -> int:
        return api.moe_workspace_status(self.ws)


def check_route(run: Run, oracle_r: dict) -> dict:
    """ids bit-exact and weights within 1e-6 relative on tokens whose margin
    exceeds 1e-4; prob_sum within 1e-5 relative."""
    ids = run.ids.cpu().numpy()
    wts = run.wts.cpu().numpy().astype(np.float64)
    safe = oracle_r["margin"] > O.SAFE_MARGIN
    assert np.array_equal(ids[safe], oracle_r["ids"][safe]), "expert ids differ on safe tokens"
    ref_w = oracle_r["weights"][safe]
    err = np.abs(wts[safe] - ref_w) / np.maximum(np.abs(ref_w), 1e-30)
    assert err.size == 0 or err.max() <= WEIGHT_RTOL, f"routing weight rel err {err.max():.3e}"
    ps = run.prob_sum.cpu().numpy().astype(np.float64)
    ref_ps = oracle_r["prob_sum"]
    perr = np.abs(ps - ref_ps) / np.maximum(np.abs(ref_ps), 1e-30)
    assert perr.max() <= PROB_RTOL, f"prob_sum rel err {perr.max():.3e}"
    return dict(n_unsafe=int((~safe).sum()), weight_err=float(err.max()) if err.size else 0.0,
                prob_err=float(perr.max()))


def check_dispatch(run: Run) -> dict:
    """The oracle's dispatch of the GPU's own ids and weights, bit-exact."""
    w = run.w
    ids = run.ids.cpu().numpy()
    wts = run.wts.cpu().numpy()
    cap = O.capacity(w.T, w.k, w.E, float(np.float32(w.capacity_factor)))
    ref = O.dispatch(ids, w.E, cap, wts)
    off = run.offsets.cpu().numpy()
    assert np.array_equal(off, ref["expert_offsets"]), "expert_offsets"
    R = int(off[-1])
    assert np.array_equal(run.perm_token.cpu().numpy()[:R], ref["perm_token"]), "perm_token"
    assert np.array_equal(run.perm_w.cpu().numpy()[:R], ref["perm_w"].astype(np.float32)), "perm_w"
    assert np.array_equal(run.slot_row.cpu().numpy(), ref["slot_row"]), "slot_row / drop set"
    assert np.array_equal(run.stats["raw_counts"].cpu().numpy(), ref["raw_counts"]), "raw_counts"
    assert np.array_equal(run.stats["kept_counts"].cpu().numpy(), ref["kept_counts"]), "kept_counts"
    assert int(run.stats["dropped"][0]) == ref["dropped"], "dropped"
    # the gather: x_perm rows are byte copies of the token rows
    xp = run.x_perm[:R]
    xs = run.inp["x"][run.perm_token[:R].long()]
    assert torch.equal(xp.view(torch.int16) if xp.dtype == torch.bfloat16 else xp,
                       xs.view(torch.int16) if xs.dtype == torch.bfloat16 else xs), "x_perm gather"
    return dict(R=R, dropped=ref["dropped"], cap=cap, ref=ref)


def check_output(run: Run, tokens=None, routing="gpu") -> float:
    """Layer output vs the oracle evaluated on `tokens` (all when None).
    routing="gpu": the oracle uses the GPU's ids and weights (checks dispatch,
    experts and combine independently of routing ties); "oracle": the oracle
    routes itself."""
    w = run.w
    shared = {k: to_host(run.inp[k]) for k in ("ws1", "ws2", "ws3")} if w.shared_F else None
    r = None
    if routing == "gpu":
        r = dict(ids=run.ids.cpu().numpy(), weights=run.wts.cpu().numpy().astype(np.float64),
                 probs=np.zeros((w.T, w.E)))
    res = O.layer_forward(to_host(run.inp["x"]), to_host(run.inp["w_router"]), HostExperts(run.inp),
                          top_k=w.k, act=w.act, capacity_factor=float(np.float32(w.capacity_factor)),
                          router=w.router, norm=w.norm_topk_prob, routed_scaling=w.routed_scaling,
                          n_group=w.n_group, topk_group=w.topk_group,
                          expert_bias=to_host(run.inp.get("expert_bias")),
                          logit_bias=to_host(run.inp.get("logit_bias")), shared=shared,
                          aux_alpha=w.aux_alpha, tokens=tokens, routing=r)
    toks = np.arange(w.T) if tokens is None else np.asarray(tokens)
    got = as_f64(run.out)[toks]
    ref = res["out"][toks]
    err = rel_max_err(got, ref)
    assert err <= out_tol(w), f"layer output rel err {err:.3e} > {out_tol(w)}"
    return err


def check_aux(run: Run, oracle_r: dict) -> float:
    """aux from the GPU stats (through moe_aux_loss) vs the oracle's."""
    w = run.w
    kept = run.stats["kept_counts"].cpu()
    ps = run.prob_sum.cpu()
    raw, _ = api.moe_aux_loss(run.cfg, kept, ps)
    cap = O.capacity(w.T, w.k, w.E, float(np.float32(w.capacity_factor)))
    ref_disp = O.dispatch(oracle_r["ids"], w.E, cap)
    oraw, _ = O.aux_loss(ref_disp["kept_counts"], oracle_r["probs"].mean(axis=0), w.T, w.E, w.aux_alpha)
    err = abs(raw - oraw) / max(abs(oraw), 1e-30)
    return err


def sample_tokens(run: Run, n: int, seed: int = 0) -> np.ndarray:
    """A seeded subset of tokens that includes every token with a dropped slot
    (up to n/2 of them) and tokens of the hottest expert."""
    rng = np.random.default_rng(seed)
    T = run.w.T
    slot = run.slot_row.cpu().numpy()
    dropped = np.nonzero((slot < 0).any(axis=1))[0]
    ids = run.ids.cpu().numpy()
    hot = np.bincount(ids.reshape(-1), minlength=run.w.E).argmax()
    hot_toks = np.nonzero((ids == hot).any(axis=1))[0]
    pick = list(dropped[: n // 2]) + list(hot_toks[: n // 4])
    rest = rng.choice(T, size=min(T, n), replace=False)
    pick += [t for t in rest if t not in set(pick)]
    return np.array(sorted(set(int(t) for t in pick[:n])))
