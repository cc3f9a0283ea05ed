"""moe_route_noalloc: the router variant for callers that cannot allocate.

Such callers (a host framework that owns all device memory, or a path that
must not allocate) call moe_route_noalloc, whose scratch is a fixed array
inside the library instead of a workspace.  Its results must match
moe_route's on the same inputs, on two calls in a row (the second with a
different problem, so nothing may leak from the first through the shared
array).  Kept in a file of its own, collected last.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_41_b200 import _lib as L
from mixture_experts_layer_41_b200 import api
from mixture_experts_layer_41_b200.inputs import make_inputs, workload
from moe_cases import cfg_of, oracle_route, router_bias_of
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

WEIGHT_RTOL = 1e-6
PROB_RTOL = 1e-5


def _route_both(w, seed):
    dev = torch.device("cuda")
    inp = make_inputs(w, seed=seed, device=dev)
    # the two calls take different router passes (moe_route may use the
    # tensor-core logits, the no-workspace call never does), so ids are
    # compared only where the oracle's selection margin is clear
    safe = oracle_route(w, inp)["margin"] > O.SAFE_MARGIN
    cfg = cfg_of(w)
    bias = router_bias_of(w, inp)
    ws = torch.empty(api.moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
    out = {}
    for name in ("ws", "noalloc"):
        ids = torch.full((w.T, w.k), -1, dtype=torch.int32, device=dev)
        wts = torch.full((w.T, w.k), float("nan"), dtype=torch.float32, device=dev)
        ps = torch.full((w.E,), float("nan"), dtype=torch.float32, device=dev)
        if name == "ws":
            api.moe_route(cfg, inp["x"], inp["w_router"], bias, ids, wts, ps, ws)
        else:
            api.moe_route_noalloc(cfg, inp["x"], inp["w_router"], bias, ids, wts, ps)
        torch.cuda.synchronize()
        out[name] = (ids.cpu().numpy(), wts.cpu().numpy().astype(np.float64), ps.cpu().numpy().astype(np.float64))
    out["safe"] = safe
    return out


def _compare(out):
    ids_a, w_a, p_a = out["ws"]
    ids_b, w_b, p_b = out["noalloc"]
    safe = out["safe"]
    assert safe.mean() > 0.9
    assert np.array_equal(ids_a[safe], ids_b[safe])
    same = safe[:, None] & (ids_a == ids_b)
    assert np.all(np.abs(w_b - w_a)[same] <= WEIGHT_RTOL * np.abs(w_a)[same])
    assert np.all(np.abs(p_b - p_a) <= PROB_RTOL * np.abs(p_a))


def test_noalloc_router_matches_workspace_router_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    # two calls in a row: a larger softmax problem, then a sigmoid-group one
    _compare(_route_both(workload("switch_top1", T=2048, d=256, F=256, E=64), seed=11))
    _compare(_route_both(workload("deepseek_v3", T=1000, d=448, F=256, E=32, n_group=8, topk_group=4,
                                  shared_F=0), seed=12))


def test_noalloc_router_rejects_oversized_problem():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    w = workload("deepseek_v3", T=16416, d=64, F=64, shared_F=0)   # ceil(16416/32)*256 > 131072
    cfg = cfg_of(w)
    dev = torch.device("cuda")
    x = torch.zeros((w.T, w.d), dtype=torch.bfloat16, device=dev)
    wr = torch.zeros((w.E, w.d), dtype=torch.float32, device=dev)
    ids = torch.empty((w.T, w.k), dtype=torch.int32, device=dev)
    wts = torch.empty((w.T, w.k), dtype=torch.float32, device=dev)
    ps = torch.empty((w.E,), dtype=torch.float32, device=dev)
    with pytest.raises(L.MoEError, match="exceed the fixed scratch"):
        api.moe_route_noalloc(cfg, x, wr, None, ids, wts, ps)
