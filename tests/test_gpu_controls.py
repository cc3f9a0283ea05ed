"""CUDA path vs the oracle for the layer's control variants, through the C ABI:
the fused gate/up weight layout, router replay (forced expert ids) and the
aux-loss-free balancing bias update.

Bars: the fused layout gives bit-identical outputs to the separate layout and
the oracle's output (split from the fused tensor) within the layer bar;
replayed ids are copied exactly, their weights within 1e-6 relative of the
oracle's and prob_sum within 1e-5; the bias update is bit-exact (an integer
decision and one fp32 add).
"""
import numpy as np
import pytest
import torch

from gpu_harness import PROB_RTOL, WEIGHT_RTOL, Run, out_tol
from mixture_experts_layer_41_b200 import _lib as L
from mixture_experts_layer_41_b200 import api
from mixture_experts_layer_41_b200.inputs import to_host, workload
from moe_cases import as_f64, cfg_of, rel_max_err
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    yield


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


# ---------------------------------------------------------------- fused gate/up layout

FUSED = {
    "fp32_swiglu": workload("tiny_fp32", T=97, d=24, F=40, E=6, k=3, act="swiglu", capacity_factor=0.0),
    "mixtral_small": workload("mixtral_prefill", T=700, d=512, F=640),
    "ragged_nk": workload("mixtral_prefill", T=333, d=200, F=136, E=4, k=2),
    "deepseek_small": workload("deepseek_v3", T=512, d=448, F=256, E=32, n_group=8, topk_group=4, shared_F=256),
    "decode_small": workload("decode_q4", T=16, d=256, F=128, E=16, k=4),
    "decode_many_rows": workload("decode_q4", T=200, d=256, F=256, E=8, k=2),
    "decode_cuda_core_shape": workload("decode_q4", T=24, d=320, F=192, E=16, k=4),
}


def _fused_weights(weights: dict) -> dict:
    """Gate over up per expert: concatenating along the output axis of the
    [E, F, ...] stacks puts expert e's up rows right after its gate rows."""
    out = dict(weights)
    out["w1"] = torch.cat([weights["w1"], weights["w2"]], dim=1).contiguous()
    del out["w2"]
    for s in ("s", "b"):
        if s + "1" in weights:
            out[s + "1"] = torch.cat([weights[s + "1"], weights[s + "2"]], dim=1).contiguous()
            del out[s + "2"]
    return out


@pytest.mark.parametrize("name", sorted(FUSED))
def test_fused_gate_up_layout(name):
    w = FUSED[name]
    run = Run(w, seed=11)
    sep = run.forward(torch.empty_like(run.out)).clone()
    assert run.status() == 0
    fused = _fused_weights(run.weights)
    cfg = cfg_of(w)
    cfg.weight_layout = L.MOE_LAYOUT_FUSED_GATE_UP
    assert api.moe_validate(cfg) == L.MOE_OK
    out = torch.empty_like(run.out)
    api.moe_forward(cfg, run.inp["x"], run.inp["w_router"], run.bias, fused, out, run.ids, run.wts, run.stats,
                    run.ws)
    torch.cuda.synchronize()
    assert run.status() == 0
    assert torch.equal(_bits(out), _bits(sep)), "fused layout changed the result"
    # the oracle reads the fused tensor and splits it itself
    q4 = "s1" in fused
    host = {k: to_host(v) for k, v in fused.items()}

    def experts(e):
        if q4:
            return dict(q13=host["w1"][e], s13=host["s1"][e], b13=host["b1"][e], q3=host["w3"][e],
                        s3=host["s3"][e], b3=host["b3"][e])
        return dict(w13=host["w1"][e], w3=host["w3"][e])
    shared = {k: host[k] for k in ("ws1", "ws2", "ws3")} if w.shared_F else None
    routing = dict(ids=run.ids.cpu().numpy(), weights=run.wts.cpu().numpy().astype(np.float64),
                   probs=np.zeros((w.T, w.E)))
    toks = np.arange(min(w.T, 96))
    res = O.layer_forward(to_host(run.inp["x"]), to_host(run.inp["w_router"]), experts, top_k=w.k, act=w.act,
                          capacity_factor=float(np.float32(w.capacity_factor)), shared=shared, tokens=toks,
                          routing=routing)
    err = rel_max_err(as_f64(out)[toks], res["out"][toks])
    assert err <= out_tol(w), err


def test_fused_layout_rejects_separate_pointers():
    w = FUSED["mixtral_small"]
    run = Run(w, seed=12)
    cfg = cfg_of(w)
    cfg.weight_layout = L.MOE_LAYOUT_FUSED_GATE_UP
    with pytest.raises(L.MoEError):        # w2 given although the layout carries up in w1
        api.moe_grouped_ffn(cfg, run.x_perm, run.offsets, run.weights, run.y_perm, run.ws)
    relu = cfg_of(workload("switch_top1", T=64, d=64, F=64, E=8))
    relu.weight_layout = L.MOE_LAYOUT_FUSED_GATE_UP
    assert api.moe_validate(relu) == L.MOE_ERR_INVALID_ARG


# ---------------------------------------------------------------- router replay

REPLAY = {
    # one per router kernel: rows (E <= 16), tiled, tiled with 8 tokens per
    # warp, hidden split + selection pass; softmax and sigmoid-group
    "rows_e8": workload("mixtral_prefill", T=777, d=1032, F=64, E=8, k=2),
    "rows_f32_sigmoid": workload("deepseek_v3", T=60, d=40, F=64, E=12, n_group=3, topk_group=2, k=3,
                                 shared_F=0, dtype="f32", weight_format="dense"),
    "tiled_e64_top1": workload("switch_top1", T=5000, d=512, F=64, E=64, k=1),
    "tiled8_e128": workload("mixtral_prefill", T=9500, d=192, F=64, E=128, k=4),
    "tiled_e256_sigmoid": workload("deepseek_v3", T=4800, d=320, F=64, shared_F=0),
    "split_e128_decode": workload("decode_q4", T=40, d=1024, F=64, k=8, weight_format="dense"),
    "split_e256_sigmoid": workload("deepseek_v3", T=70, d=2048, F=64, shared_F=0),
}


def _oracle_forced(w, inp, forced):
    return O.route_forced(to_host(inp["x"]), to_host(inp["w_router"]), forced, top_k=w.k, router=w.router,
                          norm=w.norm_topk_prob, routed_scaling=w.routed_scaling,
                          logit_bias=to_host(inp.get("logit_bias")))


def _check_weights(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    err[ref == 0.0] = np.abs(got[ref == 0.0])
    assert err.max() <= WEIGHT_RTOL, f"replayed weight rel err {err.max():.3e}"


@pytest.mark.parametrize("name", sorted(REPLAY))
def test_route_forced_parity(name):
    w = REPLAY[name]
    run = Run(w, seed=13)
    g = torch.Generator(device="cpu").manual_seed(5)
    forced = torch.argsort(torch.rand((w.T, w.E), generator=g), dim=1)[:, :w.k].to(torch.int32).contiguous()
    forced_d = forced.cuda()
    api.moe_route_forced(run.cfg, run.inp["x"], run.inp["w_router"], run.bias, forced_d, run.ids, run.wts,
                         run.prob_sum, run.ws)
    torch.cuda.synchronize()
    assert run.status() == 0
    assert torch.equal(run.ids.cpu(), forced)
    ref = _oracle_forced(w, run.inp, forced.numpy())
    _check_weights(run.wts.cpu().numpy().astype(np.float64), ref["weights"])
    ps = run.prob_sum.cpu().numpy().astype(np.float64)
    assert (np.abs(ps - ref["prob_sum"]) / np.abs(ref["prob_sum"])).max() <= PROB_RTOL


@pytest.mark.parametrize("name", sorted(REPLAY))
def test_replaying_own_route_reproduces_it(name):
    """Replaying moe_route's own choices gives back its weights bit for bit
    (same logits, same float64 score arithmetic)."""
    w = REPLAY[name]
    run = Run(w, seed=14)
    api.moe_route(run.cfg, run.inp["x"], run.inp["w_router"], run.bias, run.ids, run.wts, run.prob_sum, run.ws)
    ids0, w0, p0 = run.ids.clone(), run.wts.clone(), run.prob_sum.clone()
    ids1, w1 = torch.empty_like(ids0), torch.empty_like(w0)
    p1 = torch.empty_like(p0)
    api.moe_route_forced(run.cfg, run.inp["x"], run.inp["w_router"], run.bias, ids0, ids1, w1, p1, run.ws)
    torch.cuda.synchronize()
    assert run.status() == 0
    assert torch.equal(ids1, ids0) and torch.equal(w1, w0) and torch.equal(p1, p0)


def test_route_forced_rejects_bad_recorded_ids():
    w = REPLAY["tiled_e64_top1"].with_(k=3, T=300)
    run = Run(w, seed=15)
    g = torch.Generator(device="cpu").manual_seed(6)
    forced = torch.argsort(torch.rand((w.T, w.E), generator=g), dim=1)[:, :w.k].to(torch.int32)
    forced[7, 1] = -1                  # a missing-route sentinel
    forced[9, 2] = forced[9, 0]        # a repeat
    forced[11, 0] = w.E                # out of range
    api.moe_route_forced(run.cfg, run.inp["x"], run.inp["w_router"], run.bias, forced.cuda().contiguous(),
                         run.ids, run.wts, run.prob_sum, run.ws)
    torch.cuda.synchronize()
    assert run.status() == L.MOE_ERR_DEVICE
    ref = _oracle_forced(w, run.inp, forced.numpy())
    assert ref["bad"].sum() == 3
    got = run.wts.cpu().numpy().astype(np.float64)
    assert np.all(got[ref["bad"]] == 0.0)
    _check_weights(got, ref["weights"])


def test_layer_forward_with_replayed_routes():
    w = workload("deepseek_v3", T=256, d=448, F=256, E=32, n_group=8, topk_group=4, shared_F=256)
    run = Run(w, seed=16)
    layer = api.MoELayer(run.cfg, run.inp["w_router"], run.weights, router_bias=run.bias)
    g = torch.Generator(device="cpu").manual_seed(7)
    forced = torch.argsort(torch.rand((w.T, w.E), generator=g), dim=1)[:, :w.k].to(torch.int32)
    o = layer.forward(run.inp["x"], forced_ids=forced.cuda().contiguous())
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert torch.equal(o.topk_ids.cpu(), forced)
    ref_r = _oracle_forced(w, run.inp, forced.numpy())
    host = {k: to_host(v) for k, v in run.weights.items()}
    shared = {k: host[k] for k in ("ws1", "ws2", "ws3")}
    res = O.layer_forward(to_host(run.inp["x"]), to_host(run.inp["w_router"]),
                          lambda e: dict(w1=host["w1"][e], w2=host["w2"][e], w3=host["w3"][e]), top_k=w.k,
                          act=w.act, shared=shared, routing=ref_r)
    err = rel_max_err(as_f64(o.out), res["out"])
    assert err <= out_tol(w), err


# ---------------------------------------------------------------- balancing bias

@pytest.mark.parametrize("E", [2, 8, 64, 160, 256])
def test_update_bias_bit_exact(E):
    rng = np.random.default_rng(E)
    cfg = cfg_of(workload("deepseek_v3", T=64, d=64, F=64, E=E, n_group=1, topk_group=1, k=2, shared_F=0))
    for trial in range(4):
        if trial == 0:
            counts = np.full(E, 7, dtype=np.int32)                 # balanced: unchanged
        elif trial == 1:
            counts = np.zeros(E, dtype=np.int32)
            counts[0] = 3 * E                                      # one hot expert
        else:
            counts = rng.integers(0, 50, E).astype(np.int32)
            counts[: E // 4] = int(counts.sum() // E)              # some near the mean
        bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
        coeff = float(np.float32([1e-3, 2.0 ** -10, 0.0, 0.05][trial]))
        b_dev = torch.from_numpy(bias.copy()).cuda()
        api.moe_update_bias(cfg, torch.from_numpy(counts).cuda(), b_dev, coeff)
        torch.cuda.synchronize()
        ref = O.update_bias(bias, counts, coeff)
        assert np.array_equal(b_dev.cpu().numpy().view(np.uint32), ref.view(np.uint32)), trial


def test_update_bias_after_forward_moves_toward_balance():
    """MoELayer.update_bias applies the update to the last forward's raw
    counts; repeated steps on a skewed router shrink the busiest expert's share."""
    w = workload("deepseek_v3", T=2048, d=256, F=64, E=32, n_group=8, topk_group=4, shared_F=0)
    run = Run(w, seed=17)
    bias = torch.zeros(w.E, dtype=torch.float32, device="cuda")
    bias[:4] = 0.3                                    # skew selection toward experts 0..3
    layer = api.MoELayer(run.cfg, run.inp["w_router"], run.weights, router_bias=bias)
    layer.forward(run.inp["x"])
    first = layer.o.raw_counts.cpu().numpy().copy()
    b0 = bias.cpu().numpy().copy()
    layer.update_bias(1e-2)
    torch.cuda.synchronize()
    assert np.array_equal(bias.cpu().numpy(), O.update_bias(b0, first, 1e-2))
    for _ in range(30):
        layer.forward(run.inp["x"])
        layer.update_bias(1e-2)
    layer.forward(run.inp["x"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    last = layer.o.raw_counts.cpu().numpy()
    assert last.max() < first.max()


# ---------------------------------------------------------------- fused dispatch gather

GATHER = {
    "mixtral_small": workload("mixtral_prefill", T=700, d=512, F=640),
    "ragged_nk": workload("mixtral_prefill", T=333, d=200, F=136, E=4, k=2),
    "relu_capacity": workload("switch_top1", T=257, d=136, F=264, E=8, k=2, capacity_factor=1.25),
    "deepseek_small": workload("deepseek_v3", T=512, d=448, F=256, E=32, n_group=8, topk_group=4, shared_F=256),
}


@pytest.mark.parametrize("name", sorted(GATHER))
def test_fused_gather_matches_copy(name):
    """moe_forward with the expert rows gathered inside the grouped GEMM gives
    the copy path's output bit for bit, with a smaller workspace."""
    w = GATHER[name]
    run = Run(w, seed=21).staged()
    ref = run.out.clone()
    cfg = cfg_of(w)
    cfg.fused_gather = 1
    assert api.moe_workspace_size(cfg) < api.moe_workspace_size(run.cfg)
    ws = torch.empty(api.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(run.out)
    api.moe_forward(cfg, run.inp["x"], run.inp["w_router"], run.bias, run.weights, out, run.ids, run.wts,
                    run.stats, ws)
    torch.cuda.synchronize()
    assert api.moe_workspace_status(ws) == 0
    assert torch.equal(_bits(out), _bits(ref))


# ---------------------------------------------------------------- bf16 grouped GEMM on pairs of SMs

PAIR = dict(GATHER)
PAIR["mixtral_tail"] = workload("mixtral_prefill", T=1100, d=512, F=384, E=8, k=2)      # 256-row tiles with tails
PAIR["one_expert_rows"] = workload("switch_top1", T=130, d=264, F=200, E=2, k=1, capacity_factor=0.0)


@pytest.mark.parametrize("name", sorted(PAIR))
def test_paired_sm_gemm_matches_one_sm(name, monkeypatch):
    """MOE_TC_PAIR=1 runs the bf16 grouped FFN (and the shared expert) on
    pairs of SMs with 256-row tiles; each output element is the same chain
    of K-16 tensor-core steps as on one SM, so the layer output is identical
    bit for bit, ragged N and K, tails past the last row and all."""
    w = PAIR[name]
    monkeypatch.setenv("MOE_TC_PAIR", "0")
    one = Run(w, seed=22).staged()
    ref = one.out.clone()
    monkeypatch.setenv("MOE_TC_PAIR", "1")
    out = torch.empty_like(ref)
    api.moe_forward(one.cfg, one.inp["x"], one.inp["w_router"], one.bias, one.weights, out, one.ids, one.wts,
                    one.stats, one.ws)
    torch.cuda.synchronize()
    assert api.moe_workspace_status(one.ws) == 0
    assert torch.equal(_bits(out), _bits(ref))


# ---------------------------------------------------------------- 4-bit FFN kernels

Q4 = {
    "decode_small": workload("decode_q4", T=16, d=256, F=128, E=16, k=4),
    "decode_many_rows": workload("decode_q4", T=200, d=256, F=256, E=8, k=2),       # several token passes
    "ragged_passes": workload("decode_q4", T=90, d=384, F=256, E=4, k=3),           # pass tails in both phases
    "mostly_empty": workload("decode_q4", T=6, d=512, F=384, E=64, k=2),
    "decode_like": workload("decode_q4", T=64, d=1024, F=768, E=32, k=8),
}


@pytest.mark.parametrize("kernel", ["mma", "tc"])
@pytest.mark.parametrize("name", sorted(Q4))
def test_q4_kernels_match_oracle(name, kernel, monkeypatch):
    """Both 4-bit grouped FFN kernels (warp-level mma.sync fragments and
    tcgen05 with the weight operand in TMEM), forced in turn, against the
    oracle on every token (the GPU's own routing, so only the experts and
    the combine are compared)."""
    from gpu_harness import check_output
    monkeypatch.setenv("MOE_Q4_KERNEL", kernel)
    run = Run(Q4[name], seed=23).staged()
    assert run.status() == 0
    check_output(run)


@pytest.mark.parametrize("case", ["bf16", "bf16_pair", "q4_mma", "q4_tc"])
def test_grouped_ffn_repairs_bad_offsets(case, monkeypatch):
    """Decreasing group offsets (every value inside [0, T*k]) are clamped to a
    non-decreasing copy, the call completes, and the workspace reports the
    device-side failure."""
    if case.startswith("q4"):
        w = Q4["decode_like"]
        monkeypatch.setenv("MOE_Q4_KERNEL", case[3:])
    else:
        w = workload("mixtral_prefill", T=300, d=256, F=256, E=8, k=2)
        monkeypatch.setenv("MOE_TC_PAIR", "1" if case == "bf16_pair" else "0")
    run = Run(w, seed=24).staged()
    assert run.status() == 0
    bad = run.offsets.clone()
    bad[3] = bad[5] + 7                # a step down after index 3
    bad[3] = min(int(bad[3]), w.T * w.k)
    api.moe_grouped_ffn(run.cfg, run.x_perm, bad, run.weights, run.y_perm, run.ws)
    torch.cuda.synchronize()
    assert run.status() == L.MOE_ERR_DEVICE


# ---------------------------------------------------------------- bounded-wait failure path

@pytest.mark.parametrize("kernel", ["tc", "q4_tc"])
def test_barrier_wait_timeout_reports_and_recovers(kernel, monkeypatch):
    """The tensor-core kernels' failure path, made to run out on purpose: with
    a 1 ns bound on barrier waits the first wait that is not already
    satisfied gives up; the call reports MOE_ERR_DEVICE with the waiting
    site, the kernel lets its issued copies and MMAs land, frees its tensor
    memory and returns, so the context stays usable; with the default bound
    restored, the same workspace gives the oracle's result."""
    if kernel == "tc":
        w = workload("mixtral_prefill", T=700, d=512, F=640)
    else:
        monkeypatch.setenv("MOE_Q4_KERNEL", "tc")
        # long enough reductions that some barrier wait is still open when it is checked
        w = workload("decode_q4", T=200, d=2048, F=1024, E=8, k=2)
    from gpu_harness import check_output
    run = Run(w, seed=9)
    c = run.cfg
    api.moe_route(c, run.inp["x"], run.inp["w_router"], run.bias, run.ids, run.wts, run.prob_sum, run.ws)
    api.moe_permute(c, run.inp["x"], run.ids, run.wts, run.offsets, run.perm_token, run.perm_w, run.slot_row,
                    run.x_perm, run.stats, run.ws)
    torch.cuda.synchronize()
    assert run.status() == 0
    try:
        api.moe_set_wait_timeout_ns(1)
        api.moe_grouped_ffn(c, run.x_perm, run.offsets, run.weights, run.y_perm, run.ws)
        st = run.status()
        text = L.lib().moe_last_error().decode()
    finally:
        api.moe_set_wait_timeout_ns(0)
    assert st == L.MOE_ERR_DEVICE, st
    assert "timed out" in text, text
    # the context and the workspace are still good: a normal call succeeds
    run.staged()
    assert run.status() == 0
    check_output(run, routing="gpu")


def test_router_wait_timeout_reports_and_recovers():
    """The same failure path in the integer tensor-core router (two CTAs per
    SM sharing the tensor memory): with a 1 ns bound the router GEMM gives up,
    frees its tensor memory, and the call reports MOE_ERR_DEVICE; with the
    default bound restored the same workspace routes as the oracle does."""
    from gpu_harness import check_route
    from moe_cases import oracle_route
    w = workload("deepseek_v3", T=1024, d=2048, F=64, shared_F=0)
    run = Run(w, seed=4)
    c = run.cfg
    try:
        api.moe_set_wait_timeout_ns(1)
        api.moe_route(c, run.inp["x"], run.inp["w_router"], run.bias, run.ids, run.wts, run.prob_sum, run.ws)
        st = run.status()
        text = L.lib().moe_last_error().decode()
    finally:
        api.moe_set_wait_timeout_ns(0)
    assert st == L.MOE_ERR_DEVICE, st
    assert "timed out" in text, text
    api.moe_route(c, run.inp["x"], run.inp["w_router"], run.bias, run.ids, run.wts, run.prob_sum, run.ws)
    torch.cuda.synchronize()
    assert run.status() == 0
    check_route(run, oracle_route(w, run.inp))


# ---------------------------------------------------------------- bf16 tensor-core router (opt-in)
def test_bf16_tensor_core_router_routes_as_the_oracle():
    """MOE_ROUTER_TC=bf16 (read once per process, so run in a fresh one)
    routes bf16 batches of 512 tokens or more with the bf16 selection-grade
    tensor-core logits and an exact re-weighting of every token's chosen
    experts; ids, weights and probability sums match the oracle."""
    import os
    import subprocess
    import sys
    tests = os.path.dirname(os.path.abspath(__file__))
    code = (
        "import sys; sys.path[:0] = [%r, %r]\n"
        "import torch\n"
        "from gpu_harness import Run, check_route\n"
        "from moe_cases import oracle_route\n"
        "from mixture_experts_layer_41_b200 import api\n"
        "from mixture_experts_layer_41_b200.inputs import workload\n"
        "for w in (workload('deepseek_v3', T=1024, d=1024, F=64, shared_F=0),\n"
        "          workload('mixtral_prefill', T=600, d=512, F=64)):\n"
        "    run = Run(w, seed=7)\n"
        "    api.moe_route(run.cfg, run.inp['x'], run.inp['w_router'], run.bias, run.ids, run.wts,\n"
        "                  run.prob_sum, run.ws)\n"
        "    torch.cuda.synchronize()\n"
        "    assert run.status() == 0\n"
        "    check_route(run, oracle_route(w, run.inp))\n"
        "print('routed')\n" % (os.path.dirname(tests), tests))
    env = dict(os.environ, MOE_ROUTER_TC="bf16")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "routed" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
