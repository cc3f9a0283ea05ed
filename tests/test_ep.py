"""Expert parallelism (experts split across ranks, tokens exchanged all-to-all).

CPU (gloo, world size 2): the orchestration of mixture_experts_layer_41_b200.ep
runs with host operations built on the oracle; each rank's output must equal
the oracle's whole-layer forward of its own tokens with all experts.
GPU (one device): two shards driven in one process with the library's kernels
(ep.emulate moves the blocks); each shard's output must equal moe_forward of
the full layer on the same tokens bit for bit (a row's expert GEMM does not
depend on which other rows share its tile), and the oracle within the layer
bar.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_41_b200 import ep
from oracle import moe_oracle as O

WORLD = 2


def local_expert_ids(recv_counts: torch.Tensor) -> torch.Tensor:
    """Host reference of moe_ep_local_ids: rows from source s arrive as
    recv_counts[s, 0] rows of local expert 0, then recv_counts[s, 1] of
    expert 1, ... (the sender's expert order)."""
    world, e_local = recv_counts.shape
    ids = torch.arange(e_local, dtype=torch.int32).repeat(world)
    return torch.repeat_interleave(ids, recv_counts.reshape(-1).to(torch.int64))


def test_local_expert_ids_and_splits():
    counts = torch.tensor([[2, 0, 1], [1, 3, 0]], dtype=torch.int32)
    assert local_expert_ids(counts).tolist() == [0, 0, 2, 0, 1, 1, 1]
    recv = torch.tensor([[1, 1, 1], [0, 0, 5]], dtype=torch.int32)
    assert ep.split_sizes_pair(counts, recv) == ([3, 4], [3, 5])


@pytest.mark.gpu
def test_ep_local_ids_kernel():
    """moe_ep_local_ids against the host reference, with empty segments,
    a zero-row call and rows past the counts (-1)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from mixture_experts_layer_41_b200 import api
    gen = torch.Generator().manual_seed(3)
    for world, e_local in ((2, 4), (4, 32), (8, 32), (1, 7)):
        counts = torch.randint(0, 40, (world, e_local), generator=gen, dtype=torch.int32)
        counts[0, 1 % e_local] = 0
        n = int(counts.sum())
        ids = torch.full((n + 5, 1), 99, dtype=torch.int32, device="cuda")
        api.moe_ep_local_ids(counts.cuda(), n + 5, ids)
        torch.cuda.synchronize()
        got = ids.view(-1).cpu()
        assert torch.equal(got[:n], local_expert_ids(counts)), (world, e_local)
        assert (got[n:] == -1).all()
        api.moe_ep_local_ids(counts.cuda(), 0, ids)


# ---------------------------------------------------------------- host operations on the oracle

class OracleOps:
    """dispatch / expert / combine on the host in float64 (oracle arithmetic)."""

    def __init__(self, rank, world, w_router, experts, top_k, act, cap_factor, shared=None):
        self.rank, self.world = rank, world
        self.w_router = w_router
        self.E = w_router.shape[0]
        self.e_local = self.E // world
        self.experts = experts          # global list of (w1, w2, w3) float64
        self.k, self.act, self.cf = top_k, act, cap_factor
        self.shared = shared

    def dispatch(self, x):
        xf = x.numpy()
        r = O.route(xf, self.w_router, top_k=self.k)
        cap = O.capacity(xf.shape[0], self.k, self.E, self.cf)
        dsp = O.dispatch(r["ids"], self.E, cap, r["weights"])
        rows = torch.from_numpy(xf[dsp["perm_token"]])
        counts = torch.from_numpy(np.asarray(dsp["kept_counts"], dtype=np.int32)).view(self.world, self.e_local)
        return ep.Dispatched(rows, counts, torch.from_numpy(dsp["slot_row"]), torch.from_numpy(r["weights"]),
                             torch.from_numpy(r["ids"]), x)

    def expert(self, rows, recv_counts):
        ids = local_expert_ids(recv_counts).numpy()
        out = np.zeros(rows.shape, dtype=np.float64)
        rf = rows.numpy()
        for e in range(self.e_local):
            sel = np.nonzero(ids == e)[0]
            if sel.size:
                w1, w2, w3 = self.experts[self.rank * self.e_local + e]
                out[sel] = O.expert_mlp(rf[sel], w1, w3, self.act, w2)
        return torch.from_numpy(out)

    def combine(self, back, disp):
        b = back.numpy()
        slot = disp.slot_row.numpy()
        w = disp.topk_w.numpy()
        T, k = slot.shape
        out = np.zeros((T, b.shape[1] if b.size else disp.x.shape[1]), dtype=np.float64)
        for t in range(T):
            for j in range(k):
                if slot[t, j] >= 0:
                    out[t] += w[t, j] * b[slot[t, j]]
        if self.shared is not None:
            out += O.expert_mlp(disp.x.numpy(), self.shared[0], self.shared[2], "swiglu", self.shared[1])
        return torch.from_numpy(out)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed=0, E=8, d=12, F=10, T=40, shared=False):
    rng = np.random.default_rng(seed)
    w_router = rng.standard_normal((E, d))
    experts = [(rng.standard_normal((F, d)) * 0.3, rng.standard_normal((F, d)) * 0.3,
                rng.standard_normal((d, F)) * 0.3) for _ in range(E)]
    sh = (rng.standard_normal((F, d)) * 0.3, rng.standard_normal((F, d)) * 0.3,
          rng.standard_normal((d, F)) * 0.3) if shared else None
    xs = [rng.standard_normal((T, d)) for _ in range(WORLD)]
    return w_router, experts, sh, xs


def _ep_worker(rank, port, cf, shared, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w_router, experts, sh, xs = _layer(shared=shared)
        ops = OracleOps(rank, WORLD, w_router, experts, 2, "swiglu", cf, sh)
        out = ep.EPLayer(ops).forward(torch.from_numpy(xs[rank]))
        out_q.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cf,shared", [(0.0, False), (1.0, False), (0.0, True)])
def test_expert_parallel_gloo_matches_whole_layer(cf, shared):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, port, cf, shared, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(WORLD))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w_router, experts, sh, xs = _layer(shared=shared)
    for rank in range(WORLD):
        shared_w = dict(ws1=sh[0], ws2=sh[1], ws3=sh[2]) if shared else None
        ref = O.layer_forward(xs[rank], w_router, lambda e: dict(w1=experts[e][0], w2=experts[e][1],
                                                                   w3=experts[e][2]),
                              top_k=2, act="swiglu", capacity_factor=cf, shared=shared_w)
        assert np.allclose(got[rank], ref["out"], rtol=0, atol=1e-12), rank
        if cf > 0:
            assert ref["dispatch"]["dropped"] > 0, "the capacity case should drop slots"   # exercised, not vacuous


# ---------------------------------------------------------------- one GPU, two shards

@pytest.mark.gpu
@pytest.mark.parametrize("name", ["mixtral_like", "deepseek_like", "capacity_relu", "decode_q4_like"])
def test_expert_parallel_shards_on_one_gpu(name, monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    # the 4-bit kernel is chosen by rows per expert, which differ between the
    # whole layer and a shard's received rows: pin one so the bits can match
    monkeypatch.setenv("MOE_Q4_KERNEL", "mma")
    from gpu_harness import out_tol
    from mixture_experts_layer_41_b200 import api
    from mixture_experts_layer_41_b200.inputs import make_inputs, to_host, workload
    from moe_cases import HostExperts, as_f64, cfg_of, rel_max_err, router_bias_of, weights_of
    w = {"mixtral_like": workload("mixtral_prefill", T=600, d=256, F=384, E=8, k=2),
         "deepseek_like": workload("deepseek_v3", T=520, d=256, F=128, E=32, n_group=8, topk_group=4,
                                   shared_F=128),
         "capacity_relu": workload("switch_top1", T=700, d=256, F=256, E=16, k=2, capacity_factor=1.0),
         "decode_q4_like": workload("decode_q4", T=64, d=256, F=256, E=16, k=4)}[name]
    dev = torch.device("cuda")
    inputs = [make_inputs(w, seed=20 + r, device=dev) for r in range(WORLD)]
    base = inputs[0]                        # weights and router shared by both ranks
    full = weights_of(base)
    e_local = w.E // WORLD
    shards = []
    for r in range(WORLD):
        local = {k_: (v[r * e_local:(r + 1) * e_local] if k_ in ("w1", "w2", "w3", "s1", "s2", "s3",
                                                                  "b1", "b2", "b3") else v)
                 for k_, v in full.items()}
        shards.append(ep.DeviceOps(cfg_of(w), base["w_router"], local, WORLD,
                                   router_bias=router_bias_of(w, base), device=dev))
    outs = ep.emulate(shards, [inputs[r]["x"] for r in range(WORLD)])
    torch.cuda.synchronize()
    for r in range(WORLD):
        assert shards[r].status() == 0
        layer = api.MoELayer(cfg_of(w), base["w_router"], full, router_bias=router_bias_of(w, base))
        ref = layer.forward(inputs[r]["x"]).out
        torch.cuda.synchronize()
        bits = lambda t: t.view(torch.int16) if t.dtype == torch.bfloat16 else t
        assert torch.equal(bits(outs[r]), bits(ref)), f"rank {r}: differs from the single-GPU layer"
        host = dict(base)
        host["x"] = inputs[r]["x"]
        shared = {k_: to_host(base[k_]) for k_ in ("ws1", "ws2", "ws3")} if w.shared_F else None
        routing = dict(ids=layer.o.topk_ids.cpu().numpy(), weights=layer.o.topk_w.cpu().numpy().astype(np.float64),
                       probs=np.zeros((w.T, w.E)))
        toks = np.arange(min(w.T, 64))
        res = O.layer_forward(to_host(inputs[r]["x"]), to_host(base["w_router"]), HostExperts(base), top_k=w.k,
                              act=w.act, capacity_factor=float(np.float32(w.capacity_factor)), shared=shared,
                              tokens=toks, routing=routing)
        assert rel_max_err(as_f64(outs[r])[toks], res["out"][toks]) <= out_tol(w)
