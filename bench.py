#!/usr/bin/env python
"""MoE layer forward benchmark: routed tokens/s on B200, with the roofline.

One step = one whole layer forward (route, dispatch, grouped expert FFN,
shared expert, combine) over one batch of synthetic input already resident
in HBM.  Default workload: the DeepSeek-V3-style layer, the largest one that
fits one GPU (T=16384, hidden 7168, expert width 2048, 256 routed experts
with sigmoid group-limited top-8 routing, one shared SwiGLU expert, bf16).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs an independent
replica on its own batch (the layer has no exchange step without a capacity
limit), so the job's throughput is N * T / (slowest rank's step time).
``--impl reference`` times the CPU oracle (the plain float64 statement of the
layer) on the host cores instead, on a bounded token sample per step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd routed tokens/s on 1 B200; % of tensor/HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="deepseek_v3")
    ap.add_argument("--shape", default="",
                    help="reduced shape for profiling, e.g. E=32,T=2048 (fields of the workload; the line's "
                         "config then names the reduced shape)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-hash", action="store_true", help="skip the inputs' SHA-256 digests")
    ap.add_argument("--fused-gather", action="store_true",
                    help="bf16 experts read their token rows inside the grouped GEMM (no x_perm copy)")
    ap.add_argument("--cpu-sample", type=int, default=0, help="tokens in the oracle sample (0 = auto)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every 10 ms through
    NVML while the timed region runs (nvidia-smi's -lms loop as a fallback)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples: list[tuple[float, float, int]] = []
        self.stop_flag = threading.Event()
        self.thread = None
        self.max_mhz = None
        self.source = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            # CUDA_VISIBLE_DEVICES remaps device indices (or names GPUs by UUID)
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                ent = vis.split(",")[self.gpu].strip()
                if ent.startswith(("GPU-", "MIG-")):
                    h = pynvml.nvmlDeviceGetHandleByUUID(ent)
                else:
                    h = pynvml.nvmlDeviceGetHandleByIndex(int(ent))
            else:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.source = "nvml"

            def run():
                while not self.stop_flag.is_set():
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                        rs = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
                        self.samples.append((sm, pw, rs))
                    except Exception:  # noqa: BLE001
                        pass
                    time.sleep(0.01)
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
        except Exception:  # noqa: BLE001
            self.source = None

    def stop(self) -> dict:
        self.stop_flag.set()
        if self.thread:
            self.thread.join(timeout=2)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no clock samples"],
                    "source": self.source}
        sm = [a for a, _, _ in self.samples]
        reasons = set()
        for _, _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": self.max_mhz,
                "power_w_max": max(p for _, p, _ in self.samples), "samples": len(sm),
                "reasons": sorted(reasons), "source": self.source}


# ---------------------------------------------------------------- cost model

def layer_costs(w, R: int, touched: int) -> dict:
    """Algorithmic FLOP and bytes of the layer and of each expert GEMM.

    R = routed rows kept after the capacity cut, touched = experts with at
    least one row.  Counts the work the method must do (the touched experts'
    weights read once, x in, out written) and not the buffers it chooses."""
    es = 4 if w.dtype == "f32" else 2
    glu = 2 if w.act == "swiglu" else 1
    if w.weight_format == "q4_affine_g64":
        wbytes_per_elem = 0.5
        scale_bytes = lambda n, k: n * (k // 64) * 4       # bf16 scale + bias per group
    else:
        wbytes_per_elem = es
        scale_bytes = lambda n, k: 0
    w1 = touched * (glu * (w.F * w.d * wbytes_per_elem + scale_bytes(w.F, w.d)))
    w3 = touched * (w.d * w.F * wbytes_per_elem + scale_bytes(w.d, w.F))
    f1 = 2.0 * R * w.d * w.F * glu
    f2 = 2.0 * R * w.F * w.d
    fs = 6.0 * w.T * w.d * w.shared_F if w.shared_F else 0.0
    sbytes = 3 * w.d * w.shared_F * es if w.shared_F else 0
    router = 2.0 * w.T * w.d * w.E
    flops = f1 + f2 + fs + router
    xbytes = w.T * w.d * es
    layer_bytes = w1 + w3 + sbytes + 2 * xbytes + w.E * w.d * 4
    ffn1 = dict(flops=f1, bytes=w1 + R * w.d * es + R * w.F * es)
    ffn2 = dict(flops=f2, bytes=w3 + R * w.F * es + R * w.d * es)
    if shared_in_gemm(w):
        # the shared expert is one more group of the same two launches
        ffn1 = dict(flops=f1 + 4.0 * w.T * w.d * w.shared_F,
                    bytes=ffn1["bytes"] + 2 * w.d * w.shared_F * es + w.T * w.d * es + w.T * w.shared_F * es)
        ffn2 = dict(flops=f2 + 2.0 * w.T * w.shared_F * w.d,
                    bytes=ffn2["bytes"] + w.d * w.shared_F * es + w.T * w.shared_F * es + w.T * w.d * es)
    return dict(flops=flops, bytes=layer_bytes, ffn1=ffn1, ffn2=ffn2)


def shared_in_gemm(w) -> bool:
    """moe_forward runs a bf16 shared expert of the experts' width inside the
    grouped GEMM launches (unless the routed GEMM is forced onto SM pairs)."""
    return (w.shared_F > 0 and w.shared_F == w.F and w.dtype == "bf16" and w.weight_format == "dense"
            and os.environ.get("MOE_TC_PAIR") != "1")


def ffn_kernel_file(w) -> str:
    """Source of the grouped FFN kernel moe_forward runs for this workload
    (the library's selection: 4-bit weights on decode-sized groups, at most
    16 rows per expert, take the warp-level kernel; larger groups tcgen05;
    hidden or intermediate sizes off the 128 grid the CUDA-core kernel)."""
    if w.weight_format == "q4_affine_g64":
        if w.d % 128 or w.F % 128:
            return "ffn_q4.cu"
        kern = os.environ.get("MOE_Q4_KERNEL", "")
        if kern in ("mma", "tc"):
            return {"mma": "ffn_q4_mma.cu", "tc": "ffn_q4_tc.cu"}[kern]
        return "ffn_q4_mma.cu" if w.T * w.k <= 16 * w.E else "ffn_q4_tc.cu"
    return "ffn_simt.cu" if w.dtype == "f32" else "ffn_tc.cu"


def source_hash(path: str) -> str:
    with open(path, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current source of that kernel."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh)
    ent = rec.get(workload)
    if not ent or ent.get("source_sha256_16") != source_hash(kernel_file):
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU oracle arm

def oracle_sample_run(w, inp, n_tokens: int, seed: int = 0) -> dict:
    """The CPU oracle on a bounded sample of one layer step: the routing and
    the dispatch over the whole batch (capacity depends on every token), and
    the expert MLPs (with the combine and shared expert) on a seeded sample
    of ``n_tokens`` tokens.  Returns the three times, the sample and the
    oracle's result.  ``estimate_s`` extrapolates the sampled expert time to
    the whole batch and adds the whole-batch routing and dispatch once: the
    oracle's time for the full step."""
    import numpy as np
    from mixture_experts_layer_41_b200.inputs import to_host
    from oracle import moe_oracle as O

    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(w.T, size=min(n_tokens, w.T), replace=False))
    host = {k: to_host(v) for k, v in inp.items() if v is not None}

    def experts(e):
        out = {}
        for key in ("w1", "w2", "w3", "q1", "q2", "q3", "s1", "s2", "s3", "b1", "b2", "b3"):
            if key in host:
                out[key] = host[key][e]
        return out

    shared = {k: host[k] for k in ("ws1", "ws2", "ws3")} if w.shared_F else None
    t0 = time.perf_counter()
    routing = O.route(host["x"], host["w_router"], top_k=w.k, router=w.router, norm=w.norm_topk_prob,
                      routed_scaling=w.routed_scaling, n_group=w.n_group, topk_group=w.topk_group,
                      expert_bias=host.get("expert_bias"), logit_bias=host.get("logit_bias"))
    t1 = time.perf_counter()
    O.dispatch(np.asarray(routing["ids"]), w.E, O.capacity(w.T, w.k, w.E, w.capacity_factor), routing["weights"])
    t2 = time.perf_counter()
    res = O.layer_forward(host["x"], host["w_router"], experts, top_k=w.k, act=w.act,
                          capacity_factor=w.capacity_factor, router=w.router, norm=w.norm_topk_prob,
                          routed_scaling=w.routed_scaling, n_group=w.n_group, topk_group=w.topk_group,
                          expert_bias=host.get("expert_bias"), logit_bias=host.get("logit_bias"),
                          shared=shared, aux_alpha=w.aux_alpha, tokens=toks, routing=routing)
    t3 = time.perf_counter()
    route_s, dispatch_s = t1 - t0, t2 - t1
    experts_s = max(0.0, (t3 - t2) - dispatch_s)      # layer_forward re-runs the whole-batch dispatch
    estimate_s = route_s + dispatch_s + experts_s * w.T / len(toks)
    return dict(route_s=route_s, dispatch_s=dispatch_s, experts_s=experts_s, wall_s=t3 - t0,
                estimate_s=estimate_s, tokens=toks, result=res)


def sample_text(w, o: dict) -> str:
    return (f"oracle routing + dispatch of all {w.T} tokens ({o['route_s'] + o['dispatch_s']:.1f} s) and expert "
            f"MLPs of {len(o['tokens'])} seeded tokens ({o['experts_s']:.1f} s), extrapolated to {w.T} tokens: "
            f"value = T / (route + dispatch + experts * T / sample)")


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def auto_sample(w, per_step_s: float = 15.0) -> int:
    """Tokens in the oracle's expert sample, for about ``per_step_s`` seconds
    of host work: the oracle widens each touched expert's weights to float64
    (the dominant cost when the sample touches many experts) and evaluates
    the k expert MLPs of each sampled token."""
    per_tok = 6.0 * w.d * w.F * w.k                     # float64 MACs x 2 per sampled token
    widen = 3.0 * w.d * w.F * 4e-9                      # seconds to widen one expert (~4 ns per element)
    experts_per_tok = min(w.k, w.E)
    n = 8
    while n < w.T:
        touched = min(w.E, n * experts_per_tok)
        est = touched * widen + n * per_tok / 2e10
        if est > per_step_s:
            break
        n *= 2
    return max(4, min(w.T, n // 2 if n > 8 else n))


def run_reference(args):
    from mixture_experts_layer_41_b200.inputs import make_inputs, workload

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload_of(args)
    inp = make_inputs(w, seed=args.seed, device="cpu")
    n = args.cpu_sample or max(4, auto_sample(w, per_step_s=4.0))
    for _ in range(args.warmup):
        oracle_sample_run(w, inp, n, seed=args.seed)
    runs = [oracle_sample_run(w, inp, n, seed=args.seed + i) for i in range(args.steps)]
    sec = statistics.mean(o["estimate_s"] for o in runs)
    value = w.T / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample_text(w, runs[-1]) + "; a fresh token sample each step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_of(args):
    """The named workload, with --shape overrides (integers, floats or words)."""
    from mixture_experts_layer_41_b200.inputs import workload
    kw = {}
    for item in filter(None, args.shape.split(",")):
        key, val = item.split("=", 1)
        for conv in (int, float):
            try:
                val = conv(val)
                break
            except ValueError:
                continue
        kw[key.strip()] = val
    w = workload(args.workload, **kw)
    return w.with_(name=w.name + ("[" + args.shape + "]" if args.shape else ""))


def config_of(w, world: int) -> dict:
    return {"workload": w.name, "T": w.T, "d": w.d, "F": w.F, "E": w.E, "top_k": w.k, "act": w.act,
            "router": w.router, "capacity_factor": w.capacity_factor or None, "weights": w.weight_format,
            "shared_F": w.shared_F, "parallelism": f"replicas x{world}"}


def input_hashes(inp: dict) -> dict:
    """SHA-256 of every input tensor's bytes.  Large tensors are hashed in
    256 MiB chunks (in parallel); the tensor's digest is then the SHA-256 of
    its chunks' digests in order."""
    import concurrent.futures as cf
    chunk = 256 << 20
    out = {"scheme": "sha256 of each 256 MiB chunk of the tensor's bytes, then sha256 of the chunk digests"}

    workers = min(16, os.cpu_count() or 4)

    def digest(t):
        flat = t.detach().contiguous().view(-1).view(torch_uint8())
        offs = list(range(0, flat.numel(), chunk))
        parts = []
        with cf.ThreadPoolExecutor(max_workers=workers) as ex:
            for i in range(0, len(offs), workers):          # at most `workers` chunks on the host at once
                host = [flat[o:o + chunk].cpu().numpy() for o in offs[i:i + workers]]
                parts += list(ex.map(lambda b: hashlib.sha256(b).digest(), host))
        return hashlib.sha256(b"".join(parts)).hexdigest()

    for k in sorted(inp):
        if inp[k] is not None:
            out[k] = digest(inp[k])
    return out


def torch_uint8():
    import torch
    return torch.uint8


# ---------------------------------------------------------------- GPU arm

def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from mixture_experts_layer_41_b200 import _lib as L
    from mixture_experts_layer_41_b200 import api
    from mixture_experts_layer_41_b200.inputs import make_inputs, workload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    w = workload_of(args)
    inp = make_inputs(w, seed=args.seed + rank, device=dev)
    wf = "q4_affine_g64" if w.weight_format == "q4_affine_g64" else w.dtype
    cfg = api.make_config(num_tokens=w.T, hidden=w.d, intermediate=w.F, num_experts=w.E, top_k=w.k,
                          router=w.router, norm_topk_prob=w.norm_topk_prob,
                          routed_scaling=w.routed_scaling if w.router == "sigmoid_group" else 1.0,
                          n_group=w.n_group, topk_group=w.topk_group, capacity_factor=w.capacity_factor,
                          act=w.act, act_dtype=w.dtype, weight_dtype=wf, shared_intermediate=w.shared_F,
                          aux_alpha=w.aux_alpha, fused_gather=args.fused_gather)
    weights = {k: inp[k] for k in ("w1", "w2", "w3", "s1", "s2", "s3", "b1", "b2", "b3", "ws1", "ws2", "ws3")
               if inp.get(k) is not None}
    for i in "123":
        if inp.get("q" + i) is not None:
            weights["w" + i] = inp["q" + i]
    bias = inp["logit_bias"] if w.router == "softmax_topk" else inp["expert_bias"]
    layer = api.MoELayer(cfg, inp["w_router"], weights, router_bias=bias, device=dev)
    x = inp["x"]
    stream = torch.cuda.current_stream()

    # warm-up
    for _ in range(args.warmup):
        layer.forward(x)
    torch.cuda.synchronize()
    n0 = api.moe_kernel_launches()
    layer.forward(x)
    launches_per_step = api.moe_kernel_launches() - n0
    torch.cuda.synchronize()
    st = layer.status()
    if st != 0:
        raise SystemExit(f"device status {st}: {api.moe_status_string(st)}")

    # Eager steps with phase events recorded inside moe_forward on the
    # launching stream: the per-phase (per-kernel) times for the roofline.
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(L.MOE_PHASE_COUNT)] for _ in range(K)]
    for row in ev:              # torch creates the CUDA event on its first record
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    for i in range(K):
        api.moe_set_phase_events(ev[i])
        layer.forward(x)
    e_end.record(stream)
    torch.cuda.synchronize()
    api.moe_set_phase_events(None)
    eager_ms = e_start.elapsed_time(e_end) / K
    phases = {}
    names = ["route", "permute", "ffn1", "ffn2", "shared", "combine"]
    for p, nm in enumerate(names, start=1):
        phases[nm] = statistics.mean(ev[i][p - 1].elapsed_time(ev[i][p]) for i in range(K))

    # Headline: the same step replayed from a CUDA graph (one capture of
    # moe_forward: every kernel of the layer, launched without host overhead).
    graph = None
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            layer.forward(x)
        stream.wait_stream(side)
        with torch.cuda.graph(graph, capture_error_mode="relaxed"):
            layer.forward(x)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    except Exception as exc:  # noqa: BLE001
        graph = None
        print(f"cuda graph capture failed, timing eager launches: {exc}", file=sys.stderr)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local) if rank == 0 or world == 1 else None
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    start.record(stream)
    for i in range(K):
        if graph is not None:
            graph.replay()
        else:
            layer.forward(x)
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    st = layer.status()
    if st != 0:
        raise SystemExit(f"device status {st}: {api.moe_status_string(st)}")
    ms = start.elapsed_time(end) / K
    ms_t = torch.tensor([ms], device=dev)
    if world > 1:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())

    # routing outcome of the timed steps (identical every step)
    kept = layer.o.kept_counts.cpu().numpy()
    R = int(kept.sum())
    touched = int((kept > 0).sum())
    dropped = int(layer.o.dropped[0].item())
    aux_raw, aux = api.moe_aux_loss(cfg, layer.o.kept_counts.cpu(), layer.o.prob_sum.cpu())

    # e2e: the same layer through moe_forward_host with pinned host buffers.
    # Two streams with a workspace and result buffers each take the steps in
    # turn, as a serving loop would: step i+1's host->device copy runs while
    # step i's kernels do; every step's copies are inside the timed region.
    # The same loop on one stream is reported beside it ("serial").
    dt = x.dtype
    x_host = x.cpu().pin_memory()
    streams = [torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)]
    wss = [layer.ws, torch.empty_like(layer.ws)]
    host_out = [dict(out=torch.empty((w.T, w.d), dtype=dt).pin_memory(),
                     kc=torch.empty(w.E, dtype=torch.int32).pin_memory(),
                     ps=torch.empty(w.E, dtype=torch.float32).pin_memory(),
                     dr=torch.empty(4, dtype=torch.int32).pin_memory()) for _ in range(2)]

    def host_step(i, n_streams):
        j = i % n_streams
        h = host_out[j]
        api.moe_forward_host(cfg, x_host, inp["w_router"], bias, weights, h["out"], h["kc"], h["ps"], h["dr"],
                             wss[j], stream=streams[j])

    def timed_host_loop(n_streams):
        for i in range(max(2, args.warmup // 2) * n_streams):
            host_step(i, n_streams)
        torch.cuda.synchronize()
        barrier()
        e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_s.record(streams[0])
        streams[1].wait_event(e_s)
        for i in range(K):
            host_step(i, n_streams)
        done = torch.cuda.Event()
        done.record(streams[1])
        streams[0].wait_event(done)
        e_e.record(streams[0])
        torch.cuda.synchronize()
        t = torch.tensor([e_s.elapsed_time(e_e) / K], device=dev)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    e2e_serial_ms = timed_host_loop(1)
    e2e_ms = timed_host_loop(2)
    out_host = host_out[(K - 1) % 2]["out"]
    h2d = x_host.numel() * x_host.element_size()
    d2h = out_host.numel() * out_host.element_size() + 2 * 4 * w.E + 4
    same = torch.equal(out_host.view(torch.int16) if dt == torch.bfloat16 else out_host,
                       layer.o.out.cpu().view(torch.int16) if dt == torch.bfloat16 else layer.o.out.cpu())

    peaks, peak_src = load_peaks()
    costs = layer_costs(w, R, touched)
    # Denominators: the burst bf16 GEMM figure (a timed region of a few
    # hundred steps is seconds at most; the clocks sampled during it are in
    # "clocks"), with the fraction of the sustained (power-capped) figure
    # reported beside it.
    tensor_peak = peaks["bf16_tflops"] * 1e12
    sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * 1e12
    hbm_peak = peaks["hbm_gbs"] * 1e9
    tensor_bound = w.weight_format == "dense" and w.dtype == "bf16"

    def phase_roof(name):
        c = costs[name]
        t = phases[name] * 1e-3
        if tensor_bound and c["flops"] / tensor_peak >= c["bytes"] / hbm_peak:
            a = c["flops"] / t / 1e12
            return {"bound": "tensor", "achieved": a, "peak": tensor_peak / 1e12, "unit": "TFLOP/s",
                    "frac": a * 1e12 / tensor_peak, "frac_of_sustained": a * 1e12 / sustained, "ms": phases[name]}
        a = c["bytes"] / t / 1e9
        return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": a * 1e9 / hbm_peak, "ms": phases[name]}

    gemm_phases = {"ffn1": phase_roof("ffn1"), "ffn2": phase_roof("ffn2")}
    # dominant kernel: the longer expert GEMM phase
    dom = "ffn1" if phases["ffn1"] >= phases["ffn2"] else "ffn2"
    dk = costs[dom]
    roof = {k: v for k, v in gemm_phases[dom].items() if k != "ms"}
    kernel_file = os.path.join(ROOT, "mixture_experts_layer_41_b200", "csrc", ffn_kernel_file(w))
    roof["traffic"] = recorded_traffic(kernel_file, f"{w.name}:{dom}")
    roof["kernel"] = {"ffn1": "grouped expert GEMM, phase 1 (gate/up or in)",
                      "ffn2": "grouped expert GEMM, phase 2 (down or out)"}[dom] + \
        (" with the shared expert as one more group" if shared_in_gemm(w) else "")
    roof["peak_source"] = f"{peak_src} ({'bf16 GEMM, burst' if roof['bound'] == 'tensor' else 'HBM copy'})"
    roof["algorithmic"] = {"flop_per_launch": dk["flops"], "bytes_per_launch": dk["bytes"],
                           "ms_per_launch": phases[dom]}
    t_layer_roof = max(costs["flops"] / tensor_peak, costs["bytes"] / hbm_peak)
    t_layer_roof_sus = max(costs["flops"] / sustained, costs["bytes"] / hbm_peak)

    per_gpu = w.T / (ms_max * 1e-3)
    line = {
        "metric": METRIC, "value": per_gpu * world, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else w.dtype, "data": "synthetic",
        "config": dict(config_of(w, world),
                       l2="inputs larger than L2: every step streams all touched expert weights "
                          f"({costs['bytes'] / 1e9:.2f} GB) from HBM",
                       **({"fused_gather": True} if args.fused_gather else {}),
                       **({"paired_sms": True} if os.environ.get("MOE_TC_PAIR") == "1" else {})),
        "roofline": roof,
        "gemm_phases": gemm_phases,
        "layer_roofline": {"frac": t_layer_roof / (ms_max * 1e-3), "roof_ms": t_layer_roof * 1e3,
                           "frac_of_sustained": t_layer_roof_sus / (ms_max * 1e-3),
                           "flop": costs["flops"], "bytes": costs["bytes"],
                           "tflops": costs["flops"] / (ms_max * 1e-3) / 1e12},
        "phases_ms": {k: round(v, 4) for k, v in phases.items()},
        "routing": {"rows": R, "touched_experts": touched, "dropped": dropped, "aux_raw": aux_raw, "aux": aux},
        "e2e": {"value": world * w.T / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "streams": 2,
                "serial": {"value": world * w.T / (e2e_serial_ms * 1e-3), "ms_per_step": e2e_serial_ms,
                           "streams": 1},
                "matches_device_out": bool(same)},
        "gpu_launches": K * launches_per_step,
        "launches_per_step": launches_per_step,
        "launch": "cuda_graph" if graph is not None else "eager",
        "eager_ms_per_step": eager_ms,
        "clocks": clocks,
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = args.cpu_sample or auto_sample(w)
        o = oracle_sample_run(w, dict(inp), n, seed=args.seed)
        toks = o["tokens"]
        got = layer.o.out.float().cpu().numpy().astype(np.float64)[toks]
        ref = o["result"]["out"][toks]
        err = float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))
        line["cpu_baseline"] = {"value": w.T / o["estimate_s"], "unit": UNIT, "cores": blas_threads(),
                                "kind": "oracle", "sample": sample_text(w, o)}
        line["parity_on_sample"] = {"tokens": int(len(toks)), "rel_err": err,
                                    "tol": 1e-5 if w.dtype == "f32" else 2e-2,
                                    "ok": err <= (1e-5 if w.dtype == "f32" else 2e-2)}
    if rank == 0 and not args.no_hash:
        line["inputs_sha256"] = input_hashes(inp)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
