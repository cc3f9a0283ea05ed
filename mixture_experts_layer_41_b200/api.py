"""Python face of the C ABI in include/moe.h: the same calls, same names.

Each function converts torch tensors to raw pointers and forwards to
libmoe.so; every step of the layer runs in the library's kernels.  torch is
used for device memory and streams only.  Output tensors are caller-owned,
as in C; ``MoELayer`` is a convenience holder that allocates them.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib as L
from ._lib import check, moe_config, moe_stats, moe_weights

_ROUTERS = {"softmax_topk": L.MOE_ROUTER_SOFTMAX_TOPK, "sigmoid_group": L.MOE_ROUTER_SIGMOID_GROUP}
_ACTS = {"relu": L.MOE_ACT_RELU, "swiglu": L.MOE_ACT_SWIGLU}
_DTYPES = {"f32": L.MOE_F32, "bf16": L.MOE_BF16, "q4_affine_g64": L.MOE_Q4_AFFINE_G64}
_TORCH_DT = {L.MOE_F32: torch.float32, L.MOE_BF16: torch.bfloat16}
_LAYOUTS = {"separate": L.MOE_LAYOUT_SEPARATE, "fused_gate_up": L.MOE_LAYOUT_FUSED_GATE_UP}


def make_config(*, num_tokens: int, hidden: int, intermediate: int, num_experts: int, top_k: int,
                router: str = "softmax_topk", norm_topk_prob: bool = True, routed_scaling: float = 1.0,
                n_group: int = 1, topk_group: int = 1, capacity_factor: float = 0.0,
                act: str = "swiglu", act_dtype: str = "bf16", weight_dtype: str = "bf16",
                shared_intermediate: int = 0, aux_alpha: float = 0.01,
                weight_layout: str = "separate", fused_gather: bool = False) -> moe_config:
    return moe_config(num_tokens, hidden, intermediate, num_experts, top_k, _ROUTERS[router],
                      1 if norm_topk_prob else 0, routed_scaling, n_group, topk_group,
                      capacity_factor, _ACTS[act], _DTYPES[act_dtype], _DTYPES[weight_dtype],
                      shared_intermediate, aux_alpha, _LAYOUTS[weight_layout], 1 if fused_gather else 0)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return t.data_ptr()


def _s(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


# ---------------------------------------------------------------- host-only calls

def moe_capacity(num_tokens: int, top_k: int, num_experts: int, capacity_factor: float) -> int:
    return L.lib().moe_capacity(num_tokens, top_k, num_experts, capacity_factor)


def moe_validate(cfg: moe_config) -> int:
    return L.lib().moe_validate(C.byref(cfg))


def moe_workspace_size(cfg: moe_config) -> int:
    return L.lib().moe_workspace_size(C.byref(cfg))


def moe_aux_loss(cfg: moe_config, kept_counts_host: torch.Tensor, prob_sum_host: torch.Tensor):
    raw, scaled = C.c_double(), C.c_double()
    kc = kept_counts_host.to(torch.int32).contiguous()
    ps = prob_sum_host.to(torch.float32).contiguous()
    check(L.lib().moe_aux_loss(C.byref(cfg), kc.data_ptr(), ps.data_ptr(), C.byref(raw), C.byref(scaled)),
          "moe_aux_loss")
    return raw.value, scaled.value


def moe_routing_health(cfg: moe_config, kept_counts_host: torch.Tensor, dropped: int) -> dict:
    er, ms, df, col = C.c_double(), C.c_double(), C.c_double(), C.c_int32()
    kc = kept_counts_host.to(torch.int32).contiguous()
    check(L.lib().moe_routing_health(C.byref(cfg), kc.data_ptr(), int(dropped), C.byref(er), C.byref(ms),
                                     C.byref(df), C.byref(col)), "moe_routing_health")
    return dict(entropy_ratio=er.value, max_share=ms.value, dropped_fraction=df.value,
                collapsed=bool(col.value))


def moe_kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return L.lib().moe_kernel_launches()


def moe_set_wait_timeout_ns(ns: int) -> None:
    """Bound on the tensor-core kernels' barrier waits (0: the 2 s default)."""
    check(L.lib().moe_set_wait_timeout_ns(int(ns)), "moe_set_wait_timeout_ns")


def moe_status_string(status: int) -> str:
    return L.lib().moe_status_string(status).decode()


def moe_set_phase_events(events) -> None:
    """Register MOE_PHASE_COUNT torch.cuda.Event objects (or None to turn it off)."""
    if events is None:
        check(L.lib().moe_set_phase_events(None, 0), "moe_set_phase_events")
        return
    for e in events:
        if not e.cuda_event:
            raise ValueError("record each event once before registering it (torch creates it lazily)")
    arr = (C.c_void_p * len(events))(*[e.cuda_event for e in events])
    check(L.lib().moe_set_phase_events(arr, len(events)), "moe_set_phase_events")


def moe_workspace_status(ws: torch.Tensor, stream=None) -> int:
    return L.lib().moe_workspace_status(_p(ws), _s(stream))


_REGIONS = {"offsets": L.MOE_WS_OFFSETS, "perm_token": L.MOE_WS_PERM_TOKEN, "perm_w": L.MOE_WS_PERM_W,
            "slot_row": L.MOE_WS_SLOT_ROW, "x_perm": L.MOE_WS_X_PERM, "h": L.MOE_WS_H, "y_perm": L.MOE_WS_Y_PERM,
            "shared_h": L.MOE_WS_SHARED_H, "shared_out": L.MOE_WS_SHARED_OUT,
            "router_logits": L.MOE_WS_ROUTER_LOGITS}


def moe_workspace_region(cfg: moe_config, region: str):
    """(byte offset, bytes) of one of moe_forward's intermediates inside the workspace."""
    off, n = C.c_size_t(), C.c_size_t()
    check(L.lib().moe_workspace_region(C.byref(cfg), _REGIONS[region], C.byref(off), C.byref(n)),
          "moe_workspace_region")
    return off.value, n.value


def workspace_view(cfg: moe_config, ws: torch.Tensor, region: str, dtype: torch.dtype, cols: int = 1):
    """A tensor view of one workspace region (no copy), [bytes / (cols * itemsize), cols]."""
    off, n = moe_workspace_region(cfg, region)
    return ws[off:off + n].view(dtype).view(-1, cols)


# ---------------------------------------------------------------- device calls

def _weights_struct(w: dict) -> moe_weights:
    g = lambda k: _p(w.get(k))
    return moe_weights(g("w1"), g("w2"), g("w3"), g("s1"), g("s2"), g("s3"), g("b1"), g("b2"), g("b3"),
                       g("ws1"), g("ws2"), g("ws3"))


def _stats_struct(stats: Optional[dict]) -> Optional[moe_stats]:
    if stats is None:
        return None
    g = lambda k: _p(stats.get(k))
    return moe_stats(g("raw_counts"), g("kept_counts"), g("prob_sum"), g("dropped"))


def moe_route(cfg, x, w_router, router_bias, topk_ids, topk_w, prob_sum, ws, stream=None):
    check(L.lib().moe_route(C.byref(cfg), _p(x), _p(w_router), _p(router_bias), _p(topk_ids), _p(topk_w),
                            _p(prob_sum), _p(ws), _nbytes(ws), _s(stream)), "moe_route")


def moe_route_forced(cfg, x, w_router, router_bias, forced_ids, topk_ids, topk_w, prob_sum, ws, stream=None):
    check(L.lib().moe_route_forced(C.byref(cfg), _p(x), _p(w_router), _p(router_bias), _p(forced_ids),
                                   _p(topk_ids), _p(topk_w), _p(prob_sum), _p(ws), _nbytes(ws), _s(stream)),
          "moe_route_forced")


def moe_update_bias(cfg, counts, expert_bias, coeff: float, stream=None):
    check(L.lib().moe_update_bias(C.byref(cfg), _p(counts), _p(expert_bias), coeff, _s(stream)),
          "moe_update_bias")


def moe_route_noalloc(cfg, x, w_router, router_bias, topk_ids, topk_w, prob_sum, stream=None):
    """moe_route for callers that cannot allocate: no workspace argument; the
    router's scratch is a fixed 1 MiB device array inside the library (see
    include/moe.h for the size limit and the rule that overlapping calls race)."""
    st = L.lib().moe_route_noalloc(C.byref(cfg), _p(x), _p(w_router), _p(router_bias), _p(topk_ids),
                                   _p(topk_w), _p(prob_sum), _s(stream))
    if st != L.MOE_OK:
        raise L.MoEError(st, "moe_route_noalloc: " + L.lib().moe_last_error().decode())


def moe_permute(cfg, x, topk_ids, topk_w, expert_offsets, perm_token, perm_w, slot_row, x_perm, stats, ws,
                stream=None):
    st = _stats_struct(stats)
    check(L.lib().moe_permute(C.byref(cfg), _p(x), _p(topk_ids), _p(topk_w), _p(expert_offsets),
                              _p(perm_token), _p(perm_w), _p(slot_row), _p(x_perm),
                              C.byref(st) if st is not None else None, _p(ws), _nbytes(ws), _s(stream)),
          "moe_permute")


def moe_expert_counts(cfg, topk_ids, raw_counts, ws, stream=None):
    check(L.lib().moe_expert_counts(C.byref(cfg), _p(topk_ids), _p(raw_counts), _p(ws), _nbytes(ws),
                                    _s(stream)), "moe_expert_counts")


def moe_permute_shard(cfg, x, topk_ids, topk_w, counts_by_rank, rank, capacity, expert_offsets, perm_token,
                      perm_w, slot_row, x_perm, stats, ws, stream=None):
    """``counts_by_rank``: [world, E] int32 device tensor of every shard's
    moe_expert_counts (``exchange_counts``), or None for a single shard."""
    st = _stats_struct(stats)
    world = 1 if counts_by_rank is None else int(counts_by_rank.shape[0])
    check(L.lib().moe_permute_shard(C.byref(cfg), _p(x), _p(topk_ids), _p(topk_w), _p(counts_by_rank), world,
                                    int(rank), int(capacity), _p(expert_offsets), _p(perm_token), _p(perm_w),
                                    _p(slot_row), _p(x_perm), C.byref(st) if st is not None else None, _p(ws),
                                    _nbytes(ws), _s(stream)),
          "moe_permute_shard")


def exchange_counts(raw_counts: torch.Tensor, group=None) -> torch.Tensor:
    """The sharded layer's one exchange: all-gather every rank's per-expert
    raw counts (an E-int32 message per rank) into a [world, E] tensor on the
    same device.  Token shards must be contiguous and in rank order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    n = raw_counts.numel()
    gathered = torch.empty(world * n, dtype=raw_counts.dtype, device=raw_counts.device)
    dist.all_gather_into_tensor(gathered, raw_counts.reshape(-1).contiguous(), group=group)
    return gathered.view(world, n)


def moe_ep_local_ids(recv_counts, rows: int, ids, stream=None):
    """Local expert id of each received row (arrival order) from the
    [world, experts_per_rank] received counts."""
    world, e_local = recv_counts.shape
    check(L.lib().moe_ep_local_ids(_p(recv_counts), int(world), int(e_local), int(rows), _p(ids), _s(stream)),
          "moe_ep_local_ids")


def moe_grouped_ffn(cfg, x_perm, expert_offsets, weights: dict, y_perm, ws, stream=None):
    w = _weights_struct(weights)
    check(L.lib().moe_grouped_ffn(C.byref(cfg), _p(x_perm), _p(expert_offsets), C.byref(w), _p(y_perm),
                                  _p(ws), _nbytes(ws), _s(stream)), "moe_grouped_ffn")


def moe_shared_expert(cfg, x, weights: dict, shared_out, ws, stream=None):
    w = _weights_struct(weights)
    check(L.lib().moe_shared_expert(C.byref(cfg), _p(x), C.byref(w), _p(shared_out), _p(ws), _nbytes(ws),
                                    _s(stream)), "moe_shared_expert")


def moe_combine(cfg, y_perm, slot_row, topk_w, shared_out, out, stream=None):
    check(L.lib().moe_combine(C.byref(cfg), _p(y_perm), _p(slot_row), _p(topk_w), _p(shared_out), _p(out),
                              _s(stream)), "moe_combine")


def moe_forward(cfg, x, w_router, router_bias, weights: dict, out, topk_ids, topk_w, stats, ws, stream=None):
    w = _weights_struct(weights)
    st = _stats_struct(stats)
    check(L.lib().moe_forward(C.byref(cfg), _p(x), _p(w_router), _p(router_bias), C.byref(w), _p(out),
                              _p(topk_ids), _p(topk_w), C.byref(st) if st is not None else None, _p(ws),
                              _nbytes(ws), _s(stream)), "moe_forward")


def moe_forward_host(cfg, x_host, w_router, router_bias, weights: dict, out_host, kept_counts_host,
                     prob_sum_host, dropped_host, ws, stream=None):
    w = _weights_struct(weights)
    check(L.lib().moe_forward_host(C.byref(cfg), _p(x_host), _p(w_router), _p(router_bias), C.byref(w),
                                   _p(out_host), _p(kept_counts_host), _p(prob_sum_host), _p(dropped_host),
                                   _p(ws), _nbytes(ws), _s(stream)), "moe_forward_host")


# ---------------------------------------------------------------- convenience holder

@dataclass
class Outputs:
    out: torch.Tensor
    topk_ids: torch.Tensor
    topk_w: torch.Tensor
    raw_counts: torch.Tensor
    kept_counts: torch.Tensor
    prob_sum: torch.Tensor
    dropped: torch.Tensor


class MoELayer:
    """Holds a config, device-resident weights, a workspace and output buffers,
    and runs ``moe_forward`` on them."""

    def __init__(self, cfg: moe_config, w_router: torch.Tensor, weights: dict,
                 router_bias: Optional[torch.Tensor] = None, device=None):
        status = moe_validate(cfg)
        check(status, "moe_validate")
        self.cfg = cfg
        self.device = torch.device(device) if device is not None else w_router.device
        self.w_router = w_router
        self.router_bias = router_bias
        self.weights = weights
        self.ws = torch.empty(moe_workspace_size(cfg), dtype=torch.uint8, device=self.device)
        T, k, E, d = cfg.num_tokens, cfg.top_k, cfg.num_experts, cfg.hidden
        dt = _TORCH_DT[cfg.act_dtype]
        i32 = dict(dtype=torch.int32, device=self.device)
        self.o = Outputs(out=torch.empty((T, d), dtype=dt, device=self.device),
                         topk_ids=torch.empty((T, k), **i32),
                         topk_w=torch.empty((T, k), dtype=torch.float32, device=self.device),
                         raw_counts=torch.empty(E, **i32), kept_counts=torch.empty(E, **i32),
                         prob_sum=torch.empty(E, dtype=torch.float32, device=self.device),
                         dropped=torch.empty(4, **i32))

    def stats(self) -> dict:
        o = self.o
        return dict(raw_counts=o.raw_counts, kept_counts=o.kept_counts, prob_sum=o.prob_sum, dropped=o.dropped)

    def forward(self, x: torch.Tensor, stream=None, forced_ids: Optional[torch.Tensor] = None) -> Outputs:
        """One layer forward.  ``forced_ids`` [T, k] int32 replays recorded
        expert choices (router replay): the stages then run one by one, with
        moe_route_forced in place of the router.  Bad recorded ids surface, as
        in moe_forward, through ``status()`` (the dispatch flags them too)."""
        o = self.o
        if forced_ids is None:
            moe_forward(self.cfg, x, self.w_router, self.router_bias, self.weights, o.out, o.topk_ids,
                        o.topk_w, self.stats(), self.ws, stream)
            return o
        cfg = self.cfg
        T, k, d = cfg.num_tokens, cfg.top_k, cfg.hidden
        if not hasattr(self, "_stage"):
            i32 = dict(dtype=torch.int32, device=self.device)
            dt = _TORCH_DT[cfg.act_dtype]
            self._stage = dict(off=torch.empty(cfg.num_experts + 1, **i32), perm_token=torch.empty(T * k, **i32),
                               perm_w=torch.empty(T * k, dtype=torch.float32, device=self.device),
                               slot_row=torch.empty((T, k), **i32),
                               x_perm=torch.empty((T * k, d), dtype=dt, device=self.device),
                               y_perm=torch.empty((T * k, d), dtype=dt, device=self.device),
                               shared=torch.empty((T, d), dtype=dt, device=self.device)
                               if cfg.shared_intermediate > 0 else None)
        st = self._stage
        moe_route_forced(cfg, x, self.w_router, self.router_bias, forced_ids, o.topk_ids, o.topk_w, o.prob_sum,
                         self.ws, stream)
        moe_permute(cfg, x, o.topk_ids, o.topk_w, st["off"], st["perm_token"], st["perm_w"], st["slot_row"],
                    st["x_perm"], self.stats(), self.ws, stream)
        moe_grouped_ffn(cfg, st["x_perm"], st["off"], self.weights, st["y_perm"], self.ws, stream)
        if st["shared"] is not None:
            moe_shared_expert(cfg, x, self.weights, st["shared"], self.ws, stream)
        moe_combine(cfg, st["y_perm"], st["slot_row"], o.topk_w, st["shared"], o.out, stream)
        return o

    def update_bias(self, coeff: float, stream=None) -> None:
        """Aux-loss-free balancing step on ``router_bias`` from the last
        forward's raw per-expert counts (moe_update_bias)."""
        if self.router_bias is None:
            raise ValueError("update_bias needs a router_bias tensor")
        moe_update_bias(self.cfg, self.o.raw_counts, self.router_bias, coeff, stream)

    def status(self, stream=None) -> int:
        return moe_workspace_status(self.ws, stream)
