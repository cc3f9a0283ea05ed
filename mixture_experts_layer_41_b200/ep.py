"""Expert parallelism across GPUs: each rank holds a contiguous block of the
layer's experts, tokens travel to the rank that holds their expert and come
back ("Mixture-of-Experts" design doc, The pipeline: the expert-parallel
dispatch of step 2 and the combine of step 4).

Rank r of N holds experts [r*E/N, (r+1)*E/N) and routes its own batch of T
tokens.  One forward:

1. route over all E experts (the router weight is replicated) and dispatch
   locally (``moe_permute``; a capacity limit applies to this rank's batch).
   The dispatched rows are expert-sorted, so the rows bound for rank q are one
   contiguous block: no extra permutation before the exchange.
2. exchange: one all-to-all of the per-expert kept counts (E/N int32 per rank
   pair), then one all-to-all of the rows, each rank's block landing in the
   receiver's own memory.
3. the received rows (grouped by source, then by local expert) are grouped by
   local expert with the dispatch kernel (one slot per row, weight 1), run
   through the grouped FFN of the local experts, and put back into arrival
   order with the combine kernel (weight 1: an exact copy).
4. the reverse all-to-all returns every row to its source in the order it
   was sent, which is this rank's dispatch order: the local combine (plus the
   shared expert, computed where the token lives) finishes the layer.

The orchestration is written against a small set of operations so that the
same code runs on the device (``DeviceOps``: this library's kernels) and, in
tests, on the host.  The collectives are ``torch.distributed`` calls (NCCL on
GPUs); ``EPLayer.forward`` does them, and the phase methods let one process
drive several shards and move the blocks itself.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Sequence

import torch

from . import _lib as L
from . import api


@dataclass
class Dispatched:
    """What a rank sends: expert-sorted rows, the kept count of every expert
    (reshaped [world, E/N]: row q is what rank q receives), and what the local
    combine needs later.  ``rows`` may be longer than the kept rows (the
    dispatch buffer); the first sum(counts) rows are sent."""
    rows: torch.Tensor          # [>= R, d]
    counts: torch.Tensor        # [world, E_local] int32 (on the rows' device)
    slot_row: torch.Tensor      # [T, k]
    topk_w: torch.Tensor        # [T, k]
    topk_ids: torch.Tensor      # [T, k]
    x: torch.Tensor             # [T, d] (for the shared expert)


def split_sizes_pair(send_counts: torch.Tensor, recv_counts: torch.Tensor):
    """Rows per peer to send and to receive, from the [world, E_local] count
    tables: the one device-to-host read the row all-to-all needs (its split
    sizes are host integers)."""
    both = torch.stack([send_counts.sum(dim=1), recv_counts.sum(dim=1)]).to(torch.int64).cpu()
    return [int(v) for v in both[0].tolist()], [int(v) for v in both[1].tolist()]


class DeviceOps:
    """The layer's steps on this library's kernels, for one rank's shard."""

    def __init__(self, cfg: L.moe_config, w_router: torch.Tensor, local_weights: dict, world: int,
                 router_bias: Optional[torch.Tensor] = None, device=None):
        self.cfg = cfg
        self.world = world
        self.E = cfg.num_experts
        if self.E % world or self.E // world < 2:
            raise ValueError("expert parallelism needs E divisible by the world size, at least 2 experts per rank")
        self.e_local = self.E // world
        self.dev = torch.device(device) if device is not None else w_router.device
        self.w_router = w_router
        self.bias = router_bias
        self.weights = local_weights
        self.dt = torch.float32 if cfg.act_dtype == L.MOE_F32 else torch.bfloat16
        T, k, d = cfg.num_tokens, cfg.top_k, cfg.hidden
        i32 = dict(dtype=torch.int32, device=self.dev)
        self.ws = torch.empty(api.moe_workspace_size(cfg), dtype=torch.uint8, device=self.dev)
        self.ids = torch.empty((T, k), **i32)
        self.wts = torch.empty((T, k), dtype=torch.float32, device=self.dev)
        self.prob_sum = torch.empty(self.E, dtype=torch.float32, device=self.dev)
        self.offsets = torch.empty(self.E + 1, **i32)
        self.perm_token = torch.empty(T * k, **i32)
        self.perm_w = torch.empty(T * k, dtype=torch.float32, device=self.dev)
        self.slot_row = torch.empty((T, k), **i32)
        self.x_perm = torch.empty((T * k, d), dtype=self.dt, device=self.dev)
        self.stats = dict(raw_counts=torch.empty(self.E, **i32), kept_counts=torch.empty(self.E, **i32),
                          prob_sum=self.prob_sum, dropped=torch.empty(4, **i32))
        # the expert side: at most every row of every rank lands here
        self.max_rows = world * T * k
        self.cfg_local_max = self._local_cfg(self.max_rows)
        self.ws_local = torch.empty(api.moe_workspace_size(self.cfg_local_max), dtype=torch.uint8, device=self.dev)
        self.shared = torch.empty((T, d), dtype=self.dt, device=self.dev) if cfg.shared_intermediate > 0 else None

    def _local_cfg(self, rows: int) -> L.moe_config:
        c = self.cfg
        return L.moe_config(rows, c.hidden, c.intermediate, self.e_local, 1, L.MOE_ROUTER_SOFTMAX_TOPK, 1, 1.0,
                            1, 1, 0.0, c.act, c.act_dtype, c.weight_dtype, 0, 0.0, c.weight_layout, 0)

    def dispatch(self, x: torch.Tensor) -> Dispatched:
        c = self.cfg
        api.moe_route(c, x, self.w_router, self.bias, self.ids, self.wts, self.prob_sum, self.ws)
        api.moe_permute(c, x, self.ids, self.wts, self.offsets, self.perm_token, self.perm_w, self.slot_row,
                        self.x_perm, self.stats, self.ws)
        return Dispatched(self.x_perm, self.stats["kept_counts"].view(self.world, self.e_local), self.slot_row,
                          self.wts, self.ids, x)

    def expert(self, rows: torch.Tensor, recv_counts: torch.Tensor) -> torch.Tensor:
        n = rows.shape[0]
        out = torch.empty_like(rows)
        if n == 0:
            return out
        cfg = self._local_cfg(n)
        i32 = dict(dtype=torch.int32, device=self.dev)
        ids = torch.empty((n, 1), **i32)
        api.moe_ep_local_ids(recv_counts.to(device=self.dev, dtype=torch.int32).contiguous(), n, ids)
        ones = torch.ones((n, 1), dtype=torch.float32, device=self.dev)
        off = torch.empty(self.e_local + 1, **i32)
        perm_token = torch.empty(n, **i32)
        perm_w = torch.empty(n, dtype=torch.float32, device=self.dev)
        slot_row = torch.empty((n, 1), **i32)
        grouped = torch.empty_like(rows)
        y = torch.empty_like(rows)
        st = dict(raw_counts=torch.empty(self.e_local, **i32), kept_counts=torch.empty(self.e_local, **i32),
                  dropped=torch.empty(4, **i32))
        api.moe_permute(cfg, rows, ids, ones, off, perm_token, perm_w, slot_row, grouped, st, self.ws_local)
        api.moe_grouped_ffn(cfg, grouped, off, self.weights, y, self.ws_local)
        api.moe_combine(cfg, y, slot_row, ones, None, out)
        return out

    def combine(self, back: torch.Tensor, disp: Dispatched) -> torch.Tensor:
        c = self.cfg
        out = torch.empty((c.num_tokens, c.hidden), dtype=self.dt, device=self.dev)
        shared = None
        if self.shared is not None:
            api.moe_shared_expert(c, disp.x, self.weights, self.shared, self.ws)
            shared = self.shared
        y = back if back.shape[0] > 0 else self.x_perm[:1]
        api.moe_combine(c, y.contiguous(), disp.slot_row, disp.topk_w, shared, out)
        return out

    def status(self) -> int:
        s = api.moe_workspace_status(self.ws)
        return s if s != L.MOE_OK else api.moe_workspace_status(self.ws_local)


def exchange_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """All-to-all of the [world, E_local] kept-count tables: row q of the result
    is what rank q sends here, per local expert.  Stays on the tensors'
    device (NCCL: the GPU; gloo: the host)."""
    import torch.distributed as dist
    world, e_local = counts.shape
    send = counts.reshape(-1).to(torch.int32).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.view(world, e_local)


def exchange_rows(rows: torch.Tensor, send_sizes: Sequence[int], recv_sizes: Sequence[int],
                  group=None) -> torch.Tensor:
    """All-to-all of row blocks with per-peer sizes (rows of width d)."""
    import torch.distributed as dist
    d = rows.shape[1]
    out = torch.empty((sum(recv_sizes), d), dtype=rows.dtype, device=rows.device)
    dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=list(recv_sizes),
                           input_split_sizes=list(send_sizes), group=group)
    return out


class EPLayer:
    """One rank's share of an expert-parallel layer: ``forward`` runs the four
    steps with the collectives of ``group``."""

    def __init__(self, ops, group=None):
        self.ops = ops
        self.group = group

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        disp = self.ops.dispatch(x)
        recv_counts = exchange_counts(disp.counts, self.group)
        send_sizes, recv_sizes = split_sizes_pair(disp.counts, recv_counts)
        rows_in = exchange_rows(disp.rows[:sum(send_sizes)], send_sizes, recv_sizes, self.group)
        rows_out = self.ops.expert(rows_in, recv_counts)
        back = exchange_rows(rows_out, recv_sizes, send_sizes, self.group)
        return self.ops.combine(back, disp)


def emulate(shards: Sequence, xs: Sequence[torch.Tensor]) -> list:
    """Run an expert-parallel forward of several shards in one process: the
    same four steps as ``EPLayer.forward``, with the all-to-alls done by
    slicing and concatenating the blocks (for a single device)."""
    world = len(shards)
    disps = [s.dispatch(x) for s, x in zip(shards, xs)]
    sizes = [split_sizes_pair(dp.counts, dp.counts)[0] for dp in disps]    # sizes[src][dst]
    blocks = []
    for dp, sz in zip(disps, sizes):
        starts = [sum(sz[:q]) for q in range(world)]
        blocks.append([dp.rows[starts[q]:starts[q] + sz[q]] for q in range(world)])
    outs_back = [[None] * world for _ in range(world)]
    for dst, shard in enumerate(shards):
        recv_counts = torch.stack([disps[src].counts[dst] for src in range(world)])
        rows_in = torch.cat([blocks[src][dst] for src in range(world)], dim=0)
        rows_out = shard.expert(rows_in, recv_counts)
        off = 0
        for src in range(world):
            n = sizes[src][dst]
            outs_back[src][dst] = rows_out[off:off + n]
            off += n
    return [shard.combine(torch.cat(outs_back[src], dim=0), disps[src]) for src, shard in enumerate(shards)]
