"""Multi-process paths on CPU with the gloo backend (world size 2).

1. The token-sharded capacity exchange: each rank all-gathers the per-expert
   raw counts of its token shard and keeps a slot iff (slots of its expert on
   earlier shards + its rank on this shard) < the whole batch's capacity.  The
   union of the ranks' kept slots must equal the oracle's in-order dispatch of
   the whole batch.
2. The bench's replica timing: every rank's step time is reduced with MAX.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_41_b200 import api
from oracle import moe_oracle as O

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=__import__("datetime").timedelta(seconds=60))


def _shard_worker(rank, port, ids, cap, out_q):
    _init(rank, port)
    T, k = ids.shape
    E = int(ids.max()) + 1
    lo, hi = rank * T // WORLD, (rank + 1) * T // WORLD
    mine = ids[lo:hi]
    raw = torch.from_numpy(np.bincount(mine.reshape(-1), minlength=E).astype(np.int32))
    gathered_counts = api.exchange_counts(raw).numpy()       # [world, E], row q = shard q
    assert gathered_counts.shape == (WORLD, E) and np.array_equal(gathered_counts[rank], raw.numpy())
    base = gathered_counts[:rank].sum(axis=0)                # the prefix moe_permute_shard forms
    # this shard's kept slots under the shard rule (plain loops, token order)
    seen = np.zeros(E, dtype=np.int64)
    kept = []
    for t in range(mine.shape[0]):
        for j in range(k):
            e = int(mine[t, j])
            if cap is None or base[e] + seen[e] < cap:
                kept.append((lo + t, j))
            seen[e] += 1
    gathered = [None] * WORLD
    dist.all_gather_object(gathered, kept)
    # replica timing: max over ranks
    t = torch.tensor([1.0 + rank])
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    if rank == 0:
        out_q.put((gathered, float(t.item()), [int(v) for v in base]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("cf", [1.0, 1.25, 0.0])
def test_sharded_capacity_matches_whole_batch(cf):
    rng = np.random.default_rng(7)
    T, E, k = 90, 6, 2
    logits = rng.standard_normal((T, E)) + np.array([2.0, 1.0, 0.5, 0.0, -0.5, -1.0])
    ids, w, _, _ = O.route_softmax_topk(logits, k, True)
    cap = O.capacity(T, k, E, cf)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, port, ids, cap, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    gathered, tmax, base0 = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    union = sorted(s for part in gathered for s in part)
    ref = O.dispatch(ids, E, cap, w)
    ref_kept = sorted((int(t), int(j)) for t in range(T) for j in range(k) if ref["slot_row"][t, j] >= 0)
    assert union == ref_kept
    assert base0 == [0] * E
    assert tmax == 2.0
    if cap is not None:
        assert len(union) < T * k      # the skew makes the first expert overflow
