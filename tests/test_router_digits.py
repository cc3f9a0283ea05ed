"""The integer tensor-core router's arithmetic contract, on the CPU: the digit
model of its logits (tests/router_digits.py) stays within the stated bound of
the oracle's float64 logits, on the workloads' recipes and on rows built to
stress the split (an outlier element, a zero row, subnormal values)."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_41_b200.inputs import make_inputs, to_host, workload
from oracle import moe_oracle as O
from router_digits import logits_and_bound, rounding_correction, token_digits, weight_digits

# a chosen logit within this of exact moves a renormalised weight by at most
# twice as much relative to itself: inside the 1e-6 routing-weight bound
TAU = 2.5e-7


def _bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("name,T", [("deepseek_v3", 384), ("mixtral_prefill", 256), ("switch_top1", 256)])
def test_model_within_bound_on_recipes(name, T):
    # x and the router weight are the first draws: a small F leaves them unchanged
    w = workload(name, T=T, F=8, shared_F=0)
    inp = make_inputs(w, seed=3)
    x, wr = to_host(inp["x"]), to_host(inp["w_router"])
    ref = O.router_logits(x, wr)
    lg, bound = logits_and_bound(x, wr)
    err = np.abs(lg - ref)
    assert np.all(err <= bound * (1 + 1e-9) + 1e-300), f"bound violated by {np.max(err - bound):.3e}"
    print(f"[digits] {name}: max err {err.max():.2e}, median bound {np.median(bound):.2e}, "
          f"(t, e) with bound > tau {np.mean(bound > TAU):.4f}")
    # the recipes' logits come out far inside the routing tolerance
    assert err.max() < 3e-7
    assert np.mean(bound > TAU) < 0.05
    # with the x-rounding term added exactly, the rest of the bound holds and
    # leaves (nearly) nothing for the exact recomputation
    corr, rest, n_rounded = rounding_correction(x, wr)
    err2 = np.abs(lg + corr - ref)
    assert np.all(err2 <= rest * (1 + 1e-9) + 1e-300)
    print(f"[digits] {name}: corrected max err {err2.max():.2e}, rest bound > tau {np.mean(rest > TAU):.5f}, "
          f"rows with > 8 rounded elements {np.mean(n_rounded > 8):.4f}")
    assert np.mean(rest > TAU) < 1e-3


def test_bound_holds_on_hard_rows():
    rng = np.random.default_rng(11)
    d, E = 1024, 16
    x = rng.standard_normal((6, d))
    x[1, 7] = 3000.0                         # an outlier: the row's small values lose digits
    x[2] = 0.0                               # a zero row
    x[3] = rng.standard_normal(d) * 1e-39    # subnormal bf16 values
    x[4, ::2] = 0.0
    x[5] = rng.standard_normal(d) * 2.0 ** 40
    x = _bf16(x)
    w = (rng.standard_normal((E, d)) * 0.02).astype(np.float32)
    w[3] = 0.0
    w[4, 5] = 7.0                            # an outlier weight
    ref = O.router_logits(x, w)
    lg, bound = logits_and_bound(x, w)
    err = np.abs(lg - ref)
    assert np.all(err <= bound * (1 + 1e-9) + 1e-300)
    assert np.all(lg[2] == 0.0) and np.all(lg[:, 3] == 0.0)
    # the outlier row's bound is large: its chosen logits are recomputed exactly
    assert bound[1].max() > 100 * bound[0].max()


def test_digits_reassemble_and_fit_int8():
    rng = np.random.default_rng(5)
    x = _bf16(rng.standard_normal((8, 256)) * np.logspace(-3, 3, 8)[:, None])
    w = (rng.standard_normal((4, 256)) * 0.02).astype(np.float32)
    A, sx, vx = token_digits(x)
    B, sw, vw = weight_digits(w)
    for dgt in A + B:
        assert dgt.min() >= -128 and dgt.max() <= 127
    assert np.array_equal(A[0] * 65536 + A[1] * 256 + A[2], vx)
    assert np.array_equal(((B[0] * 256 + B[1]) * 256 + B[2]) * 256 + B[3], vw)
    assert np.abs(vx).max() <= 2 ** 22 and np.abs(vw).max() <= 2 ** 30
    # bf16 values at most 2^14 below the row maximum are represented exactly
    keep = np.abs(x) >= np.abs(x).max(1, keepdims=True) * 2.0 ** -14
    assert np.array_equal((vx * np.ldexp(1.0, -sx)[:, None])[keep], x.astype(np.float64)[keep])


def _integer_rne_digits(w: np.ndarray, sw: int) -> np.ndarray:
    """rne(w 2^sw) the way the preparation pass computes it: from the fp32
    fields with integer shifts, ties to even, no float conversion."""
    bits = w.astype(np.float32).view(np.uint32).astype(np.int64)
    fe = (bits >> 23) & 0xFF
    mant = bits & 0x7FFFFF
    m = np.where(fe > 0, mant | 0x800000, mant)
    sh = np.maximum(fe, 1) - 150 + sw
    v = np.zeros_like(m)
    up = sh >= 0
    v[up] = m[up] << sh[up]
    mid = (sh < 0) & (sh >= -25)
    k = -sh[mid]
    q = m[mid] >> k
    rem = m[mid] & ((1 << k) - 1)
    half = 1 << (k - 1)
    q = q + ((rem > half) | ((rem == half) & (q & 1 == 1)))
    v[mid] = q
    return np.where(bits >> 31 == 1, -v, v)


def test_weight_digit_integer_rounding_matches_rint():
    """The integer rounding of the router weights to their 30-bit digits
    equals round-half-even of w 2^sw in float64 over normal, subnormal, tie
    and far-below-the-row-maximum values."""
    rng = np.random.default_rng(13)
    w = (rng.standard_normal(20000) * np.exp2(rng.integers(-40, 10, 20000))).astype(np.float32)
    w[:8] = np.array([0.0, -0.0, 1e-45, -3e-42, 0.75, -0.75, 1.5, 2.5], dtype=np.float32)
    for scale in (1.0, 2.0 ** -100, 3.0e4):
        row = (w.astype(np.float64) * scale).astype(np.float32)
        _, sw, vref = weight_digits(row[None, :])
        got = _integer_rne_digits(row, int(sw[0]))
        assert np.array_equal(got, vref[0])
        # ties exercised: values exactly half a unit of 2^-sw away from an integer
        t = (np.arange(1, 200) + 0.5) * np.ldexp(1.0, -int(sw[0]))
        t = t[np.abs(t) <= np.abs(row).max()].astype(np.float32)
        t = t[t.astype(np.float64) == (np.arange(1, 200) + 0.5)[: len(t)] * np.ldexp(1.0, -int(sw[0]))]
        if len(t):
            assert np.array_equal(_integer_rne_digits(t, int(sw[0])),
                                  np.rint(t.astype(np.float64) * np.ldexp(1.0, int(sw[0]))).astype(np.int64))


def test_chunk_selection_covers_every_rounded_element():
    """The preparation pass reads again only the 8-element chunks whose
    smallest exponent field e (taken as 1 for zeros and subnormals) lies below
    the row's largest minus 14 (all chunks when the scale is clamped).  Every
    element that the digits round lies in such a chunk."""
    rng = np.random.default_rng(17)
    d = 1024
    rows = [rng.standard_normal(d), rng.standard_normal(d) * 1e-3, np.zeros(d),
            rng.standard_normal(d) * 1e-39, rng.standard_normal(d) * 2.0 ** 60]
    r = rng.standard_normal(d)
    r[5] = 4000.0                              # an outlier: far-below elements round
    rows.append(r)
    r = rng.standard_normal(d)
    r[::3] = 0.0
    rows.append(r)
    x = _bf16(np.stack(rows))
    _, sx, v = token_digits(x)
    bits = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().astype(np.int64)
    mag = bits & 0x7FFF
    rounded = x.astype(np.float64) != v * np.ldexp(1.0, -sx)[:, None]
    for t in range(x.shape[0]):
        emax = max(int(mag[t].max()) >> 7, 1)
        clamped = emax < 21                    # the scale 2^sx was capped at 2^127
        ethr = emax - 14
        chunk_min_e = np.maximum(mag[t].reshape(-1, 8).min(axis=1) >> 7, 1)
        selected = np.ones(d // 8, bool) if clamped else chunk_min_e < ethr
        assert np.all(selected[np.nonzero(rounded[t])[0] // 8]), t


def _group8_select(sel: np.ndarray, n_group: int, topk_group: int, top_k: int) -> np.ndarray:
    """The lane-per-eight-experts selection, step for step: lane l holds
    experts 8 l .. 8 l + 7; a group's two largest scores from each lane's own
    pair merged over the group's lanes by xor partners; kept groups by a rank
    count (ties to the lower group); the top k as k rounds taking the largest
    head of each lane's sorted candidates (ties to the lower lane)."""
    E = sel.shape[0]
    lanes = E // 8
    lg = E // n_group // 8
    s = sel.reshape(lanes, 8)
    a = np.sort(s, axis=1)[:, ::-1][:, :2].copy()          # (a1, a2) per lane
    o = 1
    while o < lg:
        b = a[np.arange(lanes) ^ o]
        a = np.stack([np.maximum(a[:, 0], b[:, 0]),
                      np.maximum(np.minimum(a[:, 0], b[:, 0]), np.maximum(a[:, 1], b[:, 1]))], axis=1)
        o <<= 1
    gs = a[:, 0] + a[:, 1]                                  # every lane of a group holds its score
    g = np.arange(lanes) // lg
    gscore = gs[np.arange(n_group) * lg]
    rank = np.array([np.sum((gscore > gscore[gi]) | ((gscore == gscore[gi]) & (np.arange(n_group) < gi)))
                     for gi in g])
    keep = rank < topk_group
    cand = np.where(keep[:, None], s, -np.inf)
    heads = [sorted([(-cand[l, j], j) for j in range(8)]) for l in range(lanes)]   # largest first, lower j
    chosen = []
    for _ in range(top_k):
        best = max(range(lanes), key=lambda l: (-heads[l][0][0], -l))
        chosen.append(8 * best + heads[best].pop(0)[1])
        heads[best].append((np.inf, 99))                     # an emptied slot sorts last
    return np.array(chosen)


@pytest.mark.parametrize("E,n_group,topk_group,top_k", [(256, 8, 4, 8), (64, 8, 3, 6), (96, 6, 2, 5),
                                                        (256, 4, 2, 8), (128, 1, 1, 8)])
def test_group8_selection_matches_group_routing(E, n_group, topk_group, top_k):
    """The lane-per-eight-experts selection chooses the oracle's experts, in
    its order, also when scores tie (logits on a coarse grid)."""
    rng = np.random.default_rng(E + n_group)
    for trial in range(40):
        logits = rng.integers(-8, 9, (4, E)) * 0.25 if trial % 2 else rng.standard_normal((4, E))
        bias = rng.integers(-2, 3, E) * 0.01 if trial % 3 else None
        ids, _, s, _ = O.route_sigmoid_group(logits, top_k, n_group, topk_group, 1.0, expert_bias=bias)
        sel = s + (bias if bias is not None else 0.0)
        for t in range(logits.shape[0]):
            assert np.array_equal(_group8_select(sel[t], n_group, topk_group, top_k), ids[t]), (trial, t)
