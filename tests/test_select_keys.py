"""Host model of the selection kernels' warp arg-max (a test helper, not the
oracle): a float64 score is mapped to an order-preserving unsigned 64-bit key
(negative: every bit inverted; otherwise: the sign bit set), the arg-max taken
as the largest high word, then the largest low word among those, then the
lowest index among the lanes holding both.  It must equal the arg-max of the
scores with ties to the lower index, as the oracle ranks experts."""
import numpy as np
import pytest


def _key(v: np.ndarray) -> np.ndarray:
    u = v.astype(np.float64).view(np.uint64)
    neg = (u >> np.uint64(63)) == 1
    return np.where(neg, ~u, u | np.uint64(1 << 63))


def _unkey(k: np.uint64) -> float:
    k = np.uint64(k)
    u = k & np.uint64((1 << 63) - 1) if (k >> np.uint64(63)) == 1 else ~k
    return np.array([u], dtype=np.uint64).view(np.float64)[0]


def _warp_argmax(v: np.ndarray, idx: np.ndarray):
    k = _key(v)
    hi, lo = (k >> np.uint64(32)).astype(np.uint64), (k & np.uint64(0xFFFFFFFF)).astype(np.uint64)
    mhi = hi.max()
    mlo = np.where(hi == mhi, lo, np.uint64(0)).max()
    top = (hi == mhi) & (lo == mlo)
    i = np.where(top, idx, np.iinfo(np.int64).max).min()
    return _unkey((mhi << np.uint64(32)) | mlo), int(i)


def test_key_preserves_order():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(2000) * np.exp2(rng.integers(-1070, 1000, 2000)),
                        [0.0, 5e-324, -5e-324, np.inf, -np.inf, 1.0, -1.0, 2.0 ** -1022, -(2.0 ** -1022)]])
    order = np.argsort(v, kind="stable")
    k = _key(v)[order]
    vs = v[order]
    assert np.all((k[1:] > k[:-1]) | (vs[1:] == vs[:-1]))


@pytest.mark.parametrize("trial", range(30))
def test_warp_argmax_is_argmax_with_ties_to_lower_index(trial):
    rng = np.random.default_rng(100 + trial)
    v = rng.integers(-4, 5, 32) * 0.125 if trial % 2 else rng.standard_normal(32)
    if trial % 5 == 0:
        v[rng.integers(0, 32, 6)] = -np.inf
    idx = rng.permutation(256)[:32] if trial % 3 else np.arange(32)
    got_v, got_i = _warp_argmax(v, idx)
    best = v.max()
    assert got_v == best
    assert got_i == idx[v == best].min()
