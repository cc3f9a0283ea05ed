"""Host model of the integer tensor-core router logits (a test helper, not the
oracle): the digit split and error bound that include/moe.h states for the
router's workspace logits, written out in NumPy integer arithmetic.

Token row x (bf16 values): e = the least integer with |x| < 2^e over the row
(0 for a zero row), sx = min(22 - e, 127), v = round-half-even(x 2^sx), and
u = v + 0x8080 splits v into balanced digits a0 = u >> 16, a1 = byte1(u) - 128,
a2 = byte0(u) - 128 (v = a0 2^16 + a1 2^8 + a2).  Expert row w (fp32): sw = 30 -
e_w, v = round-half-even(w 2^sw), four digits from u = v + 0x808080.  The
logit is the sum of the digit products (i, j) except (2, 3), scaled back:
  sum_{i,j} a_i . b_j 2^(8 (5 - i - j)) 2^(-sx - sw),
and it differs from x . w by at most
  |dx|_1 |w|_inf + |xhat|_2 |dw|_2 + |x2|_2 |w3|_2.
"""
from __future__ import annotations

import numpy as np

PAIRS = [(i, j) for i in range(3) for j in range(4) if (i, j) != (2, 3)]


def _f64(a) -> np.ndarray:
    """float64 values of a host array (uint16 arrays are bf16 bit patterns)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _row_exponent(a: np.ndarray) -> np.ndarray:
    mx = np.abs(a).max(axis=1)
    e = np.frexp(mx)[1].astype(np.int64)          # mx < 2**e (0 for mx == 0)
    return np.where(mx > 0, e, 0)


def token_digits(x: np.ndarray):
    """x: [T, d] float (bf16 values).  Returns digits [3][T, d], sx [T], v [T, d]."""
    x = _f64(x)
    sx = np.minimum(22 - _row_exponent(x), 127)
    v = np.rint(x * np.ldexp(1.0, sx)[:, None]).astype(np.int64)
    u = v + 0x8080
    return [u >> 16, ((u >> 8) & 255) - 128, (u & 255) - 128], sx, v


def weight_digits(w: np.ndarray):
    """w: [E, d] float32.  Returns digits [4][E, d], sw [E], v [E, d]."""
    w = _f64(w)
    sw = 30 - _row_exponent(w)
    v = np.rint(w * np.ldexp(1.0, sw)[:, None]).astype(np.int64)
    u = v + 0x808080
    return [u >> 24, ((u >> 16) & 255) - 128, ((u >> 8) & 255) - 128, (u & 255) - 128], sw, v


def logits_and_bound(x: np.ndarray, w: np.ndarray):
    """The model's logits [T, E] and the stated bound on |logit - x . w|."""
    A, sx, vx = token_digits(x)
    B, sw, vw = weight_digits(w)
    S = np.zeros((A[0].shape[0], B[0].shape[0]), dtype=np.int64)
    for i, j in PAIRS:
        c = A[i] @ B[j].T                        # exact: |c| < 2^31 for d <= 52416
        assert np.abs(c).max(initial=0) < 2 ** 31
        S += c << (8 * (4 - i - j))
    lg = S.astype(np.float64) * np.ldexp(1.0, 8 - sx[:, None] - sw[None, :])
    xs = np.ldexp(1.0, -sx)[:, None]
    ws = np.ldexp(1.0, -sw)[:, None]
    x64 = _f64(x)
    w64 = _f64(w)
    xhat, what = vx * xs, vw * ws
    bound = (np.abs(x64 - xhat).sum(1)[:, None] * np.abs(w64).max(1)[None, :]
             + np.sqrt((xhat ** 2).sum(1))[:, None] * np.sqrt(((w64 - what) ** 2).sum(1))[None, :]
             + np.sqrt(((A[2] * xs) ** 2).sum(1))[:, None] * np.sqrt(((B[3] * ws) ** 2).sum(1))[None, :])
    return lg, bound


def rounding_correction(x: np.ndarray, w: np.ndarray):
    """dx . w (the x-rounding term, which the selection pass adds exactly when
    a row lists all its rounded elements), the bound left after it, and the
    number of rounded elements per row."""
    _, sx, vx = token_digits(x)
    B, sw, vw = weight_digits(w)
    x64, w64 = _f64(x), _f64(w)
    dx = x64 - vx * np.ldexp(1.0, -sx)[:, None]
    xhat = vx * np.ldexp(1.0, -sx)[:, None]
    what = vw * np.ldexp(1.0, -sw)[:, None]
    A2 = token_digits(x)[0][2] * np.ldexp(1.0, -sx)[:, None]
    rest = (np.sqrt((xhat ** 2).sum(1))[:, None] * np.sqrt(((w64 - what) ** 2).sum(1))[None, :]
            + np.sqrt((A2 ** 2).sum(1))[:, None] * np.sqrt(((B[3] * np.ldexp(1.0, -sw)[:, None]) ** 2).sum(1))[None, :])
    return dx @ w64.T, rest, (dx != 0).sum(1)
