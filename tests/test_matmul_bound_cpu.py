"""The weight-only matmul's integer-mode error bound, checked on the CPU.

The integer mode rounds every activation row to integers at the scale
2^(29 - E), E = floor(log2 max|x|), and then sums digit x field products
exactly. So its result differs from the exact product only by that rounding:
  |y - y_exact| <= sum_k |x_k - x~_k| |w_k| <= 2^-30 max_k|x| sum_k |w_k|
(each rounding error is at most half of 2^(E - 29) <= 2^-30 max|x|). This is
the fixed-point term of the GPU parity tolerance. Here the rounding is
emulated in float64, the product with the oracle's own weight values is
taken in float64, and the result is compared with the oracle's product on
ordinary and adversarial activation rows: the bound holds, and it is not
vacuous (a 1e20 value among 1e-20 ones loses the small ones).
"""
import numpy as np
import pytest

from oracle import pq_oracle

SEQ2, TERNARY, LSQ2 = 3, 2, 5


def _bf16(v: np.ndarray) -> np.ndarray:
    """fp32 values to bf16 bit patterns (truncation; any bf16 values will do)."""
    return (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f64(xb: np.ndarray) -> np.ndarray:
    return (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rows(k, rng):
    tiny = (np.full(k, 1e-20) * rng.choice([-1, 1], k)).astype(np.float32)
    tiny[k // 3] = 1e20
    spread = (np.ldexp(1.0, rng.integers(-60, 61, k)) * rng.choice([-1.0, 1.0], k)).astype(np.float32)
    return np.stack([rng.standard_normal(k).astype(np.float32), tiny, spread,
                     np.zeros(k, np.float32)])


def _fixed_point(x: np.ndarray) -> np.ndarray:
    """x~ = rint(x * 2^(29-E)) * 2^(E-29) per row (ties to even)."""
    out = np.empty_like(x)
    for j, row in enumerate(x):
        mx = np.abs(row).max()
        e = int(np.floor(np.log2(mx))) if mx > 0 else 0
        xi = np.rint(np.ldexp(row, 29 - e))
        assert np.all(np.abs(xi) < 2.0 ** 30)
        out[j] = np.ldexp(xi, e - 29)
    return out


@pytest.mark.parametrize("q", [SEQ2, TERNARY, LSQ2])
def test_integer_mode_error_within_fixed_point_bound(q):
    rng = np.random.default_rng(q)
    k, n = 1024, 64
    O = pq_oracle.default()
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    alpha = np.abs(w).max(axis=1).astype(np.float32)
    _, _, packed = O.fwd(q, w, alpha, pack=True)
    xb = _bf16(_rows(k, rng))
    ref = O.wq_matmul(q, xb, packed, alpha, k)
    # the oracle's weight values alpha * level, read back through its own
    # product with one-hot rows (exact: one nonzero term each)
    wv = O.wq_matmul(q, _bf16(np.eye(k, dtype=np.float32)), packed, alpha, k).T
    x = _f64(xb)
    got = _fixed_point(x) @ wv.T
    bound = 2.0 ** -30 * np.outer(np.abs(x).max(axis=1), np.abs(wv).sum(axis=1))
    err = np.abs(got - ref)
    slack = 1e-12 * (np.abs(x) @ np.abs(wv).T)  # float64 summation order only
    assert np.all(err <= bound + slack), (q, float(np.max(err - bound - slack)))
    assert np.all(got[3] == 0) and np.all(ref[3] == 0)
    if q in (TERNARY, LSQ2):
        # not vacuous: where the 1e20 value meets a zero level, the row's
        # 1e-20 values decide y and are lost (far beyond the float64 noise),
        # yet the error stays within the bound
        assert np.max(err[1] - slack[1]) > 0
