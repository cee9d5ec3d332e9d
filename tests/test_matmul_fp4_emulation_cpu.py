"""The packed-fp4 form of the weight-only matmul's integer mode, emulated on
the CPU from its definition and checked against the oracle.

The emulation takes the steps that form prescribes, in float64 with exact
integers, independently of the CUDA code:
  * each code word w (16 two-bit fields, first column in the lowest bits)
    becomes two words of e2m1 nibbles, (w & 0x33333333) ^ 0x22222222 (the
    even fields) and the same of w >> 2 (the odd fields), so each nibble is
    f'/2 with f' = f xor 2, and MMA position q of every group of 16 holds
    field 2q (q < 8) or 2(q - 8) + 1;
  * each activation row becomes v = rint(x 2^(29 - E)), E = floor(log2
    max|x|), written as ten planes of balanced base-9 digits in [-4, 4],
    permuted to the same K order;
  * per plane, the products of nibble values are summed (the tensor cores'
    fp32 accumulators; exact here), the row of ones gives the plane sums
    of the digits, and the epilogue forms sum_p 9^p (2 acc_p) and
    y = alpha (P4 s + PQ Sx) 2^(E - 29).
The sums must equal sum_k v_k f'_k and sum_k v_k exactly, and y must match
the oracle within the integer mode's bound (2^-30 max|x| sum|w| beyond the
fp32 and bf16 roundings, which this float64 emulation does not take).
"""
import numpy as np
import pytest

from oracle import pq_oracle

E2M1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])
BINARY, TERNARY, SEQ2, SEQ2_B, LSQ2 = 1, 2, 3, 4, 5
# y = alpha * factor * (A * sum x f' + B * sum x) per quantizer: (A, B, factor)
AFFINE = {SEQ2: (2, -3, 0.25), SEQ2_B: (2, -3, 1 / 3), TERNARY: (2, -4, 1 / 3),
          LSQ2: (1, -2, 1.0), BINARY: (1, -2, 1.0)}


def _bf16(v):
    return (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _mma_order(k):
    """MMA position -> column index within the row (K order of the nibbles)."""
    q = np.arange(16)
    field = np.where(q < 8, 2 * q, 2 * (q - 8) + 1)
    return (np.arange(k) // 16) * 16 + field[np.arange(k) % 16]


def _weight_nibbles(packed, k):
    words = packed.view("<u4").astype(np.uint64)  # [n, k/16]
    lo = (words & 0x33333333) ^ 0x22222222
    hi = ((words >> 2) & 0x33333333) ^ 0x22222222
    out = np.empty((packed.shape[0], k), np.int64)
    for i in range(8):
        out[:, i::16] = (lo >> (4 * i)) & 15
        out[:, 8 + i::16] = (hi >> (4 * i)) & 15
    return out  # nibble at MMA position


def _fixed_point(xb):
    x = _f64(xb)
    v = np.zeros(x.shape, np.int64)
    E = np.zeros(x.shape[0], np.int64)
    for j, row in enumerate(x):
        mx = np.abs(row).max()
        E[j] = int(np.floor(np.log2(mx))) if mx > 0 else 0
        v[j] = np.rint(np.ldexp(row, int(29 - E[j]))).astype(np.int64)
    assert np.all(np.abs(v) < 2 ** 30)
    return v, E


def _planes(v):
    digits = []
    for p in range(10):
        if p < 9:
            t = v + 4
            q = np.floor_divide(t, 9)
            d = t - 9 * q - 4
            v = q
        else:
            d = v
        assert np.all(np.abs(d) <= 4)
        mag = np.abs(d)
        digits.append(np.where(mag <= 2, 2 * mag, mag + 2) | np.where(d < 0, 8, 0))
    return np.stack(digits)  # [10, m, k] nibbles, column order


@pytest.mark.parametrize("q", [BINARY, TERNARY, SEQ2, SEQ2_B, LSQ2])
@pytest.mark.parametrize("m,n,k", [(3, 40, 256), (16, 33, 384), (9, 130, 128)])
def test_fp4_form_equals_integer_sums_and_oracle(q, m, n, k):
    rng = np.random.default_rng(100 * q + m + n + k)
    O = pq_oracle.default()
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    alpha = (np.abs(w).max(axis=1) * 0.6).astype(np.float32)
    _, _, packed = O.fwd(q, w, alpha, pack=True)
    x = rng.standard_normal((m, k)) * np.exp(rng.standard_normal((m, 1)) * 3)
    x[0, : k // 2] = 0.0  # a row with zeros and a small range
    xb = _bf16(x)
    order = _mma_order(k)
    A = E2M1[_weight_nibbles(packed, k)]            # f'/2 at MMA positions
    v, E = _fixed_point(xb)
    B = E2M1[_planes(v)[:, :, order]]               # digits at MMA positions
    acc = np.einsum("nk,pmk->pnm", A, B)            # the per-plane MMA sums
    ones = B.sum(axis=2)                            # row of ones (A = 1.0)
    assert np.all(np.abs(2 * acc) < 2 ** 23)
    w9 = 9 ** np.arange(10, dtype=np.int64)
    s2 = np.einsum("p,pnm->nm", w9, np.rint(2 * acc).astype(np.int64))
    sx = np.einsum("p,pm->m", w9, np.rint(ones).astype(np.int64))
    # exact: the planes reproduce the fixed-point integers' sums
    fprime = (2 * A[:, np.argsort(order)]).astype(np.int64)  # f' in column order
    assert np.array_equal(s2, fprime @ v.T)
    assert np.array_equal(sx, v.sum(axis=1))
    a_, b_, fac = AFFINE[q]
    y = alpha[:, None].astype(np.float64) * fac * (a_ * s2 + b_ * sx[None, :]) * np.ldexp(1.0, E - 29)[None, :]
    ref = O.wq_matmul(q, xb, packed, alpha, k)  # [m, n]
    wv = O.wq_matmul(q, _bf16(np.eye(k, dtype=np.float32)), packed, alpha, k).T  # [n, k]
    xf = np.abs(_f64(xb))
    bound = 2.0 ** -30 * np.outer(xf.max(axis=1), np.abs(wv).sum(axis=1))
    slack = 1e-12 * (xf @ np.abs(wv).T)
    assert np.all(np.abs(y.T - ref) <= bound + slack), float(np.max(np.abs(y.T - ref) - bound - slack))
