"""The packed-fp4 form of the weight-only matmul's integer mode, checked on
the CPU against the definitions it rests on.

That form feeds the tensor cores e2m1 values: the weights as f'/2 (the
code's offset-binary field in the low two bits of a nibble) and the
activations' fixed-point integers v = rint(x 2^(29-E)), |v| < 2^30, as ten
planes of balanced base-9 digits in [-4, 4], every scale factor 1.0. Its
results are exact (and equal the 8-bit form's) only if
  * those nibbles decode to f'/2 and to the digits themselves under the
    e2m1 definition (sign bit, two exponent bits with bias 1, one mantissa
    bit; exponent 0 is subnormal, m/2);
  * every |v| < 2^30 has such a ten-digit expansion;
  * every product is a multiple of 1/2 and every partial sum of a plane
    stays below 2^23 in magnitude for k <= 2^20, so fp32 holds each exactly;
  * the epilogue's sum_p 9^p (2 acc_p) = sum_k v_k f'_k stays below 2^52.
Each is checked here from those definitions, not from the kernel's code.
"""
import numpy as np


def e2m1(nib: int) -> float:
    """Value of a 4-bit e2m1 code from the format's definition."""
    s, e, m = (nib >> 3) & 1, (nib >> 1) & 3, nib & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -mag if s else mag


def digit_nibble(d: int) -> int:
    """The kernel's nibble for a digit in [-4, 4]: 0,1,2,3,4 -> 0000, 0010,
    0100, 0101, 0110, sign in bit 3."""
    a = abs(d)
    return (2 * a if a <= 2 else a + 2) | (8 if d < 0 else 0)


def balanced9(v: int, planes: int = 10):
    """Digits d_0..d_{P-1} of v = sum_p 9^p d_p, d_p in [-4, 4] for p < P-1
    (floor division), the last plane taking what is left."""
    out = []
    for p in range(planes):
        if p + 1 < planes:
            t = v + 4
            q = t // 9  # Python floors, as the kernel's explicit floor does
            d = t - 9 * q - 4
            v = q
        else:
            d = v
        out.append(d)
    return out


def test_e2m1_values_of_the_kernels_nibbles():
    table = [e2m1(n) for n in range(16)]
    assert table == [0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6]
    for f in range(4):  # weights: field f' in the low two bits
        assert e2m1(f) == f / 2
    assert e2m1(0b0010) == 1.0  # the row of ones
    for d in range(-4, 5):
        assert e2m1(digit_nibble(d)) == d
    # the one-instruction decode (w & 0x33333333) ^ 0x22222222 gives, per
    # nibble, the field xor 2: offset binary of the two's-complement field
    for f in range(4):
        c = f - 4 if f >= 2 else f  # two's-complement value of the field
        assert ((f & 3) ^ 2) == c + 2


def test_balanced_base9_covers_30_bit_fixed_point():
    rng = np.random.default_rng(9)
    edge = [0, 1, -1, 4, -4, 5, -5, 2 ** 29, -2 ** 29, 2 ** 30 - 1, -(2 ** 30 - 1)]
    vals = edge + [int(v) for v in rng.integers(-(2 ** 30) + 1, 2 ** 30, 20000)]
    for v in vals:
        ds = balanced9(v)
        assert all(-4 <= d <= 4 for d in ds), (v, ds)
        assert abs(ds[-1]) <= 3, (v, ds)
        assert sum(d * 9 ** p for p, d in enumerate(ds)) == v
    # the range is not slack: 9^10 / 2 is the first magnitude ten digits miss
    assert 2 ** 30 < 9 ** 10 // 2


def test_partial_sums_stay_exact_in_fp32():
    k = 1 << 20
    # worst plane sum: every |f'/2| = 1.5 times every |d| = 4
    worst = k * 1.5 * 4
    assert worst < 2 ** 23
    # multiples of 1/2 below 2^23 are exact fp32 values: 2 s is an integer
    # below 2^24
    s = np.float32(0.0)
    for step in range(200000):
        s = np.float32(s + np.float32(6.0))
    assert s == 1_200_000.0
    half = np.float32(2 ** 23 - 0.5)
    assert float(half) == 2 ** 23 - 0.5
    # a random walk of exact products, summed in fp32 in K order, equals the
    # exact sum (the fp32 accumulators round nothing)
    rng = np.random.default_rng(4)
    f = rng.integers(0, 4, 1 << 16) / 2.0
    d = rng.integers(-4, 5, 1 << 16).astype(np.float64)
    acc = np.float32(0.0)
    for t in f * d:
        acc = np.float32(acc + np.float32(t))
    assert float(acc) == float(np.sum(f * d))


def test_epilogue_sum_fits_the_double_it_becomes():
    k = 1 << 20
    # sum_k v_k f'_k with |v| < 2^30 and f' <= 3
    assert 3 * (2 ** 30 - 1) * k < 2 ** 52
    # the plane-by-plane partial sums stay far inside int64
    assert 2 * 6 * k * (9 ** 10 - 1) // 8 < 2 ** 62
