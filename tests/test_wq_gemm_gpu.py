"""Weight-only 2-bit matmul on the tensor cores against the oracle.

Y = X (alpha * levels(codes))^T: the oracle computes it in fp64; the GPU
multiplies exact bf16 level numerators by bf16 activations with fp32
accumulation in TMEM and rounds the scaled sums once to bf16. Tolerance:
2^-8 of |Y| (bf16 output rounding) plus 1e-4 of sum_k |x_k * w_k|
(accumulation error bound, far below what a wrong tile layout gives)."""
import numpy as np
import pytest
import torch

from bit_quantization_aware_b200 import inputs as I
from bit_quantization_aware_b200 import pq
from oracle import pq_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
Q2 = [pq.PQ_SEQ2, pq.PQ_SEQ2_B, pq.PQ_TERNARY, pq.PQ_LSQ2, pq.PQ_BINARY]


def _case(q, m, n, k, seed):
    w = I.normal_weights(n, k, seed=seed, stream=0, device=DEV)
    a = I.alpha_init(w, q)
    _, packed = pq.fakequant_fwd(q, w, a, pack=True)
    x = I.normal_weights(m, k, seed=seed, stream=5, std=1.0, device=DEV).to(torch.bfloat16)
    return x, packed, a


INTEGER_ROW_WEIGHTS = 1 << 27  # one row times a lone matrix this large: integer kernel


def _integer_mode(m, n, k, grouped):
    """The integer arithmetic serves m <= 16, except one row times a lone
    matrix with k <= 32768 below INTEGER_ROW_WEIGHTS (fp32 CUDA-core kernel)."""
    if m > 16:
        return False
    return not (m == 1 and not grouped and k <= 32768 and n * k < INTEGER_ROW_WEIGHTS)


def _check(q, x, packed, a, y, grouped=False, n_total=None):
    """y against the oracle within the matmul tolerance, derived from each
    mode's arithmetic: bf16 output rounding (2^-8 |ref|) plus an accumulation
    bound (1e-4 sum_k |x w|), and
      integer arithmetic (see _integer_mode): the fixed-point conversion;
      every activation is rounded to
      a multiple of 2^(E-29) with 2^E <= max_k |x|, so |error| <=
      2^-30 max_k |x| sum_k |w|;
      bf16 and CUDA-core modes: y = alpha (P D + Q Sx) from fp32 sums over
      all k of x (1 + f'/4) and of x, whose rounding scales with
      alpha sum_k |x| (it shows where large activations meet zero levels,
      ternary and LSQ2): 2^-16 alpha sum_k |x|."""
    m, k = x.shape
    xb = x.view(torch.int16).cpu().numpy()
    pk = packed.cpu().numpy()
    an = a.cpu().numpy()
    ref = pq_oracle.default().wq_matmul(q, xb, pk, an, k)
    # sum_k |x_k * w_k| (for the tolerance only) from the dequantized weights
    wd = pq_oracle.bf16_bits_to_float(pq_oracle.dequant(q, pk, an, k)).astype(np.float64)
    xf = np.abs(x.float().cpu().numpy().astype(np.float64))
    ones = xf @ np.abs(wd).T
    got = y.float().cpu().numpy().astype(np.float64)
    tol = 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ones) + 1e-30
    if _integer_mode(m, packed.shape[0] if n_total is None else n_total, k, grouped):
        tol += 2.0 ** -30 * np.outer(xf.max(axis=1), np.abs(wd).sum(axis=1))
    else:
        tol += 2.0 ** -16 * np.outer(xf.sum(axis=1), np.abs(an).astype(np.float64))
    err = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(err / tol), err.shape)
    assert np.all(err <= tol), (f"q={q} shape={x.shape}x{packed.shape}: worst at {worst}: "
                                f"gpu={got[worst]} ref={ref[worst]} tol={tol[worst]}")


@pytest.mark.parametrize("q", Q2)
@pytest.mark.parametrize("m,n,k", [(1, 128, 128), (5, 300, 256), (16, 1024, 4096),
                                   (33, 640, 1024), (64, 2048, 2048), (128, 256, 512),
                                   (7, 4096, 14336), (20, 1000, 640), (3, 130, 384),
                                   (100, 509, 1536), (1, 300, 640), (1, 5, 128),
                                   (1, 14336, 4096), (1, 64, 32896)])
def test_wq_gemm_matches_oracle(q, m, n, k):
    x, packed, a = _case(q, m, n, k, seed=m + n + k)
    y = pq.wq_gemm(q, x, packed, a)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == 0
    _check(q, x, packed, a, y)


def test_wq_gemm_deterministic_and_repeatable():
    """Split-K reduction in a fixed order: identical bits on repeated calls
    sharing one workspace."""
    q = pq.PQ_SEQ2
    x, packed, a = _case(q, 8, 4096, 16384, seed=3)
    y1 = pq.wq_gemm(q, x, packed, a)
    y2 = pq.wq_gemm(q, x, packed, a)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_wq_gemm_rejects_bad_arguments():
    q = pq.PQ_SEQ2
    x = torch.zeros((4, 200), dtype=torch.bfloat16, device=DEV)
    packed = torch.zeros((128, 50), dtype=torch.uint8, device=DEV)
    a = torch.ones(128, device=DEV)
    y = torch.empty((4, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(pq.PQError):  # k not a multiple of 128
        pq.pq_wq_gemm(q, x, packed, a, y)
    with pytest.raises(pq.PQError):  # 4-bit codes are not served
        pq.pq_wq_gemm(pq.PQ_LSQ4, torch.zeros((4, 256), dtype=torch.bfloat16, device=DEV),
                      torch.zeros((128, 128), dtype=torch.uint8, device=DEV), a, y)


def test_wq_gemm_batch_matches_oracle():
    """One launch over matrices of different shapes (same m), including a
    ragged n, a short K tail and a matrix smaller than one row block."""
    q, m = pq.PQ_SEQ2, 5
    shapes = [(4096, 4096), (1000, 640), (100, 128), (14336, 4096), (300, 14336), (127, 512)]
    xs, pks, als = [], [], []
    for i, (n, k) in enumerate(shapes):
        x, packed, a = _case(q, m, n, k, seed=100 + i)
        xs.append(x)
        pks.append(packed)
        als.append(a)
    ys = pq.wq_gemm_batch(q, xs, pks, als)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == 0
    for x, packed, a, y in zip(xs, pks, als, ys):
        _check(q, x, packed, a, y, grouped=True)


@pytest.mark.parametrize("q", [pq.PQ_SEQ2, pq.PQ_TERNARY])
def test_rows_longer_than_fp4_exact_range(q):
    """Rows longer than 2^20 take the 8-bit MMA form of the integer mode
    (the fp4 form's fp32 sums stay exact only up to that length): a lone
    matrix with a short K tail and two row blocks (the last ragged), and a
    group in which one long matrix sends every matrix of the launch there."""
    m, n, k = 5, 130, (1 << 20) + 128
    x, packed, a = _case(q, m, n, k, seed=77)
    y = pq.wq_gemm(q, x, packed, a)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == 0
    _check(q, x, packed, a, y)
    x2, packed2, a2 = _case(q, m, 300, 1024, seed=78)
    ys = pq.wq_gemm_batch(q, [x, x2], [packed, packed2], [a, a2])
    torch.cuda.synchronize()
    assert pq.pq_device_status() == 0
    _check(q, x, packed, a, ys[0], grouped=True)
    _check(q, x2, packed2, a2, ys[1], grouped=True)


def _bf16_from_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).to(DEV).view(torch.bfloat16)


@pytest.mark.parametrize("q", Q2)
@pytest.mark.parametrize("m", [1, 6, 18])
def test_activation_value_ranges(q, m):
    """Activation rows the integer mode's fixed-point conversion (m = 6), the
    bf16 mode (m = 18, the six rows repeated) and the CUDA-core path (m = 1,
    the row with one huge value) must handle: ordinary values, an all-zero
    row, a row of subnormals only, magnitudes spread over 2^120 (far beyond
    the 2^22 the integer mode converts exactly), one huge value among tiny
    ones, and both signs of zero."""
    n, k = 1000, 2048
    rng = np.random.default_rng(17)
    rows = np.zeros((6, k), np.uint16)
    normal = (rng.standard_normal(k).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    rows[0] = normal
    rows[1] = 0
    rows[2] = rng.integers(1, 0x80, k).astype(np.uint16) | (rng.integers(0, 2, k).astype(np.uint16) << 15)
    e = rng.integers(-60, 61, k)
    spread = (np.ldexp(1.0, e) * rng.choice([-1.0, 1.0], k) * (1 + rng.random(k))).astype(np.float32)
    rows[3] = (spread.view(np.uint32) >> 16).astype(np.uint16)
    tiny = np.full(k, np.float32(1e-20), np.float32) * rng.choice([-1, 1], k).astype(np.float32)
    tiny[k // 3] = np.float32(1e20)
    rows[4] = (tiny.view(np.uint32) >> 16).astype(np.uint16)
    rows[5] = np.where(rng.random(k) < 0.5, 0x8000, 0).astype(np.uint16)  # +0 and -0
    x = _bf16_from_bits(rows[4:5] if m == 1 else np.tile(rows, (3, 1))[:m])
    w = I.normal_weights(n, k, seed=9, stream=0, device=DEV)
    a = I.alpha_init(w, q)
    _, packed = pq.fakequant_fwd(q, w, a, pack=True)
    y = pq.wq_gemm(q, x, packed, a)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == 0
    _check(q, x, packed, a, y)
    if m > 1:
        yz = y.float().cpu().numpy()
        assert np.all(yz[1::6] == 0) and np.all(yz[5::6] == 0)


def test_wq_gemm_batch_shared_activations():
    """Matrices of one launch sharing activation matrices (the integer mode
    converts each distinct one once) and ones with their own."""
    q, m = pq.PQ_SEQ2, 9
    xa = _case(q, m, 8, 4096, seed=201)[0]
    xb = _case(q, m, 8, 4096, seed=202)[0]
    xc = _case(q, m, 8, 1536, seed=203)[0]
    plan = [(xa, 4096, 1000), (xb, 4096, 640), (xa, 4096, 127), (xb, 4096, 4096),
            (xa, 4096, 300), (xc, 1536, 2000)]
    xs, pks, als = [], [], []
    for i, (x, k, n) in enumerate(plan):
        w = I.normal_weights(n, k, seed=210 + i, stream=0, device=DEV)
        a = I.alpha_init(w, q)
        _, packed = pq.fakequant_fwd(q, w, a, pack=True)
        xs.append(x)
        pks.append(packed)
        als.append(a)
    ys = pq.wq_gemm_batch(q, xs, pks, als)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == 0
    for x, packed, a, y in zip(xs, pks, als, ys):
        _check(q, x, packed, a, y, grouped=True)


@pytest.mark.parametrize("q", [pq.PQ_TERNARY, pq.PQ_SEQ2_B])
def test_wq_gemm_batch_of_64_is_deterministic(q):
    m = 16
    shapes = [(1024 + 127 * (i % 5), 512 * (1 + i % 4)) for i in range(64)]
    xs, pks, als = [], [], []
    for i, (n, k) in enumerate(shapes):
        x, packed, a = _case(q, m, n, k, seed=7 * i + 1)
        xs.append(x)
        pks.append(packed)
        als.append(a)
    y1 = pq.wq_gemm_batch(q, xs, pks, als)
    y2 = pq.wq_gemm_batch(q, xs, pks, als)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == 0
    for a_, b_ in zip(y1, y2):
        assert torch.equal(a_.view(torch.int16), b_.view(torch.int16))
    for i in (0, 17, 63):
        _check(q, xs[i], pks[i], als[i], y1[i], grouped=True)


def test_wq_gemm_batch_rejects_bad_counts():
    q = pq.PQ_SEQ2
    x = torch.zeros((2, 128), dtype=torch.bfloat16, device=DEV)
    packed = torch.zeros((127, 32), dtype=torch.uint8, device=DEV)
    a = torch.ones(127, device=DEV)
    y = torch.empty((2, 127), dtype=torch.bfloat16, device=DEV)
    one = dict(x=x, packed=packed, alpha=a, y=y)
    with pytest.raises(pq.PQError):
        pq.pq_wq_gemm_batch(q, 2, pq.gemm_problem_array([one] * 65))
    bad = dict(one)
    bad["x"] = torch.zeros((2, 200), dtype=torch.bfloat16, device=DEV)  # k not a multiple of 128
    with pytest.raises(pq.PQError):
        pq.pq_wq_gemm_batch(q, 2, pq.gemm_problem_array([one, bad]))


def test_wq_gemm_wait_timeout_reports_and_recovers():
    """With the abort switch on, the kernel's waits give up as a wait that
    reached its cap does: the device status says PQ_ERR_TIMEOUT once, and
    with the switch off the next call is correct (the context is usable)."""
    q = pq.PQ_SEQ2
    x, packed, a = _case(q, 2, 127 * 148, 4096, seed=11)  # m > 1: the tensor-core path
    assert pq.pq_device_status() == pq.PQ_OK
    try:
        pq.pq_debug_abort_waits(True)
        pq.wq_gemm(q, x, packed, a)
        torch.cuda.synchronize()
    finally:
        pq.pq_debug_abort_waits(False)
    assert pq.pq_device_status() == pq.PQ_ERR_TIMEOUT
    assert pq.pq_device_status() == pq.PQ_OK  # cleared by the read
    y = pq.wq_gemm(q, x, packed, a)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == pq.PQ_OK
    _check(q, x, packed, a, y)


def _check_rows(q, x, packed, a, y, rows, grouped=False):
    """_check on a subset of output features (the oracle runs on those rows)."""
    idx = torch.as_tensor(rows, device=packed.device)
    _check(q, x, packed.index_select(0, idx).contiguous(), a.index_select(0, idx).contiguous(),
           y.index_select(1, idx).contiguous(), grouped=grouped, n_total=packed.shape[0])


@pytest.mark.parametrize("q", [pq.PQ_SEQ2, pq.PQ_TERNARY])
@pytest.mark.parametrize("outlier", [False, True])
def test_one_row_large_lone_matrix(q, outlier):
    """One activation row times a lone matrix of 2^27 weights (the integer
    one-row kernel), with ordinary activations and with one 1e20 value among
    1e-20 ones; 128 sampled output features against the oracle."""
    m, n, k = 1, 8192, 16384
    x, packed, a = _case(q, m, n, k, seed=77)
    if outlier:
        t = np.full(k, np.float32(1e-20), np.float32) * np.random.default_rng(3).choice([-1, 1], k).astype(np.float32)
        t[k // 5] = np.float32(1e20)
        x = _bf16_from_bits((t.view(np.uint32) >> 16).astype(np.uint16)[None, :])
    y = pq.wq_gemm(q, x, packed, a)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == 0
    rows = sorted(set([0, n - 1] + list(np.random.default_rng(9).choice(n, 126, replace=False))))
    _check_rows(q, x, packed, a, y, rows)


def test_wq_gemm_full_size_grouped_sampled():
    """One Llama-3-8B layer at full size plus a 16384^2 weight, in one grouped
    launch at m = 16 (the benchmark's launch configuration); 64 sampled
    output features of every matrix (first and last included) against the
    oracle."""
    q, m = pq.PQ_SEQ2, 16
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096),
              (14336, 4096), (4096, 14336), (16384, 16384)]
    xs, pks, als = [], [], []
    for i, (n, k) in enumerate(shapes):
        x, packed, a = _case(q, m, n, k, seed=900 + i)
        xs.append(x)
        pks.append(packed)
        als.append(a)
    ys = pq.wq_gemm_batch(q, xs, pks, als)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == pq.PQ_OK
    rng = np.random.default_rng(5)
    for (n, k), x, packed, a, y in zip(shapes, xs, pks, als, ys):
        rows = sorted(set([0, n - 1] + list(rng.choice(n, 62, replace=False))))
        _check_rows(q, x, packed, a, y, rows, grouped=True)


def test_wq_gemm_batch_single_row_matches_oracle():
    """One activation row over matrices of several shapes in one launch
    (the integer tensor-core mode; a lone matrix takes the CUDA-core path)."""
    q, m = pq.PQ_SEQ2_B, 1
    shapes = [(4096, 4096), (1000, 640), (7, 128), (14336, 4096), (300, 14336)]
    xs, pks, als = [], [], []
    for i, (n, k) in enumerate(shapes):
        x, packed, a = _case(q, m, n, k, seed=300 + i)
        xs.append(x)
        pks.append(packed)
        als.append(a)
    y1 = pq.wq_gemm_batch(q, xs, pks, als)
    y2 = pq.wq_gemm_batch(q, xs, pks, als)
    torch.cuda.synchronize()
    assert pq.pq_device_status() == pq.PQ_OK
    for x, packed, a, ya, yb in zip(xs, pks, als, y1, y2):
        assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))
        _check(q, x, packed, a, ya, grouped=True)
