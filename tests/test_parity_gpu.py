"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Bit-exact for bf16 dequantized weights, packed codes and fp32 dW; d(alpha)
within 1e-4 relative (floor: 1e-6 of the row's sum of |terms|). Small cases
compare every element; the full-size workloads run in the launch
configuration of the benchmark and compare sampled rows, which the oracle
computes one by one (every output row depends only on its own inputs).
"""
import numpy as np
import pytest
import torch

from bit_quantization_aware_b200 import inputs as I
from bit_quantization_aware_b200 import pq
from bit_quantization_aware_b200.step import QuantStep
from oracle import pq_oracle
from tests.gpu_util import bits16, check_bwd, check_fwd, f32

pytestmark = pytest.mark.gpu

ALLQ = pq_oracle.ALL_QUANTIZERS
DEV = "cuda"


def make_case(rows, cols, q, seed=0, special=True):
    w = I.normal_weights(rows, cols, seed=seed, stream=1, device="cpu")
    if special and rows * cols >= 8:
        flat = w.view(-1)
        flat[0] = 0.0
        flat[1] = -0.0
        flat[2] = 1e-40           # subnormal
        flat[3] = -3e-39
    a = I.alpha_init(w, q)
    if special and rows * cols >= 8:
        # exact clip bounds for row 0 (x == lo, x == hi)
        lo, hi = {pq.PQ_BINARY: (-1.0, 1.0), pq.PQ_LSQ2: (-2.0, 1.0),
                  pq.PQ_LSQ3: (-4.0, 3.0), pq.PQ_LSQ4: (-8.0, 7.0)}.get(
                      q, (-0.99, 0.99))
        a[0] = 1.0
        w.view(-1)[4] = lo
        w.view(-1)[5] = hi
        w.view(-1)[6] = 0.5
        w.view(-1)[7] = -0.5
    g = I.grad_bf16(rows, cols, seed=seed, stream=65, device="cpu")
    return w, a, g


def run_gpu(q, w, a, g, pack, offset=0):
    """Run fwd (+pack) and bwd on the GPU; ``offset`` shifts every array by
    that many elements inside a larger buffer (misaligned pointers)."""
    rows, cols = w.shape
    n = rows * cols

    def dev(t, dtype):
        buf = torch.empty(n + offset + 8, dtype=dtype, device=DEV)
        v = buf[offset:offset + n].view(rows, cols)
        if t is not None:
            v.copy_(t)
        return v

    wd = dev(w, torch.float32)
    gd = dev(g, torch.bfloat16)
    ad = a.to(DEV)
    wq = dev(None, torch.bfloat16)
    bits = pq.pq_code_bits(q)
    pk = None
    if pack:
        pbuf = torch.zeros(n * bits // 8 + offset + 8, dtype=torch.uint8, device=DEV)
        pk = pbuf[offset:offset + n * bits // 8].view(rows, cols * bits // 8)
    pq.pq_fakequant_fwd(q, wd, ad, wq, pk, rows=rows, cols=cols)
    pk2 = None
    if pack:
        pbuf2 = torch.zeros(n * bits // 8 + offset + 8, dtype=torch.uint8, device=DEV)
        pk2 = pbuf2[offset:offset + n * bits // 8].view(rows, cols * bits // 8)
        pq.pq_pack_codes(q, wd, ad, pk2, rows=rows, cols=cols)
    dw = dev(None, torch.float32)
    da = torch.full((rows,), float("nan"), device=DEV)
    gs = pq.pq_default_grad_scale(q, cols)
    pq.pq_fakequant_bwd(q, wd, ad, gd, dw, da, gs, rows=rows, cols=cols)
    torch.cuda.synchronize()
    return wq, pk, pk2, dw, da, gs


def np_inputs(w, a, g):
    return (w.numpy(), a.numpy(), g.view(torch.int16).numpy().view(np.uint16))


SHAPES = [(1, 8), (3, 24), (5, 12), (7, 1000), (9, 1001), (33, 1032),
          (256, 1024), (2, 70000), (300, 264), (4, 4), (1, 6)]


@pytest.mark.parametrize("q", ALLQ)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_small_shapes(q, shape):
    rows, cols = shape
    w, a, g = make_case(rows, cols, q)
    pack = cols % (8 // pq.pq_code_bits(q)) == 0
    wq, pk, pk2, dw, da, gs = run_gpu(q, w, a, g, pack)
    wn, an, gn = np_inputs(w, a, g)
    check_fwd(q, wn, an, wq, pk)
    if pack:
        check_fwd(q, wn, an, None, pk2)
    check_bwd(q, wn, an, gn, gs, dw, da)


@pytest.mark.parametrize("q", ALLQ)
@pytest.mark.parametrize("offset", [1, 2, 3])
def test_misaligned_pointers(q, offset):
    w, a, g = make_case(37, 1024, q, seed=offset)
    wq, pk, pk2, dw, da, gs = run_gpu(q, w, a, g, True, offset=offset)
    wn, an, gn = np_inputs(w, a, g)
    check_fwd(q, wn, an, wq, pk)
    check_fwd(q, wn, an, None, pk2)
    check_bwd(q, wn, an, gn, gs, dw, da)


@pytest.mark.parametrize("q", [pq.PQ_SEQ2, pq.PQ_SEQ2_B])
def test_single_matrix_256x1024(q):
    """256x1024, N(0, 0.02), alpha = max|w_row|, dWq ~ N(0, 1e-3), seed 0;
    forward + packed codes + backward once, every element compared."""
    w = I.normal_weights(256, 1024, seed=0, stream=0, device="cpu")
    a = I.alpha_init(w, q)
    g = I.grad_bf16(256, 1024, seed=0, stream=64, device="cpu")
    wq, pk, pk2, dw, da, gs = run_gpu(q, w, a, g, True)
    wn, an, gn = np_inputs(w, a, g)
    check_fwd(q, wn, an, wq, pk)
    check_fwd(q, wn, an, None, pk2)
    check_bwd(q, wn, an, gn, gs, dw, da)


@pytest.mark.parametrize("q,rule", [(pq.PQ_BINARY, "lsq"), (pq.PQ_TERNARY, "lsq"),
                                    (pq.PQ_SEQ2, "lsq"), (pq.PQ_LSQ3, "lsq"),
                                    (pq.PQ_LSQ4, "lsq"), (pq.PQ_LSQ3, "max"),
                                    (pq.PQ_LSQ4, "max"), (pq.PQ_LSQ2, "lsq")])
def test_bit_width_sweep_2048x8192(q, rule):
    """One 2048x8192 N(0, 0.02) weight (seed 1) under each quantizer with
    its alpha init (LSQ: 2*mean|w|/sqrt(Qp), and max|w|/Qp as on the
    pages); every element compared."""
    w = I.normal_weights(2048, 8192, seed=1, stream=0, device="cpu")
    a = I.alpha_init(w, q, lsq_rule=rule)
    g = I.grad_bf16(2048, 8192, seed=1, stream=64, device="cpu")
    wq, pk, pk2, dw, da, gs = run_gpu(q, w, a, g, True)
    wn, an, gn = np_inputs(w, a, g)
    check_fwd(q, wn, an, wq, pk)
    check_bwd(q, wn, an, gn, gs, dw, da)


def _sampled_rows(step, rows_per_matrix, seed=0):
    rng = np.random.default_rng(seed)
    for b in step.bufs:
        r = b.m.rows
        pick = sorted(set([0, r - 1] + rng.integers(0, r, rows_per_matrix).tolist()))
        yield b, pick


def _check_step_rows(step, rows_per_matrix):
    q = step.q
    for b, pick in _sampled_rows(step, rows_per_matrix):
        idx = torch.tensor(pick, device=DEV)
        wn = f32(b.w.index_select(0, idx))
        an = f32(b.alpha.index_select(0, idx))
        gn = bits16(b.g.index_select(0, idx))
        check_fwd(q, wn, an, b.wq.index_select(0, idx),
                  b.packed.index_select(0, idx) if b.packed is not None else None)
        check_bwd(q, wn, an, gn, b.grad_scale, b.dw.index_select(0, idx),
                  b.dalpha.index_select(0, idx))


@pytest.mark.parametrize("which", ["llama_1b_stack", "llama3_8b_set"])
def test_layer_set_full_size_sampled(which):
    """The full layer sets in the benchmark's launch configuration (one
    forward over all matrices, then one backward over all), SEQ2; sampled
    rows of every matrix compared with the oracle."""
    mats = getattr(I, which)()
    step = QuantStep(mats, pq.PQ_SEQ2, device=DEV)
    step.generate(seed=2 if which == "llama_1b_stack" else 3)
    step.run()
    torch.cuda.synchronize()
    _check_step_rows(step, rows_per_matrix=3)
    del step
    torch.cuda.empty_cache()


@pytest.mark.parametrize("q", [pq.PQ_SEQ2, pq.PQ_TERNARY])
def test_student_t_16384_planted_ties(q):
    """16384x16384 Student-t(3)*0.02 with 1% of entries planted exactly on
    the clip bounds and on rounding ties; forward + packed codes + backward;
    512 sampled rows compared; most planted entries hit their target
    exactly (about 85%)."""
    mats = [I.Matrix("t3.16384", 16384, 16384, 0, 0)]
    step = QuantStep(mats, q, device=DEV, pack=True)
    step.generate(seed=4, dist="student_t")
    b = step.bufs[0]
    n, hit = I.plant_boundaries(b.w, b.alpha, frac=0.01, seed=4)
    # a target that no fp32 w reaches exactly (the quotient steps over it)
    # keeps the nearest candidate; most land exactly
    assert n > 0 and hit >= 0.5 * n, (n, hit)
    print(f"planted {n} entries, {hit} exactly on a clip bound or tie")
    step.run()
    torch.cuda.synchronize()
    _check_step_rows(step, rows_per_matrix=512)
    del step
    torch.cuda.empty_cache()


@pytest.mark.parametrize("q", ALLQ)
def test_fp32_bit_pattern_sweep(q):
    """Strided sweep of fp32 bit patterns for x in about [1e-7, 24] of
    both signs, under three scales; forward and backward compared."""
    lo_bits = np.float32(1e-7).view(np.uint32)
    hi_bits = np.float32(24.0).view(np.uint32)
    pos = np.arange(lo_bits, hi_bits, 97, dtype=np.uint32).view(np.float32)
    x = np.concatenate([pos, -pos])
    cols = 4096
    x = x[: len(x) // cols * cols].reshape(-1, cols)
    for alpha in (1.0, 0.0173, 3.7):
        w = torch.from_numpy((x * np.float32(alpha)).astype(np.float32))
        a = torch.full((w.shape[0],), alpha, dtype=torch.float32)
        g = I.grad_bf16(w.shape[0], cols, seed=5, stream=66, device="cpu")
        wq, pk, _, dw, da, gs = run_gpu(q, w, a, g, True)
        wn, an, gn = np_inputs(w, a, g)
        check_fwd(q, wn, an, wq, pk)
        check_bwd(q, wn, an, gn, gs, dw, da)


def test_determinism_and_streams():
    q = pq.PQ_SEQ2
    w, a, g = make_case(513, 4104, q, seed=6)
    r1 = run_gpu(q, w, a, g, True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        r2 = run_gpu(q, w, a, g, True)
    torch.cuda.synchronize()
    for x, y in zip(r1[:5], r2[:5]):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_empty_and_degenerate():
    q = pq.PQ_SEQ2
    z = torch.empty(0, device=DEV)
    # rows == 0 and cols == 0 launch nothing
    pq.pq_fakequant_fwd(q, z, z, z, None, rows=0, cols=8)
    da = torch.full((5,), float("nan"), device=DEV)
    pq.pq_fakequant_bwd(q, z, z, z, z, da, 1.0, rows=5, cols=0)
    torch.cuda.synchronize()
    assert torch.all(da == 0)
    # one element, one long row (generic path), one long row (vector path)
    for rows, cols in ((1, 1), (1, (1 << 22) + 4), (1, 1 << 22)):
        w, a, g = make_case(rows, cols, q, seed=7, special=False)
        pack = cols % 4 == 0
        wq, pk, pk2, dw, da, gs = run_gpu(q, w, a, g, pack)
        wn, an, gn = np_inputs(w, a, g)
        check_fwd(q, wn, an, wq, pk)
        check_bwd(q, wn, an, gn, gs, dw, da)


@pytest.mark.parametrize("q", ALLQ)
def test_idempotence_on_gpu(q):
    """Quantizing the bf16 output again with the same alpha returns it."""
    w, a, g = make_case(64, 2048, q, seed=8, special=False)
    wq, *_ = run_gpu(q, w, a, g, False)
    w2 = wq.float().cpu()
    wq2, *_ = run_gpu(q, w2, a, g, False)
    assert torch.equal(wq.view(torch.int16), wq2.view(torch.int16))
