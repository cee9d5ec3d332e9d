"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Bit-exact for bf16 dequantized weights, packed codes and fp32 dW; d(alpha)
within 1e-4 relative (floor: 1e-6 of the row's sum of |terms|). Every case
compares every element, the full-size workloads too: they run in the launch
configuration of the benchmark, come to the host one matrix at a time, and
the single-threaded oracle runs on row slices from a thread pool.
"""
import numpy as np
import pytest
import torch

from bit_quantization_aware_b200 import inputs as I
from bit_quantization_aware_b200 import pq
from bit_quantization_aware_b200.step import QuantStep
from oracle import pq_oracle
from tests.gpu_util import bits16, check_bwd, check_fwd, check_step_every_element, f32

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
@pytest.mark.parametrize("offset", [1, 2, 3, 4, 8])  # 4: fp32 16-byte aligned only; 8: 32-byte
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


@pytest.mark.parametrize("which", ["llama_1b_stack", "llama3_8b_set"])
def test_layer_set_full_size_every_element(which, oracle_pool):
    """The full layer sets in the benchmark's launch configuration (one
    batched forward over all matrices, then one batched backward), SEQ2;
    every element of every matrix compared with the oracle (the 1B-class
    stack: 1.08 G weights; the Llama-3-8B-shaped set: 6.98 G weights)."""
    mats = getattr(I, which)()
    step = QuantStep(mats, pq.PQ_SEQ2, device=DEV)
    step.generate(seed=2 if which == "llama_1b_stack" else 3)
    step.run()
    torch.cuda.synchronize()
    assert check_step_every_element(step, oracle_pool) == I.total_weights(mats)
    del step
    torch.cuda.empty_cache()


@pytest.mark.parametrize("q", [pq.PQ_SEQ2, pq.PQ_TERNARY])
def test_student_t_16384_planted_ties(q, oracle_pool):
    """16384x16384 Student-t(3)*0.02 with 1% of entries planted exactly on
    the clip bounds and on rounding ties; forward + packed codes + backward;
    every element compared (bf16 weights, packed bytes, dW, d(alpha)); most
    planted entries hit their target exactly (about 85%)."""
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
    assert check_step_every_element(step, oracle_pool) == 16384 * 16384
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


def _batch_case(q, shapes, seed, pack):
    """Inputs, outputs and descriptors for a batch of matrices; every other
    matrix is offset by one element (misaligned: element path)."""
    bits = pq.pq_code_bits(q)
    items, fwd_d, bwd_d = [], [], []
    for i, (rows, cols) in enumerate(shapes):
        off = 1 if i % 3 == 2 else 0
        w, a, g = make_case(rows, cols, q, seed=seed + i, special=rows * cols >= 8)
        n = rows * cols
        wbuf = torch.empty(n + off + 8, dtype=torch.float32, device=DEV)
        gbuf = torch.empty(n + off + 8, dtype=torch.bfloat16, device=DEV)
        qbuf = torch.empty(n + off + 8, dtype=torch.bfloat16, device=DEV)
        dbuf = torch.empty(n + off + 8, dtype=torch.float32, device=DEV)
        wd, gd = wbuf[off:off + n], gbuf[off:off + n]
        wd.copy_(w.reshape(-1)); gd.copy_(g.reshape(-1))
        ad = a.to(DEV)
        can_pack = pack and cols % (8 // bits) == 0
        pk = (torch.zeros(n * bits // 8 + 8, dtype=torch.uint8, device=DEV)[:n * bits // 8]
              if can_pack else None)
        da = torch.full((rows,), float("nan"), device=DEV)
        gs = pq.pq_default_grad_scale(q, cols)
        items.append((w, a, g, qbuf[off:off + n], pk, dbuf[off:off + n], da, gs, rows, cols))
        fwd_d.append(dict(rows=rows, cols=cols, w=wd, alpha=ad, wq=qbuf[off:off + n], packed=pk))
        bwd_d.append(dict(rows=rows, cols=cols, w=wd, alpha=ad, g=gd, dw=dbuf[off:off + n],
                          dalpha=da, grad_scale=gs))
    return items, pq.matrix_array(fwd_d), pq.matrix_array(bwd_d)


@pytest.mark.parametrize("q", ALLQ)
def test_batched_calls_match_oracle(q):
    """One batched forward and one batched backward over matrices of mixed
    shapes, alignments and empty ones; each compared with the oracle."""
    shapes = [(256, 1024), (1, 8), (3, 24), (5, 12), (64, 4096), (0, 8),
              (7, 1000), (9, 1001), (33, 1032), (2, 70000), (300, 264), (4, 0)]
    items, fd, bd = _batch_case(q, shapes, seed=20, pack=True)
    pq.pq_fakequant_fwd_batch(q, fd)
    pq.pq_fakequant_bwd_batch(q, bd)
    torch.cuda.synchronize()
    for w, a, g, wq, pk, dw, da, gs, rows, cols in items:
        if rows == 0:
            continue
        if cols == 0:
            assert torch.all(da == 0)
            continue
        wn, an, gn = np_inputs(w, a, g)
        check_fwd(q, wn, an, wq.view(rows, cols),
                  pk.view(rows, -1) if pk is not None else None)
        check_bwd(q, wn, an, gn, gs, dw.view(rows, cols), da)


def test_batch_of_more_than_256_matrices():
    """300 matrices in one call: the library splits the launches."""
    q = pq.PQ_SEQ2
    shapes = [(3 + i % 5, 8 * (1 + i % 7)) for i in range(300)]
    items, fd, bd = _batch_case(q, shapes, seed=40, pack=True)
    pq.pq_fakequant_fwd_batch(q, fd)
    pq.pq_fakequant_bwd_batch(q, bd)
    torch.cuda.synchronize()
    for w, a, g, wq, pk, dw, da, gs, rows, cols in items:
        wn, an, gn = np_inputs(w, a, g)
        check_fwd(q, wn, an, wq.view(rows, cols), pk.view(rows, -1))
        check_bwd(q, wn, an, gn, gs, dw.view(rows, cols), da)


def test_batched_step_equals_per_matrix_calls():
    """The 1B stack: batched calls give the same bits as one call per
    matrix."""
    mats = I.llama_1b_stack()[:14]
    s1 = QuantStep(mats, pq.PQ_SEQ2, device=DEV, pack=True, batched=True)
    s1.generate(seed=9)
    s2 = QuantStep(mats, pq.PQ_SEQ2, device=DEV, pack=True, batched=False)
    s2.w_all.copy_(s1.w_all); s2.g_all.copy_(s1.g_all); s2.alpha_all.copy_(s1.alpha_all)
    s1.run(); s2.run()
    torch.cuda.synchronize()
    for x, y in ((s1.wq_all, s2.wq_all), (s1.packed_all, s2.packed_all),
                 (s1.dw_all, s2.dw_all), (s1.dalpha_all, s2.dalpha_all)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def _special_alphas():
    # 1, 1-2^-24, 2-2^-23, mantissa all ones, 0.02, 2, 0.5+ulp, 2^-60 and
    # its neighbours, 2^60 and its neighbours, smallest normal, a
    # subnormal, 2^126, 0.05
    bits = [0x3F800000, 0x3F7FFFFF, 0x3FFFFFFF, 0x3C7FFFFF, 0x3CA3D70A,
            0x40000000, 0x3F000001, 0x21800000, 0x217FFFFF, 0x21800001,
            0x5D800000, 0x5D7FFFFF, 0x5D800001, 0x00800000, 0x00000400,
            0x7E800000, 0x3D4CCCCD]
    rng = np.random.default_rng(31)
    rnd = np.exp(rng.uniform(np.log(1e-30), np.log(1e30), 49)).astype(np.float32)
    return np.concatenate([np.array(bits, np.uint32).view(np.float32), rnd])


def test_scaled_weights_match_ieee_division():
    """x = fl(w/alpha) from the library's division routine equals numpy's
    IEEE fp32 division, bit for bit, over a strided sweep of all finite
    fp32 bit patterns of w (both signs, every exponent) for 64 scales,
    among them mantissas of all ones, powers of two, the edges of the
    reciprocal path's range (2^-60, 2^60), a subnormal and a huge one."""
    alphas = _special_alphas()
    stride = 2053  # odd: every residue of the low mantissa bits appears
    pos = np.arange(0, 0x7F800000, stride, dtype=np.uint32)
    pats = np.concatenate([pos, pos | np.uint32(0x80000000)]).view(np.float32)
    cols = len(pats) // 8 * 8
    pats = pats[:cols]
    w = torch.from_numpy(np.ascontiguousarray(pats)).to(DEV)
    x = torch.empty(cols, dtype=torch.float32, device=DEV)
    for a in alphas:
        ad = torch.tensor([a], dtype=torch.float32, device=DEV)
        pq.pq_scaled_weights(w, ad, x, rows=1, cols=cols)
        torch.cuda.synchronize()
        with np.errstate(over="ignore", under="ignore", divide="ignore"):
            want = (pats / np.float32(a)).astype(np.float32)
        got = x.cpu().numpy()
        bad = np.flatnonzero(got.view(np.uint32) != want.view(np.uint32))
        assert bad.size == 0, (f"alpha={a!r}: {bad.size} mismatches, e.g. "
                               f"w={pats[bad[0]]!r} gpu={got[bad[0]]!r} "
                               f"ieee={want[bad[0]]!r}")


def _threshold_targets(q):
    third = float(np.float32(1.0) / np.float32(3.0))
    base = [-0.99, 0.99, -0.5, 0.0, 0.5, -third, third, -1.0, 1.0, -0.25, 0.25]
    if q in (pq.PQ_LSQ2, pq.PQ_LSQ3, pq.PQ_LSQ4):
        b = {pq.PQ_LSQ2: 2, pq.PQ_LSQ3: 3, pq.PQ_LSQ4: 4}[q]
        lo, hi = -(2 ** (b - 1)), 2 ** (b - 1) - 1
        base += [k + 0.5 for k in range(lo - 1, hi + 1)] + [float(lo), float(hi)]
    return np.array(base, np.float32)


@pytest.mark.parametrize("q", ALLQ)
def test_weights_on_code_and_clip_boundaries(q):
    """For 512 scales, weights within 6 ulps of w = target*alpha for every
    rounding tie and clip bound of the quantizer: the places where a
    one-ulp error in w/alpha would flip a code or the STE mask."""
    rng = np.random.default_rng(37 + q)
    alphas = np.concatenate([_special_alphas()[:17],
                             np.exp(rng.uniform(np.log(1e-3), np.log(10.0), 500))]
                            ).astype(np.float32)
    tg = _threshold_targets(q)
    ks = np.arange(-6, 7)
    rows = []
    for a in alphas:
        with np.errstate(over="ignore"):
            w0 = (tg.astype(np.float32) * a).astype(np.float32)
        cand = w0[:, None].view(np.int32).astype(np.int64) + np.sign(w0[:, None] + 0).astype(
            np.int64) * ks[None, :]
        tiny = np.where(ks >= 0, ks, 0x80000000 | -ks).astype(np.int64)
        cand = np.where(w0[:, None] == 0, tiny[None, :], cand)
        row = (cand & 0xFFFFFFFF).astype(np.uint32).view(np.float32).ravel()
        row = row[np.isfinite(row)]
        rows.append(row)
    cols = max(len(r) for r in rows)
    cols = (cols + 7) // 8 * 8
    W = np.zeros((len(rows), cols), np.float32)
    for i, r in enumerate(rows):
        W[i, :len(r)] = r
    w = torch.from_numpy(W)
    a = torch.from_numpy(alphas)
    g = I.grad_bf16(len(rows), cols, seed=7, stream=77 + q, device="cpu")
    wq, pk, pk2, dw, da, gs = run_gpu(q, w, a, g, True)
    wn, an, gn = np_inputs(w, a, g)
    check_fwd(q, wn, an, wq, pk)
    check_fwd(q, wn, an, None, pk2)
    check_bwd(q, wn, an, gn, gs, dw, da)


def _dequant_gpu(q, packed_np, alpha_np, cols, offset=0):
    rows = packed_np.shape[0]
    nb = packed_np.size
    pbuf = torch.zeros(nb + offset + 16, dtype=torch.uint8, device=DEV)
    pk = pbuf[offset:offset + nb]
    pk.copy_(torch.from_numpy(packed_np.ravel()))
    qbuf = torch.empty(rows * cols + offset + 8, dtype=torch.bfloat16, device=DEV)
    out = qbuf[offset:offset + rows * cols].view(rows, cols)
    pq.pq_dequant_codes(q, pk, torch.from_numpy(alpha_np).to(DEV), out, rows=rows, cols=cols)
    torch.cuda.synchronize()
    return bits16(out)


@pytest.mark.parametrize("q", ALLQ)
@pytest.mark.parametrize("shape,offset", [((1, 32), 0), ((3, 96), 0), ((5, 12), 0),
                                          ((7, 1000), 0), ((33, 1032), 0), ((64, 4096), 0),
                                          ((9, 4096), 1), ((2, 70000), 0),
                                          # staged bulk stores: the widest row a staging
                                          # buffer holds, one row more (direct stores), and
                                          # many units per CTA (both buffers reused)
                                          ((3, 16384), 0), ((2, 16392), 0), ((20000, 1024), 0)])
def test_dequant_matches_oracle(q, shape, offset):
    """Packed codes -> bf16: every element equals the oracle's decoding
    (random bytes, so every code value of the format appears)."""
    rows, cols = shape
    bits = pq.pq_code_bits(q)
    if cols % (8 // bits):
        pytest.skip("shape not packable")
    rng = np.random.default_rng(rows * 7 + cols)
    packed = rng.integers(0, 256, (rows, cols * bits // 8), dtype=np.uint8)
    alpha = np.exp(rng.uniform(-6, 1, rows)).astype(np.float32)
    got = _dequant_gpu(q, packed, alpha, cols, offset)
    want = pq_oracle.dequant(q, packed, alpha, cols)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} mismatches, first {bad[0].tolist()}"


@pytest.mark.parametrize("q", ALLQ)
def test_dequant_inverts_forward_codes(q):
    """On 2048x8192: decoding the forward's packed codes gives the forward's
    bf16 weights, except that zero levels decode to +0."""
    w = I.normal_weights(2048, 8192, seed=11, stream=0, device=DEV)
    a = I.alpha_init(w, q)
    wq, pk = pq.fakequant_fwd(q, w, a, pack=True)
    out = torch.empty_like(wq)
    pq.pq_dequant_codes(q, pk, a, out)
    torch.cuda.synchronize()
    zero = (wq.view(torch.int16) & 0x7FFF) == 0
    assert torch.equal(out.view(torch.int16)[~zero], wq.view(torch.int16)[~zero])
    assert torch.all(out.view(torch.int16)[zero] == 0)


def test_dequant_batch_equals_single_calls():
    """A batch of mixed shapes and alignments decodes like single calls."""
    q = pq.PQ_SEQ2
    rng = np.random.default_rng(41)
    shapes = [(64, 4096), (3, 96), (5, 12), (33, 1032), (0, 8), (7, 1000)]
    descs, singles = [], []
    for rows, cols in shapes:
        packed = torch.from_numpy(rng.integers(0, 256, (rows, cols // 4), dtype=np.uint8)).to(DEV)
        alpha = torch.from_numpy(np.exp(rng.uniform(-5, 0, rows)).astype(np.float32)).to(DEV)
        o1 = torch.empty((rows, cols), dtype=torch.bfloat16, device=DEV)
        o2 = torch.empty((rows, cols), dtype=torch.bfloat16, device=DEV)
        descs.append(dict(rows=rows, cols=cols, packed=packed if rows else None,
                          alpha=alpha if rows else None, wq=o1 if rows else None))
        if rows:
            pq.pq_dequant_codes(q, packed, alpha, o2)
        singles.append((o1, o2))
    pq.pq_dequant_codes_batch(q, pq.matrix_array(descs))
    torch.cuda.synchronize()
    for o1, o2 in singles:
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def _adamw_case(q, rows, cols, seed, offset=0):
    rng = np.random.default_rng(seed)
    w, a, g = make_case(rows, cols, q, seed=seed, special=rows * cols >= 8)
    mw = rng.normal(0, 1e-4, (rows, cols)).astype(np.float32)
    vw = np.abs(rng.normal(0, 1e-7, (rows, cols))).astype(np.float32)
    ma = rng.normal(0, 1e-3, rows).astype(np.float32)
    va = np.abs(rng.normal(0, 1e-6, rows)).astype(np.float32)
    return w.numpy(), a.numpy(), g.view(torch.int16).numpy().view(np.uint16), mw, vw, ma, va


def _adamw_gpu(q, w, a, g, mw, vw, ma, va, gs, hw, ha, offset=0):
    rows, cols = w.shape
    n = rows * cols

    def dev(x, dtype):
        buf = torch.empty(n + offset + 8, dtype=dtype, device=DEV)
        t = buf[offset:offset + n]
        t.copy_(torch.from_numpy(np.ascontiguousarray(x).ravel()))
        return t

    wd = dev(w, torch.float32)
    gd = dev(g.view(np.int16), torch.int16)
    mwd, vwd = dev(mw, torch.float32), dev(vw, torch.float32)
    ad = torch.from_numpy(a.copy()).to(DEV)
    mad, vad = torch.from_numpy(ma.copy()).to(DEV), torch.from_numpy(va.copy()).to(DEV)
    da = torch.full((rows,), float("nan"), device=DEV)
    arr = pq.adamw_matrix_array([dict(rows=rows, cols=cols, w=wd, alpha=ad, g=gd, m_w=mwd,
                                      v_w=vwd, m_alpha=mad, v_alpha=vad, dalpha=da,
                                      grad_scale=gs)])
    pq.pq_fakequant_bwd_adamw(q, arr, hw, ha)
    torch.cuda.synchronize()
    f = lambda t: t.cpu().numpy().reshape(-1)
    return (f(wd).reshape(rows, cols), f(ad), f(mwd).reshape(rows, cols),
            f(vwd).reshape(rows, cols), f(mad), f(vad), f(da))


def _check_adamw(q, w, a, g, mw, vw, ma, va, gs, t, offset=0):
    from oracle.pq_oracle import AdamW
    hw_o, ha_o = AdamW.at_step(t, 2e-5, weight_decay=0.01), AdamW.at_step(t, 1e-4)
    hw, ha = pq.adamw(t, 2e-5, weight_decay=0.01), pq.adamw(t, 1e-4)
    got = _adamw_gpu(q, w, a, g, mw, vw, ma, va, gs, hw, ha, offset)
    ref = pq_oracle.default().bwd_adamw(q, w, a, g, mw, vw, ma, va, gs, hw_o, ha_o)
    for name, x, y in zip(("w", "m_w", "v_w"), (got[0], got[2], got[3]),
                          (ref[0], ref[2], ref[3])):
        bad = np.argwhere(x.view(np.uint32) != y.view(np.uint32))
        assert bad.size == 0, f"q={q} t={t} {name}: {len(bad)} mismatches, first {bad[0].tolist()}"
    # d(alpha) within the reduction-order tolerance; alpha's own AdamW step
    # from the GPU's d(alpha) is exact
    _, ref_da, row_abs = pq_oracle.bwd(q, w, a, g, gs)
    tol = 1e-4 * np.maximum(np.abs(ref_da), 1e-6 * gs * row_abs)
    assert np.all(np.abs(got[6].astype(np.float64) - ref_da) <= tol), q
    pa, pma, pva = pq_oracle.default().adamw_step(a, got[6], ma, va, ha_o)
    for x, y in ((got[1], pa), (got[4], pma), (got[5], pva)):
        assert np.array_equal(x.view(np.uint32), y.view(np.uint32)), q
    return got


@pytest.mark.parametrize("q", ALLQ)
@pytest.mark.parametrize("shape,offset", [((33, 1032), 0), ((7, 1000), 0), ((5, 12), 0),
                                          ((64, 4096), 0), ((9, 2048), 1), ((9, 2048), 4),
                                          ((9, 2048), 8), ((3, 0), 0)])
def test_bwd_adamw_two_steps(q, shape, offset):
    """Fused backward + AdamW: two consecutive steps (the second from the
    GPU's state), weights and moments bit-exact against the oracle."""
    rows, cols = shape
    w, a, g, mw, vw, ma, va = _adamw_case(q, rows, cols, seed=50 + rows)
    gs = pq.pq_default_grad_scale(q, cols) if cols else 1.0
    got = _check_adamw(q, w, a, g, mw, vw, ma, va, gs, 1, offset)
    w2, a2, mw2, vw2, ma2, va2 = got[0], got[1], got[2], got[3], got[4], got[5]
    _check_adamw(q, w2, a2, g, mw2, vw2, ma2, va2, gs, 2, offset)


def test_bwd_adamw_batch_2048x8192_and_stack():
    """Batched fused step over mixed matrices (2048x8192 and a 1B-stack
    layer) equals single-matrix calls bit for bit."""
    q = pq.PQ_SEQ2
    mats = [I.Matrix("big", 2048, 8192, 0, 0)] + I.llama_1b_stack()[:7]
    hw, ha = pq.adamw(5, 2e-5), pq.adamw(5, 1e-4)
    states = []
    for i, m in enumerate(mats):
        w = I.normal_weights(m.rows, m.cols, seed=60 + i, stream=0, device=DEV)
        a = I.alpha_init(w, q)
        g = I.grad_bf16(m.rows, m.cols, seed=60 + i, stream=64, device=DEV)
        mw = torch.randn_like(w) * 1e-4
        vw = torch.rand_like(w) * 1e-7
        ma = torch.randn_like(a) * 1e-3
        va = torch.rand_like(a) * 1e-6
        states.append([w, a, g, mw, vw, ma, va])
    clones = [[t.clone() for t in st] for st in states]

    def desc(st, m):
        w, a, g, mw, vw, ma, va = st
        return dict(rows=m.rows, cols=m.cols, w=w, alpha=a, g=g, m_w=mw, v_w=vw,
                    m_alpha=ma, v_alpha=va, grad_scale=pq.pq_default_grad_scale(q, m.cols))

    pq.pq_fakequant_bwd_adamw(q, pq.adamw_matrix_array([desc(st, m) for st, m in zip(states, mats)]), hw, ha)
    for st, m in zip(clones, mats):
        pq.pq_fakequant_bwd_adamw(q, pq.adamw_matrix_array([desc(st, m)]), hw, ha)
    torch.cuda.synchronize()
    for s1, s2 in zip(states, clones):
        for x, y in zip(s1, s2):
            assert torch.equal(x.view(torch.uint8) if x.dtype != torch.bfloat16 else x.view(torch.int16),
                               y.view(torch.uint8) if y.dtype != torch.bfloat16 else y.view(torch.int16))


def test_launch_counter_counts_batched_launches():
    """pq_launch_count: a batched forward over 300 matrices of the vector
    layout goes out as two launches (256 descriptors per launch), and a
    rejected call launches nothing."""
    q = pq.PQ_SEQ2
    shapes = [(3 + i % 5, 8 * (1 + i % 7)) for i in range(300)]
    ws = [torch.randn(r, c, device=DEV) for r, c in shapes]
    descs = [dict(rows=r, cols=c, w=w, alpha=w.abs().amax(1).clamp_min(1e-30).contiguous(),
                  wq=torch.empty(r, c, dtype=torch.bfloat16, device=DEV))
             for (r, c), w in zip(shapes, ws)]
    arr = pq.matrix_array(descs)
    n0 = pq.pq_launch_count()
    pq.pq_fakequant_fwd_batch(q, arr)
    torch.cuda.synchronize()
    assert pq.pq_launch_count() - n0 == 2
    with pytest.raises(pq.PQError):
        pq.pq_fakequant_fwd_batch(99, arr)
    assert pq.pq_launch_count() - n0 == 2
