"""Exhaustive parity: every finite fp32 weight through the CUDA quantizer.

With alpha = 1 the scaled weight x = fl(w / alpha) is w itself, so feeding
every finite fp32 bit pattern (2^32 - 2^24 values) through the forward and
the backward exercises the clip, the round-half-to-even decision, the level
table, the bf16 cast, the packed code and the straight-through mask over
their whole input domain, subnormals and both zeros included. The division
by other scales is covered by the scaled-weight tests in
``test_parity_gpu.py``.

Compared against the oracle: bf16 weights, packed codes and fp32 dW
bit-exact; d(alpha) per row (4096 consecutive bit patterns, upstream
gradient 1.0, grad_scale 1) within the tolerance of the other parity tests.
The oracle is plain single-threaded C; it runs on all host cores by calling
it from a thread pool (ctypes releases the interpreter lock during the
call), one slice of rows per call.

About 50 s per quantizer on 16 host cores: by default the two quantizers
the pages define (2-bit SEQ and ternary) run; ``PQ_EXHAUSTIVE=all`` runs
all seven.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

from bit_quantization_aware_b200 import pq
from oracle import pq_oracle
from tests.gpu_util import DALPHA_FLOOR, DALPHA_RTOL

pytestmark = pytest.mark.gpu

ROWS, COLS = 16384, 4096           # one chunk: 2^26 consecutive bit patterns
CHUNKS = (1 << 32) // (ROWS * COLS)
SLICE_ROWS = 256                   # rows per oracle call
BF16_ONE = 0x3F80


def _finite_patterns(chunk: int) -> np.ndarray:
    """Chunk ``chunk`` of all 32-bit patterns as fp32, non-finite ones
    (exponent field 255) replaced by +0.0."""
    u = np.arange(chunk * ROWS * COLS, (chunk + 1) * ROWS * COLS, dtype=np.uint64).astype(np.uint32)
    u[((u >> 23) & 0xFF) == 0xFF] = 0
    return u.view(np.float32).reshape(ROWS, COLS)


@pytest.fixture(scope="module")
def pool():
    with ThreadPoolExecutor(max(1, min(64, os.cpu_count() or 1))) as ex:
        yield ex


DEFAULT_QUANTIZERS = (pq.PQ_SEQ2, pq.PQ_TERNARY)


@pytest.mark.parametrize("q", pq_oracle.ALL_QUANTIZERS)
def test_every_finite_fp32_weight(q, pool):
    if q not in DEFAULT_QUANTIZERS and os.environ.get("PQ_EXHAUSTIVE") != "all":
        pytest.skip("set PQ_EXHAUSTIVE=all to sweep every quantizer")
    O = pq_oracle.default()
    bits = pq.pq_code_bits(q)
    dev = "cuda"
    alpha = np.ones(ROWS, np.float32)
    g_np = np.full((ROWS, COLS), BF16_ONE, np.uint16)
    wd = torch.empty((ROWS, COLS), dtype=torch.float32, device=dev)
    ad = torch.ones(ROWS, dtype=torch.float32, device=dev)
    gd = torch.from_numpy(g_np.view(np.int16)).to(dev).view(torch.bfloat16)
    wq = torch.empty((ROWS, COLS), dtype=torch.bfloat16, device=dev)
    pk = torch.empty((ROWS, COLS * bits // 8), dtype=torch.uint8, device=dev)
    dw = torch.empty((ROWS, COLS), dtype=torch.float32, device=dev)
    da = torch.empty(ROWS, dtype=torch.float32, device=dev)
    slices = [slice(r, r + SLICE_ROWS) for r in range(0, ROWS, SLICE_ROWS)]
    checked = 0
    for chunk in range(CHUNKS):
        w_np = _finite_patterns(chunk)
        wd.copy_(torch.from_numpy(w_np))
        pq.pq_fakequant_fwd(q, wd, ad, wq, pk, rows=ROWS, cols=COLS)
        pq.pq_fakequant_bwd(q, wd, ad, gd, dw, da, 1.0, rows=ROWS, cols=COLS)

        def oracle_slice(s):
            ref_wq, _, ref_pk = O.fwd(q, w_np[s], alpha[s], pack=True)
            ref_dw, ref_da, row_abs = O.bwd(q, w_np[s], alpha[s], g_np[s], 1.0)
            return s, ref_wq, ref_pk, ref_dw, ref_da, row_abs

        futures = [pool.submit(oracle_slice, s) for s in slices]
        got_wq = wq.view(torch.int16).cpu().numpy().view(np.uint16)
        got_pk = pk.cpu().numpy()
        got_dw = dw.cpu().numpy().view(np.uint32)
        got_da = da.cpu().numpy().astype(np.float64)
        for f in futures:
            s, ref_wq, ref_pk, ref_dw, ref_da, row_abs = f.result()
            for name, got, ref, per in (("bf16 weight", got_wq[s], ref_wq, 1),
                                        ("packed byte", got_pk[s], ref_pk, 8 // bits),
                                        ("dW", got_dw[s], ref_dw.view(np.uint32), 1)):
                bad = np.argwhere(got != ref)
                if bad.size:
                    r, c = bad[0]
                    pytest.fail(f"q={q}: {len(bad)} {name} mismatches in chunk {chunk}; first at "
                                f"w bits {w_np[s.start + r, c * per].view(np.uint32):#010x}: "
                                f"gpu {got[r, c]:#x} oracle {ref[r, c]:#x}")
            tol = DALPHA_RTOL * np.maximum(np.abs(ref_da).astype(np.float64), DALPHA_FLOOR * row_abs)
            err = np.abs(got_da[s] - ref_da.astype(np.float64))
            assert np.all(err <= tol), f"q={q}: d(alpha) out of tolerance in chunk {chunk}"
        checked += ROWS * COLS
    assert checked == 1 << 32
