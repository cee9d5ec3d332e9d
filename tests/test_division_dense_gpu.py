"""Dense check of the quantizer's division x = fl(w / alpha) on the GPU.

The library divides by a per-row reciprocal with two remainder corrections
(IEEE division outside a guarded range), which must give the same bits as
IEEE round-to-nearest division. Here 2^31 random (w, alpha) pairs, drawn on
the device from a counter-based hash, go through ``pq_scaled_weights`` and
through CUDA's ``__fdiv_rn`` in a separate test-only kernel
(``tests/csrc/fdiv_ref.cu``); every quotient must match bit for bit. Half
the batches draw both operands from every finite fp32 value (all
exponents, subnormals, zeros of both signs for w; positive values for
alpha); the other half keep both in [2^-60, 2^61), the range of the fast
reciprocal path and its upper edge.
"""
import pytest
import torch

from bit_quantization_aware_b200 import pq
from tests import fdiv_ref

pytestmark = pytest.mark.gpu

ROWS, COLS = 1 << 17, 2048        # 2^28 pairs per batch, one alpha per row
BATCHES = [(seed, mode) for seed in range(4) for mode in (0, 1)]  # 2^31 pairs


def test_division_matches_ieee_on_random_pairs():
    L = fdiv_ref.load()
    dev = "cuda"
    s = torch.cuda.current_stream().cuda_stream
    w = torch.empty((ROWS, COLS), dtype=torch.int32, device=dev)
    a = torch.empty(ROWS, dtype=torch.int32, device=dev)
    x = torch.empty((ROWS, COLS), dtype=torch.float32, device=dev)
    ref = torch.empty((ROWS, COLS), dtype=torch.float32, device=dev)
    total = 0
    for seed, mode in BATCHES:
        assert L.fdiv_draw(w.data_ptr(), w.numel(), 2 * seed + 1, mode, 0, s) == 0
        assert L.fdiv_draw(a.data_ptr(), a.numel(), 2 * seed + 2, mode, 1, s) == 0
        wf, af = w.view(torch.float32), a.view(torch.float32)
        pq.pq_scaled_weights(wf, af, x)
        assert L.fdiv_ref(wf.data_ptr(), af.data_ptr(), ref.data_ptr(), ROWS, COLS, s) == 0
        bad = x.view(torch.int32) != ref.view(torch.int32)
        nbad = int(bad.sum())
        if nbad:
            r, c = (int(v) for v in bad.nonzero()[0])
            pytest.fail(f"batch (seed {seed}, mode {mode}): {nbad} quotients differ; first "
                        f"w={wf[r, c].item()!r} alpha={af[r].item()!r}: "
                        f"library {x[r, c].item()!r} IEEE {ref[r, c].item()!r}")
        total += w.numel()
    assert total == 1 << 31
