"""pq_wq_gemm_noalloc (fixed library scratch, no allocation) against the
existing pq_wq_gemm entry point (caller workspace), on two consecutive
calls each: the second call reuses the scratch the first one left.

Both entry points run the same kernel with the same split plan, so the
outputs must be the same bits; the check also applies the tolerance of the
weight-only matmul tests (2^-8 of |Y| plus 1e-4 of sum_k |x_k * w_k|) so
that a failure says how far off a result is. This file is collected last
so that it also runs after every other GPU test in the same process."""
import numpy as np
import pytest
import torch

from bit_quantization_aware_b200 import inputs as I
from bit_quantization_aware_b200 import pq
from oracle import pq_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(q, m, n, k, seed):
    w = I.normal_weights(n, k, seed=seed, stream=0, device=DEV)
    a = I.alpha_init(w, q)
    _, packed = pq.fakequant_fwd(q, w, a, pack=True)
    x = I.normal_weights(m, k, seed=seed, stream=5, std=1.0, device=DEV).to(torch.bfloat16)
    return x, packed, a


def _tolerance(q, x, packed, a, ref):
    k = x.shape[1]
    wd = pq_oracle.bf16_bits_to_float(
        pq_oracle.dequant(q, packed.cpu().numpy(), a.cpu().numpy(), k)).astype(np.float64)
    absum = np.abs(x.float().cpu().numpy().astype(np.float64)) @ np.abs(wd).T
    return 2.0 ** -8 * np.abs(ref) + 1e-4 * absum + 1e-30


@pytest.mark.parametrize("q,m,n,k", [(pq.PQ_SEQ2, 8, 4096, 8192),     # split-K: scratch used
                                     (pq.PQ_TERNARY, 33, 1000, 2048),  # split-K, ragged n
                                     (pq.PQ_SEQ2_B, 4, 16384, 512)])   # one segment: no scratch
def test_noalloc_matches_workspace_entry_point(q, m, n, k):
    need = pq.pq_wq_gemm_workspace_bytes(q, m, n, k)
    assert 0 <= need <= pq.WQ_GEMM_NOALLOC_SCRATCH_BYTES
    x, packed, a = _case(q, m, n, k, seed=m * 7 + n + k)
    ref = pq.wq_gemm(q, x, packed, a)
    torch.cuda.synchronize()
    ref64 = ref.float().cpu().numpy().astype(np.float64)
    tol = _tolerance(q, x, packed, a, ref64)
    for call in range(2):
        y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        pq.pq_wq_gemm_noalloc(q, x, packed, a, y)
        torch.cuda.synchronize()
        assert pq.pq_device_status() == 0
        got = y.float().cpu().numpy().astype(np.float64)
        err = np.abs(got - ref64)
        assert np.all(err <= tol), f"call {call}: max error {err.max()} over tolerance"
        same = torch.equal(y.view(torch.int16), ref.view(torch.int16))
        assert same, f"call {call}: {int((y.view(torch.int16) != ref.view(torch.int16)).sum())} " \
                     "outputs differ in their bits from pq_wq_gemm"


def test_noalloc_rejects_problems_over_the_scratch_limit():
    q, m, n, k = pq.PQ_SEQ2, 128, 14336, 4096
    assert pq.pq_wq_gemm_workspace_bytes(q, m, n, k) > pq.WQ_GEMM_NOALLOC_SCRATCH_BYTES
    x = torch.zeros((m, k), dtype=torch.bfloat16, device=DEV)
    packed = torch.zeros((n, k // 4), dtype=torch.uint8, device=DEV)
    a = torch.ones(n, device=DEV)
    y = torch.full((m, n), 7.0, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(pq.PQError, match="scratch"):
        pq.pq_wq_gemm_noalloc(q, x, packed, a, y)
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())  # nothing was enqueued
