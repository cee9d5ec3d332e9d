"""Helpers for the GPU parity tests: move tensors to numpy and compare the
CUDA library's outputs with the oracle's."""
from __future__ import annotations

import numpy as np
import torch

from oracle import pq_oracle

# d(alpha) tolerance: 1e-4 relative, with a floor of 1e-6 of the row's
# sum of |terms| (times grad_scale) for rows whose sum cancels to ~0. Both
# sides accumulate fp32-identical terms in fp64; only the order differs.
DALPHA_RTOL = 1e-4
DALPHA_FLOOR = 1e-6


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns."""
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.uint8)


def check_fwd(q, w_np, a_np, wq_gpu, packed_gpu=None, rows=None):
    """Bit-exact comparison of bf16 weights (and packed codes)."""
    ref_wq, _, ref_pk = pq_oracle.fwd(q, w_np, a_np, pack=packed_gpu is not None)
    got = bits16(wq_gpu) if wq_gpu is not None else None
    if got is not None:
        bad = np.argwhere(got != ref_wq)
        assert bad.size == 0, (
            f"q={q}: {len(bad)} bf16 mismatches, first at {bad[0].tolist()}: "
            f"w={w_np[tuple(bad[0])]!r} alpha={a_np[bad[0][0]]!r} "
            f"gpu={got[tuple(bad[0])]:#06x} ref={ref_wq[tuple(bad[0])]:#06x}")
    if packed_gpu is not None:
        gp = u8(packed_gpu)
        bad = np.argwhere(gp != ref_pk)
        assert bad.size == 0, f"q={q}: {len(bad)} packed byte mismatches, first {bad[0].tolist()}"


def check_bwd(q, w_np, a_np, g_np, gs, dw_gpu, da_gpu):
    """dW bit-exact, d(alpha) within the stated tolerance."""
    ref_dw, ref_da, row_abs = pq_oracle.bwd(q, w_np, a_np, g_np, gs)
    got = f32(dw_gpu)
    bad = np.argwhere(got.view(np.uint32) != ref_dw.view(np.uint32))
    assert bad.size == 0, f"q={q}: {len(bad)} dW mismatches, first {bad[0].tolist()}"
    da = f32(da_gpu)
    tol = DALPHA_RTOL * np.maximum(np.abs(ref_da).astype(np.float64),
                                   DALPHA_FLOOR * abs(gs) * row_abs)
    err = np.abs(da.astype(np.float64) - ref_da.astype(np.float64))
    worst = int(np.argmax(err - tol)) if len(err) else 0
    assert np.all(err <= tol), (
        f"q={q}: dalpha row {worst}: gpu={da[worst]!r} ref={ref_da[worst]!r}")
    return float(np.max(err / np.maximum(np.abs(ref_da), 1e-30))) if len(err) else 0.0
