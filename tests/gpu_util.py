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


def compare_rows(q, w, a, g, gs, wq_bits, packed, dw_bits, da):
    """The oracle's forward (+ packed codes) and backward of these rows
    against the GPU's outputs (host arrays). Returns a list of mismatch
    descriptions, empty when bf16 weights, packed bytes and dW are
    bit-exact and d(alpha) is within tolerance."""
    errs = []
    ref_wq, _, ref_pk = pq_oracle.fwd(q, w, a, pack=packed is not None)
    if wq_bits is not None:
        bad = np.argwhere(wq_bits != ref_wq)
        if bad.size:
            r, c = bad[0]
            errs.append(f"{len(bad)} bf16 weights differ, first at ({r}, {c}): "
                        f"gpu {wq_bits[r, c]:#06x} oracle {ref_wq[r, c]:#06x}")
    if packed is not None:
        bad = np.argwhere(packed != ref_pk)
        if bad.size:
            errs.append(f"{len(bad)} packed bytes differ, first at {bad[0].tolist()}")
    ref_dw, ref_da, row_abs = pq_oracle.bwd(q, w, a, g, gs)
    bad = np.argwhere(dw_bits != ref_dw.view(np.uint32))
    if bad.size:
        errs.append(f"{len(bad)} dW values differ, first at {bad[0].tolist()}")
    tol = DALPHA_RTOL * np.maximum(np.abs(ref_da).astype(np.float64),
                                   DALPHA_FLOOR * abs(gs) * row_abs)
    err = np.abs(da.astype(np.float64) - ref_da.astype(np.float64))
    if not np.all(err <= tol):
        r = int(np.argmax(err - tol))
        errs.append(f"d(alpha) row {r}: gpu {da[r]!r} oracle {ref_da[r]!r}")
    return errs


def check_step_every_element(step, pool, task_weights=1 << 22):
    """Every element of every matrix of a QuantStep (after one forward and
    one backward) against the oracle: bf16 weights, packed codes (if the
    step packs) and dW bit-exact, d(alpha) within tolerance. Matrices come
    to the host one at a time; the oracle runs on slices of about
    ``task_weights`` weights in ``pool`` (ctypes releases the interpreter
    lock), at most two matrices in flight. Returns the number of weights
    compared."""
    q = step.q
    pending, checked = [], 0

    def drain(items):
        for name, r0, fut in items:
            errs = fut.result()
            assert not errs, f"{name} rows from {r0}: " + "; ".join(errs)

    for b in step.bufs:
        w, a, g = f32(b.w), f32(b.alpha), bits16(b.g)
        wq = bits16(b.wq)
        pk = u8(b.packed) if b.packed is not None else None
        dw = f32(b.dw).view(np.uint32)
        da = f32(b.dalpha)
        per = max(1, task_weights // max(1, b.m.cols))
        futs = []
        for r0 in range(0, b.m.rows, per):
            s = slice(r0, min(b.m.rows, r0 + per))
            futs.append((b.m.name, r0, pool.submit(
                compare_rows, q, w[s], a[s], g[s], b.grad_scale, wq[s],
                None if pk is None else pk[s], dw[s], da[s])))
        drain(pending)
        pending = futs
        checked += b.m.numel
    drain(pending)
    return checked
