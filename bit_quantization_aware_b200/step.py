"""One quantizer step over a set of weight matrices (a model's linear layers).

A step is what QAT runs for every linear layer in one training iteration:
the forward fake-quantization of every matrix (bf16 dequantized weights,
optionally packed codes), then, after the model's matmuls, the STE backward
of every matrix (fp32 dW and the per-row scale gradient). All buffers of the
set live in a handful of flat device allocations, one per tensor kind, with
per-matrix views, so that the step's launches touch resident HBM only.

The arithmetic runs in the CUDA library through the C ABI (``pq``).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import inputs as I
from . import pq


def _align(n: int, a: int = 64) -> int:
    return (n + a - 1) // a * a


@dataclass
class MatrixBuffers:
    m: I.Matrix
    w: torch.Tensor
    alpha: torch.Tensor
    g: torch.Tensor
    wq: torch.Tensor
    dw: torch.Tensor
    dalpha: torch.Tensor
    packed: torch.Tensor | None
    grad_scale: float


class QuantStep:
    """Buffers and launches for one quantizer over a list of matrices."""

    def __init__(self, mats, q: int, device="cuda", pack: bool = False,
                 alloc_outputs: bool = True, batched: bool = True):
        self.batched = batched
        self.mats = list(mats)
        self.q = q
        self.pack = pack
        self.device = torch.device(device)
        bits = pq.pq_code_bits(q)
        offs, n = [], 0
        for m in self.mats:
            offs.append(n)
            n += _align(m.numel)
        roffs, nr = [], 0
        for m in self.mats:
            roffs.append(nr)
            nr += _align(m.rows)
        poffs, npk = [], 0
        for m in self.mats:
            poffs.append(npk)
            npk += _align(m.numel * bits // 8)
        dev = self.device
        self.w_all = torch.empty(n, dtype=torch.float32, device=dev)
        self.g_all = torch.empty(n, dtype=torch.bfloat16, device=dev)
        self.alpha_all = torch.empty(nr, dtype=torch.float32, device=dev)
        self.wq_all = torch.empty(n, dtype=torch.bfloat16, device=dev) if alloc_outputs else None
        self.dw_all = torch.empty(n, dtype=torch.float32, device=dev) if alloc_outputs else None
        self.dalpha_all = torch.empty(nr, dtype=torch.float32, device=dev)
        self.packed_all = (torch.empty(npk, dtype=torch.uint8, device=dev)
                           if pack else None)
        self.bufs = []
        for m, o, ro, po in zip(self.mats, offs, roffs, poffs):
            v2 = lambda t: t[o:o + m.numel].view(m.rows, m.cols)
            self.bufs.append(MatrixBuffers(
                m=m, w=v2(self.w_all), alpha=self.alpha_all[ro:ro + m.rows],
                g=v2(self.g_all),
                wq=v2(self.wq_all) if alloc_outputs else None,
                dw=v2(self.dw_all) if alloc_outputs else None,
                dalpha=self.dalpha_all[ro:ro + m.rows],
                packed=(self.packed_all[po:po + m.numel * bits // 8].view(
                    m.rows, m.cols * bits // 8) if pack else None),
                grad_scale=pq.pq_default_grad_scale(q, m.cols)))

        self._fwd_descs = pq.matrix_array([
            dict(rows=b.m.rows, cols=b.m.cols, w=b.w, alpha=b.alpha, wq=b.wq,
                 packed=b.packed) for b in self.bufs])
        self._bwd_descs = pq.matrix_array([
            dict(rows=b.m.rows, cols=b.m.cols, w=b.w, alpha=b.alpha, g=b.g,
                 dw=b.dw, dalpha=b.dalpha, grad_scale=b.grad_scale)
            for b in self.bufs])

    @property
    def weights(self) -> int:
        return sum(m.numel for m in self.mats)

    def bytes_fwd(self) -> int:
        bits = pq.pq_code_bits(self.q) if self.pack else 0
        return sum(m.numel * 6 + m.numel * bits // 8 + m.rows * 4 for m in self.mats)

    def bytes_bwd(self) -> int:
        return sum(m.numel * 10 + m.rows * 8 for m in self.mats)

    def generate(self, seed: int = 0, dist: str = "normal", lsq_rule="lsq"):
        """Draw W, alpha and G for every matrix on the device."""
        for b in self.bufs:
            sid = 8 * b.m.layer + b.m.proj
            if dist == "normal":
                I.normal_weights(b.m.rows, b.m.cols, seed=seed, stream=sid,
                                 device=self.device, out=b.w)
            else:
                b.w.copy_(I.student_t3_weights(b.m.rows, b.m.cols, seed=seed,
                                               stream=sid, device=self.device))
            b.alpha.copy_(I.alpha_init(b.w, self.q, lsq_rule=lsq_rule))
            I.grad_bf16(b.m.rows, b.m.cols, seed=seed, stream=sid + 64,
                        device=self.device, out=b.g)

    def fwd_all(self, stream=None):
        """Forward of every matrix: one batched call (or one call each)."""
        if self.batched:
            pq.pq_fakequant_fwd_batch(self.q, self._fwd_descs, stream)
            return
        for b in self.bufs:
            pq.pq_fakequant_fwd(self.q, b.w, b.alpha, b.wq, b.packed, stream)

    def bwd_all(self, stream=None):
        """Backward of every matrix: one batched call (or one call each)."""
        if self.batched:
            pq.pq_fakequant_bwd_batch(self.q, self._bwd_descs, stream)
            return
        for b in self.bufs:
            pq.pq_fakequant_bwd(self.q, b.w, b.alpha, b.g, b.dw, b.dalpha,
                                b.grad_scale, stream)

    def run(self, stream=None):
        self.fwd_all(stream)
        self.bwd_all(stream)

    @property
    def launches_per_step(self) -> int:
        """Kernel launches of one step (all matrices use the vector layout:
        one launch per 256 matrices per phase when batched)."""
        if self.batched:
            return 2 * ((len(self.mats) + 255) // 256)
        return 2 * len(self.mats)
