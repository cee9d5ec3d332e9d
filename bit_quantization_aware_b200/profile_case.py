"""Run one weight matrix through the quantizer a few times (for profilers).

    python -m bit_quantization_aware_b200.profile_case --rows 14336 --cols 4096 \
        --quant seq2 --iters 3 [--pack]
    python -m bit_quantization_aware_b200.profile_case --rows 16384 --cols 16384 \
        --quant seq2 --iters 3 --gemm-m 1
    python -m bit_quantization_aware_b200.profile_case ... --op dequant | bwd_adamw
    python -m bit_quantization_aware_b200.profile_case --set llama3_8b --iters 2

Draws seeded synthetic inputs on the device (N(0, 0.02) weights, alpha =
max|w_row| or the quantizer's init, bf16 N(0, 1e-3) upstream gradient),
then runs forward and backward ``iters`` times on the current stream and
prints the per-iteration CUDA-event times. Sized by the caller; a
14336x4096 matrix moves about 0.9 GB per iteration, more than L2.

``--op dequant`` runs the packed-code dequantization instead (codes from a
forward), ``--op bwd_adamw`` the backward fused with one AdamW step, and
``--gemm-m M`` the weight-only matmul with M activation rows on seeded
random codes (only codes, scales, X and Y are allocated).

``--set llama3_8b`` (or ``llama_1b``) runs the benchmark's batched forward
and backward over a whole layer set instead of one matrix: one launch per
phase, about 84 GB resident for the Llama-3-8B-shaped set. Its backward
moves 70 GB per launch, so an L2-sized tail of dirty lines left after the
kernel is below 0.2% of its writes (for one-pass DRAM counters only).
"""
from __future__ import annotations

import argparse

import torch

from . import inputs as I
from . import pq


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--rows", type=int, default=14336)
    p.add_argument("--cols", type=int, default=4096)
    p.add_argument("--quant", default="seq2", choices=sorted(pq.QUANTIZERS))
    p.add_argument("--iters", type=int, default=3)
    p.add_argument("--pack", action="store_true")
    p.add_argument("--gemm-m", type=int, default=0,
                   help="run the weight-only matmul with this many activation rows")
    p.add_argument("--op", default="quantizer", choices=["quantizer", "dequant", "bwd_adamw"])
    p.add_argument("--set", default="", choices=["", "llama3_8b", "llama_1b"],
                   help="a whole layer set in the benchmark's batched launches")
    a = p.parse_args()
    q = pq.QUANTIZERS[a.quant]
    dev = torch.device("cuda")
    if a.set:
        return set_case(a, q, dev)
    if a.gemm_m:
        return gemm_case(a, q, dev)
    if a.op != "quantizer":
        return next_case(a, q, dev)
    w = I.normal_weights(a.rows, a.cols, seed=0, stream=0, device=dev)
    alpha = I.alpha_init(w, q)
    g = I.grad_bf16(a.rows, a.cols, seed=0, stream=64, device=dev)
    wq = torch.empty((a.rows, a.cols), dtype=torch.bfloat16, device=dev)
    packed = (torch.empty((a.rows, a.cols * pq.pq_code_bits(q) // 8),
                          dtype=torch.uint8, device=dev) if a.pack else None)
    dw = torch.empty((a.rows, a.cols), dtype=torch.float32, device=dev)
    da = torch.empty((a.rows,), dtype=torch.float32, device=dev)
    gs = pq.pq_default_grad_scale(q, a.cols)
    torch.cuda.synchronize()
    for i in range(a.iters):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        pq.pq_fakequant_fwd(q, w, alpha, wq, packed)
        e[1].record()
        pq.pq_fakequant_bwd(q, w, alpha, g, dw, da, gs)
        e[2].record()
        torch.cuda.synchronize()
        n = a.rows * a.cols
        tf, tb = e[0].elapsed_time(e[1]) * 1e-3, e[1].elapsed_time(e[2]) * 1e-3
        fb = 6 + (pq.pq_code_bits(q) / 8 if a.pack else 0)
        print(f"iter {i}: fwd {tf * 1e6:.1f} us ({n * fb / tf / 1e9:.0f} GB/s), "
              f"bwd {tb * 1e6:.1f} us ({n * 10 / tb / 1e9:.0f} GB/s)")


def set_case(a, q, dev):
    from .step import QuantStep
    mats = I.llama3_8b_set() if a.set == "llama3_8b" else I.llama_1b_stack()
    step = QuantStep(mats, q, device=dev, pack=a.pack)
    step.generate(seed=3)
    torch.cuda.synchronize()
    for i in range(a.iters):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        step.fwd_all()
        e[1].record()
        step.bwd_all()
        e[2].record()
        torch.cuda.synchronize()
        tf, tb = e[0].elapsed_time(e[1]) * 1e-3, e[1].elapsed_time(e[2]) * 1e-3
        print(f"iter {i}: fwd {tf * 1e3:.3f} ms ({step.bytes_fwd() / tf / 1e9:.0f} GB/s), "
              f"bwd {tb * 1e3:.3f} ms ({step.bytes_bwd() / tb / 1e9:.0f} GB/s)")


def next_case(a, q, dev):
    w = I.normal_weights(a.rows, a.cols, seed=0, stream=0, device=dev)
    alpha = I.alpha_init(w, q)
    n = a.rows * a.cols
    if a.op == "dequant":
        wq, packed = pq.fakequant_fwd(q, w, alpha, pack=True)
        out = torch.empty_like(wq)
        nbytes = n * 2 + packed.numel() + a.rows * 4

        def go():
            pq.pq_dequant_codes(q, packed, alpha, out)
    else:
        g = I.grad_bf16(a.rows, a.cols, seed=0, stream=64, device=dev)
        m_w, v_w = torch.zeros_like(w), torch.zeros_like(w)
        m_a, v_a = torch.zeros_like(alpha), torch.zeros_like(alpha)
        arr = pq.adamw_matrix_array([dict(rows=a.rows, cols=a.cols, w=w, alpha=alpha, g=g,
                                          m_w=m_w, v_w=v_w, m_alpha=m_a, v_alpha=v_a,
                                          grad_scale=pq.pq_default_grad_scale(q, a.cols))])
        nbytes = 26 * n + 24 * a.rows
        t = [0]

        def go():
            t[0] += 1
            pq.pq_fakequant_bwd_adamw(q, arr, pq.adamw(t[0], 2e-5), pq.adamw(t[0], 2e-5))
    torch.cuda.synchronize()
    for i in range(a.iters):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record()
        go()
        e[1].record()
        torch.cuda.synchronize()
        dt = e[0].elapsed_time(e[1]) * 1e-3
        print(f"iter {i}: {a.op} {dt * 1e6:.1f} us ({nbytes / dt / 1e9:.0f} GB/s algorithmic)")


def gemm_case(a, q, dev):
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    bits = pq.pq_code_bits(q)
    packed = torch.randint(0, 256, (a.rows, a.cols * bits // 8), dtype=torch.uint8,
                           device=dev, generator=g)
    alpha = torch.rand(a.rows, device=dev, generator=g) + 0.5
    x = torch.randn(a.gemm_m, a.cols, device=dev, generator=g).to(torch.bfloat16)
    y = torch.empty((a.gemm_m, a.rows), dtype=torch.bfloat16, device=dev)
    need = pq.pq_wq_gemm_workspace_bytes(q, a.gemm_m, a.rows, a.cols)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    for i in range(a.iters):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record()
        pq.pq_wq_gemm(q, x, packed, alpha, y, ws)
        e[1].record()
        torch.cuda.synchronize()
        t = e[0].elapsed_time(e[1]) * 1e-3
        print(f"iter {i}: wq_gemm {t * 1e6:.1f} us ({packed.numel() / t / 1e9:.0f} GB/s of codes)")
    if pq.pq_device_status() != 0:
        raise RuntimeError("a bounded device wait gave up")


if __name__ == "__main__":
    main()
