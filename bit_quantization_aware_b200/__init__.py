"""B200-native ParetoQ-style per-output-channel weight fake-quantizer.

The hot path (forward quantize + bf16 dequant + packed codes, STE backward
with the per-row scale gradient) runs in hand-written CUDA kernels for
sm_100a behind the C ABI declared in ``include/pq.h``; ``pq`` is the thin
ctypes binding over it. ``inputs`` draws seeded synthetic workloads.
"""
