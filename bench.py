"""Benchmark of the quantizer step: forward + STE backward over the
Llama-3-8B-shaped linear set (32 layers of q/o 4096x4096, k/v 1024x4096,
gate/up 14336x4096, down 4096x14336; 2-bit SEQ, bf16 dequant output).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--op quantizer|dequant|bwd_adamw|wq_gemm|sharded] [--no-extras]

One step = one forward over every matrix, then one backward over every
matrix, with all inputs resident in HBM (synthetic, seeded; about 84 GB per
GPU, far larger than L2, so no flush is needed between steps). Each rank
runs the full set on its own GPU (weak scaling; the quantizer shards by
matrix and row and needs no collective). Rank 0 prints one JSON line.

With one GPU the default run adds to that line, after the headline's timed
region:

* ``per_config``: forward, backward and forward + backward of the other
  four workloads (one 256x1024 weight with packed codes under both 2-bit SEQ
  readings; one 2048x8192 weight under five quantizers; the 1B-class stack;
  one 16384x16384 heavy-tailed weight with planted ties and clip bounds,
  fused packed export and the standalone packer), each phase timed after an
  L2 flush, with the CPU oracle's rate on the same kind of input beside it;
* ``next``: the rows built on the quantizer, on the same Llama-3-8B-shaped
  set: dequantization of packed codes, the backward fused with AdamW (and
  the unfused backward + torch AdamW beside it), the weight-only 2-bit
  matmul at 1, 16 and 128 activation rows (and cuBLAS bf16 on the
  dequantized weights beside it), and the row-sharded step with two ranks
  emulated on the one GPU.

``--impl reference`` times the CPU oracle (the plain C reference used by
the tests) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantizer fwd+bwd Gweights/s per step and % of B200 HBM roofline"
UNIT = "Gweights/s"
WORKLOAD = "llama3_8b_linear_set_seq2_fwd_ste_bwd"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 2 ** 20
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (the roofline uses the measured copy peak)
MAX_SHARDED_WORLD = 16  # gradient sources one reduce launch accepts


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--op", choices=["quantizer", "dequant", "bwd_adamw", "wq_gemm", "sharded"],
                   default="quantizer",
                   help="quantizer: the forward+backward step (the headline); "
                        "dequant: packed codes -> bf16 over the same layer set; "
                        "bwd_adamw: the backward fused with the AdamW step; "
                        "wq_gemm: Y = X W^T from the packed 2-bit codes on the tensor cores; "
                        "sharded: the row-sharded step with its ranks emulated on one GPU")
    p.add_argument("--no-extras", action="store_true",
                   help="quantizer: print the headline only (no per_config, no next)")
    p.add_argument("--config-steps", type=int, default=20,
                   help="timed iterations of each per_config measurement (median reported)")
    p.add_argument("--extra-steps", type=int, default=10,
                   help="timed iterations of each next-row measurement")
    p.add_argument("--world", type=int, default=2,
                   help=f"sharded: emulated ranks (buffer sets on the one GPU), 1..{MAX_SHARDED_WORLD}")
    p.add_argument("--layers", type=int, default=8,
                   help="sharded: layers of the Llama-3-8B-shaped set (memory grows with world)")
    p.add_argument("--m", type=int, default=16,
                   help="wq_gemm: activation rows (tokens of a decode batch), 1..128")
    p.add_argument("--shape", default="llama3_8b", choices=["llama3_8b", "16384"],
                   help="wq_gemm: every matrix of the Llama-3-8B-shaped set, or one "
                        "16384x16384 weight (the size the pages compare kernels at)")
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="target CPU time of the oracle baseline sample")
    a = p.parse_args(argv)
    if not 1 <= a.world <= MAX_SHARDED_WORLD:
        p.error(f"--world must be between 1 and {MAX_SHARDED_WORLD} "
                f"(the gradient sources one reduce launch sums), got {a.world}")
    if not 1 <= a.layers <= 32:
        p.error(f"--layers must be between 1 and 32, got {a.layers}")
    if not 1 <= a.m <= 128:
        p.error(f"--m must be between 1 and 128, got {a.m}")
    return a


def config_dict(n_gpus, weights_per_gpu):
    return {"workload": WORKLOAD,
            "matrices": "32 layers x {q,o 4096x4096; k,v 1024x4096; "
                        "gate,up 14336x4096; down 4096x14336}",
            "quantizer": "seq2 (2-bit SEQ, levels +-0.25, +-0.75 alpha)",
            "weights_per_gpu": weights_per_gpu,
            "global_weights": weights_per_gpu * n_gpus,
            "parallelism": f"replicas x{n_gpus} (each GPU its own layer set)",
            "l2": "inputs larger than L2 (about 84 GB resident per GPU)"}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


QUANTIZER_KERNEL_SOURCES = ("pq.cu", "pq_quant.cuh")  # define the step's kernels


def kernel_source_hash():
    """Hash of the sources that define the quantizer step's kernels."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantization_aware_b200", "csrc")
    for name in QUANTIZER_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per weight of the backward kernel from an ncu capture,
    valid only while the kernel sources are unchanged."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    return d


# ------------------------------------------------------------- rank logic
def reduce_max(values, device, world):
    """Element-wise max over ranks (timings: the slowest rank decides)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def step_throughput(weights_per_rank, world, ms_per_step):
    """Whole-job Gweights/s: the weights every rank processed in one step
    over the (max-over-ranks) step time."""
    return weights_per_rank * world / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clocks and throttle reasons during the timed
    region (read only; no GPU setting is changed)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
            os.unlink(self.path)
        except Exception:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "samples": len(sm), "reasons": sorted(reasons)}


def physical_gpu_index(local):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return int(vis.split(",")[local])
        except (ValueError, IndexError):
            pass
    return local


# ---------------------------------------------------------------- reference
def workload_weights():
    from bit_quantization_aware_b200 import inputs as I
    return I.total_weights(I.llama3_8b_set())


def oracle_seconds_per_weight(q, cols, pack=False):
    """Single-thread oracle time per weight of forward (+ packed codes) +
    backward, calibrated on 8 full-width rows."""
    import numpy as np
    import torch

    from bit_quantization_aware_b200 import inputs as I
    from oracle import pq_oracle
    w = I.normal_weights(8, cols, seed=0, stream=6, device="cpu")
    a = I.alpha_init(w, q)
    g = I.grad_bf16(8, cols, seed=0, stream=70, device="cpu")
    gn = g.view(torch.int16).numpy().view(np.uint16)
    t0 = time.perf_counter()
    pq_oracle.fwd(q, w.numpy(), a.numpy(), pack=pack)
    pq_oracle.bwd(q, w.numpy(), a.numpy(), gn, 1.0)
    return (time.perf_counter() - t0) / w.numel()


def oracle_sample(mats, q, seconds, *, seed=0, dist="normal", lsq_rule="lsq",
                  plant=False, pack=False):
    """Full-width rows of every matrix in ``mats`` (the same draws and
    scales as the GPU inputs of that workload, on the host) so that the
    oracle's forward + backward takes about ``seconds`` on one core; whole
    matrices when they fit."""
    import numpy as np
    import torch

    from bit_quantization_aware_b200 import inputs as I
    per_weight = oracle_seconds_per_weight(q, max(m.cols for m in mats), pack)
    per_mat = seconds / max(per_weight, 1e-12) / len(mats)
    sample = []
    for m in mats:
        rows = max(1, min(m.rows, int(per_mat // m.cols)))
        sid = 8 * m.layer + m.proj
        if dist == "normal":
            wm = I.normal_weights(rows, m.cols, seed=seed, stream=sid, device="cpu")
        else:
            wm = I.student_t3_weights(rows, m.cols, seed=seed, stream=sid, device="cpu")
        am = I.alpha_init(wm, q, lsq_rule=lsq_rule)
        if plant:
            I.plant_boundaries(wm, am, frac=0.01, seed=seed)
        gm = I.grad_bf16(rows, m.cols, seed=seed, stream=sid + 64, device="cpu")
        sample.append((m, wm.numpy(), am.numpy(), gm.view(torch.int16).numpy().view(np.uint16)))
    return sample


def sample_rows_for_oracle(cpu_seconds):
    """Rows drawn from every matrix kind of one layer of the Llama-3-8B-shaped
    set so that the oracle's forward + backward takes about ``cpu_seconds``
    on one core."""
    from bit_quantization_aware_b200 import inputs as I
    mats = [m for m in I.llama3_8b_set() if m.layer == 0]
    return oracle_sample(mats, I.SEQ2, cpu_seconds)


def time_oracle(sample, q=3, pack=False):
    """Runs the oracle's forward (+ packed codes) and backward over a sample;
    returns (weights, seconds)."""
    from oracle import pq_oracle
    t0 = time.perf_counter()
    n = 0
    for m, w, a, g in sample:
        pq_oracle.fwd(q, w, a, pack=pack)
        pq_oracle.bwd(q, w, a, g, pq_oracle.default_grad_scale(q, m.cols))
        n += w.size
    dt = time.perf_counter() - t0
    return n, dt


def describe_sample(sample):
    rows = {m.name.split(".")[-1]: w.shape[0] for m, w, _, _ in sample}
    n = sum(w.size for _, w, _, _ in sample)
    return (f"{n} weights: rows {rows} of layer 0's matrices (full width), "
            f"SEQ2 forward + backward, single thread")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # each step is a bounded sample: the whole run stays near two minutes
    per_step = max(0.5, min(10.0, 120.0 / max(1, args.steps)))
    sample = sample_rows_for_oracle(per_step)
    for _ in range(args.warmup):
        time_oracle(sample[:1])
    times, n = [], 0
    for _ in range(args.steps):
        n, dt = time_oracle(sample)
        times.append(dt)
    total = sum(times)
    value = n * args.steps / total / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config_dict(args.gpus, workload_weights()),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1,
                             "kind": "oracle", "sample": describe_sample(sample)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------- timing helpers
class L2Flush:
    """Reads a buffer of twice the L2 size (a sum), so that the next kernel
    finds none of its inputs in L2 (a real step runs a matmul between the
    quantizer's phases). A read leaves only clean lines behind: a written
    flush buffer would leave up to an L2 of dirty lines whose write-back
    lands in the next kernel's time (for a 268 MB phase, up to half again
    its own traffic)."""

    def __init__(self, device):
        import torch
        self.buf = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
        self.out = torch.empty((), dtype=torch.float32, device=device)

    def __call__(self):
        import torch
        torch.sum(self.buf, dim=0, out=self.out)


def timed_phases(fns, steps, warmup, flush):
    """Runs ``fns`` (name -> callable) in order ``warmup + steps`` times,
    each call bracketed by CUDA events on the current stream and preceded
    by an L2 flush (outside the events). Returns, per name, the median
    milliseconds over the timed iterations, the medians of the sums over
    all phases, and the library's kernel launches per iteration."""
    import torch

    from bit_quantization_aware_b200 import pq
    names = list(fns)
    for _ in range(max(warmup, 1)):
        for n in names:
            flush()
            fns[n]()
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in names] for _ in range(steps)]
    l0 = pq.pq_launch_count()
    for it in range(steps):
        for j, n in enumerate(names):
            flush()
            ev[it][j][0].record()
            fns[n]()
            ev[it][j][1].record()
    torch.cuda.synchronize()
    launches = (pq.pq_launch_count() - l0) / steps
    per = {n: [ev[it][j][0].elapsed_time(ev[it][j][1]) for it in range(steps)]
           for j, n in enumerate(names)}
    med = {n: statistics.median(v) for n, v in per.items()}
    return med, per, launches


def phase_entry(ms, weights, nbytes, peak):
    sec = ms * 1e-3
    return {"ms": ms, "Gweights_s": weights / sec / 1e9, "GB_s": nbytes / sec / 1e9,
            "frac_of_peak": nbytes / sec / 1e9 / peak, "algorithmic_bytes": nbytes}


def time_graph(fn, steps, warmup):
    """Captures ``fn`` in a CUDA graph (after two eager runs on a side
    stream) and times ``steps`` replays; returns (ms per replay, graph,
    library kernel launches per replay)."""
    import torch

    from bit_quantization_aware_b200 import pq
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    l0 = pq.pq_launch_count()
    with torch.cuda.graph(g):
        fn()
    launches = pq.pq_launch_count() - l0
    for _ in range(max(warmup, 3)):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, g, launches


def time_eager(fn, steps, warmup):
    """Times ``steps`` back-to-back calls of ``fn`` with CUDA events on the
    current stream; returns (ms per call, library launches per call)."""
    import torch

    from bit_quantization_aware_b200 import pq
    for _ in range(max(warmup, 1)):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0 = pq.pq_launch_count()
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, (pq.pq_launch_count() - l0) / steps


# ---------------------------------------------------------------- per config
def per_config_cases():
    """The four workloads besides the headline, with the seeds, draws and
    scale initialisations of their parity tests (seed = workload number - 1)."""
    from bit_quantization_aware_b200 import inputs as I
    return [
        dict(key="1_single_256x1024_pack", mats=[I.Matrix("w", 256, 1024, 0, 0)],
             quantizers=[("seq2", I.SEQ2, "lsq"), ("seq2_b", I.SEQ2_B, "lsq")],
             pack=True, dist="normal", seed=0, plant=False, standalone_pack=False,
             what="one 256x1024 N(0,0.02) weight, alpha = max|w_row|, forward with packed "
                  "codes + backward; launch-bound and L2-resident (a parity case)"),
        dict(key="2_bit_width_sweep_2048x8192", mats=[I.Matrix("w", 2048, 8192, 0, 0)],
             quantizers=[("binary", I.BINARY, "lsq"), ("ternary", I.TERNARY, "lsq"),
                         ("seq2", I.SEQ2, "lsq"), ("lsq3", I.LSQ3, "lsq"),
                         ("lsq4", I.LSQ4, "lsq")],
             pack=False, dist="normal", seed=1, plant=False, standalone_pack=False,
             what="one 2048x8192 N(0,0.02) weight; alpha = mean|w_row| (binary), "
                  "max|w_row| (ternary, seq2), 2 mean|w_row|/sqrt(Qp) (lsq3, lsq4)"),
        dict(key="3_llama_1b_stack", mats=I.llama_1b_stack(),
             quantizers=[("seq2", I.SEQ2, "lsq")],
             pack=False, dist="normal", seed=2, plant=False, standalone_pack=False,
             what="24 layers: q,o 2048x2048; k,v 512x2048; gate,up 5632x2048; "
                  "down 2048x5632; one batched launch per phase"),
        dict(key="5_student_t_16384_planted_pack", mats=[I.Matrix("t3.16384", 16384, 16384, 0, 0)],
             quantizers=[("seq2", I.SEQ2, "lsq"), ("ternary", I.TERNARY, "lsq")],
             pack=True, dist="student_t", seed=4, plant=True, standalone_pack=True,
             what="one 16384x16384 Student-t(3)*0.02 weight, 1% of entries planted on "
                  "clip bounds and rounding ties; forward with fused packed codes + "
                  "backward; the standalone packer timed beside it"),
    ]


def measure_case(case, steps, warmup, peak, device, flush, oracle_seconds):
    """One per_config workload: every quantizer's forward, backward and
    forward + backward (median of ``steps`` after an L2 flush each), the
    standalone packer where asked, and the oracle's rate on a sample."""
    import torch

    from bit_quantization_aware_b200 import inputs as I
    from bit_quantization_aware_b200 import pq
    from bit_quantization_aware_b200.step import QuantStep
    out = {"what": case["what"], "weights": I.total_weights(case["mats"]),
           "l2_flush": "before every phase (a buffer of twice the L2 size is read)"}
    for name, q, rule in case["quantizers"]:
        step = QuantStep(case["mats"], q, device=device, pack=case["pack"])
        step.generate(seed=case["seed"], dist=case["dist"], lsq_rule=rule)
        planted = None
        if case["plant"]:
            b = step.bufs[0]
            n, hit = I.plant_boundaries(b.w, b.alpha, frac=0.01, seed=case["seed"])
            planted = {"entries": n, "exactly_on_target": hit}
        fns = {"fwd": step.fwd_all, "bwd": step.bwd_all}
        if case["standalone_pack"]:  # one matrix: pq_pack_codes into its own buffer
            b0 = step.bufs[0]
            pk_alone = torch.empty_like(b0.packed)
            fns["pack_standalone"] = lambda: pq.pq_pack_codes(step.q, b0.w, b0.alpha, pk_alone)
        med, per, launches = timed_phases(fns, steps, warmup, flush)
        fb = statistics.median([f + g for f, g in zip(per["fwd"], per["bwd"])])
        w = step.weights
        entry = {"fwd": phase_entry(med["fwd"], w, step.bytes_fwd(), peak),
                 "bwd": phase_entry(med["bwd"], w, step.bytes_bwd(), peak),
                 "fwd_bwd": phase_entry(fb, w, step.bytes_fwd() + step.bytes_bwd(), peak),
                 "launches_per_iteration": launches,
                 "packed_codes": bool(case["pack"])}
        if case["standalone_pack"]:
            rows = sum(m.rows for m in case["mats"])
            nb = w * 4 + w * pq.pq_code_bits(q) // 8 + rows * 4
            entry["pack_standalone"] = phase_entry(med["pack_standalone"], w, nb, peak)
        if planted:
            entry["planted"] = planted
        # free this quantizer's buffers before the next one allocates
        del step, fns
        if case["standalone_pack"]:
            del b0, pk_alone
        if case["plant"]:
            del b
        torch.cuda.empty_cache()
        if oracle_seconds > 0:
            sample = oracle_sample(case["mats"], q, oracle_seconds, seed=case["seed"],
                                   dist=case["dist"], lsq_rule=rule, plant=case["plant"],
                                   pack=case["pack"])
            n, dt = time_oracle(sample, q=q, pack=case["pack"])
            whole = all(wm.shape[0] == m.rows for m, wm, _, _ in sample)
            entry["oracle"] = {"Gweights_s": n / dt / 1e9, "cores": 1, "seconds": dt,
                               "weights": n,
                               "sample": ("the whole workload" if whole else
                                          "full-width rows of every matrix"),
                               "gpu_speedup_fwd_bwd": entry["fwd_bwd"]["Gweights_s"]
                               / (n / dt / 1e9)}
        out[name] = entry
    return out


def run_per_config(args, peak, device, oracle_seconds=1.5):
    flush = L2Flush(device)
    res = {}
    for case in per_config_cases():
        res[case["key"]] = measure_case(case, args.config_steps, args.warmup, peak, device,
                                        flush, oracle_seconds)
    del flush
    return res


# ---------------------------------------------------------------- next rows
def packed_views(step, packed_all):
    """Per-matrix views of one flat packed-code buffer (2-bit codes)."""
    views, o = [], 0
    for b in step.bufs:
        n = b.m.numel // 4
        views.append(packed_all[o:o + n].view(b.m.rows, b.m.cols // 4))
        o += (n + 255) // 256 * 256
    return views


def packed_bytes(step):
    return sum((b.m.numel // 4 + 255) // 256 * 256 for b in step.bufs)


def measure_dequant(step, packed, out, steps, warmup, peak):
    """Packed codes + alpha -> bf16 for every matrix of the step, one batched
    call (2.25 B per weight + 4 B per row)."""
    from bit_quantization_aware_b200 import pq
    descs = [dict(rows=b.m.rows, cols=b.m.cols, alpha=b.alpha, packed=pk, wq=o)
             for b, pk, o in zip(step.bufs, packed, out)]
    mats = pq.matrix_array(descs)
    ms, launches = time_eager(lambda: pq.pq_dequant_codes_batch(step.q, mats), steps, warmup)
    nbytes = sum(b.m.numel * 2 + b.m.numel // 4 + b.m.rows * 4 for b in step.bufs)
    achieved = nbytes / (ms * 1e-3) / 1e9
    return {"ms": ms, "Gweights_s": step.weights / (ms * 1e-3) / 1e9,
            "launches_per_call": launches,
            "roofline": {"bound": "hbm", "kernel": "pq::dequant_units_kernel<SEQ2, vector layout>",
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "algorithmic_bytes": nbytes}}


def measure_bwd_adamw(step, steps, warmup, peak):
    """The backward fused with one AdamW step over every matrix (one batched
    launch; 26 B per weight + 24 B per row), then, for context, the unfused
    sequence: the batched backward writing dW, then torch's fused AdamW. The
    step's weights and scales are updated in place."""
    import torch

    from bit_quantization_aware_b200 import pq
    m_w = torch.zeros_like(step.w_all)
    v_w = torch.zeros_like(step.w_all)
    m_a = torch.zeros_like(step.alpha_all)
    v_a = torch.zeros_like(step.alpha_all)
    descs = []
    for b in step.bufs:
        o = b.w.data_ptr() - step.w_all.data_ptr()
        o //= 4
        ro = (b.alpha.data_ptr() - step.alpha_all.data_ptr()) // 4
        n = b.m.numel
        descs.append(dict(rows=b.m.rows, cols=b.m.cols, w=b.w, alpha=b.alpha, g=b.g,
                          m_w=m_w[o:o + n], v_w=v_w[o:o + n], m_alpha=m_a[ro:ro + b.m.rows],
                          v_alpha=v_a[ro:ro + b.m.rows], grad_scale=b.grad_scale))
    arr = pq.adamw_matrix_array(descs)
    t = [0]

    def fused():
        t[0] += 1
        pq.pq_fakequant_bwd_adamw(step.q, arr, pq.adamw(t[0], 2e-5), pq.adamw(t[0], 2e-5))

    ms, launches = time_eager(fused, steps, warmup)
    del arr, descs, m_w, v_w, m_a, v_a
    torch.cuda.empty_cache()
    # context: backward (dW to memory) + torch fused AdamW on the same data
    params = []
    for b in step.bufs:
        prm = torch.nn.Parameter(b.w, requires_grad=True)
        prm.grad = b.dw
        params.append(prm)
    opt = torch.optim.AdamW(params, lr=2e-5, weight_decay=0.0, fused=True)

    def unfused():
        step.bwd_all()
        opt.step()

    ms_unfused, _ = time_eager(unfused, steps, warmup)
    del opt, params
    torch.cuda.empty_cache()
    rows = sum(b.m.rows for b in step.bufs)
    nbytes = 26 * step.weights + 24 * rows
    achieved = nbytes / (ms * 1e-3) / 1e9
    return {"ms": ms, "Gweights_s": step.weights / (ms * 1e-3) / 1e9,
            "launches_per_call": launches,
            "roofline": {"bound": "hbm", "kernel": "pq::bwd_adamw_units_kernel<SEQ2, vector layout>",
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "algorithmic_bytes": nbytes},
            "unfused": {"ms": ms_unfused,
                        "what": "pq_fakequant_bwd_batch (dW to memory) + "
                                "torch.optim.AdamW(fused=True)",
                        "speedup_of_fused": ms_unfused / ms}}


def wq_gemm_kernel_name(m, gsize, max_k):
    """The kernel a grouped launch of ``gsize`` matrices with ``m`` activation
    rows runs, and its arithmetic: one row times a lone matrix (k <= 32768)
    takes the CUDA-core kernel; 1..16 rows otherwise the exact fixed-point
    mode after its activation digit-plane pre-pass, on packed fp4 MMAs while
    every k <= 2^20 and on 8-bit MMAs beyond; more rows the bf16 mode."""
    if m == 1 and gsize == 1 and max_k <= 32768:
        return "pqg::pqv::gemv_kernel<MAXP> (CUDA cores, paired fp32 FMA)", "bf16 x 2-bit codes, f32 FMA"
    if m <= 16 and max_k <= (1 << 20):
        return ("pqg::wq_gemm_kernel<NT, MAXP, kModeF4> (tcgen05.mma kind::mxf4 block-scaled, unit scales, "
                "TMEM accumulator) after pqg::xplanes_kernel<true>",
                "e2m1 base-9 digit planes of bf16 activations x e2m1 f'/2 code nibbles, "
                "f32 accumulate (exact integers)")
    if m <= 16:
        return ("pqg::wq_gemm_kernel<NT, MAXP, kModeI8> (tcgen05.mma kind::i8, TMEM accumulator)"
                " after pqg::xplanes_kernel<false>",
                "s8 digit planes of bf16 activations x u8 2-bit code fields, s32 accumulate")
    return ("pqg::wq_gemm_kernel<NT, MAXP, kModeBF16> (tcgen05.mma kind::f16, TMEM accumulator)",
            "bf16 x 2-bit codes, f32 accumulate")


def measure_wq_gemm(bufs, packed, q, m, steps, warmup, device, with_single=False):
    """Weight-only 2-bit matmul Y = X (alpha * levels)^T for every matrix in
    ``bufs`` (grouped launches of up to 64 matrices, captured in one CUDA
    graph), against cuBLAS (torch.matmul) on the dense bf16 dequantized
    weights, also graph-captured."""
    import torch

    from bit_quantization_aware_b200 import pq
    ks = sorted({b.m.cols for b in bufs})
    ns = sorted({b.m.rows for b in bufs})
    gen = torch.Generator(device=device)
    gen.manual_seed(11)
    xs = {k: torch.randn((m, k), generator=gen, device=device).to(torch.bfloat16) for k in ks}
    ys = {n: torch.empty((m, n), dtype=torch.bfloat16, device=device) for n in ns}
    ys_ref = {n: torch.empty((m, n), dtype=torch.bfloat16, device=device) for n in ns}
    ngroups = (len(bufs) + 63) // 64
    gsize = (len(bufs) + ngroups - 1) // ngroups
    groups = [pq.gemm_problem_array([dict(x=xs[b.m.cols], packed=pk, alpha=b.alpha,
                                          y=ys[b.m.rows])
                                     for b, pk in zip(bufs[i:i + gsize], packed[i:i + gsize])])
              for i in range(0, len(bufs), gsize)]
    gneed = max(pq.pq_wq_gemm_batch_workspace_bytes(q, m, g) for g in groups)
    gws = torch.empty(max(gneed, 256), dtype=torch.uint8, device=device)

    def ours():
        for g in groups:
            pq.pq_wq_gemm_batch(q, m, g, gws)

    def dense():
        for b in bufs:
            torch.matmul(xs[b.m.cols], b.wq.t(), out=ys_ref[b.m.rows])

    ms, g_ours, launches = time_graph(ours, steps, warmup)
    res = {}
    if with_single:
        need = max(pq.pq_wq_gemm_workspace_bytes(q, m, b.m.rows, b.m.cols) for b in bufs)
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device)

        def ours_single():
            for b, pk in zip(bufs, packed):
                pq.pq_wq_gemm(q, xs[b.m.cols], pk, b.alpha, ys[b.m.rows], ws)
        ms_single, g_single, l_single = time_graph(ours_single, steps, warmup)
        res["per_matrix_launches"] = {"ms": ms_single, "launches_per_step": l_single,
                                      "what": "pq_wq_gemm once per matrix, CUDA graph"}
        del g_single
    ms_dense, g_dense, _ = time_graph(dense, steps, warmup)
    status = pq.pq_device_status()
    if status != 0:
        raise RuntimeError(f"weight-only matmul: a bounded device wait gave up ({status})")
    # the last matrix of the set, both ways (same weights, fp32 sums)
    b = bufs[-1]
    yo, yr = ys[b.m.rows].float(), ys_ref[b.m.rows].float()
    rel = float((yo - yr).abs().max() / yr.abs().max().clamp_min(1e-30))
    del g_ours, g_dense
    weights = sum(b.m.numel for b in bufs)
    nbytes = sum(b.m.numel // 4 + b.m.rows * 4 + m * b.m.cols * 2 + m * b.m.rows * 2
                 for b in bufs)
    flops = 2 * m * weights
    hbm, hbm_kind = measured_peaks()
    tflops, tf_kind = measured_tensor_peak()
    if nbytes / (hbm * 1e9) >= flops / (tflops * 1e12):
        roof = {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm,
                "unit": "GB/s", "peak_source": f"{hbm_kind} hbm_gbs",
                "algorithmic_bytes": nbytes}
    else:
        roof = {"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": tflops,
                "unit": "TFLOP/s", "peak_source": f"{tf_kind} bf16_tflops (burst)",
                "algorithmic_flops": flops}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"], arith = wq_gemm_kernel_name(m, gsize, max(ks))
    res.update({"m": m, "ms": ms, "Gweights_s": weights / (ms * 1e-3) / 1e9,
                "tflops": flops / (ms * 1e-3) / 1e12, "launches_per_step": launches,
                "grouped_launches": len(groups), "matrices_per_launch": gsize,
                "dtype": arith,
                "roofline": roof,
                "cublas_bf16_dense": {"ms": ms_dense, "speedup_of_ours": ms_dense / ms,
                                      "what": "torch.matmul(x, W_bf16.t()) per matrix, CUDA graph",
                                      "max_rel_diff_last_matrix": rel}})
    return res


def sharded_bytes(weights: int, world: int) -> dict:
    """Algorithmic bytes of one row-sharded step over `weights` weights (all
    ranks together; scales and d(alpha) are per-row and negligible): pack
    reads each owned fp32 weight and writes 0.25 B of codes; every rank's
    gather + dequantization reads all codes and writes all bf16 weights;
    the reduce step reads `world` bf16 gradient rows per owned weight plus
    w, m, v and writes w, m, v."""
    return {"pack": int(4.25 * weights),
            "gather_dequant": int(world * 2.25 * weights),
            "reduce_bwd_adamw": int((2 * world + 24) * weights)}


def measure_sharded(world, layers, steps, warmup, peak, device):
    """The row-sharded owner-computes step (pack own rows; gather + dequantize
    everyone's codes; reduce the replicas' gradients + backward + AdamW on
    own rows) for ``world`` ranks emulated as buffer sets on one GPU, over
    the first ``layers`` layers of the Llama-3-8B-shaped set. Peer buffers
    are local device memory here, so this measures the kernels' HBM
    efficiency, not NVLink. Each phase runs for every rank in turn, timed by
    CUDA events."""
    import torch

    from bit_quantization_aware_b200 import inputs as I
    from bit_quantization_aware_b200 import pq
    from bit_quantization_aware_b200.sharded import LocalPeers, ShardedQuantStep
    q = pq.PQ_SEQ2
    mats = I.llama3_8b_set()[: 7 * layers]
    peers = LocalPeers(world)
    ranks = [ShardedQuantStep(mats, q, k, world, peers, device=device) for k in range(world)]
    for i, m in enumerate(mats):
        w = I.normal_weights(m.rows, m.cols, seed=3, stream=i, device=device)
        a = I.alpha_init(w, q)
        for r in ranks:
            r.load_full(i, w, a)
        del w, a
    for k, r in enumerate(ranks):
        for i, m in enumerate(mats):
            r.g(i).copy_(I.grad_bf16(m.rows, m.cols, seed=4 + k, stream=64 + i, device=device))
    torch.cuda.synchronize()
    t = [0]

    def phase(fn):
        for r in ranks:
            fn(r)

    def step_fns():
        t[0] += 1
        hw, ha = pq.adamw(t[0], 2e-5), pq.adamw(t[0], 1e-4)
        return [("pack", lambda r: r.pack_shards()),
                ("gather_dequant", lambda r: r.gather_dequant()),
                ("reduce_bwd_adamw", lambda r: r.reduce_step(hw, ha))]

    for _ in range(max(warmup, 1)):
        for _, fn in step_fns():
            phase(fn)
    torch.cuda.synchronize()
    names = ["pack", "gather_dequant", "reduce_bwd_adamw"]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4 * steps)]
    l0 = pq.pq_launch_count()
    for s_ in range(steps):
        for j, (_, fn) in enumerate(step_fns()):
            ev[4 * s_ + j].record()
            phase(fn)
        ev[4 * s_ + 3].record()
    torch.cuda.synchronize()
    launches = pq.pq_launch_count() - l0
    ms = {n: sum(ev[4 * s_ + j].elapsed_time(ev[4 * s_ + j + 1]) for s_ in range(steps)) / steps
          for j, n in enumerate(names)}
    total = sum(ms.values())
    weights = I.total_weights(mats)
    nbytes = sharded_bytes(weights, world)
    phases = {n: {"ms": ms[n], "algorithmic_bytes": nbytes[n],
                  "GB_s": nbytes[n] / (ms[n] * 1e-3) / 1e9,
                  "frac_of_peak": nbytes[n] / (ms[n] * 1e-3) / 1e9 / peak} for n in names}
    allb = sum(nbytes.values())
    del ranks, peers
    torch.cuda.empty_cache()
    return {"ms": total, "Gweights_s": weights / (total * 1e-3) / 1e9, "weights": weights,
            "world": world, "layers": layers, "launches_per_step": launches / steps,
            "workload": f"llama3_8b_first{layers}layers_seq2_sharded_world{world}_emulated",
            "note": "all ranks' work on one GPU in turn; peer reads are local HBM reads",
            "roofline": {"bound": "hbm", "kernel": "pack, dequant and reduce_bwd_adamw units kernels",
                         "achieved": allb / (total * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": allb / (total * 1e-3) / 1e9 / peak,
                         "algorithmic_bytes": allb},
            "phases": phases, "launches_total": launches}


def run_next_rows(step, args, peak, device):
    """The rows built on the quantizer, on the headline's Llama-3-8B-shaped
    buffers: packed export -> dequantization -> weight-only matmul at 1, 16
    and 128 activation rows, then the backward fused with AdamW (which
    updates the weights in place, so it runs last)."""
    import torch

    from bit_quantization_aware_b200 import pq
    res = {}
    packed_all = torch.empty(packed_bytes(step), dtype=torch.uint8, device=device)
    packed = packed_views(step, packed_all)
    # one forward that writes bf16 weights and packed codes
    pq.pq_fakequant_fwd_batch(step.q, pq.matrix_array([
        dict(rows=b.m.rows, cols=b.m.cols, w=b.w, alpha=b.alpha, wq=b.wq, packed=pk)
        for b, pk in zip(step.bufs, packed)]))
    torch.cuda.synchronize()
    deq_all = torch.empty_like(step.wq_all)
    deq_out = [deq_all[(b.wq.data_ptr() - step.wq_all.data_ptr()) // 2:][: b.m.numel]
               .view(b.m.rows, b.m.cols) for b in step.bufs]
    res["dequant"] = measure_dequant(step, packed, deq_out, args.extra_steps, args.warmup, peak)
    same = all(torch.equal(o.view(torch.int16), b.wq.view(torch.int16))
               for o, b in zip(deq_out, step.bufs))
    res["dequant"]["equals_forward_bf16"] = bool(same)
    res["wq_gemm"] = {}
    for m in (1, 16, 128):
        res["wq_gemm"][f"m{m}"] = measure_wq_gemm(step.bufs, packed, step.q, m,
                                                   2 * args.extra_steps, args.warmup, device)
    del packed, packed_all, deq_out, deq_all
    torch.cuda.empty_cache()
    res["bwd_adamw"] = measure_bwd_adamw(step, args.extra_steps, args.warmup, peak)
    return res


# --------------------------------------------------------------------- ours
def run_ours(args):
    import torch
    import torch.distributed as dist

    from bit_quantization_aware_b200 import inputs as I
    from bit_quantization_aware_b200 import pq
    from bit_quantization_aware_b200.step import QuantStep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    pq.lib()  # fail loudly if the CUDA library is missing

    mats = I.llama3_8b_set()
    step = QuantStep(mats, pq.PQ_SEQ2, device=device)
    step.generate(seed=3 + rank)
    stream = torch.cuda.current_stream()
    weights = step.weights

    def barrier():
        if world > 1:
            dist.barrier()

    n_b = step.launches_per_step // 2  # backward launches per step
    ev_start = torch.cuda.Event(enable_timing=True)
    ev_end = torch.cuda.Event(enable_timing=True)
    bwd_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    fwd_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    time.sleep(0.3)
    # warm-up right before the timed region: after an idle gap the first
    # few launches run slower while the clocks come back up
    for _ in range(max(args.warmup, 0)):
        step.run()
    torch.cuda.synchronize()

    barrier()
    torch.cuda.synchronize()
    l0 = pq.pq_launch_count()
    ev_start.record(stream)
    for k in range(args.steps):
        fwd_ev[k].record(stream)
        step.fwd_all()
        bwd_ev[k][0].record(stream)
        step.bwd_all()
        bwd_ev[k][1].record(stream)
    ev_end.record(stream)
    torch.cuda.synchronize()
    launches = pq.pq_launch_count() - l0
    barrier()
    clocks = sampler.stop()

    ms_total = ev_start.elapsed_time(ev_end)
    bwd_ms = sum(a.elapsed_time(b) for a, b in bwd_ev)
    fwd_ms = sum(a.elapsed_time(b[0]) for a, b in zip(fwd_ev, bwd_ev))
    ms_total, bwd_ms, fwd_ms = reduce_max([ms_total, bwd_ms, fwd_ms], device, world)
    ms_step = ms_total / args.steps
    value = step_throughput(weights, world, ms_step)

    # roofline of the dominant kernel (the backward: 10 of 16 bytes/weight;
    # one batched launch covers all matrices of the step)
    peak, peak_kind = measured_peaks()
    bwd_bytes_step = step.bytes_bwd()
    bwd_s_step = bwd_ms * 1e-3 / args.steps
    achieved = bwd_bytes_step / bwd_s_step / 1e9
    tr = recorded_traffic()
    traffic = None
    if tr is not None:
        traffic = tr["dram_bytes_per_weight"] * weights / n_b
    roofline = {"bound": "hbm", "kernel": "pq::bwd_units_kernel<SEQ2, vector layout>",
                "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peak_kind} hbm_gbs (STREAM-style copy)",
                "algorithmic_bytes_per_launch": bwd_bytes_step / n_b,
                "avg_launch_us": bwd_s_step / n_b * 1e6,
                "fwd_bwd_frac_of_peak": (step.bytes_fwd() + bwd_bytes_step)
                / (ms_step * 1e-3) / 1e9 / peak,
                "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                "traffic_frac_of_peak": (None if traffic is None
                                         else traffic / bwd_s_step * n_b / 1e9 / peak)}

    def phase(ms_per_step, nbytes):
        sec = ms_per_step * 1e-3
        return {"ms_per_step": ms_per_step, "Gweights_s": step_throughput(weights, world, ms_per_step),
                "GB_s": nbytes / sec / 1e9, "frac_of_peak": nbytes / sec / 1e9 / peak,
                "frac_of_nominal": nbytes / sec / 1e9 / NOMINAL_HBM_GBS,
                "algorithmic_bytes": nbytes}
    phases = {"fwd": phase(fwd_ms / args.steps, step.bytes_fwd()),
              "bwd": phase(bwd_ms / args.steps, bwd_bytes_step),
              "fwd_bwd": phase(ms_step, step.bytes_fwd() + bwd_bytes_step),
              "peak_GB_s": peak, "nominal_GB_s": NOMINAL_HBM_GBS}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(step, args, local, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = sample_rows_for_oracle(args.cpu_seconds)
        n, dt = time_oracle(sample)
        cpu = {"value": n / dt / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": describe_sample(sample), "seconds": dt,
               "host_cores": os.cpu_count()}

    per_config = nxt = extras_clocks = None
    if world == 1 and not args.no_extras:
        # after the headline's timed region: the NEXT rows on its buffers,
        # then the other workloads and the sharded step on fresh buffers
        xs = ClockSampler(physical_gpu_index(local))
        xs.start()
        nxt = run_next_rows(step, args, peak, device)
        del step
        torch.cuda.empty_cache()
        nxt["sharded"] = measure_sharded(2, 8, args.extra_steps, args.warmup, peak, device)
        per_config = run_per_config(args, peak, device)
        extras_clocks = xs.stop()
        per_config["4_llama3_8b_set"] = {
            "see": "the line's phases (the headline workload)",
            "oracle": None if cpu is None else
            {"Gweights_s": cpu["value"], "cores": 1, "seconds": cpu["seconds"],
             "sample": cpu["sample"],
             "gpu_speedup_fwd_bwd": phases["fwd_bwd"]["Gweights_s"] / cpu["value"]}}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic (seeded N(0,0.02) weights, "
                "bf16 N(0,1e-3) upstream grads, alpha = max|w_row|)",
                "config": config_dict(world, weights),
                "gpu_launches": launches,
                "roofline": roofline, "phases": phases, "cpu_baseline": cpu, "e2e": e2e,
                "clocks": clocks}
        if per_config is not None:
            line["per_config"] = per_config
            line["next"] = nxt
            line["extras_clocks"] = extras_clocks
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def bind_to_gpu_numa_node(device_index):
    """Pin this process to the CPUs next to the GPU (sysfs local_cpulist), so
    that pinned host buffers are first touched on the GPU's NUMA node."""
    try:
        import torch
        p = torch.cuda.get_device_properties(device_index)
        bus = f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        with open(f"/sys/bus/pci/devices/{bus}/local_cpulist") as f:
            spec = f.read().strip()
        cpus = set()
        for part in spec.split(","):
            a, _, b = part.partition("-")
            cpus.update(range(int(a), int(b or a) + 1))
        if cpus:
            os.sched_setaffinity(0, cpus)
            return spec
    except Exception:
        return None
    return None


def run_e2e(step, args, local, world):
    """Same metric through the public API from host buffers: every step
    copies each layer's W and dWq from pinned host memory, runs the batched
    forward and backward calls for the layer's matrices, and copies Wq, dW
    and d(alpha) back to pinned host memory. Copies in, compute and copies
    out run on three streams, so layer l's outputs travel while layer l+1's
    inputs arrive."""
    import torch
    import torch.distributed as dist

    from bit_quantization_aware_b200 import pq

    numa = bind_to_gpu_numa_node(local)
    layers = sorted({b.m.layer for b in step.bufs})
    by_layer = {l: [b for b in step.bufs if b.m.layer == l] for l in layers}
    n_layer = sum(b.m.numel for b in by_layer[layers[0]])
    rows_layer = sum(b.m.rows for b in by_layer[layers[0]])
    pin = dict(pin_memory=True)
    h_w = torch.empty(n_layer, dtype=torch.float32, **pin)
    h_g = torch.empty(n_layer, dtype=torch.bfloat16, **pin)
    h_wq = torch.empty(n_layer, dtype=torch.bfloat16, **pin)
    h_dw = torch.empty(n_layer, dtype=torch.float32, **pin)
    h_da = torch.empty(rows_layer, dtype=torch.float32, **pin)
    # host inputs: the device data of layer 0 (realistic values)
    o = 0
    for b in by_layer[layers[0]]:
        h_w[o:o + b.m.numel].copy_(b.w.reshape(-1))
        h_g[o:o + b.m.numel].copy_(b.g.reshape(-1))
        o += b.m.numel
    fwd_d = {l: pq.matrix_array([dict(rows=b.m.rows, cols=b.m.cols, w=b.w, alpha=b.alpha,
                                      wq=b.wq) for b in by_layer[l]]) for l in layers}
    bwd_d = {l: pq.matrix_array([dict(rows=b.m.rows, cols=b.m.cols, w=b.w, alpha=b.alpha,
                                      g=b.g, dw=b.dw, dalpha=b.dalpha,
                                      grad_scale=b.grad_scale) for b in by_layer[l]])
             for l in layers}
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def one_step():
        for l in layers:
            with torch.cuda.stream(s_in):
                o = 0
                for b in by_layer[l]:
                    b.w.view(-1).copy_(h_w[o:o + b.m.numel], non_blocking=True)
                    b.g.view(-1).copy_(h_g[o:o + b.m.numel], non_blocking=True)
                    o += b.m.numel
            s_cmp.wait_stream(s_in)
            pq.pq_fakequant_fwd_batch(step.q, fwd_d[l], s_cmp)
            pq.pq_fakequant_bwd_batch(step.q, bwd_d[l], s_cmp)
            s_out.wait_stream(s_cmp)
            with torch.cuda.stream(s_out):
                o, ro = 0, 0
                for b in by_layer[l]:
                    h_wq[o:o + b.m.numel].copy_(b.wq.view(-1), non_blocking=True)
                    h_dw[o:o + b.m.numel].copy_(b.dw.view(-1), non_blocking=True)
                    h_da[ro:ro + b.m.rows].copy_(b.dalpha, non_blocking=True)
                    o += b.m.numel
                    ro += b.m.rows

    one_step()
    torch.cuda.synchronize()
    k = max(1, args.e2e_steps)
    if world > 1:
        dist.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    start.record(s_in)
    for _ in range(k):
        one_step()
        # the next step's inputs may only land after this step's outputs left
        s_in.wait_stream(s_out)
    end.record(s_in)
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) * 1e3
    ms = reduce_max([start.elapsed_time(end)], f"cuda:{local}", world)[0]
    ms_step = ms / k
    bi = sum(b.m.numel * 6 for b in step.bufs)
    bo = sum(b.m.numel * 6 + b.m.rows * 4 for b in step.bufs)
    return {"value": step_throughput(step.weights, world, ms_step), "unit": UNIT,
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "ms_per_step": ms_step, "steps": k, "wall_ms_per_step": wall / k,
            "pcie_GBs": (bi + bo) / (ms_step * 1e-3) / 1e9, "numa_cpus": numa,
            "how": "pinned host W, dWq -> device; pq_fakequant_fwd_batch/bwd_batch per layer; "
                   "Wq, dW, dalpha -> pinned host; three streams, layer-pipelined"}


# ------------------------------------------------------- single-row modes
def _llama_step_with_codes(device):
    """The Llama-3-8B-shaped set with bf16 weights and packed codes from
    one forward (inputs of the dequantization and matmul modes)."""
    import torch

    from bit_quantization_aware_b200 import inputs as I
    from bit_quantization_aware_b200 import pq
    from bit_quantization_aware_b200.step import QuantStep
    step = QuantStep(I.llama3_8b_set(), pq.PQ_SEQ2, device=device, pack=True)
    step.generate(seed=3)
    step.fwd_all()
    torch.cuda.synchronize()
    return step


def run_dequant(args):
    """Packed 2-bit codes + alpha -> bf16 weights for every matrix of the
    Llama-3-8B-shaped set (the export path's consumer), one batched call,
    1 GPU. Prints one JSON line with its own roofline (2.25 B/weight)."""
    import torch
    torch.cuda.set_device(0)
    step = _llama_step_with_codes("cuda:0")
    out = [torch.empty_like(b.wq) for b in step.bufs]
    peak, kind = measured_peaks()
    r = measure_dequant(step, [b.packed for b in step.bufs], out, args.steps, args.warmup, peak)
    r["roofline"].update(peak_source=f"{kind} hbm_gbs", traffic=None)
    print(json.dumps({
        "metric": "packed-code dequantization Gweights/s", "op": "dequant",
        "value": r["Gweights_s"], "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"],
        "higher_is_better": True, "dtype": "u8->bf16", "data": "synthetic",
        "config": {"workload": "llama3_8b_linear_set_seq2_dequant",
                   "weights": step.weights, "launches_per_step": r["launches_per_call"]},
        "gpu_launches": r["launches_per_call"] * args.steps,
        "roofline": r["roofline"]}), flush=True)
    return 0


def run_bwd_adamw(args):
    """The backward fused with one AdamW step over every matrix of the
    Llama-3-8B-shaped set (one batched launch per step), 1 GPU; beside it,
    for context, the unfused sequence: the batched backward writing dW, then
    torch's fused AdamW over the same weights. Prints one JSON line."""
    import torch

    from bit_quantization_aware_b200 import inputs as I
    from bit_quantization_aware_b200 import pq
    from bit_quantization_aware_b200.step import QuantStep
    torch.cuda.set_device(0)
    step = QuantStep(I.llama3_8b_set(), pq.PQ_SEQ2, device="cuda:0")
    step.generate(seed=3)
    peak, kind = measured_peaks()
    r = measure_bwd_adamw(step, args.steps, args.warmup, peak)
    r["roofline"].update(peak_source=f"{kind} hbm_gbs", traffic=None)
    print(json.dumps({
        "metric": "backward + AdamW step Gweights/s", "op": "bwd_adamw",
        "value": r["Gweights_s"], "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"],
        "higher_is_better": True, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "llama3_8b_linear_set_seq2_bwd_adamw", "weights": step.weights,
                   "launches_per_step": r["launches_per_call"]},
        "gpu_launches": r["launches_per_call"] * args.steps,
        "roofline": r["roofline"], "unfused": r["unfused"]}), flush=True)
    return 0


def run_wq_gemm(args):
    """Weight-only 2-bit matmul for every matrix of the Llama-3-8B-shaped set
    (or four 16384x16384 weights, so that every replay reads its codes from
    HBM), X of --m rows, 1 GPU; beside it one launch per matrix and cuBLAS
    bf16 on the dequantized weights. Prints one JSON line."""
    import torch

    from bit_quantization_aware_b200 import inputs as I
    from bit_quantization_aware_b200 import pq
    from bit_quantization_aware_b200.step import QuantStep
    torch.cuda.set_device(0)
    if args.shape == "16384":
        mats = [I.Matrix(f"w{i}", 16384, 16384, i, 0) for i in range(4)]
        step = QuantStep(mats, pq.PQ_SEQ2, device="cuda:0", pack=True)
        step.generate(seed=3)
        step.fwd_all()
        torch.cuda.synchronize()
        workload = f"4x16384x16384_seq2_wq_gemm_m{args.m}"
    else:
        step = _llama_step_with_codes("cuda:0")
        workload = f"llama3_8b_linear_set_seq2_wq_gemm_m{args.m}"
    r = measure_wq_gemm(step.bufs, [b.packed for b in step.bufs], step.q, args.m, args.steps,
                        args.warmup, "cuda:0", with_single=True)
    r["roofline"]["traffic"] = None
    print(json.dumps({
        "metric": "weight-only 2-bit matmul Gweights/s", "op": "wq_gemm",
        "value": r["Gweights_s"], "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"],
        "higher_is_better": True, "dtype": r["dtype"], "data": "synthetic",
        "config": {"workload": workload, "m": args.m, "weights": step.weights,
                   "launches_per_step": r["launches_per_step"],
                   "matrices_per_launch": r["matrices_per_launch"],
                   "l2": f"codes {step.weights / 4e9:.2f} GB per step, larger than L2"},
        "roofline": r["roofline"],
        "gpu_launches": r["launches_per_step"] * args.steps,
        "tflops": r["tflops"],
        "per_matrix_launches": r["per_matrix_launches"],
        "cublas_bf16_dense": r["cublas_bf16_dense"]}), flush=True)
    return 0


def run_sharded(args):
    """The row-sharded step for ``--world`` ranks emulated on one GPU over
    the first ``--layers`` layers; prints one JSON line."""
    import torch
    torch.cuda.set_device(0)
    peak, kind = measured_peaks()
    r = measure_sharded(args.world, args.layers, args.steps, args.warmup, peak, "cuda:0")
    r["roofline"].update(peak_source=f"{kind} hbm_gbs", traffic=None)
    print(json.dumps({
        "metric": "row-sharded step (ranks emulated on one GPU) Gweights/s", "op": "sharded",
        "value": r["Gweights_s"], "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"],
        "higher_is_better": True, "dtype": "f32", "data": "synthetic",
        "config": {"workload": r["workload"], "weights": r["weights"], "world": r["world"],
                   "note": r["note"]},
        "roofline": r["roofline"], "phases": r["phases"],
        "gpu_launches": r["launches_total"]}), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "dequant":
        return run_dequant(args)
    if args.op == "bwd_adamw":
        return run_bwd_adamw(args)
    if args.op == "wq_gemm":
        return run_wq_gemm(args)
    if args.op == "sharded":
        return run_sharded(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
