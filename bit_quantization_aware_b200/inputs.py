"""Seeded synthetic inputs for the weight fake-quantizer.

This module is shared by the tests, the smoke check and the benchmark: it
makes the same tensors for the CUDA library and for the CPU oracle. It holds
none of the quantizer's arithmetic (no division by alpha, no clipping, no
rounding to a level set); it only draws weights, upstream gradients and the
initial per-row scales, with the shapes and distributions of the workloads:

* shadow weights W: fp32, row-major [rows, cols], N(0, 0.02^2), or a
  heavy-tailed Student-t with 3 degrees of freedom times 0.02;
* upstream gradient dWq: bf16 [rows, cols], N(0, 1e-3^2) rounded to bf16;
* per-row scale alpha: fp32 [rows], max|w_row| (SEQ, ternary), mean|w_row|
  (binary), 2*mean|w_row|/sqrt(Qp) or max|w_row|/Qp (LSQ).

Random streams are torch generators seeded from (seed, stream id); the
stream id of layer l, projection p is 8*l + p and the gradient of the same
matrix uses stream id + 64. Generation runs on whatever device is asked for
(the big layer sets are drawn directly in HBM).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

# projection order inside one transformer layer
PROJ = ("q", "k", "v", "o", "gate", "up", "down")

# Quantizer identifiers of the library's C ABI (see include/pq.h).
BINARY, TERNARY, SEQ2, SEQ2_B, LSQ2, LSQ3, LSQ4 = 1, 2, 3, 4, 5, 6, 7
QUANT_NAMES = {BINARY: "binary", TERNARY: "ternary", SEQ2: "seq2",
               SEQ2_B: "seq2_b", LSQ2: "lsq2", LSQ3: "lsq3", LSQ4: "lsq4"}
# Q_p of the LSQ integer grids, used here only to initialise alpha.
_LSQ_QP = {LSQ2: 1.0, LSQ3: 3.0, LSQ4: 7.0}


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 7_919 + 12_345) % (1 << 63))
    return g


def normal_weights(rows, cols, *, seed=0, stream=0, std=0.02, device="cpu",
                   out=None):
    """fp32 [rows, cols] ~ N(0, std^2)."""
    g = _gen(device, seed, stream)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32, device=device)
    out.normal_(0.0, std, generator=g)
    return out


def student_t3_weights(rows, cols, *, seed=0, stream=0, scale=0.02,
                       device="cpu"):
    """fp32 [rows, cols] = scale * z / sqrt(chi2_3 / 3), chi2_3 the sum of
    three squared standard normals (Student-t, nu = 3)."""
    g = _gen(device, seed, stream)
    z = torch.randn((rows, cols), generator=g, device=device)
    chi = torch.zeros_like(z)
    for _ in range(3):
        n = torch.randn((rows, cols), generator=g, device=device)
        chi.addcmul_(n, n)
    z.div_(torch.sqrt(chi.div_(3.0)).clamp_min_(1e-30)).mul_(scale)
    return z


def grad_bf16(rows, cols, *, seed=0, stream=64, std=1e-3, device="cpu",
              out=None):
    """bf16 [rows, cols] ~ N(0, std^2) rounded to bf16."""
    g = _gen(device, seed, stream)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
    # draw in fp32 one row block at a time to bound the temporary
    step = max(1, (1 << 26) // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        tmp = torch.empty((r1 - r0, cols), dtype=torch.float32, device=device)
        tmp.normal_(0.0, std, generator=g)
        out[r0:r1].copy_(tmp)
    return out


def alpha_init(w: torch.Tensor, q: int, *, lsq_rule: str = "lsq") -> torch.Tensor:
    """Initial per-row scale (fp32 [rows]).

    SEQ2, SEQ2_B, ternary: max|w_row|. Binary: mean|w_row|. LSQ: the LSQ
    paper's 2*mean|w_row|/sqrt(Qp) (``lsq_rule="lsq"``) or max|w_row|/Qp
    (``lsq_rule="max"``).
    """
    if w.shape[1] == 0:  # empty rows: any positive scale
        return torch.ones(w.shape[0], dtype=torch.float32, device=w.device)
    a = w.abs()
    if q in (SEQ2, SEQ2_B, TERNARY):
        out = a.amax(dim=1)
    elif q == BINARY:
        out = a.mean(dim=1, dtype=torch.float64).float()
    elif q in _LSQ_QP:
        qp = _LSQ_QP[q]
        if lsq_rule == "lsq":
            out = (2.0 * a.mean(dim=1, dtype=torch.float64) / math.sqrt(qp)).float()
        else:
            out = (a.amax(dim=1).double() / qp).float()
    else:
        raise ValueError(f"unknown quantizer {q}")
    return out.clamp_min_(1e-30).contiguous()


def plant_boundaries(w: torch.Tensor, alpha: torch.Tensor, *, frac=0.01,
                     seed=0, stream=99):
    """Overwrite ``frac`` of the entries so that fl(w/alpha) lands exactly on
    chosen targets: half on the clip bounds +-0.99f, half on values that put
    the SEQ or ternary rounding argument exactly on a half-integer
    (x in {-0.5, 0, +0.5} and x = +-fl(1/3)). Each w is found by trying
    fl(target*alpha) and its neighbours up to 4 ulps away in fp32 and keeping
    the first whose fp32 quotient by alpha equals the target. Returns the
    number of entries planted and the number that hit their target."""
    rows, cols = w.shape
    dev = w.device
    g = _gen(dev, seed, stream)
    n = int(rows * cols * frac)
    if n == 0:
        return 0, 0
    flat_idx = torch.randint(0, rows * cols, (n,), generator=g, device=dev)
    kind = torch.randint(0, 2, (n,), generator=g, device=dev)
    clip_t = torch.tensor([-0.99, 0.99], dtype=torch.float32, device=dev)
    third = torch.tensor(1.0, dtype=torch.float32) / torch.tensor(3.0, dtype=torch.float32)
    tie_t = torch.tensor([-0.5, 0.0, 0.5, -third.item(), third.item()],
                         dtype=torch.float32, device=dev)
    pick_c = torch.randint(0, 2, (n,), generator=g, device=dev)
    pick_t = torch.randint(0, 5, (n,), generator=g, device=dev)
    target = torch.where(kind == 0, clip_t[pick_c], tie_t[pick_t])
    a = alpha[flat_idx // cols]
    base = target * a
    best = base.clone()
    found = torch.zeros(n, dtype=torch.bool, device=dev)
    up = torch.full_like(base, float("inf"))
    down = torch.full_like(base, float("-inf"))
    cand_up = base.clone()
    cand_dn = base.clone()
    for k in range(0, 5):
        for cand in ((cand_up,) if k == 0 else (cand_up, cand_dn)):
            ok = (~found) & ((cand / a) == target)
            best = torch.where(ok, cand, best)
            found |= ok
        cand_up = torch.nextafter(cand_up, up)
        cand_dn = torch.nextafter(cand_dn, down)
    wf = w.view(-1)
    wf[flat_idx] = best
    return n, int(found.sum().item())


@dataclass(frozen=True)
class Matrix:
    name: str
    rows: int
    cols: int
    layer: int
    proj: int

    @property
    def numel(self) -> int:
        return self.rows * self.cols


def layer_set(n_layers: int, hidden: int, kv: int, ffn: int, prefix: str):
    """The seven linear weights of each layer: q/o hidden x hidden, k/v
    kv x hidden, gate/up ffn x hidden, down hidden x ffn (rows = output
    features)."""
    shapes = {"q": (hidden, hidden), "k": (kv, hidden), "v": (kv, hidden),
              "o": (hidden, hidden), "gate": (ffn, hidden),
              "up": (ffn, hidden), "down": (hidden, ffn)}
    mats = []
    for l in range(n_layers):
        for p, name in enumerate(PROJ):
            r, c = shapes[name]
            mats.append(Matrix(f"{prefix}.{l}.{name}", r, c, l, p))
    return mats


def llama3_8b_set():
    """Llama-3-8B-shaped linear set: 32 layers, q/o 4096x4096, k/v 1024x4096,
    gate/up 14336x4096, down 4096x14336."""
    return layer_set(32, 4096, 1024, 14336, "llama3_8b")


def llama_1b_stack():
    """1B-class stack: 24 layers, q/o 2048x2048, k/v 512x2048, gate/up
    5632x2048, down 2048x5632."""
    return layer_set(24, 2048, 512, 5632, "llama_1b")


def total_weights(mats) -> int:
    return sum(m.numel for m in mats)
