"""The element-wise parity checker used by the full-size GPU tests, run on
the CPU with the oracle's own outputs standing in for the GPU's: it accepts
them, and it reports a single changed bit in any output kind."""
from concurrent.futures import ThreadPoolExecutor
from types import SimpleNamespace

import numpy as np
import pytest
import torch

from bit_quantization_aware_b200 import inputs as I
from oracle import pq_oracle
from tests.gpu_util import check_step_every_element


def _fake_step(q, shapes, pack):
    bufs = []
    for i, (rows, cols) in enumerate(shapes):
        m = I.Matrix(f"m{i}", rows, cols, 0, i)
        w = I.normal_weights(rows, cols, seed=9, stream=i, device="cpu")
        a = I.alpha_init(w, q)
        g = I.grad_bf16(rows, cols, seed=9, stream=64 + i, device="cpu")
        gn = g.view(torch.int16).numpy().view(np.uint16)
        gs = pq_oracle.default_grad_scale(q, cols)
        wq, _, pk = pq_oracle.fwd(q, w.numpy(), a.numpy(), pack=pack)
        dw, da, _ = pq_oracle.bwd(q, w.numpy(), a.numpy(), gn, gs)
        bufs.append(SimpleNamespace(
            m=m, w=w, alpha=a, g=g, grad_scale=gs,
            wq=torch.from_numpy(wq.view(np.int16)).view(torch.bfloat16),
            packed=torch.from_numpy(pk) if pack else None,
            dw=torch.from_numpy(dw), dalpha=torch.from_numpy(da)))
    return SimpleNamespace(q=q, bufs=bufs)


@pytest.fixture(scope="module")
def pool():
    with ThreadPoolExecutor(4) as ex:
        yield ex


SHAPES = [(37, 64), (5, 1000), (300, 16)]


def test_accepts_the_oracles_outputs(pool):
    step = _fake_step(pq_oracle.SEQ2, SHAPES, pack=True)
    n = check_step_every_element(step, pool, task_weights=4096)
    assert n == sum(r * c for r, c in SHAPES)


@pytest.mark.parametrize("what", ["wq", "packed", "dw", "dalpha"])
def test_reports_one_changed_value(pool, what):
    step = _fake_step(pq_oracle.TERNARY, SHAPES, pack=True)
    b = step.bufs[2]
    t = getattr(b, what)
    if what == "wq":
        t.view(torch.int16)[299, 15] ^= 1
    elif what == "packed":
        t[123, 3] ^= 0x40
    elif what == "dw":
        t.view(torch.int32)[7, 9] ^= 1
    else:
        t[211] *= 1.01
    with pytest.raises(AssertionError, match="m2 rows from"):
        check_step_every_element(step, pool, task_weights=4096)
