"""Row-sharded quantizer step with several GPUs emulated on one device.

The ranks' buffer sets live on one GPU and their phases run in stream order
(no kernel waits on another). Each rank's gathered bf16 weights must equal
the unsharded forward, and each rank's updated shard must equal the
unsharded reduce + backward + AdamW over the same replicas' gradients."""
import numpy as np
import pytest
import torch

from bit_quantization_aware_b200 import inputs as I
from bit_quantization_aware_b200 import pq
from bit_quantization_aware_b200.sharded import LocalPeers, ShardedQuantStep
from oracle import pq_oracle
from oracle.pq_oracle import AdamW
from tests.gpu_util import DALPHA_FLOOR, DALPHA_RTOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _mats():
    return I.llama_1b_stack()[:7] + [I.Matrix("odd", 1000, 264, 1, 0), I.Matrix("few", 3, 64, 1, 1)]


@pytest.mark.parametrize("q", [pq.PQ_SEQ2, pq.PQ_LSQ4, pq.PQ_TERNARY])
@pytest.mark.parametrize("world", [1, 2, 3])
def test_sharded_step_equals_unsharded(q, world):
    mats = _mats()
    peers = LocalPeers(world)
    ranks = [ShardedQuantStep(mats, q, k, world, peers, device=DEV) for k in range(world)]
    full = []
    for i, m in enumerate(mats):
        w = I.normal_weights(m.rows, m.cols, seed=70 + i, stream=0, device=DEV)
        a = I.alpha_init(w, q)
        full.append((w, a))
        for r in ranks:
            r.load_full(i, w, a)
    # forward: every rank packs its rows, then every rank gathers + decodes
    for r in ranks:
        r.pack_shards()
    for r in ranks:
        r.gather_dequant()
    torch.cuda.synchronize()
    for i, (w, a) in enumerate(full):
        ref, _ = pq.fakequant_fwd(q, w, a)
        rb = ref.view(torch.int16)
        zero = (rb & 0x7FFF) == 0  # codes do not keep the sign of a zero level
        for r in ranks:
            got = r.wq(i).view(torch.int16)
            assert torch.equal(got[~zero], rb[~zero]), (i, r.rank)
            assert torch.all(got[zero] == 0)
    # backward: each replica has its own gradient of every matrix
    for k, r in enumerate(ranks):
        for i, m in enumerate(mats):
            r.g(i).copy_(I.grad_bf16(m.rows, m.cols, seed=80 + k, stream=64 + i, device=DEV))
    hw, ha = pq.adamw(1, 2e-5, weight_decay=0.01), pq.adamw(1, 1e-4)
    for r in ranks:
        r.reduce_step(hw, ha)
    torch.cuda.synchronize()
    # unsharded reference: the whole matrix as one shard, same sources
    for i, (w, a) in enumerate(full):
        m = mats[i]
        wr, ar = w.clone(), a.clone()
        mw, vw = torch.zeros_like(wr), torch.zeros_like(wr)
        ma, va, da = torch.zeros_like(ar), torch.zeros_like(ar), torch.zeros_like(ar)
        e0 = ranks[0].full[i][0]
        sh = pq.shard_array([dict(rows=m.rows, cols=m.cols, w=wr, alpha=ar, m_w=mw, v_w=vw,
                                  m_alpha=ma, v_alpha=va, dalpha=da, g_offset=e0,
                                  grad_scale=pq.pq_default_grad_scale(q, m.cols))])
        pq.pq_reduce_bwd_adamw(q, [r.g_full for r in ranks], 1.0 / world, sh, hw, ha)
        torch.cuda.synchronize()
        for r in ranks:
            b, e = r.my_rows(i)
            assert torch.equal(r.w_shard(i).view(torch.int32), wr[b:e].view(torch.int32)), (i, r.rank)
            assert torch.equal(r.alpha_rows(i, b, e).view(torch.int32), ar[b:e].view(torch.int32))
            r0 = r.full[i][1]
            assert torch.equal(r.m_a[r0 + b:r0 + e].view(torch.int32), ma[b:e].view(torch.int32))
            s0 = r.sh[i]
            assert torch.equal(r.m_w[s0:s0 + (e - b) * m.cols].view(torch.int32),
                               mw[b:e].reshape(-1).view(torch.int32))


@pytest.mark.parametrize("q", [pq.PQ_SEQ2, pq.PQ_BINARY])
def test_reduce_bwd_adamw_matches_oracle(q):
    """pq_reduce_bwd_adamw with 3 gradient sources against the oracle:
    weights and moments bit-exact; d(alpha) within tolerance and alpha's
    own step exact given the GPU's d(alpha)."""
    rows, cols = 37, 1032
    w = I.normal_weights(rows, cols, seed=90, stream=0, device="cpu")
    a = I.alpha_init(w, q) * 0.8
    gs = [I.grad_bf16(rows, cols, seed=91 + k, stream=64, device="cpu") for k in range(3)]
    hw_o, ha_o = AdamW.at_step(4, 2e-5), AdamW.at_step(4, 1e-4)
    rng = np.random.default_rng(92)
    mw = rng.normal(0, 1e-4, (rows, cols)).astype(np.float32)
    vw = np.abs(rng.normal(0, 1e-7, (rows, cols))).astype(np.float32)
    ma = rng.normal(0, 1e-3, rows).astype(np.float32)
    va = np.abs(rng.normal(0, 1e-6, rows)).astype(np.float32)
    gsc = pq.pq_default_grad_scale(q, cols)
    ref = pq_oracle.default().reduce_bwd_adamw(
        q, w.numpy(), a.numpy(), [g.view(torch.int16).numpy() for g in gs], 1 / 3,
        mw, vw, ma, va, gsc, hw_o, ha_o)
    wd, ad = w.to(DEV), a.to(DEV)
    mwd, vwd = torch.from_numpy(mw).to(DEV), torch.from_numpy(vw).to(DEV)
    mad, vad = torch.from_numpy(ma).to(DEV), torch.from_numpy(va).to(DEV)
    dad = torch.zeros(rows, device=DEV)
    srcs = [g.to(DEV) for g in gs]
    sh = pq.shard_array([dict(rows=rows, cols=cols, w=wd, alpha=ad, m_w=mwd, v_w=vwd,
                              m_alpha=mad, v_alpha=vad, dalpha=dad, g_offset=0, grad_scale=gsc)])
    pq.pq_reduce_bwd_adamw(q, srcs, 1 / 3, sh, pq.adamw(4, 2e-5), pq.adamw(4, 1e-4))
    torch.cuda.synchronize()
    for x, y in ((wd, ref[0]), (mwd, ref[2]), (vwd, ref[3])):
        assert np.array_equal(x.cpu().numpy().view(np.uint32), y.view(np.uint32))
    da = dad.cpu().numpy()
    # the d(alpha) tolerance of every parity test: 1e-4 relative, floored at
    # 1e-6 of the row's sum of |terms| times grad_scale
    tol = DALPHA_RTOL * np.maximum(np.abs(ref[6]).astype(np.float64),
                                   DALPHA_FLOOR * abs(gsc) * ref[7])
    assert np.all(np.abs(da.astype(np.float64) - ref[6].astype(np.float64)) <= tol)
    pa, pma, pva = pq_oracle.default().adamw_step(a.numpy(), da, ma, va, ha_o)
    assert np.array_equal(ad.cpu().numpy().view(np.uint32), pa.view(np.uint32))
