"""Row-sharded step across two processes whose peer buffers are shared by
CUDA IPC (``IpcPeers``), both processes on the one GPU.

Each process is one rank: it owns a row shard of every matrix, exports its
packed-code, scale and gradient buffers, and maps the other rank's with
``pq_ipc_open``. The phases run through ``ShardedQuantStep.forward`` and
``backward`` with a device synchronise plus a gloo barrier as the barrier,
so the ranks' kernels never wait on one another. Checked against the
oracle: every rank's gathered bf16 weights (every element) and every
rank's shard after the reduce + backward + AdamW (weights and moments
bit-exact, d(alpha) within the parity tolerance).

Every rank takes the same barriers in the same order, also after an error
(it then skips its work but still waits), and unmaps and frees nothing
before both ranks have passed the last barrier with their kernels done."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

WORLD = 2
BARRIERS = 4  # forward, after the forward check, backward, after the backward check


def _mats():
    from bit_quantization_aware_b200 import inputs as I
    return [I.Matrix("q", 512, 1024, 0, 0), I.Matrix("odd", 1000, 264, 0, 1),
            I.Matrix("few", 3, 64, 0, 2), I.Matrix("down", 256, 2816, 0, 3)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, out):
    import torch.distributed as dist

    from bit_quantization_aware_b200 import inputs as I
    from bit_quantization_aware_b200 import pq
    from bit_quantization_aware_b200.sharded import IpcPeers, ShardedQuantStep
    from oracle import pq_oracle
    from oracle.pq_oracle import AdamW
    from tests.gpu_util import DALPHA_FLOOR, DALPHA_RTOL

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=timedelta(seconds=120))
    torch.cuda.set_device(0)
    res = {"rank": rank, "errors": [], "gathered": 0, "shards": 0}
    done = [0]

    def barrier():
        torch.cuda.synchronize()
        dist.barrier()
        done[0] += 1

    peers = st = None
    q, mats = pq.PQ_SEQ2, _mats()
    try:
        peers = IpcPeers()
        st = ShardedQuantStep(mats, q, rank, WORLD, peers, device="cuda:0")
        full = []
        for i, m in enumerate(mats):
            w = I.normal_weights(m.rows, m.cols, seed=90 + i, stream=0, device="cpu")
            a = I.alpha_init(w, q)
            full.append((w, a))
            st.load_full(i, w.cuda(), a.cuda())
        grads = [[I.grad_bf16(m.rows, m.cols, seed=95 + k, stream=64 + i, device="cpu")
                  for i, m in enumerate(mats)] for k in range(WORLD)]
        for i in range(len(mats)):
            st.g(i).copy_(grads[rank][i].cuda())
        st.forward(barrier)
        barrier()
        for i, (w, a) in enumerate(full):
            ref, _, _ = pq_oracle.fwd(q, w.numpy(), a.numpy())
            got = st.wq(i).view(torch.int16).cpu().numpy().view(np.uint16)
            if not np.array_equal(got, ref):
                res["errors"].append(f"gathered weights of matrix {i} differ")
            res["gathered"] += got.size
        hw, ha = pq.adamw(1, 2e-5), pq.adamw(1, 1e-4)
        st.backward(barrier, hw, ha)
        barrier()
        O = pq_oracle.default()
        for i, (w, a) in enumerate(full):
            m = mats[i]
            b, e = st.my_rows(i)
            if e == b:
                continue
            z = np.zeros((e - b, m.cols), np.float32)
            zr = np.zeros(e - b, np.float32)
            gs = pq.pq_default_grad_scale(q, m.cols)
            srcs = [grads[k][i][b:e].contiguous().view(torch.int16).numpy() for k in range(WORLD)]
            ref = O.reduce_bwd_adamw(q, w[b:e].numpy(), a[b:e].numpy(), srcs, 1.0 / WORLD,
                                     z, z, zr, zr, gs, AdamW.at_step(1, 2e-5),
                                     AdamW.at_step(1, 1e-4))
            s0, r0 = st.sh[i], st.full[i][1]
            n = (e - b) * m.cols
            got = [st.w_shard(i).cpu().numpy(), st.alpha_rows(i, b, e).cpu().numpy(),
                   st.m_w[s0:s0 + n].view(e - b, m.cols).cpu().numpy(),
                   st.v_w[s0:s0 + n].view(e - b, m.cols).cpu().numpy()]
            for name, x, y in zip(("w", "alpha", "m_w", "v_w"), got, ref[:4]):
                if not np.array_equal(x.view(np.uint32), y.view(np.uint32)):
                    res["errors"].append(f"{name} of matrix {i}, rows {b}..{e} differ")
            da = st.dalpha[r0 + b:r0 + e].cpu().numpy().astype(np.float64)
            tol = DALPHA_RTOL * np.maximum(np.abs(ref[6]).astype(np.float64),
                                           DALPHA_FLOOR * abs(gs) * ref[7])
            if not np.all(np.abs(da - ref[6]) <= tol):
                res["errors"].append(f"d(alpha) of matrix {i} out of tolerance")
            res["shards"] += 1
    except Exception as ex:  # recorded; the barriers below still run
        res["errors"].append(repr(ex))
    finally:
        while done[0] < BARRIERS:
            barrier()
        if peers is not None:
            peers.close()
        barrier()
        del st, peers
        dist.destroy_process_group()
    out.put(res)


def test_two_processes_share_buffers_by_ipc():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r["rank"])
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.exitcode is None:
                p.kill()
    for r in res:
        assert not r["errors"], r
    n = sum(m.numel for m in _mats())
    assert [r["gathered"] for r in res] == [n, n]
    assert sum(r["shards"] for r in res) >= len(_mats())
    for p in procs:
        assert p.exitcode == 0
