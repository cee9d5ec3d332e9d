"""Phase ordering of the row-sharded step with two processes (gloo, CPU).

The ranks' peer buffers are file-backed shared CPU tensors, and the library
is replaced by a host stand-in that keeps only the data movement of each
phase (no quantizer arithmetic): the pack writes each owned row's global
row number into that row's codes, the gather-dequantize copies every
rank's code rows into this rank's full weights, and the reduce writes the
fp32 sum of every replica's gradient rows over this rank's shard. With
``forward``/``backward`` (pack -> barrier -> gather; gradient -> barrier
-> reduce) every rank sees every other rank's writes; a run that gathers
before a peer has packed sees that peer's rows still zero, which shows the
check can tell the orders apart."""
import os
import socket
import tempfile

import pytest
import torch
import torch.multiprocessing as mp

from bit_quantization_aware_b200 import inputs as I
from bit_quantization_aware_b200.sharded import ShardedQuantStep


class HostLib:
    """Stand-in for the library binding: descriptors stay dicts, each call
    runs at once on the CPU."""

    @staticmethod
    def pq_code_bits(q):
        return 2

    @staticmethod
    def pq_default_grad_scale(q, cols):
        return 1.0

    @staticmethod
    def matrix_array(descs):
        return list(descs)

    shard_array = matrix_array

    @staticmethod
    def pq_fakequant_fwd_batch(q, descs, stream=None):
        for d in descs:
            r, c = d["rows"], d["cols"]
            w = d["w"].view(r, c)
            d["packed"].view(r, c // 4)[:] = (w[:, :1].long() % 256).to(torch.uint8)

    @staticmethod
    def pq_dequant_codes_batch(q, descs, stream=None):
        for d in descs:
            r, c = d["rows"], d["cols"]
            d["wq"].view(r, c)[:] = d["packed"].view(r, c // 4)[:, :1].float()

    @staticmethod
    def pq_reduce_bwd_adamw(q, sources, mult, shards, hp_w, hp_a, stream=None):
        for s in shards:
            n = s["rows"] * s["cols"]
            o = s["g_offset"]
            acc = torch.zeros(n, dtype=torch.float32)
            for src in sources:
                acc += src[o:o + n].float()
            s["w"].view(-1)[:] = acc * mult


class ShmPeers:
    """Every rank's buffer is a file under a directory both processes see,
    mapped shared; a rank reads another rank's buffer through its file."""

    def __init__(self, root, rank):
        self.root, self.rank = root, rank

    def _path(self, rank, name):
        return os.path.join(self.root, f"{rank}.{name}")

    def allocate(self, rank, name, numel, dtype, device):
        nbytes = numel * torch.empty((), dtype=dtype).element_size()
        with open(self._path(rank, name), "wb") as f:
            f.truncate(nbytes)
        return self.get(rank, name)

    def get(self, rank, name):
        nbytes = os.path.getsize(self._path(rank, name))
        t = torch.from_file(self._path(rank, name), shared=True, size=nbytes, dtype=torch.uint8)
        return t if name == "packed" else t.view({"alpha": torch.float32,
                                                  "g": torch.bfloat16}[name])


MATS = [I.Matrix("a", 37, 64, 0, 0), I.Matrix("b", 5, 16, 0, 1), I.Matrix("c", 130, 8, 0, 2)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, root, ordered, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        peers = ShmPeers(root, rank)
        # every rank allocates its files before any rank opens a peer's
        st = ShardedQuantStep(MATS, 3, rank, world, peers, device="cpu", lib=HostLib)
        dist.barrier()
        for i, m in enumerate(MATS):
            rows = torch.arange(1, m.rows + 1, dtype=torch.float32)
            st.load_full(i, rows[:, None].expand(m.rows, m.cols).contiguous(),
                         torch.ones(m.rows))
            # replica k's gradient: (k + 1) * (row % 7 + 1), exact in bf16
            g = (rank + 1) * (torch.arange(m.rows) % 7 + 1).float()
            st.g(i).copy_(g[:, None].expand(m.rows, m.cols))
        if ordered:
            st.forward(dist.barrier)
            st.backward(dist.barrier, None, None)
        else:
            # the gather of rank 0 runs before rank 1 has packed
            if rank == 0:
                st.pack_shards()
                st.gather_dequant()
                dist.barrier()
            else:
                dist.barrier()
                st.pack_shards()
                st.gather_dequant()
        dist.barrier()
        gathered = all(torch.equal(st.wq(i).float(),
                                   (torch.arange(1, m.rows + 1).float() % 256)[:, None]
                                   .expand(m.rows, m.cols))
                       for i, m in enumerate(MATS))
        reduced = True
        if ordered:
            for i, m in enumerate(MATS):
                b, e = st.my_rows(i)
                want = sum(k + 1 for k in range(world)) / world * \
                    (torch.arange(b, e) % 7 + 1).float()
                reduced &= torch.equal(st.w_shard(i), want[:, None].expand(e - b, m.cols))
        out.put((rank, gathered, reduced))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(ordered):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    with tempfile.TemporaryDirectory() as root:
        procs = [ctx.Process(target=_worker, args=(r, 2, port, root, ordered, q))
                 for r in range(2)]
        for p in procs:
            p.start()
        res = sorted(q.get(timeout=120) for _ in procs)
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    return res


def test_forward_backward_order_every_write_is_seen():
    assert _run(ordered=True) == [(0, True, True), (1, True, True)]


def test_gather_before_a_peer_packs_sees_zeros():
    res = dict((r, g) for r, g, _ in _run(ordered=False))
    assert res[0] is False and res[1] is True
