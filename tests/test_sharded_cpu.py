"""Host logic of the row-sharded step: row partitions and buffer layout
(no GPU), and a 2-rank gloo check that the ranks' shards cover every row of
every matrix exactly once."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from bit_quantization_aware_b200 import inputs as I
from bit_quantization_aware_b200.sharded import Layout, row_partition


@pytest.mark.parametrize("rows", [0, 1, 3, 7, 1000, 14336])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_row_partition(rows, world):
    parts = row_partition(rows, world)
    assert len(parts) == world and parts[0][0] == 0 and parts[-1][1] == rows
    for (b0, e0), (b1, e1) in zip(parts, parts[1:]):
        assert e0 == b1
    sizes = [e - b for b, e in parts]
    assert max(sizes) - min(sizes) <= 1


def test_layout_offsets_do_not_overlap():
    mats = I.llama_1b_stack()[:7] + [I.Matrix("odd", 1000, 264, 1, 0)]
    for world in (1, 2, 3, 4):
        for rank in range(world):
            L = Layout(tuple(mats), world, rank, 2)
            full, (ne, nr, npk) = L.full_offsets()
            for (e0, r0, p0), m, nxt in zip(full, mats, full[1:] + [(ne, nr, npk)]):
                assert e0 + m.numel <= nxt[0] and r0 + m.rows <= nxt[1]
                assert p0 + m.numel * 2 // 8 <= nxt[2]
                assert e0 % 64 == 0  # 16-byte aligned fp32/bf16 views
            sh, nsh = L.shard_offsets()
            ends = sh[1:] + [nsh]
            for s0, s1, m, part in zip(sh, ends, mats, L.parts):
                b, e = part[rank]
                assert s0 + (e - b) * m.cols <= s1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mats = I.llama_1b_stack()[:7] + [I.Matrix("odd", 1001, 264, 1, 0)]
        L = Layout(tuple(mats), world, rank, 2)
        mine = torch.tensor([[i, *L.parts[i][rank]] for i in range(len(mats))])
        allr = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(allr, mine)
        if rank == 0:
            cover = {}
            for t in allr:
                for i, b, e in t.tolist():
                    for r in range(b, e):
                        cover[(i, r)] = cover.get((i, r), 0) + 1
            ok = all(cover.get((i, r), 0) == 1 for i, m in enumerate(mats) for r in range(m.rows))
            out.put(ok and len(cover) == sum(m.rows for m in mats))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_cover_every_row_once():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    assert q.get(timeout=120) is True
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
