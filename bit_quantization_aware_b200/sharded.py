"""Row-sharded (owner-computes) quantizer step across data-parallel GPUs.

Every GPU owns a contiguous row shard of each weight matrix: the shard's
fp32 shadow weights, its per-row scales and the AdamW moments. One training
step, per GPU:

1. ``pack_shards``: quantize the owned rows to packed codes (0.25 B/weight
   at 2 bits), written into this GPU's copy of a buffer that every GPU can
   read (the owned rows only).
2. after every GPU's pack is complete (the caller orders it, e.g. a barrier
   or collective on the stream), ``gather_dequant``: one batched
   dequantization whose descriptors point at every GPU's packed shard and
   scale shard, so the codes cross NVLink (8x fewer bytes than bf16 weights)
   and are decoded straight into this GPU's full bf16 weights. The
   all-gather is fused into the dequantization kernel: there is no gathered
   copy of the codes.
3. the model's matmuls write this GPU's full upstream gradient dWq (bf16)
   into a readable buffer; after every GPU's gradient is complete,
   ``reduce_step``: each GPU sums every replica's gradient rows of the
   shards it owns (fp32, fixed replica order, times 1/world) and applies
   the STE backward, d(alpha) and AdamW to them, in one kernel
   (the reduce-scatter is fused into the backward).

Ordering: ``forward`` and ``backward`` put the caller's barrier between the
phases (pack -> barrier -> gather; the model writes the gradient ->
barrier -> reduce). Two barriers per step suffice when the barrier is a
stream-ordered collective (or a device synchronise plus a host barrier):
a rank passes the forward barrier of step t+1 only after every rank's
reduce of step t is done, and the backward barrier only after every
rank's gather is done, so no phase overwrites a buffer a peer still reads.

Peer buffers come from a provider: ``IpcPeers`` (CUDA IPC across
processes, one GPU each; point-to-point mappings, no multicast object) or
``LocalPeers`` (several buffer sets on one GPU standing in for GPUs, for
tests). The arithmetic runs in the CUDA library (``pq``); this module only
lays out buffers and descriptors.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import pq


def row_partition(rows: int, world: int):
    """Contiguous near-equal row ranges [(begin, end)] for ranks 0..world-1
    (the first rows % world ranks get one extra row)."""
    base, extra = divmod(rows, world)
    out, b = [], 0
    for k in range(world):
        e = b + base + (1 if k < extra else 0)
        out.append((b, e))
        b = e
    return out


def _align(n: int, a: int = 64) -> int:
    return (n + a - 1) // a * a


@dataclass(frozen=True)
class Layout:
    """Offsets of every matrix in the full-size buffers (identical on every
    GPU) and of this rank's shards in its local shard buffers."""
    mats: tuple
    world: int
    rank: int
    bits: int

    @property
    def parts(self):
        return [row_partition(m.rows, self.world) for m in self.mats]

    def full_offsets(self):
        """(elements, rows, packed bytes) offsets of each matrix and totals."""
        e, r, p, out = 0, 0, 0, []
        for m in self.mats:
            out.append((e, r, p))
            e += _align(m.numel)
            r += _align(m.rows)
            p += _align(m.numel * self.bits // 8)
        return out, (e, r, p)

    def shard_offsets(self):
        """Element offset of this rank's shard of each matrix in the local
        shard buffers, and the total."""
        e, out = 0, []
        for m, part in zip(self.mats, self.parts):
            b, en = part[self.rank]
            out.append(e)
            e += _align((en - b) * m.cols)
        return out, e


class LocalPeers:
    """Stand-in for several GPUs on one device: every rank's buffers are
    ordinary local tensors, and a rank reads another rank's copy directly."""

    def __init__(self, world: int):
        self.world = world
        self.bufs = [dict() for _ in range(world)]

    def allocate(self, rank, name, numel, dtype, device):
        t = torch.zeros(numel, dtype=dtype, device=device)
        self.bufs[rank][name] = t
        return t

    def get(self, rank, name):
        return self.bufs[rank][name]


class PeerSpan:
    """A contiguous 1-D range of another process's device memory, mapped by
    CUDA IPC, typed like a tensor of ``dtype``. Slicing gives a sub-range;
    the library's kernels take it wherever they take a device tensor. It is
    never a torch tensor, so nothing reads or copies it on the host."""

    is_cuda = True

    def __init__(self, ptr: int, numel: int, dtype):
        self.ptr, self.n, self.dtype = int(ptr), int(numel), dtype
        self.itemsize = torch.empty((), dtype=dtype).element_size()

    def data_ptr(self) -> int:
        return self.ptr

    def numel(self) -> int:
        return self.n

    def is_contiguous(self) -> bool:
        return True

    def __getitem__(self, s):
        if not isinstance(s, slice) or s.step not in (None, 1):
            raise TypeError("a peer range takes contiguous slices only")
        b, e, _ = s.indices(self.n)
        return PeerSpan(self.ptr + b * self.itemsize, max(0, e - b), self.dtype)


class IpcPeers:
    """Peer buffers for one process per GPU, shared by CUDA IPC: each rank
    allocates its buffer as an ordinary device tensor, the ranks exchange
    the IPC handle of the allocation holding it and the buffer's offset (an
    all-gather of small host objects over the process group), and every
    rank maps the others' allocations with ``pq.ipc_open`` (once per
    allocation). These are point-to-point peer mappings over NVLink: no
    NVLink multicast object is created, so no rank's memory is bound to one.

    Lifetime: a rank's tensors must outlive every other rank's reads. Call
    ``close`` on every rank after the last kernel that reads a peer buffer
    has completed on every rank (synchronise, then a barrier); it unmaps the
    peers' allocations. Only then may the owners free their tensors."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.local = {}
        self.views = {}
        self.mapped = {}  # handle bytes -> base address in this process

    def allocate(self, rank, name, numel, dtype, device):
        assert rank == self.rank
        t = torch.zeros(numel, dtype=dtype, device=device)
        handle, offset = pq.ipc_export(t)
        info = [None] * self.world
        self.dist.all_gather_object(info, (handle, offset, numel), group=self.group)
        views = []
        for k, (h, off, n) in enumerate(info):
            if k == self.rank:
                views.append(t)
                continue
            if h not in self.mapped:
                self.mapped[h] = pq.ipc_open(h)
            views.append(PeerSpan(self.mapped[h] + off, n, dtype))
        self.local[name] = t
        self.views[name] = views
        return t

    def get(self, rank, name):
        return self.views[name][rank]

    def close(self):
        for base in self.mapped.values():
            pq.ipc_close(base)
        self.mapped.clear()
        self.views.clear()


class ShardedQuantStep:
    """One GPU's part of the row-sharded quantizer step over ``mats``."""

    def __init__(self, mats, q: int, rank: int, world: int, peers, device="cuda", lib=pq):
        self.q, self.rank, self.world, self.peers = q, rank, world, peers
        self.lib = lib  # the library binding (a stand-in in host-only tests)
        self.device = torch.device(device)
        self.bits = lib.pq_code_bits(q)
        self.layout = Layout(tuple(mats), world, rank, self.bits)
        self.mats = list(mats)
        full, (ne, nr, npk) = self.layout.full_offsets()
        sh, nsh = self.layout.shard_offsets()
        self.full, self.sh = full, sh
        dev = self.device
        # readable by every GPU: codes, scales (owned rows), gradients
        self.packed_full = peers.allocate(rank, "packed", npk, torch.uint8, dev)
        self.alpha_full = peers.allocate(rank, "alpha", nr, torch.float32, dev)
        self.g_full = peers.allocate(rank, "g", ne, torch.bfloat16, dev)
        # local
        self.wq_full = torch.zeros(ne, dtype=torch.bfloat16, device=dev)
        self.w_sh = torch.zeros(nsh, dtype=torch.float32, device=dev)
        self.m_w = torch.zeros(nsh, dtype=torch.float32, device=dev)
        self.v_w = torch.zeros(nsh, dtype=torch.float32, device=dev)
        self.m_a = torch.zeros(nr, dtype=torch.float32, device=dev)
        self.v_a = torch.zeros(nr, dtype=torch.float32, device=dev)
        self.dalpha = torch.zeros(nr, dtype=torch.float32, device=dev)

    # ---------------------------------------------------------- views
    def my_rows(self, i):
        return self.layout.parts[i][self.rank]

    def w_shard(self, i):
        m, (b, e) = self.mats[i], self.my_rows(i)
        return self.w_sh[self.sh[i]:self.sh[i] + (e - b) * m.cols].view(e - b, m.cols)

    def alpha_rows(self, i, b, e, rank=None):
        src = self.alpha_full if rank is None else self.peers.get(rank, "alpha")
        r0 = self.full[i][1]
        return src[r0 + b:r0 + e]

    def wq(self, i):
        m = self.mats[i]
        e0 = self.full[i][0]
        return self.wq_full[e0:e0 + m.numel].view(m.rows, m.cols)

    def g(self, i):
        m = self.mats[i]
        e0 = self.full[i][0]
        return self.g_full[e0:e0 + m.numel].view(m.rows, m.cols)

    def load_full(self, i, w_full, alpha_full):
        """Take this rank's rows of a full matrix and its scales."""
        b, e = self.my_rows(i)
        self.w_shard(i).copy_(w_full[b:e])
        self.alpha_rows(i, b, e).copy_(alpha_full[b:e])

    # ---------------------------------------------------------- phases
    def pack_shards(self, stream=None):
        descs = []
        for i, m in enumerate(self.mats):
            b, e = self.my_rows(i)
            p0 = self.full[i][2] + b * m.cols * self.bits // 8
            descs.append(dict(rows=e - b, cols=m.cols, w=self.w_shard(i),
                              alpha=self.alpha_rows(i, b, e),
                              packed=self.packed_full[p0:p0 + (e - b) * m.cols * self.bits // 8]))
        self.lib.pq_fakequant_fwd_batch(self.q, self.lib.matrix_array(descs), stream)

    def gather_dequant(self, stream=None):
        descs = []
        for i, m in enumerate(self.mats):
            e0, r0, p0 = self.full[i]
            for k, (b, e) in enumerate(self.layout.parts[i]):
                if e == b:
                    continue
                pk = self.peers.get(k, "packed")
                pb = p0 + b * m.cols * self.bits // 8
                descs.append(dict(rows=e - b, cols=m.cols,
                                  packed=pk[pb:pb + (e - b) * m.cols * self.bits // 8],
                                  alpha=self.alpha_rows(i, b, e, rank=k),
                                  wq=self.wq_full[e0 + b * m.cols:e0 + e * m.cols]))
        self.lib.pq_dequant_codes_batch(self.q, self.lib.matrix_array(descs), stream)

    def reduce_step(self, hp_w, hp_alpha, grad_mult=None, stream=None):
        sources = [self.peers.get(k, "g") for k in range(self.world)]
        shards = []
        for i, m in enumerate(self.mats):
            b, e = self.my_rows(i)
            if e == b:
                continue
            e0, r0, _ = self.full[i]
            s0 = self.sh[i]
            n = (e - b) * m.cols
            shards.append(dict(rows=e - b, cols=m.cols, w=self.w_shard(i),
                               alpha=self.alpha_rows(i, b, e),
                               m_w=self.m_w[s0:s0 + n], v_w=self.v_w[s0:s0 + n],
                               m_alpha=self.m_a[r0 + b:r0 + e], v_alpha=self.v_a[r0 + b:r0 + e],
                               dalpha=self.dalpha[r0 + b:r0 + e], g_offset=e0 + b * m.cols,
                               grad_scale=self.lib.pq_default_grad_scale(self.q, m.cols)))
        mult = 1.0 / self.world if grad_mult is None else grad_mult
        self.lib.pq_reduce_bwd_adamw(self.q, sources, mult, self.lib.shard_array(shards), hp_w,
                                     hp_alpha, stream)

    # ---------------------------------------------------------- one step
    def forward(self, barrier, stream=None):
        """Forward of one step: pack the owned rows, wait at ``barrier``
        until every rank's codes are written, then gather + dequantize all
        rows into this rank's bf16 weights."""
        self.pack_shards(stream)
        barrier()
        self.gather_dequant(stream)

    def backward(self, barrier, hp_w, hp_alpha, grad_mult=None, stream=None):
        """Backward of one step, after the model wrote this rank's full
        upstream gradient into ``g``: wait at ``barrier`` until every
        rank's gradient is written, then reduce + backward + AdamW on the
        owned shards."""
        barrier()
        self.reduce_step(hp_w, hp_alpha, grad_mult, stream)
