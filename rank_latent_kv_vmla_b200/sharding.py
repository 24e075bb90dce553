"""One sequence on several GPUs, one process per GPU: the query rows of each chunk are sharded across
the ranks and every rank keeps a full replica of the layer's latent cache (VideoMLA technical summary,
Problem definition: one fixed-size sliding window per sequence; the latent cache is small, 448 bytes
per token at the Wan shapes, so replicating it is cheap).

Per chunk, rank r
  1. compresses its token range of the chunk and stores the rows into every replica: its own and,
     through peer mappings, every other rank's (vmla_compress_append_rows; the exchange of the new
     latents rides on the compress kernel's stores, no separate all-gather);
  2. waits, on the stream that carries the kernels, until every rank's rows are in place (a one-element
     all-reduce: it completes only after every rank's compress kernel has completed);
  3. advances frames_written of its replica records and attends with its own query rows
     (vmla_latent_attention_fused_rows); attention itself needs no exchange;
  4. waits, again on the kernels' stream, until every rank's attention of this chunk has completed
     (a second one-element all-reduce) before its next compress may start.

Step 4 closes a write-after-read race between ranks: once the window is full, the next chunk's frames
go to the ring slots of the oldest frames, and those frames are still inside this chunk's window.  A
rank's compress writes into every replica, so without step 4 a rank that finished its attention early
could overwrite rows that a slower rank's attention still reads.  With it, a replica is only ever
written while no rank reads it: the compress of chunk k+1 on any rank is ordered after the attention of
chunk k on every rank, and the attention of chunk k after the compress of chunk k on every rank.

The communicator and the device operations are injectable (``comm``, ``ops``), so the protocol is
exercised by multi-process CPU tests with stand-ins; on GPUs ``TorchComm`` (NCCL) and the library are
used.  With one rank this is an ordinary layer step.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple


def token_shards(n_tokens: int, world: int, align: int = 128) -> List[Tuple[int, int]]:
    """Contiguous (begin, count) token ranges of a chunk, one per rank, split at multiples of ``align``
    (128 = one attention tile) and balanced to within one unit: the last ranks take the extra units,
    so the partial last unit sits with a rank that has one more unit than the others; ranks left
    without a unit get (begin, 0)."""
    if n_tokens < 0 or world < 1 or align < 1:
        raise ValueError("n_tokens >= 0, world >= 1, align >= 1 required")
    units = -(-n_tokens // align)
    base, extra = divmod(units, world)
    out, begin = [], 0
    for r in range(world):
        u = base + (1 if r >= world - extra else 0)
        count = max(0, min(u * align, n_tokens - begin))
        out.append((begin, count))
        begin += count
    return out


class TorchComm:
    """torch.distributed: object all-gather for the handle exchange, a one-element all-reduce on the
    current stream as the device-side barrier, and a host barrier."""

    def __init__(self, group=None, device=None):
        import torch
        import torch.distributed as dist
        self._dist, self._group = dist, group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self._flag = torch.zeros(1, dtype=torch.float32, device=device) if self.world > 1 else None

    def all_gather_object(self, obj) -> list:
        if self.world == 1:
            return [obj]
        out = [None] * self.world
        self._dist.all_gather_object(out, obj, group=self._group)
        return out

    def device_barrier(self) -> None:
        if self.world > 1:
            self._dist.all_reduce(self._flag, group=self._group)

    def barrier(self) -> None:
        if self.world > 1:
            self._dist.barrier(group=self._group)


class ShardedLayer:
    """One layer of one (or a batch of) sequence(s) whose chunk query rows are split across ranks."""

    def __init__(self, cfg, batch: int, comm, device=None, ops=None, align: int = 128):
        if ops is None:
            from . import vmla as ops
        self.cfg, self.batch, self.comm, self.ops = cfg, batch, comm, ops
        self.rank, self.world = comm.rank, comm.world
        self.cache = ops.LatentCache(cfg, batch, device=device)
        own = (ops.ipc_export(self.cache.c), ops.ipc_export(self.cache.k_r)) if self.world > 1 else None
        handles = comm.all_gather_object(own)
        self._imported: List[int] = []
        self.replicas = []
        for r in range(self.world):
            if r == self.rank:
                c, k = self.cache.c.data_ptr(), self.cache.k_r.data_ptr()
            else:
                c, k = ops.ipc_import(handles[r][0]), ops.ipc_import(handles[r][1])
                self._imported += [c, k]
            self.replicas.append(ops.CCache(c, k, batch, 0, self.cache.frames_written))
        self.shards = token_shards(cfg.chunk_tokens, self.world, align)
        self.begin, self.count = self.shards[self.rank]

    @property
    def frames_written(self) -> int:
        return self.cache.frames_written

    def step(self, x_rows, q_nope_rows, q_rope_rows, w_dkv_kr, w_uk, w_uv, out=None):
        """One streaming step: this rank's rows of the chunk (x_rows [B, count, D], q rows [B, count, H, *])
        in, this rank's output rows [B, count, H, d_v] out (None when the rank holds no rows)."""
        cfg, ops = self.cfg, self.ops
        f0 = self.cache.frames_written
        if self.count:
            ops.compress_append_rows(cfg, x_rows, w_dkv_kr, f0, self.begin, self.replicas, self.batch)
        self.comm.device_barrier()
        for rep in self.replicas:
            rep.frames_written = f0 + cfg.chunk_frames
        self.cache.struct.frames_written = f0 + cfg.chunk_frames
        o = None
        if self.count:
            o = ops.latent_attention_fused_rows(cfg, q_nope_rows, q_rope_rows, w_uk, w_uv, self.cache, f0,
                                                self.begin, out=out)
        # no rank's next compress may overwrite ring rows before every rank has read this chunk's window
        self.comm.device_barrier()
        return o

    def close(self) -> None:
        """Unmap the peers' replicas once every rank is done with them."""
        self.comm.barrier()
        for p in self._imported:
            self.ops.ipc_release(p)
        self._imported = []
        self.comm.barrier()


__all__ = ["token_shards", "TorchComm", "ShardedLayer"]
