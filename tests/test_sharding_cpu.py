"""Query-row sharding of one sequence (rank_latent_kv_vmla_b200.sharding) on the CPU.

The host protocol runs in world-size-2 and world-size-3 gloo process groups with stand-ins for the
device: a replica plane is a file-backed shared mapping (np.memmap), so a store into another rank's
replica lands in that rank's memory at once, as a store through an NVLink peer mapping does;
compression and attention are the float64 oracle's.  One rank is delayed on the host before every
attention, so the other ranks run ahead as far as the protocol lets them.  Every rank's attention must
see exactly the oracle's ring for its chunk, its output rows must equal the oracle's layer output, and
after the last chunk every replica must equal the oracle's ring.  The same run with the release barrier
after attention left out must see a peer overwrite rows that the delayed rank still reads."""
import os
import pickle
import socket
import time

import numpy as np
import pytest
import torch.multiprocessing as mp

from rank_latent_kv_vmla_b200.sharding import token_shards


def test_token_shards_cover_the_chunk_in_aligned_pieces():
    for n, world, align in ((4680, 2, 128), (4680, 3, 128), (4680, 8, 128), (480, 3, 128), (16, 2, 8),
                            (100, 8, 128), (0, 2, 128), (1, 1, 1)):
        shards = token_shards(n, world, align)
        assert len(shards) == world
        begin = 0
        for b, c in shards:
            assert b == begin and c >= 0
            if c and b + c < n:
                assert c % align == 0
            begin += c
        assert begin == n
        counts = [c for _, c in shards]
        assert max(counts) - min(counts) <= align           # balanced to one unit
    with pytest.raises(ValueError):
        token_shards(10, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _Ptr:
    """Stand-in device pointer: (owning rank, plane) and the mapped array."""
    def __init__(self, owner, plane, arr):
        self.owner, self.plane, self.arr = owner, plane, arr


class _Plane:
    def __init__(self, arr, ptr):
        self.arr, self._ptr = arr, ptr

    def data_ptr(self):
        return self._ptr


class _Struct:
    def __init__(self, c, k_r, batch, reserved, frames_written):
        self.c, self.k_r, self.batch, self.frames_written = c, k_r, batch, frames_written


def _mapped(path, shape, create):
    if create:
        a = np.lib.format.open_memmap(path, mode="w+", dtype=np.float64, shape=shape)
        a[...] = np.nan
        a.flush()
        return a
    return np.lib.format.open_memmap(path, mode="r+")


class _Ops:
    """CPU stand-in of the library calls ShardedLayer makes.  Replica planes live in shared file
    mappings: a store into a peer's replica is visible to the peer immediately.  The rank
    ``delay_rank`` sleeps ``delay_s`` before each attention whose window a later chunk overwrites."""

    def __init__(self, rank, O, pairs, shm_dir, delay_rank=-1, delay_s=0.0):
        self.rank, self.O, self.pairs, self.shm_dir = rank, O, pairs, shm_dir
        self.delay_rank, self.delay_s = delay_rank, delay_s
        self.CCache = _Struct
        self.seen = None

    def LatentCache(self, cfg, batch, device=None):
        rank = self.rank

        class _Cache:
            pass
        cache = _Cache()
        for plane, d in (("c", cfg.d_c), ("k_r", cfg.d_rope)):
            arr = _mapped(os.path.join(self.shm_dir, f"r{rank}_{plane}.npy"), (batch, cfg.window_tokens, d), True)
            setattr(cache, plane, _Plane(arr, _Ptr(rank, plane, arr)))
        cache.struct = _Struct(cache.c.data_ptr(), cache.k_r.data_ptr(), batch, 0, 0)
        cache.batch = batch
        type(cache).frames_written = property(lambda s: s.struct.frames_written)
        self.local = cache
        return cache

    def ipc_export(self, plane):
        p = plane.data_ptr()
        return pickle.dumps((p.owner, p.plane))

    def ipc_import(self, handle):
        owner, plane = pickle.loads(handle)
        assert owner != self.rank
        return _Ptr(owner, plane, _mapped(os.path.join(self.shm_dir, f"r{owner}_{plane}.npy"), None, False))

    def ipc_release(self, ptr):
        assert ptr.owner != self.rank
        ptr.arr.flush()

    def compress_append_rows(self, cfg, x_rows, w, f0, begin, replicas, batch):
        O = self.O
        n = x_rows.shape[1]
        pos = O.token_positions(f0, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)[begin:begin + n]
        tok = np.arange(begin, begin + n)
        rows = ((f0 + tok // cfg.tokens_per_frame) % cfg.window_frames) * cfg.tokens_per_frame + \
            tok % cfg.tokens_per_frame
        for r in replicas:
            assert r.frames_written == f0
        for b in range(batch):
            c, k_r = O.compress(x_rows[b], w, cfg.d_c, pos, self.pairs, cfg.rope_theta)
            for r in replicas:                      # stores land in the target replica at once
                r.c.arr[b, rows] = c
                r.k_r.arr[b, rows] = k_r

    def latent_attention_fused_rows(self, cfg, qn, qr, w_uk, w_uv, cache, f0, begin, out=None):
        O = self.O
        if self.rank == self.delay_rank and f0 + 2 * cfg.chunk_frames > cfg.window_frames:
            time.sleep(self.delay_s)                # the next chunk evicts frames of this window
        n = qn.shape[1]
        fw = cache.frames_written
        key_frames = np.repeat([O.frame_of_slot(s, fw, cfg.window_frames) for s in range(cfg.window_frames)],
                               cfg.tokens_per_frame)
        pos = O.token_positions(f0, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)[begin:begin + n]
        hi = O.query_chunk_end(f0, cfg.chunk_tokens, cfg.chunk_frames, cfg.tokens_per_frame)[begin:begin + n]
        mask = O.visible(hi, key_frames, cfg.window_frames) & (key_frames >= 0)[None, :]
        self.seen = (np.array(cache.c.arr), np.array(cache.k_r.arr))     # what this attention reads
        outs = []
        for b in range(qn.shape[0]):
            q_abs = O.absorbed_query(qn[b], O.rotate_query(qr[b], pos, self.pairs, cfg.rope_theta), w_uk)
            c = np.nan_to_num(self.seen[0][b])
            k_r = np.nan_to_num(self.seen[1][b])
            o_lat, _ = O.latent_attention(q_abs, c, k_r, mask, cfg.scale)
            outs.append(O.value_up(o_lat, w_uv))
        return np.stack(outs)


class _Comm:
    """gloo collectives.  The device barrier is a host all-reduce: the stand-in's stores are made
    synchronously, so every store issued before it has landed when it returns.  ``release_barrier``
    False turns every second device barrier (the one after attention) into a no-op on every rank."""

    def __init__(self, dist, release_barrier=True):
        import torch
        self.dist, self.torch = dist, torch
        self.world, self.rank = dist.get_world_size(), dist.get_rank()
        self.release_barrier = release_barrier
        self.n_barriers = 0
        self._calls = 0

    def all_gather_object(self, obj):
        out = [None] * self.world
        self.dist.all_gather_object(out, obj)
        return out

    def device_barrier(self):
        self._calls += 1
        if not self.release_barrier and self._calls % 2 == 0:
            return
        self.dist.all_reduce(self.torch.zeros(1))
        self.n_barriers += 1

    def barrier(self):
        self.dist.barrier()


def _worker(rank, world, port, root, shm_dir, release_barrier, q):
    import sys
    sys.path.insert(0, root)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from oracle import vmla_oracle as O
        from rank_latent_kv_vmla_b200.config import TINY
        from rank_latent_kv_vmla_b200.sharding import ShardedLayer
        import synthetic
        cfg = TINY.replace(grid_h=4, grid_w=6, chunk_frames=1, window_frames=3)     # 24 tokens per chunk
        pairs = (cfg.rope_pairs_t, cfg.rope_pairs_h, cfg.rope_pairs_w)
        ops = _Ops(rank, O, pairs, shm_dir, delay_rank=0, delay_s=0.4)
        comm = _Comm(dist, release_barrier)
        B, n_chunks = 2, 5
        layer = ShardedLayer(cfg, B, comm, ops=ops, align=8)
        w = synthetic.draw_weights(cfg, 5)
        w, w_uk, w_uv = (t.double().numpy() for t in w)
        hists = [O.History(cfg.d_c, cfg.d_rope) for _ in range(B)]
        report, seen_err, out_err = [], 0.0, 0.0
        for k in range(n_chunks):
            x, qn, qr = (t.double().numpy() for t in synthetic.draw_chunk(cfg, B, 50 + k))
            f0 = layer.frames_written
            b0, cnt = layer.begin, layer.count
            o = layer.step(x[:, b0:b0 + cnt], qn[:, b0:b0 + cnt], qr[:, b0:b0 + cnt], w, w_uk, w_uv)
            pos = O.token_positions(f0, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)
            for b in range(B):
                c, k_r = O.compress(x[b], w, cfg.d_c, pos, pairs, cfg.rope_theta)
                hists[b].append(c, k_r, pos[:, 0])
            if cnt:
                # the replica this rank's attention read, and its output rows, against the oracle
                for b in range(B):
                    for plane, hist in ((0, hists[b].c), (1, hists[b].k_r)):
                        ref, written = O.ring_from_history(hist, layer.frames_written, cfg.window_frames,
                                                           cfg.tokens_per_frame)
                        got = ops.seen[plane][b]
                        seen_err = max(seen_err, float(np.nan_to_num(np.abs(got[written] - ref[written]),
                                                                     nan=np.inf).max()))
                        assert np.isnan(got[~written]).all()
                    ref = O.layer_reference(hists[b], qn[b], qr[b], w_uk, w_uv, first_frame=f0,
                                            query_rows=np.arange(b0, b0 + cnt), chunk_frames=cfg.chunk_frames,
                                            window_frames=cfg.window_frames, grid_h=cfg.grid_h,
                                            grid_w=cfg.grid_w, pairs=pairs, theta=cfg.rope_theta, scale=cfg.scale)
                    out_err = max(out_err, float(np.abs(o[b] - ref["o"]).max()))
            report.append((k, b0, cnt, layer.frames_written))
        layer.close()
        # after the last chunk (close() holds two barriers) every replica equals the oracle's ring
        final_err = 0.0
        for b in range(B):
            for arr, hist in ((ops.local.c.arr, hists[b].c), (ops.local.k_r.arr, hists[b].k_r)):
                ref, written = O.ring_from_history(hist, layer.frames_written, cfg.window_frames,
                                                   cfg.tokens_per_frame)
                final_err = max(final_err, float(np.abs(arr[b][written] - ref[written]).max()))
        q.put((rank, report, comm.n_barriers, [r.frames_written for r in layer.replicas],
               seen_err, out_err, final_err))
    finally:
        dist.destroy_process_group()


def _run(world, tmp_path, release_barrier):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    procs = [ctx.Process(target=_worker, args=(r, world, port, root, str(tmp_path), release_barrier, q))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    return sorted(q.get(timeout=5) for _ in range(world))


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_layer_protocol_gloo(world, tmp_path):
    """Rank 0 is delayed before every attention; the other ranks' next compress must still wait."""
    got = _run(world, tmp_path, release_barrier=True)
    shards = token_shards(24, world, 8)
    for rank, report, n_barriers, replica_frames, seen_err, out_err, final_err in got:
        assert n_barriers == 2 * 5                      # two device barriers per chunk on every rank
        assert replica_frames == [5] * world
        assert [(b, c) for _, b, c, _ in report] == [shards[rank]] * 5
        assert [f for *_, f in report][:5] == [1, 2, 3, 4, 5]
        assert seen_err <= 1e-12, (rank, seen_err)      # the attention read exactly the oracle's ring
        assert out_err <= 1e-10, (rank, out_err)
        assert final_err <= 1e-12, (rank, final_err)


def test_without_the_release_barrier_a_peer_overwrites_a_window_in_use(tmp_path):
    """The protocol with only the barrier after the compress: while rank 0 sleeps before its attention,
    rank 1 compresses the next chunk into rank 0's replica, evicting frames of the window rank 0 is
    about to read.  The stand-ins detect it (this is the race the release barrier closes)."""
    got = _run(2, tmp_path, release_barrier=False)
    seen_err = {rank: e for rank, _, _, _, e, _, _ in got}
    out_err = {rank: e for rank, _, _, _, _, e, _ in got}
    assert seen_err[0] > 1e-3 and out_err[0] > 1e-6
    # the rank that is never delayed reads correct windows (nobody writes into its window early)
    assert seen_err[1] <= 1e-12
