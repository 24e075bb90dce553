"""Query-row sharding of one sequence (rank_latent_kv_vmla_b200.sharding) on the CPU.

The host protocol runs in world-size-2 and world-size-3 gloo process groups with stand-ins for the
device: a replica plane is a NumPy array; a store into another rank's replica is queued and delivered
at the device barrier (which is where the real peer stores are known to have landed); compression and
attention are the float64 oracle's.  After every streamed chunk each rank's replica must equal the
oracle's ring, and the ranks' output rows together must equal the oracle's layer output."""
import os
import pickle
import socket

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
    """Stand-in device pointer: (owning rank, plane)."""
    def __init__(self, owner, plane):
        self.owner, self.plane = owner, plane


class _Plane:
    def __init__(self, arr, ptr):
        self.arr, self._ptr = arr, ptr

    def data_ptr(self):
        return self._ptr


class _Struct:
    def __init__(self, c, k_r, batch, reserved, frames_written):
        self.c, self.k_r, self.batch, self.frames_written = c, k_r, batch, frames_written


class _Ops:
    """CPU stand-in of the library calls ShardedLayer makes."""

    def __init__(self, rank, O, pairs):
        self.rank, self.O, self.pairs = rank, O, pairs
        self.outbox = []
        self.CCache = _Struct

    def LatentCache(self, cfg, batch, device=None):
        rank = self.rank

        class _Cache:
            pass
        cache = _Cache()
        cache.c = _Plane(np.full((batch, cfg.window_tokens, cfg.d_c), np.nan), _Ptr(rank, "c"))
        cache.k_r = _Plane(np.full((batch, cfg.window_tokens, cfg.d_rope), np.nan), _Ptr(rank, "k_r"))
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
        return _Ptr(owner, plane)

    def ipc_release(self, ptr):
        assert ptr.owner != self.rank

    def _store(self, ptr, b, rows, vals):
        if ptr.owner == self.rank:
            getattr(self.local, ptr.plane).arr[b, rows] = vals
        else:
            self.outbox.append((ptr.owner, ptr.plane, b, rows, vals))

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
            for r in replicas:
                self._store(r.c, b, rows, c)
                self._store(r.k_r, b, rows, k_r)

    def deliver(self, incoming):
        for owner, plane, b, rows, vals in incoming:
            assert owner == self.rank
            getattr(self.local, plane).arr[b, rows] = vals

    def latent_attention_fused_rows(self, cfg, qn, qr, w_uk, w_uv, cache, f0, begin, out=None):
        O = self.O
        n = qn.shape[1]
        fw = cache.frames_written
        key_frames = np.repeat([O.frame_of_slot(s, fw, cfg.window_frames) for s in range(cfg.window_frames)],
                               cfg.tokens_per_frame)
        pos = O.token_positions(f0, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)[begin:begin + n]
        hi = O.query_chunk_end(f0, cfg.chunk_tokens, cfg.chunk_frames, cfg.tokens_per_frame)[begin:begin + n]
        mask = O.visible(hi, key_frames, cfg.window_frames) & (key_frames >= 0)[None, :]
        outs = []
        for b in range(qn.shape[0]):
            q_abs = O.absorbed_query(qn[b], O.rotate_query(qr[b], pos, self.pairs, cfg.rope_theta), w_uk)
            c = np.nan_to_num(cache.c.arr[b])
            k_r = np.nan_to_num(cache.k_r.arr[b])
            o_lat, _ = O.latent_attention(q_abs, c, k_r, mask, cfg.scale)
            outs.append(O.value_up(o_lat, w_uv))
        return np.stack(outs)


class _Comm:
    """gloo collectives; queued peer stores are delivered at the device barrier."""

    def __init__(self, dist, ops):
        self.dist, self.ops = dist, ops
        self.world, self.rank = dist.get_world_size(), dist.get_rank()
        self.n_barriers = 0

    def all_gather_object(self, obj):
        out = [None] * self.world
        self.dist.all_gather_object(out, obj)
        return out

    def device_barrier(self):
        boxes = self.all_gather_object(self.ops.outbox)
        self.ops.outbox = []
        self.ops.deliver([m for box in boxes for m in box if m[0] == self.rank])
        self.n_barriers += 1

    def barrier(self):
        self.dist.barrier()


def _worker(rank, world, port, root, q):
    import sys
    sys.path.insert(0, root)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import vmla_oracle as O
        from rank_latent_kv_vmla_b200.config import TINY
        from rank_latent_kv_vmla_b200.sharding import ShardedLayer
        import synthetic
        cfg = TINY.replace(grid_h=4, grid_w=6, chunk_frames=1, window_frames=3)     # 24 tokens per chunk
        pairs = (cfg.rope_pairs_t, cfg.rope_pairs_h, cfg.rope_pairs_w)
        ops = _Ops(rank, O, pairs)
        comm = _Comm(dist, ops)
        B, n_chunks = 2, 5
        layer = ShardedLayer(cfg, B, comm, ops=ops, align=8)
        w = synthetic.draw_weights(cfg, 5)
        w, w_uk, w_uv = (t.double().numpy() for t in w)
        hists = [O.History(cfg.d_c, cfg.d_rope) for _ in range(B)]
        report = []
        for k in range(n_chunks):
            x, qn, qr = (t.double().numpy() for t in synthetic.draw_chunk(cfg, B, 50 + k))
            f0 = layer.frames_written
            b0, cnt = layer.begin, layer.count
            o = layer.step(x[:, b0:b0 + cnt], qn[:, b0:b0 + cnt], qr[:, b0:b0 + cnt], w, w_uk, w_uv)
            pos = O.token_positions(f0, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)
            for b in range(B):
                c, k_r = O.compress(x[b], w, cfg.d_c, pos, pairs, cfg.rope_theta)
                hists[b].append(c, k_r, pos[:, 0])
            for b in range(B):
                c_ref, written = O.ring_from_history(hists[b].c, layer.frames_written, cfg.window_frames,
                                                     cfg.tokens_per_frame)
                kr_ref, _ = O.ring_from_history(hists[b].k_r, layer.frames_written, cfg.window_frames,
                                                cfg.tokens_per_frame)
                np.testing.assert_allclose(ops.local.c.arr[b][written], c_ref[written], rtol=0, atol=1e-12)
                np.testing.assert_allclose(ops.local.k_r.arr[b][written], kr_ref[written], rtol=0, atol=1e-12)
                assert np.isnan(ops.local.c.arr[b][~written]).all()
            # this rank's output rows against the oracle's whole-layer reference
            if cnt:
                for b in range(B):
                    ref = O.layer_reference(hists[b], qn[b], qr[b], w_uk, w_uv, first_frame=f0,
                                            query_rows=np.arange(b0, b0 + cnt), chunk_frames=cfg.chunk_frames,
                                            window_frames=cfg.window_frames, grid_h=cfg.grid_h,
                                            grid_w=cfg.grid_w, pairs=pairs, theta=cfg.rope_theta, scale=cfg.scale)
                    np.testing.assert_allclose(o[b], ref["o"], rtol=1e-10, atol=1e-12)
            report.append((k, b0, cnt, layer.frames_written))
        layer.close()
        q.put((rank, report, comm.n_barriers, [r.frames_written for r in layer.replicas]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_layer_protocol_gloo(repo_root, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, repo_root, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    shards = token_shards(24, world, 8)
    for rank, report, n_barriers, replica_frames in got:
        assert n_barriers == 5                          # one device barrier per chunk on every rank
        assert replica_frames == [5] * world
        assert [(b, c) for _, b, c, _ in report] == [shards[rank]] * 5
        assert [f for *_, f in report] == [1, 2, 3, 4, 5]
