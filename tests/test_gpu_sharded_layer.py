"""ShardedLayer end to end with two processes on one GPU (gloo process group): each rank exports its
replica of the latent cache, imports the other's, compresses its token range of every chunk into both
(through the CUDA IPC mapping), passes the device barrier (a gloo all-reduce of a device tensor, which
completes only after both ranks' compress kernels), attends with its own query rows on its own
replica and passes the second device barrier (after both ranks' attention) before its next compress.
Rank 0 sleeps on the host before every attention whose window the next chunk overwrites, so rank 1
runs ahead as far as the protocol lets it: its next compress, which stores into rank 0's replica, must
still wait for rank 0's attention.  The ranks' output rows together must equal the unsharded fused call
and the float64 oracle, and both replicas must equal the oracle's ring.  No kernel waits on the other
process."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N_CHUNKS = 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _pack(t):
    """A bf16 tensor as an int16 numpy array: pickled by value, so it outlives the sending process
    (torch tensors in a multiprocessing queue travel as shared memory owned by the sender)."""
    return t.cpu().view(torch.int16).numpy().copy()


def _unpack(a):
    return torch.from_numpy(a).view(torch.bfloat16)


class _DelayedOps:
    """The library calls as they are, except that rank 0 sleeps on the host before launching each
    attention whose window the next chunk evicts frames of."""

    def __init__(self, V, rank, delay_s=0.5):
        self._V, self._rank, self._delay = V, rank, delay_s

    def __getattr__(self, name):
        return getattr(self._V, name)

    def latent_attention_fused_rows(self, cfg, *args, **kw):
        import time
        f0 = args[5]
        if self._rank == 0 and f0 + 2 * cfg.chunk_frames > cfg.window_frames:
            time.sleep(self._delay)
        return self._V.latent_attention_fused_rows(cfg, *args, **kw)


def _rank(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import datetime
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from rank_latent_kv_vmla_b200 import vmla as V
        from rank_latent_kv_vmla_b200.sharding import ShardedLayer, TorchComm
        import synthetic
        from parity import MID
        cfg, B = MID, 2
        torch.cuda.set_device(0)
        layer = ShardedLayer(cfg, B, TorchComm(device="cuda"), device="cuda", align=8, ops=_DelayedOps(V, rank))
        w, wuk, wuv = (t.cuda() for t in synthetic.draw_weights(cfg, 51))
        outs = []
        for k in range(N_CHUNKS):
            x, qn, qr = (t.cuda() for t in synthetic.draw_chunk(cfg, B, 500 + k))
            b0, n = layer.begin, layer.count
            rows = lambda t: t[:, b0:b0 + n].contiguous()
            o = layer.step(rows(x), rows(qn), rows(qr), w, wuk, wuv)
            torch.cuda.synchronize()
            outs.append(_pack(o))
        assert V.device_status() == 0
        q.put((rank, layer.shards, outs, _pack(layer.cache.c), _pack(layer.cache.k_r), layer.frames_written))
        layer.close()
    except Exception as e:
        q.put((rank, "error", repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def test_sharded_layer_two_processes_one_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            item = q.get(timeout=600)
            assert item[1] != "error", item
            got[item[0]] = item
    finally:
        for p in procs:
            p.join(timeout=300)
            if p.is_alive():
                p.terminate()
    assert all(p.exitcode == 0 for p in procs)
    got = {r: (it[0], it[1], [_unpack(a) for a in it[2]], _unpack(it[3]), _unpack(it[4]), it[5])
           for r, it in got.items()}

    # reference: the unsharded fused call on a cache filled by plain appends, and the oracle
    from rank_latent_kv_vmla_b200 import vmla as V
    import synthetic
    from parity import MID, OracleLayer, assert_close, errors, f64
    cfg, B = MID, 2
    inp = synthetic.draw_layer(cfg, batch=B, seed=1, n_chunks=0)
    w, wuk, wuv = (t.cuda() for t in synthetic.draw_weights(cfg, 51))
    ref = V.LatentCache(cfg, B, device="cuda")
    orc = OracleLayer(cfg, inp, B)
    orc.w, orc.w_uk, orc.w_uv = (f64(t) for t in synthetic.draw_weights(cfg, 51))
    shards = got[0][1]
    for k in range(N_CHUNKS):
        x, qn, qr = synthetic.draw_chunk(cfg, B, 500 + k)
        o_ref = V.layer_step(cfg, x.cuda(), qn.cuda(), qr.cuda(), w, wuk, wuv, ref, fused=True).cpu()
        f0 = orc.frames_written
        orc.append(x)
        o = torch.cat([got[r][2][k] for r in range(world) if shards[r][1]], dim=1)
        for b in range(B):
            rel_l2, _ = errors(f64(o[b]), f64(o_ref[b]))
            assert rel_l2 <= 2e-3, (k, b, rel_l2)
            assert_close(f64(o[b]), orc.reference(b, qn, qr, f0)["o"], cfg, f"chunk {k} sharded o b{b}")
    for r in range(world):
        assert got[r][5] == N_CHUNKS * cfg.chunk_frames
        for b in range(B):
            c_ref, kr_ref, written = orc.ring(b)
            assert_close(f64(got[r][3][b])[written], c_ref[written], cfg, f"rank {r} replica c b{b}")
            assert_close(f64(got[r][4][b])[written], kr_ref[written], cfg, f"rank {r} replica k_r b{b}")
    # 4 chunks of 2 frames fill the 5-frame ring: every row written, and both replicas hold the same bits
    assert torch.equal(got[0][3].view(torch.int16), got[1][3].view(torch.int16))
    assert torch.equal(got[0][4].view(torch.int16), got[1][4].view(torch.int16))
