"""CUDA IPC path of query-row sharding, on one GPU with two processes: the parent exports its replica of
the latent cache (vmla_ipc_export); a child process imports it (vmla_ipc_import), compresses its token
range of each chunk into both its own replica and the parent's through the imported mapping
(vmla_compress_append_rows), synchronises, releases the mapping and reports.  The parent compresses the
other token range into both replicas the same way (the child's replica is exported to the parent in
turn).  The two replicas must then be bit-identical and equal a cache filled by plain
vmla_compress_append.  No kernel waits on another process: the two processes are ordered on the host."""
import os

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N_CHUNKS = 3


def _bits(t):
    return t.view(torch.int16)


def _child(q_in, q_out):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    from rank_latent_kv_vmla_b200 import vmla as V
    from rank_latent_kv_vmla_b200.sharding import token_shards
    import synthetic
    from parity import MID
    try:
        cfg, B = MID, 2
        own = V.LatentCache(cfg, B, device="cuda", fill=float("nan"))
        q_out.put(("handles", V.ipc_export(own.c), V.ipc_export(own.k_r)))
        hc, hk = q_in.get(timeout=120)
        pc, pk = V.ipc_import(hc), V.ipc_import(hk)
        peer = V.CCache(pc, pk, B, 0, 0)
        w = synthetic.draw_weights(cfg, 41)[0].cuda()
        (b0, n), _ = token_shards(cfg.chunk_tokens, 2, align=8)[::-1]   # the child takes the second range
        for k in range(N_CHUNKS):
            assert q_in.get(timeout=120) == ("chunk", k)
            x = synthetic.draw_chunk(cfg, B, 400 + k)[0].cuda()
            f0 = own.frames_written
            V.compress_append_rows(cfg, x[:, b0:b0 + n].contiguous(), w, f0, b0, [own.struct, peer], B)
            torch.cuda.synchronize()
            own.struct.frames_written = peer.frames_written = f0 + cfg.chunk_frames
            q_out.put(("done", k))
        assert V.device_status() == 0
        q_out.put(("own", own.c.cpu(), own.k_r.cpu()))
        assert q_in.get(timeout=120) == "release"
        V.ipc_release(pc)
        V.ipc_release(pk)
        q_out.put(("released",))
        assert q_in.get(timeout=120) == "exit"        # keep own planes mapped until the parent released them
    except Exception as e:                          # report instead of leaving the parent waiting
        q_out.put(("error", repr(e)))


def test_two_processes_share_replicas_through_ipc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from rank_latent_kv_vmla_b200 import vmla as V
    from rank_latent_kv_vmla_b200.sharding import token_shards
    import synthetic
    from parity import MID
    cfg, B = MID, 2
    ctx = mp.get_context("spawn")
    q_in, q_out = ctx.Queue(), ctx.Queue()
    child = ctx.Process(target=_child, args=(q_in, q_out))
    child.start()
    try:
        own = V.LatentCache(cfg, B, device="cuda", fill=float("nan"))
        ref = V.LatentCache(cfg, B, device="cuda", fill=float("nan"))
        msg = q_out.get(timeout=300)
        assert msg[0] == "handles", msg
        pc, pk = V.ipc_import(msg[1]), V.ipc_import(msg[2])
        peer = V.CCache(pc, pk, B, 0, 0)
        q_in.put((V.ipc_export(own.c), V.ipc_export(own.k_r)))
        w = synthetic.draw_weights(cfg, 41)[0].cuda()
        b0, n = token_shards(cfg.chunk_tokens, 2, align=8)[0]            # the parent takes the first range
        for k in range(N_CHUNKS):
            x = synthetic.draw_chunk(cfg, B, 400 + k)[0].cuda()
            f0 = own.frames_written
            V.compress_append_rows(cfg, x[:, b0:b0 + n].contiguous(), w, f0, b0, [own.struct, peer], B)
            V.compress_append(cfg, x, w, ref)
            torch.cuda.synchronize()
            q_in.put(("chunk", k))
            msg = q_out.get(timeout=300)
            assert msg == ("done", k), msg
            own.struct.frames_written = peer.frames_written = f0 + cfg.chunk_frames
        assert V.device_status() == 0
        msg = q_out.get(timeout=300)
        assert msg[0] == "own", msg
        child_c, child_kr = msg[1], msg[2]
        # both replicas received the same stores: identical bits
        assert torch.equal(_bits(own.c), _bits(child_c.cuda())) and torch.equal(_bits(own.k_r), _bits(child_kr.cuda()))
        # and they equal a plain compress of the whole chunks (tile shapes differ: bf16-rounding agreement)
        from parity import errors, f64
        for name, a, b in (("c", own.c, ref.c), ("k_r", own.k_r, ref.k_r)):
            rel_l2, max_rel = errors(f64(a), f64(b))
            assert rel_l2 <= 1e-3 and max_rel <= 1e-2, (name, rel_l2, max_rel)
        V.ipc_release(pc)
        V.ipc_release(pk)
        q_in.put("release")
        assert q_out.get(timeout=300) == ("released",)
        q_in.put("exit")
    finally:
        child.join(timeout=300)
        if child.is_alive():
            child.terminate()
    assert child.exitcode == 0
