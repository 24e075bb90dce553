"""The streaming executor (host buffers in and out, copies overlapped with the kernels) against the
synchronous device path on the same inputs: two layers with their own caches and weights, stepped
alternately for several chunks, so that both staging slots are reused and the ring wraps."""
import pytest
import torch

import synthetic
from parity import MID

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from rank_latent_kv_vmla_b200 import vmla
    return vmla


def test_executor_matches_synchronous_path(V):
    cfg, B, n_layers, n_chunks = MID, 2, 2, 5
    weights = [tuple(t.to(DEV) for t in synthetic.draw_weights(cfg, 70 + l)) for l in range(n_layers)]
    inputs = [[synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(71, l, k)) for k in range(n_chunks)]
              for l in range(n_layers)]
    ref_caches = [V.LatentCache(cfg, B, device=DEV) for _ in range(n_layers)]
    ex_caches = [V.LatentCache(cfg, B, device=DEV) for _ in range(n_layers)]
    ref_out, ex_out = {}, {}
    for k in range(n_chunks):
        for l in range(n_layers):
            x, qn, qr = inputs[l][k]
            wd, wuk, wuv = weights[l]
            ref_out[(l, k)] = V.layer_step(cfg, x.to(DEV), qn.to(DEV), qr.to(DEV), wd, wuk, wuv, ref_caches[l],
                                           fused=True).cpu()
    torch.cuda.synchronize()
    with V.Executor(cfg, B) as ex:
        hosts = {}
        for k in range(n_chunks):
            for l in range(n_layers):
                x, qn, qr = inputs[l][k]
                hx, hqn, hqr = (t.pin_memory() for t in (x, qn, qr))
                ho = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16).pin_memory()
                wd, wuk, wuv = weights[l]
                ex.submit(ex_caches[l], wd, wuk, wuv, hx, hqn, hqr, ho)
                hosts[(l, k)] = (hx, hqn, hqr, ho)
        ex.wait()
        for key, (_, _, _, ho) in hosts.items():
            assert torch.equal(ho, ref_out[key]), key
    for l in range(n_layers):
        assert ex_caches[l].frames_written == ref_caches[l].frames_written == n_chunks * cfg.chunk_frames
        assert torch.equal(ex_caches[l].c, ref_caches[l].c)
        assert torch.equal(ex_caches[l].k_r, ref_caches[l].k_r)
    assert V.device_status() == 0


def test_executor_rejects_bad_submissions(V):
    cfg = MID
    w, wuk, wuv = (t.to(DEV) for t in synthetic.draw_weights(cfg, 72))
    x, qn, qr = (t.pin_memory() for t in synthetic.draw_chunk(cfg, 2, 73))
    ho = torch.empty((2, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16).pin_memory()
    with V.Executor(cfg, 2) as ex:
        with pytest.raises(V.VmlaError):
            ex.submit(V.LatentCache(cfg, 1, device=DEV), w, wuk, wuv, x, qn, qr, ho)     # batch 1 cache
        with pytest.raises(ValueError):
            ex.submit(V.LatentCache(cfg, 2, device=DEV), w, wuk, wuv, x.cuda(), qn, qr, ho)   # device input
        cache = V.LatentCache(cfg, 2, device=DEV)
        # refused on the host by a check of the inner fused call (a misaligned W^V_up): nothing is
        # enqueued, the cache is not advanced and no ring row is written
        import ctypes
        st = V.LIB.vmla_executor_submit(ex._h, ctypes.byref(cache.struct), w.data_ptr(), wuk.data_ptr(),
                                        wuv.data_ptr() + 2, x.data_ptr(), qn.data_ptr(), qr.data_ptr(),
                                        ho.data_ptr())
        assert st == V.VMLA_ERR_MISALIGNED
        assert cache.frames_written == 0
        ex.submit(cache, w, wuk, wuv, x, qn, qr, ho)          # the executor still works afterwards
        ex.wait()
        assert cache.frames_written == cfg.chunk_frames
        ref = V.LatentCache(cfg, 2, device=DEV)
        o_ref = V.layer_step(cfg, x.to(DEV), qn.to(DEV), qr.to(DEV), w, wuk, wuv, ref, fused=True).cpu()
        assert torch.equal(ho, o_ref)
        n = cfg.chunk_tokens                                  # the rows of frames 0 .. F-1
        assert torch.equal(ref.c[:, :n], cache.c[:, :n]) and torch.equal(ref.k_r[:, :n], cache.k_r[:, :n])
    assert V.device_status() == 0


def test_executor_wan_batch4_matches_synchronous_path(V):
    """The Wan-1.3B layer at B = 4 through the executor (the compress on CTA pairs, 28.8 MB of inputs per
    step staged through the workspace): outputs and caches bit-identical to the synchronous path."""
    from rank_latent_kv_vmla_b200.config import WAN
    cfg, B, n_chunks = WAN, 4, 3
    wd, wuk, wuv = (t.to(DEV) for t in synthetic.draw_weights(cfg, 80))
    inputs = [synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(81, 0, k)) for k in range(n_chunks)]
    ref_cache = V.LatentCache(cfg, B, device=DEV, fill=float("nan"))
    ex_cache = V.LatentCache(cfg, B, device=DEV, fill=float("nan"))
    ref_out = []
    for x, qn, qr in inputs:
        ref_out.append(V.layer_step(cfg, x.to(DEV), qn.to(DEV), qr.to(DEV), wd, wuk, wuv, ref_cache,
                                    fused=True).cpu())
    torch.cuda.synchronize()
    with V.Executor(cfg, B) as ex:
        outs = []
        for x, qn, qr in inputs:
            ho = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16).pin_memory()
            ex.submit(ex_cache, wd, wuk, wuv, x.pin_memory(), qn.pin_memory(), qr.pin_memory(), ho)
            outs.append(ho)
        ex.wait()
    for k in range(n_chunks):
        assert torch.equal(outs[k], ref_out[k]), k
    bits = lambda t: t.view(torch.int16)      # the rows not yet written are NaN: compare bit patterns
    assert torch.equal(bits(ex_cache.c), bits(ref_cache.c)) and torch.equal(bits(ex_cache.k_r), bits(ref_cache.k_r))
    assert V.device_status() == 0
