"""Device path of query-row sharding on one GPU: three virtual ranks, each with its own replica of
the latent cache in this GPU's memory.  Every rank compresses its token range of each chunk into all
three replicas (vmla_compress_append_rows) and attends with its own rows on its own replica
(vmla_latent_attention_fused_rows).  The replicas must be identical and equal the oracle's ring; the
ranks' rows together must equal the oracle's layer output and the unsharded fused call.  (On several
GPUs the other replicas are peer mappings and the same kernels store through them; the host protocol
is tested across processes in test_sharding_cpu.)"""
import numpy as np
import pytest
import torch

import synthetic
from parity import MID, OracleLayer, assert_close, errors, f64
from rank_latent_kv_vmla_b200.sharding import token_shards

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from rank_latent_kv_vmla_b200 import vmla
    return vmla


def _to(t):
    return t.to(DEV).contiguous()


@pytest.mark.parametrize("world", [3, 2])
def test_virtual_ranks_one_gpu(V, world):
    cfg, B, n_chunks = MID, 2, 4
    inp = synthetic.draw_layer(cfg, batch=B, seed=900 + world, n_chunks=0)
    w, w_uk, w_uv = _to(inp.w_dkv_kr), _to(inp.w_uk), _to(inp.w_uv)
    orc = OracleLayer(cfg, inp, B)
    reps = [V.LatentCache(cfg, B, device=DEV, fill=float("nan")) for _ in range(world)]
    ref = V.LatentCache(cfg, B, device=DEV, fill=float("nan"))
    # 120 tokens per chunk: shards split at multiples of 8 (40 + 40 + 40, or 64 + 56), so every virtual
    # rank holds rows and the ranges start inside 128-token tiles
    shards = token_shards(cfg.chunk_tokens, world, align=8)
    assert all(cnt > 0 for _, cnt in shards)
    for k in range(n_chunks):
        x, qn, qr = (_to(t) for t in synthetic.draw_chunk(cfg, B, 950 + 10 * world + k))
        f0 = ref.frames_written
        for b0, cnt in shards:
            if cnt:
                V.compress_append_rows(cfg, x[:, b0:b0 + cnt].contiguous(), w, f0, b0, [r.struct for r in reps], B)
        for r in reps:
            r.struct.frames_written = f0 + cfg.chunk_frames
        V.compress_append(cfg, x, w, ref)
        orc.append(x.cpu())
        outs = []
        for g, (b0, cnt) in enumerate(shards):
            if cnt:
                outs.append(V.latent_attention_fused_rows(cfg, qn[:, b0:b0 + cnt].contiguous(),
                                                          qr[:, b0:b0 + cnt].contiguous(), w_uk, w_uv, reps[g],
                                                          f0, b0))
        o = torch.cat(outs, dim=1)
        o_ref = V.latent_attention_fused(cfg, qn, qr, w_uk, w_uv, ref, f0)
        torch.cuda.synchronize()
        assert V.device_status() == 0
        bits = lambda t: t.view(torch.int16)                 # unwritten rows are NaN: compare bit patterns
        for r in reps[1:]:
            assert torch.equal(bits(r.c), bits(reps[0].c)) and torch.equal(bits(r.k_r), bits(reps[0].k_r))
        for b in range(B):
            c_ref, kr_ref, written = orc.ring(b)
            assert written.any()
            assert_close(f64(reps[0].c[b])[written], c_ref[written], cfg, f"chunk {k} replica c b{b}")
            assert_close(f64(reps[0].k_r[b])[written], kr_ref[written], cfg, f"chunk {k} replica k_r b{b}")
            assert np.isnan(f64(reps[0].c[b])[~written]).all()
            rel_l2, _ = errors(f64(reps[0].c[b])[written], f64(ref.c[b])[written])
            assert rel_l2 <= 1e-3
            layer = orc.reference(b, qn.cpu(), qr.cpu(), f0)
            assert_close(f64(o[b]), layer["o"], cfg, f"chunk {k} sharded o b{b}")
            rel_l2, _ = errors(f64(o[b]), f64(o_ref[b]))
            assert rel_l2 <= 2e-3


def test_rows_calls_reject_bad_ranges(V):
    cfg = MID
    cache = V.LatentCache(cfg, 1, device=DEV)
    x = torch.zeros((1, 64, cfg.dim), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((cfg.d_c + cfg.d_rope, cfg.dim), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(V.VmlaError):
        V.compress_append_rows(cfg, x, w, 0, cfg.chunk_tokens - 32, [cache.struct], 1)   # past the chunk
    with pytest.raises(V.VmlaError):
        V.compress_append_rows(cfg, x, w, 1, 0, [cache.struct], 1)                       # frames_written is 0
    V.compress_append_rows(cfg, x, w, 0, 0, [cache.struct], 1)
    cache.struct.frames_written = cfg.chunk_frames
    qn = torch.zeros((1, 64, cfg.n_heads, cfg.d_nope), dtype=torch.bfloat16, device=DEV)
    qr = torch.zeros((1, 64, cfg.n_heads, cfg.d_rope), dtype=torch.bfloat16, device=DEV)
    wuk = torch.zeros((cfg.n_heads, cfg.d_nope, cfg.d_c), dtype=torch.bfloat16, device=DEV)
    wuv = torch.zeros((cfg.n_heads, cfg.d_v, cfg.d_c), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(V.VmlaError):
        V.latent_attention_fused_rows(cfg, qn, qr, wuk, wuv, cache, 0, cfg.chunk_tokens - 32)
    torch.cuda.synchronize()
    assert V.device_status() == 0


def test_paired_compress_into_two_replicas_equals_single_call(V):
    """At Wan shapes with B = 4 the compress runs on CTA pairs (M = 256 MMAs).  With two destination
    rings (as when one replica is another GPU's; here both in this GPU's memory) every store of the
    epilogue goes to both: the whole-chunk call into two replicas equals the one-destination call bit
    for bit.  The same chunk split unevenly into two calls, as two ranks would issue them (narrower
    tiles, no pairs), agrees within bf16 rounding."""
    from rank_latent_kv_vmla_b200.config import WAN
    cfg, B = WAN, 4
    inp = synthetic.draw_layer(cfg, batch=B, seed=4242, n_chunks=2)
    w = _to(inp.w_dkv_kr)
    single = V.LatentCache(cfg, B, device=DEV, fill=float("nan"))
    whole = [V.LatentCache(cfg, B, device=DEV, fill=float("nan")) for _ in range(2)]
    split = [V.LatentCache(cfg, B, device=DEV, fill=float("nan")) for _ in range(2)]
    cut = 2600                                 # not a multiple of 128 or 256
    for x in inp.x_chunks:
        f0 = single.frames_written
        xd = _to(x)
        V.compress_append(cfg, xd, w, single)
        V.compress_append_rows(cfg, xd, w, f0, 0, [r.struct for r in whole], B)
        for b0, cnt in ((0, cut), (cut, cfg.chunk_tokens - cut)):
            V.compress_append_rows(cfg, xd[:, b0:b0 + cnt].contiguous(), w, f0, b0, [r.struct for r in split], B)
        for r in whole + split:
            r.struct.frames_written = single.frames_written
    torch.cuda.synchronize()
    assert V.device_status() == 0
    rows = 2 * cfg.chunk_tokens
    bits = lambda t: t.view(torch.int16)      # the unwritten rows are NaN: compare bit patterns
    for r in whole:
        assert torch.equal(bits(r.c), bits(single.c)) and torch.equal(bits(r.k_r), bits(single.k_r))
    assert torch.equal(bits(split[0].c), bits(split[1].c)) and torch.equal(bits(split[0].k_r), bits(split[1].k_r))
    for b in (0, B - 1):
        for got, ref in ((split[0].c[b, :rows], single.c[b, :rows]), (split[0].k_r[b, :rows], single.k_r[b, :rows])):
            rel_l2, _ = errors(f64(got), f64(ref))
            assert rel_l2 <= 1e-3
    assert torch.isnan(split[0].c[:, rows:].float()).all()
