"""GPU parity of few-step generation: each chunk is denoised over several steps; the first step
appends it, later steps rewrite its cache rows in place (vmla_compress_rewrite / vmla_dense_rewrite),
and every step attends with its own queries.  Every call is checked against the float64 oracle, whose
history replaces the chunk's entries, and the rows of older frames must stay bit-identical."""
import numpy as np
import pytest
import torch

from rank_latent_kv_vmla_b200.config import TINY
import synthetic
from parity import MID, OracleLayer, assert_close, dense_weights_from_latent, f64, round_to

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


def _bits(t):
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32)


def _chunk_rows(cfg, first_frame):
    """Ring rows (within a batch element) of the chunk whose first frame is first_frame."""
    rows = []
    for f in range(first_frame, first_frame + cfg.chunk_frames):
        s = f % cfg.window_frames
        rows.extend(range(s * cfg.tokens_per_frame, (s + 1) * cfg.tokens_per_frame))
    return np.asarray(rows)


def _fewstep(V, cfg, batch, n_chunks, n_denoise, seed):
    inp = synthetic.draw_layer(cfg, batch=batch, seed=seed, n_chunks=0)
    orc = OracleLayer(cfg, inp, batch)
    cache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    w, w_uk, w_uv = _to(inp.w_dkv_kr), _to(inp.w_uk), _to(inp.w_uv)
    for k in range(n_chunks):
        for s in range(n_denoise):
            x, qn, qr = synthetic.draw_chunk(cfg, batch, synthetic.rollout_seed(seed, 0, k * n_denoise + s))
            if s == 0:
                f0 = cache.frames_written
                V.compress_append(cfg, _to(x), w, cache)
                orc.append(x)
            else:
                before_c, before_k = cache.c.clone(), cache.k_r.clone()
                V.compress_rewrite(cfg, _to(x), w, cache)
                orc.rewrite(x)
                assert cache.frames_written == f0 + cfg.chunk_frames
                keep = np.setdiff1d(np.arange(cfg.window_tokens), _chunk_rows(cfg, f0))
                torch.cuda.synchronize()
                assert torch.equal(_bits(cache.c[:, keep]), _bits(before_c[:, keep])), "older c rows changed"
                assert torch.equal(_bits(cache.k_r[:, keep]), _bits(before_k[:, keep])), "older k_r rows changed"
            q_abs = V.absorb_q(cfg, _to(qn), _to(qr), w_uk, f0)
            o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, want_lse=True)
            o = V.value_up(cfg, o_lat, w_uv)
            torch.cuda.synchronize()
            assert V.device_status() == 0
            for b in range(batch):
                c_ref, kr_ref, written = orc.ring(b)
                tag = f"chunk {k} step {s} b{b}"
                assert_close(f64(cache.c[b])[written], c_ref[written], cfg, f"{tag} c plane")
                assert_close(f64(cache.k_r[b])[written], kr_ref[written], cfg, f"{tag} k_r plane")
                ref = orc.reference(b, qn, qr, f0)
                assert_close(f64(o_lat[b]), ref["o_latent"], cfg, f"{tag} o_latent")
                assert_close(f64(lse[b]), ref["lse"], cfg, f"{tag} lse")
                assert_close(f64(o[b]), ref["o"], cfg, f"{tag} o")


def test_tiny_fp32_fewstep(V):
    """5 one-frame chunks x 3 denoising steps into a 3-frame window (rewrites after eviction)."""
    _fewstep(V, TINY, batch=2, n_chunks=5, n_denoise=3, seed=4321)


def test_mid_bf16_fewstep(V):
    """4 two-frame chunks x 3 steps into a 5-frame window: the third chunk wraps the ring."""
    _fewstep(V, MID, batch=2, n_chunks=4, n_denoise=3, seed=555)


def test_mid_bf16_dense_rewrite_matches_latent(V):
    """The dense rewrite with W_K,h = [W^K_up,h W^KV_down ; W^KR], W_V,h = W^V_up,h W^KV_down gives the
    latent path's output at every denoising step."""
    cfg, batch = MID, 1
    inp = synthetic.draw_layer(cfg, batch=batch, seed=99, n_chunks=0)
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    orc = OracleLayer(cfg, inp, batch)
    dcache = V.DenseCache(cfg, batch, device=DEV, fill=float("nan"))
    lcache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    for k in range(3):
        for s in range(2):
            x, qn, qr = synthetic.draw_chunk(cfg, batch, synthetic.rollout_seed(99, 1, 2 * k + s))
            if s == 0:
                f0 = dcache.frames_written
                V.dense_append(cfg, _to(x), w_kv, dcache)
                V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), lcache)
                orc.append(x)
            else:
                V.dense_rewrite(cfg, _to(x), w_kv, dcache)
                V.compress_rewrite(cfg, _to(x), _to(inp.w_dkv_kr), lcache)
                orc.rewrite(x)
            o_d = V.dense_mha(cfg, V.rope_q(cfg, _to(qn), _to(qr), f0), dcache, f0)
            o_l = V.value_up(cfg, V.latent_attention(
                cfg, V.absorb_q(cfg, _to(qn), _to(qr), _to(inp.w_uk), f0), lcache, f0), _to(inp.w_uv))
            torch.cuda.synchronize()
            ref = orc.reference(0, qn, qr, f0)
            assert_close(f64(o_d[0]), ref["o"], cfg, f"dense chunk {k} step {s}")
            assert_close(f64(o_l[0]), ref["o"], cfg, f"latent chunk {k} step {s}")
