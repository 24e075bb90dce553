"""GPU parity at the full sizes of the larger workloads: the Wan-1.3B layer at batch 8 with the dense
per-head layer on identical inputs, the lower-rank latents at batch 16, and a long streaming rollout
whose ring wraps many times (frame indices up to 240).  At batch 8 and 16 both the three-call path and
the fused call (the one the bench times there) are checked.  The oracle checks sampled query rows of batch
elements {0, B-1} and whole cache planes; the dense and latent paths are also compared in full."""
import numpy as np
import pytest
import torch

from oracle import vmla_oracle as O
from rank_latent_kv_vmla_b200.config import WAN
import synthetic
from parity import OracleLayer, assert_close, dense_weights_from_latent, errors, f64, round_to, pairs, paths_rel_tol

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


def _rows(cfg, n=48):
    T = cfg.tokens_per_frame
    picks = {0, 1, 11, 12, cfg.chunk_tokens - 1, cfg.chunk_tokens - 12, T - 1, T, 2 * T - 1, 2 * T}
    picks.update(int(v) for v in np.linspace(0, cfg.chunk_tokens - 1, n - len(picks)))
    return np.array(sorted(p for p in picks if 0 <= p < cfg.chunk_tokens))


def test_wan_batch8_latent_and_dense_agree_with_oracle(V):
    cfg, B = WAN, 8
    n_chunks = 7                                     # frames 0..20: the full window, no eviction
    inp = synthetic.draw_layer(cfg, batch=B, seed=1234 + 2, n_chunks=n_chunks)
    lc = V.LatentCache(cfg, B, device=DEV, fill=float("nan"))
    dc = V.DenseCache(cfg, B, device=DEV, fill=float("nan"))
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    for x in inp.x_chunks:
        f0 = lc.frames_written
        xd = _to(x)
        V.compress_append(cfg, xd, _to(inp.w_dkv_kr), lc)
        V.dense_append(cfg, xd, w_kv, dc)
    qn, qr = _to(inp.q_nope), _to(inp.q_rope)
    o_lat = V.latent_attention(cfg, V.absorb_q(cfg, qn, qr, _to(inp.w_uk), f0), lc, f0)
    o_l = V.value_up(cfg, o_lat, _to(inp.w_uv))
    o_d = V.dense_mha(cfg, V.rope_q(cfg, qn, qr, f0), dc, f0)
    # the fused call (absorb + attention + value-up in one launch), as the batch-8 bench times it
    o_f, lse_f = V.latent_attention_fused(cfg, qn, qr, _to(inp.w_uk), _to(inp.w_uv), lc, f0, want_lse=True)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    # the paths, all rows, against each other
    for b in range(B):
        assert_close(f64(o_d[b]), f64(o_l[b]), cfg, f"dense vs latent b{b}")
        rel_l2, max_ratio = errors(f64(o_f[b]), f64(o_l[b]))
        assert rel_l2 <= paths_rel_tol(cfg) and max_ratio <= 1e-2, (b, rel_l2, max_ratio)
    # and sampled rows of the first and last sequence against the oracle
    orc = OracleLayer(cfg, inp, B)
    rows = _rows(cfg)
    for x in inp.x_chunks:
        orc.append(x)
    for b in (0, B - 1):
        ref = orc.reference(b, inp.q_nope, inp.q_rope, f0, rows=rows)
        assert_close(f64(o_l[b][rows]), ref["o"], cfg, f"latent o b{b}")
        assert_close(f64(o_f[b][rows]), ref["o"], cfg, f"fused o b{b}")
        assert_close(f64(lse_f[b][rows]), ref["lse"], cfg, f"fused lse b{b}")
        assert_close(f64(o_d[b][rows]), ref["o"], cfg, f"dense o b{b}")
        c_ref, kr_ref, written = orc.ring(b)
        assert written.all()
        assert_close(f64(lc.c[b]), c_ref, cfg, f"c plane b{b}")


@pytest.mark.parametrize("d_c", [64, 128, 192])
def test_wan_lower_rank_batch16(V, d_c):
    cfg, B = WAN.replace(d_c=d_c), 16
    n_chunks = 3
    inp = synthetic.draw_layer(cfg, batch=B, seed=1234 + 3 + d_c, n_chunks=n_chunks)
    cache = V.LatentCache(cfg, B, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), cache)
    q_abs = V.absorb_q(cfg, _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), f0)
    o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, want_lse=True)
    o = V.value_up(cfg, o_lat, _to(inp.w_uv))
    # the fused call, as the d_c sweep of the bench times it at this batch
    fused = V.fused_supported(cfg)
    assert fused or d_c == 64
    if fused:
        o_f, lse_f = V.latent_attention_fused(cfg, _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk),
                                              _to(inp.w_uv), cache, f0, want_lse=True)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    assert cache.nbytes() == V.latent_cache_bytes(cfg, B)
    for b in range(B if fused else 0):
        rel_l2, max_ratio = errors(f64(o_f[b]), f64(o[b]))
        assert rel_l2 <= paths_rel_tol(cfg) and max_ratio <= 1e-2, (b, rel_l2, max_ratio)
    orc = OracleLayer(cfg, inp, B)
    for x in inp.x_chunks:
        orc.append(x)
    rows = _rows(cfg, 32)
    for b in (0, B - 1):
        ref = orc.reference(b, inp.q_nope, inp.q_rope, f0, rows=rows)
        assert_close(f64(o_lat[b][rows]), ref["o_latent"], cfg, f"o_latent b{b}")
        assert_close(f64(lse[b][rows]), ref["lse"], cfg, f"lse b{b}")
        assert_close(f64(o[b][rows]), ref["o"], cfg, f"o b{b}")
        if fused:
            assert_close(f64(o_f[b][rows]), ref["o"], cfg, f"fused o b{b}")
            assert_close(f64(lse_f[b][rows]), ref["lse"], cfg, f"fused lse b{b}")


def test_streaming_rollout_80_chunks(V):
    """Two layers of the Wan-shaped rollout at batch 4: 80 chunks of 3 frames each (frames 0..239,
    the 21-frame ring wraps 11 times); the last chunk of each layer is checked against the oracle,
    which rebuilds the window from the last 7 chunks' inputs."""
    cfg, B, n_chunks, base = WAN, 4, 80, 5
    keep = cfg.window_frames // cfg.chunk_frames
    for layer in range(2):
        w_dkv_kr, w_uk, w_uv = synthetic.draw_weights(cfg, synthetic.rollout_seed(base, layer, -1))
        wd, wukd, wuvd = _to(w_dkv_kr), _to(w_uk), _to(w_uv)
        cache = V.LatentCache(cfg, B, device=DEV)
        for k in range(n_chunks):
            x, qn, qr = synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(base, layer, k))
            f0 = cache.frames_written
            o = V.layer_step(cfg, _to(x), _to(qn), _to(qr), wd, wukd, wuvd, cache)
        torch.cuda.synchronize()
        assert V.device_status() == 0
        assert cache.frames_written == 3 * n_chunks
        # oracle: the window holds chunks n_chunks-7 .. n_chunks-1 (frames 219..239)
        for b in (0, B - 1):
            hist = O.History(cfg.d_c, cfg.d_rope)
            for k in range(n_chunks - keep, n_chunks):
                x, _, _ = synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(base, layer, k))
                pos = O.token_positions(k * cfg.chunk_frames, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)
                c, k_r = O.compress(f64(x[b]), f64(w_dkv_kr), cfg.d_c, pos, pairs(cfg), cfg.rope_theta)
                hist.append(c, k_r, pos[:, 0])
            _, qn, qr = synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(base, layer, n_chunks - 1))
            rows = _rows(cfg, 24)
            ref = O.layer_reference(hist, f64(qn[b]), f64(qr[b]), f64(w_uk), f64(w_uv), first_frame=f0,
                                    query_rows=rows, chunk_frames=cfg.chunk_frames,
                                    window_frames=cfg.window_frames, grid_h=cfg.grid_h, grid_w=cfg.grid_w,
                                    pairs=pairs(cfg), theta=cfg.rope_theta, scale=cfg.scale)
            assert_close(f64(o[b][rows]), ref["o"], cfg, f"rollout layer {layer} o b{b}")
            # the ring rows of the newest frame equal the oracle's compression of that chunk
            slot0 = (f0 % cfg.window_frames) * cfg.tokens_per_frame
            c_new = hist.c[-cfg.chunk_tokens:]
            got = f64(cache.c[b][slot0:slot0 + cfg.tokens_per_frame])
            assert_close(got, c_new[:cfg.tokens_per_frame], cfg, f"rollout layer {layer} newest ring rows b{b}")
