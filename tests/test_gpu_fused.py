"""GPU parity of the fused call (absorbed query + latent attention + value up-projection in one
kernel): against the float64 oracle on every streamed chunk, and against the three-call path on the
same inputs.  Tiles are 128 tokens of one head: the mid config's 120-token chunks are one ragged tile
per head, a 12 x 12 grid gives 288-token chunks (2.25 tiles per head), and the Wan-shaped layer (37
tiles per head) is checked at full size on sampled tokens."""
import numpy as np
import pytest
import torch

from rank_latent_kv_vmla_b200.config import WAN
import synthetic
from parity import MID, OracleLayer, assert_close, errors, f64, paths_rel_tol

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


def _three_calls(V, cfg, qn, qr, w_uk, w_uv, cache, f0, n_query_chunks=1):
    q_abs = V.absorb_q(cfg, qn, qr, w_uk, f0, n_query_chunks=n_query_chunks)
    o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, n_query_chunks=n_query_chunks, want_lse=True)
    return V.value_up(cfg, o_lat, w_uv), lse


def _stream_fused(V, cfg, batch, n_steps, seed, rows=None):
    inp = synthetic.draw_layer(cfg, batch=batch, seed=seed, n_chunks=n_steps)
    orc = OracleLayer(cfg, inp, batch)
    cache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    w, w_uk, w_uv = _to(inp.w_dkv_kr), _to(inp.w_uk), _to(inp.w_uv)
    for k in range(n_steps):
        f0 = cache.frames_written
        V.compress_append(cfg, _to(inp.x_chunks[k]), w, cache)
        orc.append(inp.x_chunks[k])
        qn, qr = synthetic.draw_queries(cfg, batch, seed * 100 + k)
        out = torch.full((batch, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), float("nan"), dtype=torch.bfloat16,
                         device=DEV)
        o, lse = V.latent_attention_fused(cfg, _to(qn), _to(qr), w_uk, w_uv, cache, f0, out=out, want_lse=True)
        o3, lse3 = _three_calls(V, cfg, _to(qn), _to(qr), w_uk, w_uv, cache, f0)
        torch.cuda.synchronize()
        assert V.device_status() == 0
        assert torch.isfinite(o.float()).all()
        for b in sorted({0, batch - 1}):
            ref = orc.reference(b, qn, qr, f0, rows=rows)
            sel = slice(None) if rows is None else rows
            assert_close(f64(o[b][sel]), ref["o"], cfg, f"step {k} fused o b{b}")
            assert_close(f64(lse[b][sel]), ref["lse"], cfg, f"step {k} fused lse b{b}")
            # the three-call path rounds q~ and the latent output to bf16 at the same points
            rel_l2, max_rel = errors(f64(o[b]), f64(o3[b]))
            assert rel_l2 <= paths_rel_tol(cfg), (k, b, max_rel, rel_l2)
            np.testing.assert_allclose(f64(lse[b]), f64(lse3[b]), rtol=0, atol=1e-3)


def test_mid_fused_streaming(V):
    """4 two-frame chunks into a 5-frame window (partial, full, wrapping), B = 2, every call."""
    _stream_fused(V, MID, batch=2, n_steps=4, seed=3030)


def test_mid_fused_streaming_multitile(V):
    """288-token chunks (12 x 12 grid, F = 2): two full tiles and a ragged third per head, 4 chunks into a
    5-frame window (the ring wraps), B = 2."""
    _stream_fused(V, MID.replace(grid_h=12, grid_w=12), batch=2, n_steps=4, seed=3050)


@pytest.mark.parametrize("d_c", [64, 128, 256])
def test_mid_fused_latent_sizes(V, d_c):
    _stream_fused(V, MID.replace(d_c=d_c), batch=1, n_steps=3, seed=3100 + d_c)


def test_mid_fused_lowest_rank_multitile(V):
    """d_c = 64 (one latent box; q^nope still staged in two boxes) with 288-token chunks, B = 2, the
    ring wrapping."""
    _stream_fused(V, MID.replace(d_c=64, grid_h=12, grid_w=12), batch=2, n_steps=4, seed=3150)


def test_mid_fused_narrow_heads(V):
    """d_nope = 64 (one q^nope box) and d_v = 64 (half-width value up-projection)."""
    _stream_fused(V, MID.replace(d_nope=64, d_v=64), batch=1, n_steps=3, seed=3200)


@pytest.mark.parametrize("d_c", [192, 64, 128])
def test_mid_fused_block_causal_multichunk(V, d_c):
    cfg = MID.replace(window_frames=8, d_c=d_c)
    n = 3
    inp = synthetic.draw_layer(cfg, batch=1, seed=3300, n_chunks=n, n_query_chunks=n)
    orc = OracleLayer(cfg, inp, 1)
    cache = V.LatentCache(cfg, 1, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), cache)
        orc.append(x)
    o, lse = V.latent_attention_fused(cfg, _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), _to(inp.w_uv),
                                      cache, 0, n_query_chunks=n, want_lse=True)
    torch.cuda.synchronize()
    ref = orc.reference(0, inp.q_nope, inp.q_rope, 0)
    assert_close(f64(o[0]), ref["o"], cfg, "o")
    assert_close(f64(lse[0]), ref["lse"], cfg, "lse")


@pytest.mark.parametrize("d_c", [192, 64])
def test_mid_fused_peaked_softmax(V, d_c):
    """Logits x8: the running max moves and O is rescaled; compared with the three-call path on the
    same cache (the oracle comparison of this case is made call by call in test_gpu_parity)."""
    cfg = MID.replace(d_c=d_c)
    inp = synthetic.draw_layer(cfg, batch=1, seed=3400, n_chunks=3, q_gain=8.0)
    cache = V.LatentCache(cfg, 1, device=DEV)
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), cache)
    args = (_to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), _to(inp.w_uv))
    o, lse = V.latent_attention_fused(cfg, *args, cache, f0, want_lse=True)
    o3, lse3 = _three_calls(V, cfg, *args, cache, f0)
    torch.cuda.synchronize()
    rel_l2, max_rel = errors(f64(o[0]), f64(o3[0]))
    assert rel_l2 <= 5e-3 and max_rel <= 1e-2, (max_rel, rel_l2)
    np.testing.assert_allclose(f64(lse[0]), f64(lse3[0]), rtol=0, atol=1e-2)


def _sample_tokens(cfg, n=64):
    nq, T = cfg.chunk_tokens, cfg.tokens_per_frame
    picks = {0, 1, 127, 128, 255, nq - 1, nq - 2, nq - 128, T - 1, T, 2 * T - 1, 2 * T}
    picks.update(int(s) for s in np.linspace(0, nq - 1, n - len(picks), dtype=np.int64))
    return np.array(sorted(p for p in picks if 0 <= p < nq))


def test_wan_fused_full_size_sampled(V):
    """Wan-1.3B-shaped layer, 8 chunks into the 21-frame window, B = 2: sampled tokens of both batch
    elements (first / last 128-token tiles, frame boundaries, a spread)."""
    cfg, batch = WAN, 2
    inp = synthetic.draw_layer(cfg, batch=batch, seed=3500, n_chunks=8)
    orc = OracleLayer(cfg, inp, batch)
    cache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), cache)
        orc.append(x)
    args = (_to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), _to(inp.w_uv))
    o, lse = V.latent_attention_fused(cfg, *args, cache, f0, want_lse=True)
    o3, _ = _three_calls(V, cfg, *args, cache, f0)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    rows = _sample_tokens(cfg)
    for b in range(batch):
        ref = orc.reference(b, inp.q_nope, inp.q_rope, f0, rows=rows)
        assert_close(f64(o[b][rows]), ref["o"], cfg, f"o b{b}")
        assert_close(f64(lse[b][rows]), ref["lse"], cfg, f"lse b{b}")
        rel_l2, max_rel = errors(f64(o[b]), f64(o3[b]))
        assert rel_l2 <= paths_rel_tol(cfg), (b, max_rel, rel_l2)


@pytest.mark.parametrize("d_c", [192, 64, 128])
def test_fused_bounded_wait_reports_timeout_and_context_survives(V, d_c):
    """A KV tile the fused kernel never loads: the bounded wait runs out, every role winds down (the
    up-projection weights are not loaded, no output is written), vmla_device_status reports the code,
    and the next fused call on the same context is correct.  d_c = 64 / 128 run the key-split kernel."""
    cfg = MID.replace(d_c=d_c)
    inp = synthetic.draw_layer(cfg, batch=1, seed=3600, n_chunks=3)
    cache = V.LatentCache(cfg, 1, device=DEV)
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), cache)
    args = (_to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), _to(inp.w_uv))
    torch.cuda.synchronize()
    assert V.device_status() == 0
    old = V.set_wait_timeout_ms(20)
    try:
        V.debug_drop_kv_tile(1)
        V.latent_attention_fused(cfg, *args, cache, f0)
        torch.cuda.synchronize()
        assert V.device_status() != 0
        assert V.device_status() == 0          # reading clears it
    finally:
        V.debug_drop_kv_tile(-1)
        V.set_wait_timeout_ms(old)
    o = V.latent_attention_fused(cfg, *args, cache, f0)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    orc = OracleLayer(cfg, inp, 1)
    for x in inp.x_chunks:
        orc.append(x)
    ref = orc.reference(0, inp.q_nope, inp.q_rope, f0)
    assert_close(f64(o[0]), ref["o"], cfg, "fused o after a timed-out launch")
