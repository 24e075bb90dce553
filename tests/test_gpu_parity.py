"""GPU parity: every C-ABI call against the float64 oracle on the same seeded inputs.

Sizes span several 128-row tiles with ragged tails; the Wan-shaped layer is checked at full size on
sampled query rows (first/last tiles, frame and chunk boundaries) and whole cache planes.
"""
import numpy as np
import pytest
import torch

from oracle import vmla_oracle as O
from rank_latent_kv_vmla_b200.config import TINY, WAN, VMLA_BF16
import synthetic
from parity import (MID, OracleLayer, assert_close, dense_weights_from_latent, f64, round_to, sample_rows,
                    pairs)

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


def _stream_and_check(V, cfg, batch, n_steps, seed, q_gain=1.0, check_every_step=True):
    """Stream n_steps chunks through the GPU path (append -> absorb -> attend -> value-up) and check
    every call's output against the oracle.  Caches and outputs start NaN-poisoned."""
    inp = synthetic.draw_layer(cfg, batch=batch, seed=seed, n_chunks=n_steps)
    orc = OracleLayer(cfg, inp, batch)
    cache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    w, w_uk, w_uv = _to(inp.w_dkv_kr), _to(inp.w_uk), _to(inp.w_uv)
    report = []
    for k in range(n_steps):
        x = _to(inp.x_chunks[k])
        f0 = cache.frames_written
        V.compress_append(cfg, x, w, cache)
        orc.append(inp.x_chunks[k])
        assert cache.frames_written == orc.frames_written
        if not (check_every_step or k == n_steps - 1):
            continue
        qn, qr = synthetic.draw_queries(cfg, batch, seed * 100 + k, q_gain=q_gain)
        q_abs = V.absorb_q(cfg, _to(qn), _to(qr), w_uk, f0)
        o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, want_lse=True)
        o = V.value_up(cfg, o_lat, w_uv)
        torch.cuda.synchronize()
        assert V.device_status() == 0
        for b in range(batch):
            c_ref, kr_ref, written = orc.ring(b)
            assert_close(f64(cache.c[b])[written], c_ref[written], cfg, f"step {k} c plane b{b}")
            assert_close(f64(cache.k_r[b])[written], kr_ref[written], cfg, f"step {k} k_r plane b{b}")
            ref = orc.reference(b, qn, qr, f0)
            assert_close(f64(q_abs[b]), ref["q_abs"], cfg, f"step {k} q_abs b{b}")
            assert_close(f64(o_lat[b]), ref["o_latent"], cfg, f"step {k} o_latent b{b}")
            assert_close(f64(lse[b]), ref["lse"], cfg, f"step {k} lse b{b}")
            report.append(assert_close(f64(o[b]), ref["o"], cfg, f"step {k} o b{b}"))
    return report


def test_tiny_fp32_streaming_every_call(V):
    """6 one-frame chunks into a 3-frame window (eviction from step 3), fp32, every call checked."""
    _stream_and_check(V, TINY, batch=1, n_steps=6, seed=1234)


def test_tiny_fp32_batch3(V):
    _stream_and_check(V, TINY, batch=3, n_steps=4, seed=77)


@pytest.mark.parametrize("batch", [1, 2])
def test_mid_bf16_streaming_every_call(V, batch):
    """4 two-frame chunks into a 5-frame window: partial window, full window, wrap inside a chunk."""
    _stream_and_check(V, MID, batch=batch, n_steps=4, seed=2024 + batch)


@pytest.mark.parametrize("d_c", [192, 64])
def test_mid_bf16_peaked_softmax_isolated(V, d_c):
    """Queries x8 (peaked attention, exercises the running-max rescale).  Each call is fed the
    oracle's own bf16-rounded inputs, so only that call's arithmetic is measured: through the whole
    chain the x8 logits would amplify the bf16 storage rounding of q_abs and c beyond the tolerance."""
    _isolated_attention_and_value_up(V, MID.replace(d_c=d_c), seed=31, q_gain=8.0)


def _isolated_attention_and_value_up(V, cfg, seed, q_gain=1.0, batch=2, n_chunks=4):
    inp = synthetic.draw_layer(cfg, batch=batch, seed=seed, n_chunks=n_chunks)
    orc = OracleLayer(cfg, inp, batch)
    for x in inp.x_chunks:
        orc.append(x)
    f0 = orc.frames_written - cfg.chunk_frames
    cache = V.LatentCache(cfg, batch, device=DEV)
    for b in range(batch):
        c_ref, kr_ref, _ = orc.ring(b)
        cache.c[b].copy_(round_to(cfg, c_ref))
        cache.k_r[b].copy_(round_to(cfg, kr_ref))
    cache.struct.frames_written = orc.frames_written
    qn, qr = synthetic.draw_queries(cfg, batch, seed + 4242, q_gain=q_gain)
    q_abs = _to(round_to(cfg, orc.q_abs(qn, qr, f0)))
    o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, want_lse=True)
    torch.cuda.synchronize()
    key_frames = orc.key_frames_of_ring()
    hi = O.query_chunk_end(f0, cfg.chunk_tokens, cfg.chunk_frames, cfg.tokens_per_frame)
    mask = O.visible(hi, np.where(key_frames >= 0, key_frames, -10 ** 9), cfg.window_frames)
    refs = []
    for b in range(batch):
        c_in, kr_in = f64(cache.c[b]), f64(cache.k_r[b])
        ref_lat, ref_lse = O.latent_attention(f64(q_abs[b]), np.nan_to_num(c_in), np.nan_to_num(kr_in),
                                              mask, cfg.scale)
        assert_close(f64(o_lat[b]), ref_lat, cfg, f"o_latent b{b}")
        assert_close(f64(lse[b]), ref_lse, cfg, f"lse b{b}")
        refs.append(ref_lat)
    # value up-projection alone, on the oracle's latent output rounded to bf16
    o_lat_in = _to(round_to(cfg, np.stack(refs)))
    o = V.value_up(cfg, o_lat_in, _to(inp.w_uv))
    torch.cuda.synchronize()
    for b in range(batch):
        assert_close(f64(o[b]), O.value_up(f64(o_lat_in[b]), f64(inp.w_uv)), cfg, f"value_up b{b}")


@pytest.mark.parametrize("d_c", [64, 128, 256])
def test_mid_bf16_latent_sizes(V, d_c):
    cfg = MID.replace(d_c=d_c)
    _stream_and_check(V, cfg, batch=1, n_steps=3, seed=500 + d_c, check_every_step=False)


def test_mid_bf16_attention_isolated(V):
    """Latent attention and value up-projection alone, each fed with the oracle's own bf16-rounded
    inputs (cache planes, absorbed queries, latent outputs)."""
    _isolated_attention_and_value_up(V, MID, seed=99)


@pytest.mark.parametrize("d_c", [64, 128, 256])
def test_mid_bf16_attention_isolated_latent_sizes(V, d_c):
    _isolated_attention_and_value_up(V, MID.replace(d_c=d_c), seed=98 + d_c, batch=1)


@pytest.mark.parametrize("d_c", [192, 64, 128])
def test_mid_bf16_block_causal_multichunk(V, d_c):
    """One call over 3 query chunks (bidirectional inside a chunk, causal across chunks)."""
    cfg = MID.replace(window_frames=8, d_c=d_c)
    n = 3
    inp = synthetic.draw_layer(cfg, batch=1, seed=7, n_chunks=n, n_query_chunks=n)
    orc = OracleLayer(cfg, inp, 1)
    cache = V.LatentCache(cfg, 1, device=DEV, fill=float("nan"))
    w = _to(inp.w_dkv_kr)
    for x in inp.x_chunks:
        V.compress_append(cfg, _to(x), w, cache)
        orc.append(x)
    q_abs = V.absorb_q(cfg, _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), 0, n_query_chunks=n)
    o_lat, lse = V.latent_attention(cfg, q_abs, cache, 0, n_query_chunks=n, want_lse=True)
    o = V.value_up(cfg, o_lat, _to(inp.w_uv))
    torch.cuda.synchronize()
    ref = orc.reference(0, inp.q_nope, inp.q_rope, 0)
    assert_close(f64(o_lat[0]), ref["o_latent"], cfg, "o_latent")
    assert_close(f64(lse[0]), ref["lse"], cfg, "lse")
    assert_close(f64(o[0]), ref["o"], cfg, "o")


def test_mid_bf16_deterministic_and_fully_written(V):
    cfg = MID
    inp = synthetic.draw_layer(cfg, batch=2, seed=5, n_chunks=3)
    outs = []
    for _ in range(2):
        cache = V.LatentCache(cfg, 2, device=DEV, fill=float("nan"))
        for x in inp.x_chunks:
            V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), cache)
        f0 = cache.frames_written - cfg.chunk_frames
        q_abs = torch.full((2, cfg.chunk_tokens, cfg.n_heads, cfg.d_qk), float("nan"), dtype=torch.bfloat16, device=DEV)
        V.absorb_q(cfg, _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), f0, out=q_abs)
        o_lat = torch.full((2, cfg.chunk_tokens, cfg.n_heads, cfg.d_c), float("nan"), dtype=torch.bfloat16, device=DEV)
        lse = torch.full((2, cfg.chunk_tokens, cfg.n_heads), float("nan"), dtype=torch.float32, device=DEV)
        V.latent_attention(cfg, q_abs, cache, f0, out=o_lat, lse=lse)
        o = torch.full((2, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), float("nan"), dtype=torch.bfloat16, device=DEV)
        V.value_up(cfg, o_lat, _to(inp.w_uv), out=o)
        torch.cuda.synchronize()
        for t in (q_abs, o_lat, lse, o):
            assert torch.isfinite(t.float()).all()
        outs.append([t.clone() for t in (cache.c, cache.k_r, q_abs, o_lat, lse, o)])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_dense_path_matches_oracle_and_latent_path(V):
    """Dense comparison layer with weights W_K,h = [W^K_up,h W^KV_down ; W^KR], W_V,h = W^V_up,h W^KV_down
    equals the latent layer (both against the oracle, and against each other)."""
    cfg = MID
    batch, n_steps = 2, 4
    inp = synthetic.draw_layer(cfg, batch=batch, seed=808, n_chunks=n_steps)
    orc = OracleLayer(cfg, inp, batch)
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    dcache = V.DenseCache(cfg, batch, device=DEV, fill=float("nan"))
    lcache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        f0 = dcache.frames_written
        V.dense_append(cfg, _to(x), w_kv, dcache)
        V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), lcache)
        orc.append(x)
    q = V.rope_q(cfg, _to(inp.q_nope), _to(inp.q_rope), f0)
    o_d, lse_d = V.dense_mha(cfg, q, dcache, f0, want_lse=True)
    o_lat = V.latent_attention(cfg, V.absorb_q(cfg, _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), f0),
                               lcache, f0)
    o_l = V.value_up(cfg, o_lat, _to(inp.w_uv))
    torch.cuda.synchronize()
    pos = O.token_positions(f0, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)
    for b in range(batch):
        ref = orc.reference(b, inp.q_nope, inp.q_rope, f0)
        qr = O.rotate_query(f64(inp.q_rope[b]), pos, pairs(cfg), cfg.rope_theta)
        assert_close(f64(q[b]), np.concatenate([f64(inp.q_nope[b]), qr], -1), cfg, "dense q")
        assert_close(f64(o_d[b]), ref["o"], cfg, f"dense o b{b}")
        assert_close(f64(lse_d[b]), ref["lse"], cfg, f"dense lse b{b}")
        assert_close(f64(o_d[b]), f64(o_l[b]), cfg, f"dense vs latent b{b}")


def test_tiny_fp32_dense_path(V):
    cfg = TINY
    inp = synthetic.draw_layer(cfg, batch=1, seed=3, n_chunks=5)
    orc = OracleLayer(cfg, inp, 1)
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    dcache = V.DenseCache(cfg, 1, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        f0 = dcache.frames_written
        V.dense_append(cfg, _to(x), w_kv, dcache)
        orc.append(x)
    q = V.rope_q(cfg, _to(inp.q_nope), _to(inp.q_rope), f0)
    o_d = V.dense_mha(cfg, q, dcache, f0)
    torch.cuda.synchronize()
    ref = orc.reference(0, inp.q_nope, inp.q_rope, f0)
    assert_close(f64(o_d[0]), ref["o"], cfg, "dense o")


@pytest.mark.parametrize("batch", [1, 2, 4])
def test_wan_full_size_sampled(V, batch):
    """The Wan-1.3B-shaped layer at full size: 8 chunks streamed into the 21-frame window (the last
    one evicts frames 0-2); whole cache planes and all absorbed queries are checked, attention and
    the final output on sampled rows of batch elements {0, B-1}."""
    cfg = WAN
    n_steps = 8
    inp = synthetic.draw_layer(cfg, batch=batch, seed=1235, n_chunks=n_steps)
    orc = OracleLayer(cfg, inp, batch)
    cache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    w = _to(inp.w_dkv_kr)
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.compress_append(cfg, _to(x), w, cache)
        orc.append(x)
    q_abs = V.absorb_q(cfg, _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), f0)
    o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, want_lse=True)
    o = V.value_up(cfg, o_lat, _to(inp.w_uv))
    torch.cuda.synchronize()
    assert V.device_status() == 0
    rows = sample_rows(cfg, cfg.chunk_tokens)
    q_ref = orc.q_abs(inp.q_nope, inp.q_rope, f0)
    for b in sorted({0, batch - 1}):
        c_ref, kr_ref, written = orc.ring(b)
        assert written.all()
        assert_close(f64(cache.c[b]), c_ref, cfg, f"c plane b{b}")
        assert_close(f64(cache.k_r[b]), kr_ref, cfg, f"k_r plane b{b}")
        assert_close(f64(q_abs[b]), q_ref[b], cfg, f"q_abs b{b}")
        ref = orc.reference(b, inp.q_nope, inp.q_rope, f0, rows=rows)
        assert_close(f64(o_lat[b][rows]), ref["o_latent"], cfg, f"o_latent b{b}")
        assert_close(f64(lse[b][rows]), ref["lse"], cfg, f"lse b{b}")
        assert_close(f64(o[b][rows]), ref["o"], cfg, f"o b{b}")


def test_native_kernels_launched(V):
    before = V.launch_count()
    cfg = MID
    inp = synthetic.draw_layer(cfg, batch=1, seed=1, n_chunks=1)
    cache = V.LatentCache(cfg, 1, device=DEV)
    V.layer_step(cfg, _to(inp.x_chunks[0]), _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_dkv_kr),
                 _to(inp.w_uk), _to(inp.w_uv), cache)
    torch.cuda.synchronize()
    assert V.launch_count() > before


@pytest.mark.parametrize("d_c", [192, 64])
def test_bounded_wait_reports_timeout_and_context_survives(V, d_c):
    """A KV tile that is never loaded makes the consumer's bounded wait run out: the kernel returns,
    vmla_device_status reports a nonzero code, and the next call on the same context is correct
    (d_c = 64 runs the kernel whose tile keys are split between two softmax warpgroups)."""
    cfg = MID.replace(d_c=d_c)
    inp = synthetic.draw_layer(cfg, batch=1, seed=404, n_chunks=3)
    cache = V.LatentCache(cfg, 1, device=DEV)
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), cache)
    q_abs = V.absorb_q(cfg, _to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), f0)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    old = V.set_wait_timeout_ms(20)
    try:
        V.debug_drop_kv_tile(1)
        V.latent_attention(cfg, q_abs, cache, f0)
        torch.cuda.synchronize()
        code = V.device_status()
        assert code != 0
        assert V.device_status() == 0          # reading clears it
    finally:
        V.debug_drop_kv_tile(-1)
        V.set_wait_timeout_ms(old)
    o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, want_lse=True)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    orc = OracleLayer(cfg, inp, 1)
    for x in inp.x_chunks:
        orc.append(x)
    ref = orc.reference(0, inp.q_nope, inp.q_rope, f0)
    assert_close(f64(o_lat[0]), ref["o_latent"], cfg, "o_latent after a timed-out launch")
