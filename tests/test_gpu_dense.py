"""GPU parity of the dense comparison layer's attention kernel on the shapes that stress its key split
(two softmax warpgroups per 128-key tile, each with its own max, sum and O, merged at the end):
  * one-token frames: 1-3 visible keys, so the second half of the only tile is fully masked;
  * a window of many tiles with a ragged last tile (the second half of the last tile masked);
  * the whole window as one block-causal multi-chunk query set (rows of one tile see different ends);
  * a batch of several sequences;
  * the Wan-1.3B shapes at full size (256 KV tiles, a ragged 37th query tile per head), sampled rows.
The dense weights are W_K,h = [W^K_up,h W^KV_down ; W^KR] and W_V,h = W^V_up,h W^KV_down, so the
float64 oracle's latent layer is the reference for o and the log-sum-exp."""
import pytest
import torch

import synthetic
from parity import MID, OracleLayer, assert_close, dense_weights_from_latent, f64, round_to, sample_rows
from rank_latent_kv_vmla_b200.config import WAN

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


def _stream(V, cfg, batch, n_chunks, seed, check_from=0):
    """Append n_chunks chunks to a dense cache; from chunk check_from on attend with the chunk's
    queries and compare o and lse with the oracle."""
    inp = synthetic.draw_layer(cfg, batch=batch, seed=seed, n_chunks=0)
    orc = OracleLayer(cfg, inp, batch)
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    cache = V.DenseCache(cfg, batch, device=DEV, fill=float("nan"))
    for k in range(n_chunks):
        x, qn, qr = synthetic.draw_chunk(cfg, batch, seed * 17 + k)
        f0 = cache.frames_written
        V.dense_append(cfg, _to(x), w_kv, cache)
        orc.append(x)
        if k < check_from:
            continue
        q = V.rope_q(cfg, _to(qn), _to(qr), f0)
        o, lse = V.dense_mha(cfg, q, cache, f0, want_lse=True)
        torch.cuda.synchronize()
        assert V.device_status() == 0
        for b in range(batch):
            ref = orc.reference(b, qn, qr, f0)
            assert_close(f64(o[b]), ref["o"], cfg, f"chunk {k} dense o b{b}")
            assert_close(f64(lse[b]), ref["lse"], cfg, f"chunk {k} dense lse b{b}")


def test_one_token_frames(V):
    cfg = MID.replace(grid_h=1, grid_w=1, chunk_frames=1, window_frames=3)
    _stream(V, cfg, batch=3, n_chunks=5, seed=71)


def test_many_tiles_ragged_window(V):
    # 12 frames x 60 tokens = 720 keys: 5 full tiles and a last tile of 80 keys (its second half
    # holds 16 visible keys), 120 query tokens (one full and one partial query tile per head)
    cfg = MID.replace(window_frames=12)
    _stream(V, cfg, batch=2, n_chunks=7, seed=72, check_from=2)


def test_ragged_tail_half_masked(V):
    # 5 frames x 60 = 300 keys: the last tile holds 44 keys, so its second half is fully masked
    _stream(V, MID, batch=2, n_chunks=4, seed=73, check_from=2)


def test_whole_window_block_causal(V):
    cfg = MID.replace(window_frames=8)
    n = cfg.window_frames // cfg.chunk_frames
    inp = synthetic.draw_layer(cfg, batch=2, seed=74, n_chunks=n, n_query_chunks=n)
    orc = OracleLayer(cfg, inp, 2)
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    cache = V.DenseCache(cfg, 2, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        V.dense_append(cfg, _to(x), w_kv, cache)
        orc.append(x)
    q = V.rope_q(cfg, _to(inp.q_nope), _to(inp.q_rope), 0, n_query_chunks=n)
    o, lse = V.dense_mha(cfg, q, cache, 0, n_query_chunks=n, want_lse=True)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    for b in range(2):
        ref = orc.reference(b, inp.q_nope, inp.q_rope, 0)
        assert_close(f64(o[b]), ref["o"], cfg, f"dense o b{b}")
        assert_close(f64(lse[b]), ref["lse"], cfg, f"dense lse b{b}")


def test_batch_of_eight_runs_are_bit_identical(V):
    """Eight sequences; the kernel's result does not depend on scheduling (two launches agree bit for
    bit) and matches the oracle."""
    cfg = MID.replace(grid_h=3, grid_w=8)
    inp = synthetic.draw_layer(cfg, batch=8, seed=75, n_chunks=3)
    orc = OracleLayer(cfg, inp, 8)
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    cache = V.DenseCache(cfg, 8, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.dense_append(cfg, _to(x), w_kv, cache)
        orc.append(x)
    q = V.rope_q(cfg, _to(inp.q_nope), _to(inp.q_rope), f0)
    o1 = V.dense_mha(cfg, q, cache, f0)
    o2 = V.dense_mha(cfg, q, cache, f0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    for b in range(8):
        assert_close(f64(o1[b]), orc.reference(b, inp.q_nope, inp.q_rope, f0)["o"], cfg, f"dense o b{b}")


def test_bounded_wait_reports_timeout_and_context_survives(V):
    """A KV tile the dense kernel never loads: the MMA warp's wait for it runs out, both softmax halves
    and the producer wind down (the producer does not wait for the missing copy), vmla_device_status
    reports the code, and the next call on the same context is correct."""
    cfg = MID
    inp = synthetic.draw_layer(cfg, batch=1, seed=76, n_chunks=3)
    orc = OracleLayer(cfg, inp, 1)
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    cache = V.DenseCache(cfg, 1, device=DEV)
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.dense_append(cfg, _to(x), w_kv, cache)
        orc.append(x)
    q = V.rope_q(cfg, _to(inp.q_nope), _to(inp.q_rope), f0)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    old = V.set_wait_timeout_ms(20)
    try:
        V.debug_drop_kv_tile(1)
        V.dense_mha(cfg, q, cache, f0)
        torch.cuda.synchronize()
        assert V.device_status() != 0
        assert V.device_status() == 0          # reading clears it
    finally:
        V.debug_drop_kv_tile(-1)
        V.set_wait_timeout_ms(old)
    o = V.dense_mha(cfg, q, cache, f0)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    assert_close(f64(o[0]), orc.reference(0, inp.q_nope, inp.q_rope, f0)["o"], cfg, "dense o after a timed-out launch")


def test_wan_full_size_sampled(V):
    """The dense layer at the Wan-1.3B shapes the bench times: 8 chunks streamed into the 21-frame
    window (the last evicts frames 0-2), then the newest chunk's queries over all 32760 keys; o and the
    log-sum-exp on sampled rows (first and last tiles, frame boundaries, a spread) of every head."""
    cfg = WAN
    inp = synthetic.draw_layer(cfg, batch=1, seed=1236, n_chunks=8)
    orc = OracleLayer(cfg, inp, 1)
    w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
    cache = V.DenseCache(cfg, 1, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        f0 = cache.frames_written
        V.dense_append(cfg, _to(x), w_kv, cache)
        orc.append(x)
    q = V.rope_q(cfg, _to(inp.q_nope), _to(inp.q_rope), f0)
    o, lse = V.dense_mha(cfg, q, cache, f0, want_lse=True)
    torch.cuda.synchronize()
    assert V.device_status() == 0
    rows = sample_rows(cfg, cfg.chunk_tokens)
    ref = orc.reference(0, inp.q_nope, inp.q_rope, f0, rows=rows)
    assert_close(f64(o[0][rows]), ref["o"], cfg, "dense o")
    assert_close(f64(lse[0][rows]), ref["lse"], cfg, "dense lse")

