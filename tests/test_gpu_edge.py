"""GPU parity on the degenerate cases of the method, every call against the float64 oracle:
  * a window of exactly one chunk (each chunk evicts the previous one and sees only itself);
  * one-token frames (grid 1 x 1): a single valid row in every 128-row tile;
  * very large absolute frame indices (the RoPE angles reach ~1e6 rad and are reduced exactly);
  * the whole window as one block-causal multi-chunk query set;
  * a batch of 16 short sequences.
Both the three-call path and the fused call are checked (bf16), and the fp32 path where it applies."""
import numpy as np
import pytest
import torch

from oracle import vmla_oracle as O
from rank_latent_kv_vmla_b200.config import TINY, VMLA_BF16
import synthetic
from parity import MID, OracleLayer, assert_close, f64

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


def _isolated_lse(orc, cfg, q_abs, c_ring, kr_ring, f0):
    """The oracle's latent attention on the given q_abs [Nq, H, d_qk] and ring planes (masked by the
    frames the ring holds): its log-sum-exp [Nq, H]."""
    key_frames = orc.key_frames_of_ring()
    hi = O.query_chunk_end(f0, q_abs.shape[0], cfg.chunk_frames, cfg.tokens_per_frame)
    mask = O.visible(hi, key_frames, cfg.window_frames) & (key_frames >= 0)[None, :]
    _, lse = O.latent_attention(q_abs, np.nan_to_num(c_ring), np.nan_to_num(kr_ring), mask, cfg.scale)
    return lse


def _run(V, cfg, batch, n_chunks, seed, first_frame=0, check_from=0, fused=None):
    """Stream n_chunks chunks starting at absolute frame first_frame; from chunk check_from on, attend
    with fresh queries and check cache planes, o (three-call path) and, for bf16, the fused call."""
    if fused is None:
        fused = cfg.dtype == VMLA_BF16
    inp = synthetic.draw_layer(cfg, batch=batch, seed=seed, n_chunks=0)
    orc = OracleLayer(cfg, inp, batch)
    orc.frames_written = first_frame
    cache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    cache.struct.frames_written = first_frame
    w, w_uk, w_uv = _to(inp.w_dkv_kr), _to(inp.w_uk), _to(inp.w_uv)
    for k in range(n_chunks):
        x, qn, qr = synthetic.draw_chunk(cfg, batch, seed * 31 + k)
        f0 = cache.frames_written
        V.compress_append(cfg, _to(x), w, cache)
        orc.append(x)
        if k < check_from:
            continue
        q_abs = V.absorb_q(cfg, _to(qn), _to(qr), w_uk, f0)
        o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, want_lse=True)
        o = V.value_up(cfg, o_lat, w_uv)
        o_f = V.latent_attention_fused(cfg, _to(qn), _to(qr), w_uk, w_uv, cache, f0) if fused else None
        torch.cuda.synchronize()
        assert V.device_status() == 0
        for b in range(batch):
            c_ref, kr_ref, written = orc.ring(b)
            assert_close(f64(cache.c[b])[written], c_ref[written], cfg, f"chunk {k} c b{b}")
            assert_close(f64(cache.k_r[b])[written], kr_ref[written], cfg, f"chunk {k} k_r b{b}")
            ref = orc.reference(b, qn, qr, f0)
            assert_close(f64(o[b]), ref["o"], cfg, f"chunk {k} o b{b}")
            # lse on the GPU's own stored (rounded) q_abs and ring: with one visible key lse is that key's
            # score, whose relative error after bf16 storage of its operands is not bounded by the output
            # tolerance, so the kernel's arithmetic is measured on its own inputs
            assert_close(f64(lse[b]), _isolated_lse(orc, cfg, f64(q_abs[b]), f64(cache.c[b]),
                                                    f64(cache.k_r[b]), f0), cfg, f"chunk {k} lse b{b}")
            if fused:
                assert_close(f64(o_f[b]), ref["o"], cfg, f"chunk {k} fused o b{b}")


@pytest.mark.parametrize("d_c", [192, 64])
def test_window_of_one_chunk(V, d_c):
    _run(V, MID.replace(window_frames=MID.chunk_frames, d_c=d_c), batch=2, n_chunks=3, seed=61)


def test_window_of_one_chunk_fp32(V):
    _run(V, TINY.replace(window_frames=1), batch=2, n_chunks=3, seed=62)


@pytest.mark.parametrize("d_c", [192, 64, 128])
def test_one_token_frames(V, d_c):
    """Three visible keys at most: at d_c = 64 / 128 the second key half of every tile is fully
    masked (that warpgroup keeps m = -inf and contributes nothing to the merge)."""
    cfg = MID.replace(grid_h=1, grid_w=1, chunk_frames=1, window_frames=3, d_c=d_c)
    _run(V, cfg, batch=3, n_chunks=5, seed=63)


def test_one_token_frames_fp32(V):
    _run(V, TINY.replace(grid_h=1, grid_w=1), batch=2, n_chunks=5, seed=64)


@pytest.mark.parametrize("first_frame", [999_999, 3_000_001])
def test_large_frame_index(V, first_frame):
    """Absolute frame indices far beyond any training length: keys are rotated once with their absolute
    index, queries likewise; the ring is filled before the first attention call."""
    cfg = MID
    n_fill = cfg.window_frames // cfg.chunk_frames + 1
    f0 = first_frame - first_frame % cfg.chunk_frames
    _run(V, cfg, batch=1, n_chunks=n_fill + 1, seed=65, first_frame=f0, check_from=n_fill)


def test_large_frame_index_fp32(V):
    cfg = TINY
    _run(V, cfg, batch=1, n_chunks=cfg.window_frames + 1, seed=66, first_frame=2_000_000,
         check_from=cfg.window_frames)


@pytest.mark.parametrize("d_c", [192, 64])
def test_whole_window_block_causal(V, d_c):
    """All W/F chunks of a window as one query set: chunk k sees chunks 0..k only."""
    cfg = MID.replace(window_frames=6, d_c=d_c)
    n = cfg.window_frames // cfg.chunk_frames
    inp = synthetic.draw_layer(cfg, batch=2, seed=67, n_chunks=n, n_query_chunks=n)
    orc = OracleLayer(cfg, inp, 2)
    cache = V.LatentCache(cfg, 2, device=DEV, fill=float("nan"))
    for x in inp.x_chunks:
        V.compress_append(cfg, _to(x), _to(inp.w_dkv_kr), cache)
        orc.append(x)
    args = (_to(inp.q_nope), _to(inp.q_rope), _to(inp.w_uk), _to(inp.w_uv))
    q_abs = V.absorb_q(cfg, args[0], args[1], args[2], 0, n_query_chunks=n)
    o = V.value_up(cfg, V.latent_attention(cfg, q_abs, cache, 0, n_query_chunks=n), args[3])
    o_f = V.latent_attention_fused(cfg, *args, cache, 0, n_query_chunks=n)
    torch.cuda.synchronize()
    for b in range(2):
        ref = orc.reference(b, inp.q_nope, inp.q_rope, 0)
        assert_close(f64(o[b]), ref["o"], cfg, f"o b{b}")
        assert_close(f64(o_f[b]), ref["o"], cfg, f"fused o b{b}")
        # the first chunk's rows see only the first chunk's keys
        assert ref["mask"][0].sum() == cfg.chunk_tokens


def test_batch_of_sixteen(V):
    cfg = MID.replace(grid_h=3, grid_w=8)
    _run(V, cfg, batch=16, n_chunks=3, seed=68, check_from=2)
