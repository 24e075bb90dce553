"""Seeded sweep over layer shapes: for each drawn configuration, stream chunks through the ring until it
wraps and check every call of the bf16 path against the float64 oracle on the same inputs.

Each case draws the latent rank d_c in {64, 128, 192, 256} (both attention kernels and, where the fused
call supports the shapes, both fused kernels), the per-head sizes d_nope and d_v, 1-5 heads, a frame
grid of 3-9 x 5-17 tokens (ragged query and key tiles), 1-3 frames per chunk, a window of chunk + 1 to
7 frames, a model width D that is a multiple of 8 but not always of the 64-column k-tile, a 3D-RoPE pair
split, and a batch of 1-3.  Per streamed chunk: the ring planes (every row, including the not yet
written NaN-filled ones), the absorbed queries, the latent output, the log-sum-exp and the final output
of the three-call path, and the fused call's output and log-sum-exp.  On the last chunk, where the
head shapes allow the dense kernel (d_h = d_v = 128), the dense layer built from the latent weights is
checked as well (VideoMLA technical summary, Method items 1-4: the absorbed form equals per-head
attention with W_K,h = [W^K_up,h W^KV_down ; W^KR], W_V,h = W^V_up,h W^KV_down)."""
import numpy as np
import pytest
import torch

from rank_latent_kv_vmla_b200.config import VMLA_BF16, VmlaConfig
import synthetic
from parity import (OracleLayer, assert_close, dense_weights_from_latent, errors, f64, paths_rel_tol,
                    round_to, sample_rows)

DEV = "cuda"
N_CASES = 24


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from rank_latent_kv_vmla_b200 import vmla
    return vmla


def _to(t):
    return t.to(DEV).contiguous()


def draw_config(case: int):
    """Configuration and batch of sweep case `case` (a pure function of the index)."""
    r = np.random.default_rng(9000 + case)
    d_c = int((64, 128, 192, 256)[case % 4])
    d_nope = int(r.choice([32, 64, 96, 128]))
    d_v = int(r.choice([64, 128]))
    if case % 3 == 0:                       # every third case has the dense kernel's head shapes
        d_nope, d_v = 96, 128
    chunk = int(r.integers(1, 4))
    window = int(r.integers(chunk + 1, 8))
    pt = int(r.integers(1, 15))
    ph = int(r.integers(1, 16 - pt))
    cfg = VmlaConfig(dim=int(r.choice([192, 200, 256, 328])), n_heads=int(r.integers(1, 6)), d_nope=d_nope,
                     d_rope=32, d_c=d_c, d_v=d_v, grid_h=int(r.integers(3, 10)), grid_w=int(r.integers(5, 18)),
                     chunk_frames=chunk, window_frames=window, rope_pairs_t=pt, rope_pairs_h=ph,
                     rope_pairs_w=16 - pt - ph, dtype=VMLA_BF16)
    return cfg, int(r.integers(1, 4))


def test_sweep_configs_are_valid_and_varied():
    cfgs = [draw_config(i)[0] for i in range(N_CASES)]
    assert {c.d_c for c in cfgs} == {64, 128, 192, 256}
    assert any(c.dim % 64 for c in cfgs)                       # a ragged reduction tile
    assert any(c.chunk_tokens % 128 for c in cfgs)
    for c in cfgs:
        assert c.rope_pairs_t + c.rope_pairs_h + c.rope_pairs_w == c.d_rope // 2
        assert min(c.rope_pairs_t, c.rope_pairs_h, c.rope_pairs_w) >= 1
        assert c.window_frames > c.chunk_frames


@pytest.mark.gpu
@pytest.mark.parametrize("case", range(N_CASES))
def test_sweep_case_against_oracle(V, case):
    cfg, batch = draw_config(case)
    n_steps = cfg.window_frames // cfg.chunk_frames + 2        # the ring wraps at least once
    inp = synthetic.draw_layer(cfg, batch=batch, seed=7100 + case, n_chunks=n_steps)
    orc = OracleLayer(cfg, inp, batch)
    cache = V.LatentCache(cfg, batch, device=DEV, fill=float("nan"))
    w, w_uk, w_uv = _to(inp.w_dkv_kr), _to(inp.w_uk), _to(inp.w_uv)
    fused = V.fused_supported(cfg)
    rows = None if cfg.chunk_tokens <= 160 else sample_rows(cfg, cfg.chunk_tokens, n=48)
    sel = slice(None) if rows is None else rows
    tag = (f"case {case}: d_c {cfg.d_c} d_nope {cfg.d_nope} d_v {cfg.d_v} H {cfg.n_heads} D {cfg.dim} "
           f"grid {cfg.grid_h}x{cfg.grid_w} F {cfg.chunk_frames} W {cfg.window_frames} B {batch}")
    for k in range(n_steps):
        f0 = cache.frames_written
        V.compress_append(cfg, _to(inp.x_chunks[k]), w, cache)
        orc.append(inp.x_chunks[k])
        qn, qr = synthetic.draw_queries(cfg, batch, 7100 * 100 + case * 10 + k)
        q_abs = V.absorb_q(cfg, _to(qn), _to(qr), w_uk, f0)
        o_lat, lse = V.latent_attention(cfg, q_abs, cache, f0, want_lse=True)
        o = V.value_up(cfg, o_lat, w_uv)
        if fused:
            o_f, lse_f = V.latent_attention_fused(cfg, _to(qn), _to(qr), w_uk, w_uv, cache, f0, want_lse=True)
        torch.cuda.synchronize()
        assert V.device_status() == 0, tag
        q_ref = orc.q_abs(qn, qr, f0)
        for b in sorted({0, batch - 1}):
            c_ref, kr_ref, written = orc.ring(b)
            got_c, got_kr = f64(cache.c[b]), f64(cache.k_r[b])
            assert np.isnan(got_c[~written]).all(), f"{tag} step {k}: a ring row outside the written frames changed"
            assert_close(got_c[written], c_ref[written], cfg, f"{tag} step {k} c plane b{b}")
            assert_close(got_kr[written], kr_ref[written], cfg, f"{tag} step {k} k_r plane b{b}")
            assert_close(f64(q_abs[b]), q_ref[b], cfg, f"{tag} step {k} q_abs b{b}")
            ref = orc.reference(b, qn, qr, f0, rows=rows)
            assert_close(f64(o_lat[b][sel]), ref["o_latent"], cfg, f"{tag} step {k} o_latent b{b}")
            assert_close(f64(lse[b][sel]), ref["lse"], cfg, f"{tag} step {k} lse b{b}")
            assert_close(f64(o[b][sel]), ref["o"], cfg, f"{tag} step {k} o b{b}")
            if fused:
                assert_close(f64(o_f[b][sel]), ref["o"], cfg, f"{tag} step {k} fused o b{b}")
                assert_close(f64(lse_f[b][sel]), ref["lse"], cfg, f"{tag} step {k} fused lse b{b}")
                rel_l2, _ = errors(f64(o_f[b]), f64(o[b]))
                assert rel_l2 <= paths_rel_tol(cfg), f"{tag} step {k}: fused vs three calls rel-L2 {rel_l2:.2e}"
    if cfg.d_nope + cfg.d_rope == 128 and cfg.d_v == 128:
        # the dense comparison layer built from the latent weights, fed the same chunks
        w_kv = _to(round_to(cfg, dense_weights_from_latent(inp, cfg)))
        dcache = V.DenseCache(cfg, batch, device=DEV, fill=float("nan"))
        for x in inp.x_chunks:
            fd = dcache.frames_written
            V.dense_append(cfg, _to(x), w_kv, dcache)
        q = V.rope_q(cfg, _to(qn), _to(qr), fd)
        o_d, lse_d = V.dense_mha(cfg, q, dcache, fd, want_lse=True)
        torch.cuda.synchronize()
        assert V.device_status() == 0, tag
        for b in sorted({0, batch - 1}):
            ref = orc.reference(b, qn, qr, fd, rows=rows)
            assert_close(f64(o_d[b][sel]), ref["o"], cfg, f"{tag} dense o b{b}")
            assert_close(f64(lse_d[b][sel]), ref["lse"], cfg, f"{tag} dense lse b{b}")
