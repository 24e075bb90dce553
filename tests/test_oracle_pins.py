"""Pins of the float64 oracle against what the VideoMLA pages and the mathematics fix.

Each test checks the oracle against something other than itself: figures printed on the pages
(tests/golden/paper_figures.json), closed forms, the textbook complex-number form of 1-D RoPE,
brute-force scalar loops on tiny inputs, an operational simulation of the streaming window, and
torch's float64 scaled_dot_product_attention for the MLA == MHA identity.
"""
import itertools
import json
import math
import os
from collections import deque

import numpy as np
import pytest
import torch

from oracle import vmla_oracle as O
from rank_latent_kv_vmla_b200.config import TINY, WAN
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paper_figures.json")


def _tiny_kwargs(cfg):
    return dict(d_c=cfg.d_c, d_rope=cfg.d_rope, chunk_frames=cfg.chunk_frames, grid_h=cfg.grid_h,
                grid_w=cfg.grid_w, pairs=(cfg.rope_pairs_t, cfg.rope_pairs_h, cfg.rope_pairs_w),
                theta=cfg.rope_theta)


def _f64(t):
    return t.double().numpy()


# ------------------------------------------------------------------------------------------------
# Cache arithmetic printed on the pages
# ------------------------------------------------------------------------------------------------
def test_cache_arithmetic_matches_printed_figures():
    g = json.load(open(GOLDEN))
    n_h, d_h, d_c, d_r = g["n_heads"]["value"], g["d_h"]["value"], g["d_c"]["value"], g["d_rope"]["value"]
    assert n_h * d_h == g["per_head_k_scalars_all_heads"]["value"]
    assert O.dense_scalars_per_token(n_h, d_h) == 3072
    assert O.latent_scalars_per_token(d_c, d_r) == 224
    red = 100.0 * O.memory_reduction(n_h, d_h, d_c, d_r)
    assert round(red, g["reduction_percent"]["decimals"]) == g["reduction_percent"]["value"]
    # ~6.0 GB dense cache for 21 latent frames of Wan-1.3B under the stated reading
    tokens = 21 * 30 * 52
    gb = 30 * tokens * O.dense_scalars_per_token(n_h, d_h) * 2 / 1e9
    assert round(gb, 1) == g["dense_cache_gb_21_frames"]["value"]
    # the config presets carry the same figures
    assert WAN.dense_scalars_per_token() == 3072 and WAN.latent_scalars_per_token() == 224


def test_memory_reduction_changes_with_each_term():
    base = O.memory_reduction(12, 128, 192, 32)
    assert O.memory_reduction(12, 128, 128, 32) > base      # smaller latent -> larger saving
    assert O.memory_reduction(12, 128, 192, 64) < base      # larger rope key -> smaller saving
    assert O.memory_reduction(24, 128, 192, 32) > base      # more heads in the dense layout
    assert O.memory_reduction(12, 64, 192, 32) < base       # narrower heads


# ------------------------------------------------------------------------------------------------
# Positions
# ------------------------------------------------------------------------------------------------
def test_token_positions_raster_enumeration():
    gh, gw, f0, nframes = 3, 5, 7, 2
    expect = [(f, i, j) for f in range(f0, f0 + nframes) for i in range(gh) for j in range(gw)]
    got = O.token_positions(f0, nframes * gh * gw, gh, gw)
    assert [tuple(r) for r in got.tolist()] == expect


# ------------------------------------------------------------------------------------------------
# 3D-RoPE
# ------------------------------------------------------------------------------------------------
def test_rope_hand_values():
    # pairs (2, 1, 1), theta = 1e4: frame pairs turn at 1 and 1e4^(-1/2) = 0.01; row and column at 1
    u = np.array([1.0, 0.0] * 4)
    out = O.rope3d(u, np.array([3, 2, 1]), (2, 1, 1), 1e4)
    expect = [math.cos(3), math.sin(3), math.cos(0.03), math.sin(0.03),
              math.cos(2), math.sin(2), math.cos(1), math.sin(1)]
    np.testing.assert_allclose(out, expect, rtol=0, atol=1e-15)
    # the second component of a pair turns the same way: (0, 1) -> (-sin, cos)
    out2 = O.rope3d(np.array([0.0, 1.0] * 4), np.array([3, 2, 1]), (2, 1, 1), 1e4)
    np.testing.assert_allclose(out2[0:2], [-math.sin(3), math.cos(3)], atol=1e-15)


def test_rope_single_axis_is_textbook_1d_rope():
    """With all pairs on the frame axis, 3D-RoPE is 1-D RoPE: pair m is the complex number
    u[2m] + i u[2m+1] multiplied by exp(i * pos * theta^(-2m/d))."""
    rng = np.random.default_rng(0)
    d = 16
    u = rng.standard_normal((5, d))
    pos = np.array([[0, 0, 0], [1, 0, 0], [7, 0, 0], [100, 0, 0], [12345, 0, 0]])
    got = O.rope3d(u, pos, (d // 2, 0, 0), 10000.0)
    z = u[:, 0::2] + 1j * u[:, 1::2]
    m = np.arange(d // 2)
    zr = z * np.exp(1j * pos[:, :1] * 10000.0 ** (-2.0 * m / d))
    np.testing.assert_allclose(got[:, 0::2], zr.real, atol=1e-12)
    np.testing.assert_allclose(got[:, 1::2], zr.imag, atol=1e-12)


def test_rope_zero_position_identity_and_norm():
    rng = np.random.default_rng(1)
    u = rng.standard_normal((50, 32))
    pairs = (6, 5, 5)
    np.testing.assert_array_equal(O.rope3d(u, np.zeros(3, dtype=np.int64), pairs, 1e4), u)
    pos = rng.integers(0, 300, size=(50, 3))
    r = O.rope3d(u, pos, pairs, 1e4)
    # each pair keeps its length (a rotation), hence the vector keeps its norm
    np.testing.assert_allclose(np.hypot(r[:, 0::2], r[:, 1::2]), np.hypot(u[:, 0::2], u[:, 1::2]),
                               rtol=1e-13)


def test_rope_relative_position_invariance():
    """q(p) . k(p') depends only on p - p': shifting both positions by any (df, di, dj) leaves it."""
    rng = np.random.default_rng(2)
    pairs = (6, 5, 5)
    q = rng.standard_normal((200, 32))
    k = rng.standard_normal((200, 32))
    pq = rng.integers(0, 60, size=(200, 3))
    pk = rng.integers(0, 60, size=(200, 3))
    s0 = np.sum(O.rope3d(q, pq, pairs, 1e4) * O.rope3d(k, pk, pairs, 1e4), axis=-1)
    for shift in ([5, 0, 0], [0, 3, 0], [0, 0, 11], [17, -4, 9]):
        sh = np.array(shift)
        s1 = np.sum(O.rope3d(q, pq + sh, pairs, 1e4) * O.rope3d(k, pk + sh, pairs, 1e4), axis=-1)
        np.testing.assert_allclose(s1, s0, rtol=1e-10, atol=1e-10)
    # and it is not invariant to a shift of only one side (so the test can fail)
    s2 = np.sum(O.rope3d(q, pq + np.array([1, 1, 1]), pairs, 1e4) * O.rope3d(k, pk, pairs, 1e4), axis=-1)
    assert np.max(np.abs(s2 - s0)) > 1e-2


def test_rope_axis_blocks_follow_t_h_w_order():
    """Moving only the row index turns only the P_h row pairs (pairs P_t .. P_t+P_h-1)."""
    u = np.ones(32)
    pairs = (6, 5, 5)
    base = O.rope3d(u, np.array([4, 2, 9]), pairs, 1e4)
    moved = O.rope3d(u, np.array([4, 3, 9]), pairs, 1e4)
    changed = np.nonzero(np.abs(moved - base) > 1e-14)[0] // 2
    assert set(changed.tolist()) == set(range(6, 11))


# ------------------------------------------------------------------------------------------------
# Compression, cache and sliding window (brute force)
# ------------------------------------------------------------------------------------------------
def test_compress_against_scalar_loops():
    cfg = TINY
    inp = synthetic.draw_layer(cfg, batch=1, seed=11, n_chunks=1)
    x = _f64(inp.x_chunks[0][0])
    w = _f64(inp.w_dkv_kr)
    pos = O.token_positions(5, x.shape[0], cfg.grid_h, cfg.grid_w)
    pairs = (cfg.rope_pairs_t, cfg.rope_pairs_h, cfg.rope_pairs_w)
    c, k_r = O.compress(x, w, cfg.d_c, pos, pairs, cfg.rope_theta)
    for t in range(x.shape[0]):
        for r in range(cfg.d_c):
            ref = sum(w[r, d] * x[t, d] for d in range(cfg.dim))
            assert abs(c[t, r] - ref) < 1e-12
        raw = [sum(w[cfg.d_c + r, d] * x[t, d] for d in range(cfg.dim)) for r in range(cfg.d_rope)]
        f, i, j = pos[t]
        axis_pos = [f] * cfg.rope_pairs_t + [i] * cfg.rope_pairs_h + [j] * cfg.rope_pairs_w
        local = list(range(cfg.rope_pairs_t)) + list(range(cfg.rope_pairs_h)) + list(range(cfg.rope_pairs_w))
        size = [cfg.rope_pairs_t] * cfg.rope_pairs_t + [cfg.rope_pairs_h] * cfg.rope_pairs_h + \
               [cfg.rope_pairs_w] * cfg.rope_pairs_w
        for p in range(cfg.d_rope // 2):
            ang = axis_pos[p] * cfg.rope_theta ** (-local[p] / size[p])
            a, b = raw[2 * p], raw[2 * p + 1]
            assert abs(k_r[t, 2 * p] - (a * math.cos(ang) - b * math.sin(ang))) < 1e-12
            assert abs(k_r[t, 2 * p + 1] - (a * math.sin(ang) + b * math.cos(ang))) < 1e-12


def test_ring_matches_explicit_ring_writes():
    """Append 6 one-frame chunks into a 3-frame window: the expected ring equals an explicit ring that
    writes frame f into slot f mod W (evicting f - W), checked after every append."""
    W, T, d = 3, 4, 2
    hist = np.arange(6 * T * d, dtype=np.float64).reshape(6 * T, d)
    ring = np.full((W * T, d), np.nan)
    for fw in range(1, 7):
        f = fw - 1
        s = f % W
        ring[s * T:(s + 1) * T] = hist[f * T:(f + 1) * T]
        plane, written = O.ring_from_history(hist[:fw * T], fw, W, T)
        np.testing.assert_array_equal(np.isnan(plane[:, 0]), np.isnan(ring[:, 0]))
        np.testing.assert_array_equal(plane[written], ring[written])
        assert written.sum() == min(fw, W) * T
    assert [O.frame_of_slot(s, 6, W) for s in range(W)] == [3, 4, 5]
    assert [O.frame_of_slot(s, 2, W) for s in range(W)] == [0, 1, -1]
    assert O.frame_of_slot(0, 0, W) == -1
    # a history that starts at a late absolute frame F0: the same explicit ring, slots by f mod W
    F0 = 1_000_004
    ring = np.full((W * T, d), np.nan)
    for fw in range(F0 + 1, F0 + 6):
        f = fw - 1
        s = f % W
        r = f - F0
        ring[s * T:(s + 1) * T] = hist[r * T:(r + 1) * T]
        plane, written = O.ring_from_history(hist[:(fw - F0) * T], fw, W, T, first_frame=F0)
        np.testing.assert_array_equal(np.isnan(plane[:, 0]), np.isnan(ring[:, 0]))
        np.testing.assert_array_equal(plane[written], ring[written])
        assert written.sum() == min(fw - F0, W) * T


def test_window_mask_matches_streaming_simulation():
    """The block-causal + window mask equals what a streaming generator sees: chunk k attends, right
    after appending its own frames, to exactly the frames held in a W-frame sliding window."""
    F, T = 2, 3
    for W in (2, 3, 4, 5, 8, 20):
        n_chunks = 5
        key_frames = np.repeat(np.arange(n_chunks * F), T)
        hi = O.query_chunk_end(0, n_chunks * F * T, F, T)
        mask = O.visible(hi, key_frames, W)
        window = deque(maxlen=W)
        for k in range(n_chunks):
            for f in range(k * F, (k + 1) * F):
                window.append(f)
            allowed = set(window)
            rows = range(k * F * T, (k + 1) * F * T)
            for n in rows:
                got = {int(key_frames[t]) for t in np.nonzero(mask[n])[0]}
                assert got == allowed, (W, k, n)


# ------------------------------------------------------------------------------------------------
# Attention: brute force, special cases, absorbed == reconstructed, MLA == MHA (library routine)
# ------------------------------------------------------------------------------------------------
def _tiny_history(cfg, seed, n_chunks, q_gain=1.0):
    inp = synthetic.draw_layer(cfg, batch=1, seed=seed, n_chunks=n_chunks, q_gain=q_gain)
    hist = O.build_history([_f64(x) for x in inp.x_chunks], _f64(inp.w_dkv_kr), 0, **_tiny_kwargs(cfg))
    return inp, hist


def _ref(cfg, inp, hist, first_frame, rows=None, q_nope=None, q_rope=None):
    qn = _f64(inp.q_nope[0]) if q_nope is None else q_nope
    qr = _f64(inp.q_rope[0]) if q_rope is None else q_rope
    rows = np.arange(qn.shape[0]) if rows is None else rows
    return O.layer_reference(hist, qn, qr, _f64(inp.w_uk), _f64(inp.w_uv), first_frame=first_frame,
                             query_rows=rows, chunk_frames=cfg.chunk_frames,
                             window_frames=cfg.window_frames, grid_h=cfg.grid_h, grid_w=cfg.grid_w,
                             pairs=(cfg.rope_pairs_t, cfg.rope_pairs_h, cfg.rope_pairs_w),
                             theta=cfg.rope_theta, scale=cfg.scale)


def test_attention_against_scalar_loops():
    cfg = TINY
    n_chunks = 5                     # frames 0..4, window 3: frames 0, 1 evicted
    inp, hist = _tiny_history(cfg, 21, n_chunks)
    f0 = (n_chunks - 1) * cfg.chunk_frames
    ref = _ref(cfg, inp, hist, f0)
    qn, qr = _f64(inp.q_nope[0]), _f64(inp.q_rope[0])
    wuk, wuv = _f64(inp.w_uk), _f64(inp.w_uv)
    T = cfg.tokens_per_frame
    for n in range(qn.shape[0]):
        f, i, j = f0 + n // T, (n % T) // cfg.grid_w, n % cfg.grid_w
        for h in range(cfg.n_heads):
            # rotate the query by explicit pair loops
            qrot = []
            for p in range(cfg.d_rope // 2):
                if p < cfg.rope_pairs_t:
                    ang = f * cfg.rope_theta ** (-p / cfg.rope_pairs_t)
                elif p < cfg.rope_pairs_t + cfg.rope_pairs_h:
                    ang = i * cfg.rope_theta ** (-(p - cfg.rope_pairs_t) / cfg.rope_pairs_h)
                else:
                    ang = j * cfg.rope_theta ** (-(p - cfg.rope_pairs_t - cfg.rope_pairs_h) / cfg.rope_pairs_w)
                a, b = qr[n, h, 2 * p], qr[n, h, 2 * p + 1]
                qrot += [a * math.cos(ang) - b * math.sin(ang), a * math.sin(ang) + b * math.cos(ang)]
            scores, vals = [], []
            for t in range(hist.c.shape[0]):
                kf = hist.frames[t]
                if not (f0 + cfg.chunk_frames - cfg.window_frames <= kf < f0 + cfg.chunk_frames):
                    continue
                knope = [sum(wuk[h, r, m] * hist.c[t, m] for m in range(cfg.d_c)) for r in range(cfg.d_nope)]
                s = sum(qn[n, h, r] * knope[r] for r in range(cfg.d_nope))
                s += sum(qrot[r] * hist.k_r[t, r] for r in range(cfg.d_rope))
                scores.append(s * cfg.scale)
                vals.append([sum(wuv[h, r, m] * hist.c[t, m] for m in range(cfg.d_c)) for r in range(cfg.d_v)])
            mx = max(scores)
            e = [math.exp(s - mx) for s in scores]
            z = sum(e)
            o = [sum(e[t] * vals[t][r] for t in range(len(e))) / z for r in range(cfg.d_v)]
            np.testing.assert_allclose(ref["o"][n, h], o, rtol=1e-11, atol=1e-12)
            assert abs(ref["lse"][n, h] - (math.log(z) + mx)) < 1e-11
        assert len(scores) == cfg.window_frames * T


def test_softmax_rows_sum_to_one_and_lse():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((7, 3, 8))
    k = rng.standard_normal((20, 3, 8))
    v = rng.standard_normal((20, 3, 4))
    mask = rng.random((7, 20)) < 0.6
    mask[:, 0] = True
    o, lse, p = O.mha(q, k, v, mask, 0.3)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-14)
    assert np.all(p[np.broadcast_to(~mask[:, None, :], p.shape)] == 0)
    s = np.einsum('nhd,thd->nht', q, k) * 0.3
    np.testing.assert_allclose(lse, np.log(np.sum(np.where(mask[:, None, :], np.exp(s), 0), -1)), rtol=1e-13)


def test_single_visible_key_returns_its_value():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((4, 2, 8)) * 30.0
    k = rng.standard_normal((9, 2, 8))
    v = rng.standard_normal((9, 2, 5))
    mask = np.zeros((4, 9), dtype=bool)
    mask[np.arange(4), [0, 3, 8, 5]] = True
    o, _, _ = O.mha(q, k, v, mask, 1.0)
    np.testing.assert_allclose(o, v[[0, 3, 8, 5]], rtol=1e-14)


def test_zero_query_gives_mean_of_visible_values():
    cfg = TINY
    inp, hist = _tiny_history(cfg, 31, 4)
    f0 = 3 * cfg.chunk_frames
    qn = np.zeros_like(_f64(inp.q_nope[0]))
    qr = np.zeros_like(_f64(inp.q_rope[0]))
    ref = _ref(cfg, inp, hist, f0, q_nope=qn, q_rope=qr)
    vis = (hist.frames >= f0 + 1 - cfg.window_frames) & (hist.frames < f0 + 1)
    v = np.einsum('hvc,tc->thv', _f64(inp.w_uv), hist.c[vis])
    np.testing.assert_allclose(ref["o"], np.broadcast_to(v.mean(0), ref["o"].shape), rtol=1e-12)
    np.testing.assert_allclose(ref["o_latent"], np.broadcast_to(hist.c[vis].mean(0), ref["o_latent"].shape),
                               rtol=1e-12)


@pytest.mark.parametrize("q_gain", [1.0, 8.0])
def test_absorbed_equals_reconstructed(q_gain):
    cfg = TINY
    inp, hist = _tiny_history(cfg, 41, 4, q_gain=q_gain)
    f0 = 3 * cfg.chunk_frames
    ref = _ref(cfg, inp, hist, f0)
    o_lat, lse = O.latent_attention(ref["q_abs"], hist.c, hist.k_r, ref["mask"], cfg.scale)
    np.testing.assert_allclose(o_lat, ref["o_latent"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, ref["lse"], rtol=1e-12)
    np.testing.assert_allclose(O.value_up(o_lat, _f64(inp.w_uv)), ref["o"], rtol=1e-11, atol=1e-13)


def test_mla_equals_textbook_mha_via_torch_sdpa():
    """With dense per-head weights built as W_K,h = [W^K_up,h W^KV_down ; W^KR] (rope rows rotated)
    and W_V,h = W^V_up,h W^KV_down, the MLA layer is ordinary MHA: compare against torch's float64
    scaled_dot_product_attention (default scale 1/sqrt(d_h)) with an explicit boolean mask."""
    cfg = TINY.replace(window_frames=2, chunk_frames=1)
    n_chunks = 4
    inp, hist = _tiny_history(cfg, 51, n_chunks)
    f0 = (n_chunks - 1) * cfg.chunk_frames
    ref = _ref(cfg, inp, hist, f0)

    w = torch.from_numpy(_f64(inp.w_dkv_kr))
    w_dkv, w_kr = w[:cfg.d_c], w[cfg.d_c:]
    wuk, wuv = torch.from_numpy(_f64(inp.w_uk)), torch.from_numpy(_f64(inp.w_uv))
    xs = torch.cat([torch.from_numpy(_f64(x[0])) for x in inp.x_chunks])          # [T_all, D]
    pairs = (cfg.rope_pairs_t, cfg.rope_pairs_h, cfg.rope_pairs_w)
    pos_k = np.concatenate([O.token_positions(k * cfg.chunk_frames, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)
                            for k in range(n_chunks)])
    k_heads, v_heads = [], []
    for h in range(cfg.n_heads):
        wk_h = wuk[h] @ w_dkv                                                       # [d_nope, D]
        k_nope = xs @ wk_h.T
        k_rope = torch.from_numpy(O.rope3d((xs @ w_kr.T).numpy(), pos_k, pairs, cfg.rope_theta))
        k_heads.append(torch.cat([k_nope, k_rope], -1))
        v_heads.append(xs @ (wuv[h] @ w_dkv).T)
    K = torch.stack(k_heads, 0)                                                     # [H, T, d_h]
    V = torch.stack(v_heads, 0)
    pos_q = O.token_positions(f0, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)
    q_rot = O.rotate_query(_f64(inp.q_rope[0]), pos_q, pairs, cfg.rope_theta)
    Q = torch.cat([torch.from_numpy(_f64(inp.q_nope[0])), torch.from_numpy(q_rot)], -1).transpose(0, 1)
    key_frames = torch.from_numpy(pos_k[:, 0])
    allowed = (key_frames >= f0 + cfg.chunk_frames - cfg.window_frames) & (key_frames < f0 + cfg.chunk_frames)
    attn_mask = allowed[None, None, :].expand(cfg.n_heads, cfg.chunk_tokens, -1)
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=attn_mask)
    np.testing.assert_allclose(ref["o"], o.transpose(0, 1).numpy(), rtol=1e-10, atol=1e-12)


def test_streaming_calls_equal_one_block_causal_call():
    """With a window that holds every frame, one call over 4 chunks (block-causal) equals 4 streaming
    calls, each made right after appending its own chunk."""
    cfg = TINY.replace(window_frames=8)
    n_chunks = 4
    inp = synthetic.draw_layer(cfg, batch=1, seed=61, n_chunks=n_chunks, n_query_chunks=n_chunks)
    hist = O.build_history([_f64(x) for x in inp.x_chunks], _f64(inp.w_dkv_kr), 0, **_tiny_kwargs(cfg))
    qn, qr = _f64(inp.q_nope[0]), _f64(inp.q_rope[0])
    whole = _ref(cfg, inp, hist, 0, q_nope=qn, q_rope=qr)
    per = cfg.chunk_tokens
    for k in range(n_chunks):
        part = O.build_history([_f64(x) for x in inp.x_chunks[:k + 1]], _f64(inp.w_dkv_kr), 0, **_tiny_kwargs(cfg))
        one = _ref(cfg, inp, part, k * cfg.chunk_frames, q_nope=qn[k * per:(k + 1) * per],
                   q_rope=qr[k * per:(k + 1) * per])
        np.testing.assert_allclose(whole["o"][k * per:(k + 1) * per], one["o"], rtol=1e-12, atol=1e-14)
    # chunk 0 sees only itself; the last chunk sees everything
    assert whole["mask"][0].sum() == per and whole["mask"][-1].sum() == n_chunks * per


def test_layer_reference_row_sampling_is_consistent():
    cfg = TINY
    inp, hist = _tiny_history(cfg, 71, 3)
    full = _ref(cfg, inp, hist, 2)
    rows = np.array([0, 5, 15])
    part = _ref(cfg, inp, hist, 2, rows=rows)
    for key in ("o", "o_latent", "lse", "q_abs"):
        np.testing.assert_array_equal(part[key], full[key][rows])


# ------------------------------------------------------------------------------------------------
# Few-step generation: in-place rewrite of the newest chunk
# ------------------------------------------------------------------------------------------------
def test_rewrite_newest_equals_history_built_with_that_chunk():
    """Rewriting the newest chunk with x' gives exactly the history built from the chunk list whose last
    entry is x'; rewriting with the same x changes nothing; only the newest tokens can be rewritten."""
    cfg = TINY
    inp = synthetic.draw_layer(cfg, batch=1, seed=91, n_chunks=5)
    xs = [_f64(x) for x in inp.x_chunks]
    w = _f64(inp.w_dkv_kr)
    kw = _tiny_kwargs(cfg)
    hist = O.build_history(xs[:4], w, 0, **kw)
    before_c, before_k = hist.c.copy(), hist.k_r.copy()
    pos = O.token_positions(3 * cfg.chunk_frames, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)
    c, k_r = O.compress(xs[3][0], w, cfg.d_c, pos, kw["pairs"], cfg.rope_theta)
    hist.rewrite_newest(c, k_r, pos[:, 0])
    np.testing.assert_array_equal(hist.c, before_c)
    np.testing.assert_array_equal(hist.k_r, before_k)
    c2, k2 = O.compress(xs[4][0], w, cfg.d_c, pos, kw["pairs"], cfg.rope_theta)
    hist.rewrite_newest(c2, k2, pos[:, 0])
    other = O.build_history(xs[:3] + [xs[4]], w, 0, **kw)
    np.testing.assert_array_equal(hist.c, other.c)
    np.testing.assert_array_equal(hist.k_r, other.k_r)
    np.testing.assert_array_equal(hist.frames, other.frames)
    n = cfg.chunk_tokens
    np.testing.assert_array_equal(hist.c[:-n], before_c[:-n])
    old_pos = O.token_positions(2 * cfg.chunk_frames, n, cfg.grid_h, cfg.grid_w)
    with pytest.raises(ValueError):
        hist.rewrite_newest(c2, k2, old_pos[:, 0])


# ------------------------------------------------------------------------------------------------
# Batch capacity at a fixed memory budget
# ------------------------------------------------------------------------------------------------
def _wan_capacity_kwargs(**over):
    kw = dict(n_layers=30, window_tokens=WAN.window_tokens, elt_bytes=2, fixed_bytes=0,
              extra_bytes_per_seq=0, dim=WAN.dim, n_heads=WAN.n_heads, d_nope=WAN.d_nope,
              d_rope=WAN.d_rope, d_c=WAN.d_c, d_v=WAN.d_v, tokens_per_chunk=WAN.chunk_tokens)
    kw.update(over)
    return kw


def test_capacity_cache_terms_match_printed_figures():
    """The per-sequence growth of memory_bytes, less one layer step's tensors, is the cache: the dense
    one is the printed ~6.0 GB (30 layers, bf16, 21 frames), the latent one 7.3 % of it (92.7 %)."""
    g = json.load(open(GOLDEN))
    per_seq = {}
    for dense in (False, True):
        kw = _wan_capacity_kwargs(dense=dense)
        grow = O.memory_bytes(2, **kw) - O.memory_bytes(1, **kw)
        step = (O.memory_bytes(1, **kw) - O.memory_bytes(0, **kw)) - grow    # 0: linear in the batch
        assert step == 0
        shape = {k: kw[k] for k in ("dim", "n_heads", "d_nope", "d_rope", "d_c", "d_v", "tokens_per_chunk")}
        tensors = sum(int(np.prod(v)) for v in O.step_tensors(1, dense=dense, **shape).values()) * 2
        per_seq[dense] = grow - tensors
    assert round(per_seq[True] / 1e9, 1) == g["dense_cache_gb_21_frames"]["value"]
    red = 100 * (1 - per_seq[False] / per_seq[True])
    assert round(red, 1) == g["reduction_percent"]["value"]
    # the printed batch ratios lie below the cache-only ratio 3072 / 224
    assert g["batch_ratio_dc192"]["value"] < per_seq[True] / per_seq[False]
    assert g["batch_ratio_lower_dc_max"]["value"] < 3072 / (64 + 32)


def test_capacity_search_is_exact_and_matches_a_linear_scan():
    kw = _wan_capacity_kwargs(fixed_bytes=3_000_000_000, extra_bytes_per_seq=123_456_789)
    for dense in (False, True):
        for k in (0, 1, 7, 29, 300):
            exact = O.memory_bytes(k, dense=dense, **kw)
            assert O.batch_capacity(exact, dense=dense, **kw) == k
            if k > 0:
                assert O.batch_capacity(exact - 1, dense=dense, **kw) == k - 1
    assert O.batch_capacity(O.memory_bytes(0, dense=False, **kw) - 1, dense=False, **kw) == 0
    tiny = dict(n_layers=2, window_tokens=TINY.window_tokens, elt_bytes=4, fixed_bytes=1000,
                extra_bytes_per_seq=10, dim=TINY.dim, n_heads=TINY.n_heads, d_nope=TINY.d_nope,
                d_rope=TINY.d_rope, d_c=TINY.d_c, d_v=TINY.d_v, tokens_per_chunk=TINY.chunk_tokens)
    for dense in (False, True):
        for budget in range(0, 400_000, 9_973):
            scan = 0
            while O.memory_bytes(scan + 1, dense=dense, **tiny) <= budget:
                scan += 1
            if O.memory_bytes(0, dense=dense, **tiny) > budget:
                scan = 0
            assert O.batch_capacity(budget, dense=dense, **tiny) == scan


def test_capacity_grows_as_the_latent_shrinks():
    caps = [O.batch_capacity(180 * 10**9, dense=False, **_wan_capacity_kwargs(d_c=d)) for d in (64, 128, 192)]
    dense = O.batch_capacity(180 * 10**9, dense=True, **_wan_capacity_kwargs())
    assert caps[0] > caps[1] > caps[2] > dense > 0


def _weight_cases():
    return [("wan", WAN), ("wan_dc64", WAN.replace(d_c=64)), ("tiny", TINY)]


def _shape_kw(cfg):
    return dict(dim=cfg.dim, n_heads=cfg.n_heads, d_nope=cfg.d_nope, d_rope=cfg.d_rope, d_c=cfg.d_c,
                d_v=cfg.d_v)


@pytest.mark.parametrize("name,cfg", _weight_cases())
def test_layer_weights_are_the_drawn_weights(name, cfg):
    """layer_weights lists exactly the tensors the seeded input recipe draws for one layer (shapes and
    order: W^KV_down || W^KR, W^K_up, W^V_up; dense: the per-head K/V projection).  The recipe states
    its shapes itself and holds none of the oracle's arithmetic, so a dropped weight, a missing head
    axis or a d_nope / d_c swap in layer_weights fails here."""
    drawn = synthetic.draw_weights(cfg, 7)
    lw = O.layer_weights(dense=False, **_shape_kw(cfg))
    assert [tuple(t.shape) for t in drawn] == list(lw.values())
    dense = O.layer_weights(dense=True, **_shape_kw(cfg))
    assert list(dense.values()) == [tuple(synthetic.draw_dense_weights(cfg, 7).shape)]


@pytest.mark.parametrize("name,cfg", _weight_cases())
def test_layer_weight_shapes_produce_the_printed_token_state(name, cfg):
    """Weights of layer_weights' shapes, run through the oracle's own projections, give per token the
    state the pages print: the stacked down-projection yields d_c + d_rope cached scalars (224 at the
    defaults, Method item 4), the dense projection 2 n_h d_h scalars (3072), and the per-head keys and
    values rebuilt from the latent have the dense head widths (d_nope + d_rope = d_h, and d_v)."""
    rng = np.random.default_rng(3)
    lw = O.layer_weights(dense=False, **_shape_kw(cfg))
    w = {k: rng.standard_normal(v) for k, v in lw.items()}
    T = 5
    x = rng.standard_normal((T, cfg.dim))
    pos = O.token_positions(0, T, cfg.grid_h, cfg.grid_w)
    pairs = (cfg.rope_pairs_t, cfg.rope_pairs_h, cfg.rope_pairs_w)
    c, k_r = O.compress(x, w["w_dkv_kr"], cfg.d_c, pos, pairs, cfg.rope_theta)
    assert c.shape[-1] + k_r.shape[-1] == O.latent_scalars_per_token(cfg.d_c, cfg.d_rope)
    k, v = O.reconstruct_kv(c, k_r, w["w_uk"], w["w_uv"])
    assert k.shape == (T, cfg.n_heads, cfg.d_h) and v.shape == (T, cfg.n_heads, cfg.d_v)
    q = O.absorbed_query(rng.standard_normal((T, cfg.n_heads, cfg.d_nope)),
                         rng.standard_normal((T, cfg.n_heads, cfg.d_rope)), w["w_uk"])
    assert q.shape == (T, cfg.n_heads, cfg.d_c + cfg.d_rope)
    (rows, cols), = O.layer_weights(dense=True, **_shape_kw(cfg)).values()
    assert cols == cfg.dim and rows == cfg.n_heads * (cfg.d_h + cfg.d_v)
    if name == "wan":
        g = json.load(open(GOLDEN))
        assert c.shape[-1] + k_r.shape[-1] == 224
        assert rows == 2 * g["n_heads"]["value"] * g["d_h"]["value"] == 3072


@pytest.mark.parametrize("dense", [False, True])
def test_memory_bytes_without_sequences_is_the_weights_and_fixed_bytes(dense):
    """memory_bytes(0) holds no cache and no step tensor: it is n_layers times one layer's drawn
    weights (counted from the seeded recipe's tensors) times the element size, plus the fixed bytes."""
    for cfg, n_layers, fixed in ((WAN, 30, 0), (WAN.replace(d_c=64), 30, 12345), (TINY, 2, 1000)):
        if dense:
            numel = synthetic.draw_dense_weights(cfg, 1).numel()
        else:
            numel = sum(t.numel() for t in synthetic.draw_weights(cfg, 1))
        kw = dict(n_layers=n_layers, window_tokens=cfg.window_tokens, elt_bytes=cfg.elt_bytes,
                  fixed_bytes=fixed, extra_bytes_per_seq=777, tokens_per_chunk=cfg.chunk_tokens,
                  **_shape_kw(cfg))
        assert O.memory_bytes(0, dense=dense, **kw) == n_layers * numel * cfg.elt_bytes + fixed
        # and one sequence adds its caches (every layer), its step tensors and its extra bytes
        per_tok = cfg.dense_scalars_per_token() if dense else cfg.latent_scalars_per_token()
        cache = n_layers * cfg.window_tokens * per_tok * cfg.elt_bytes
        B, N, H = 1, cfg.chunk_tokens, cfg.n_heads
        if dense:
            step = N * cfg.dim + N * H * cfg.d_h + N * H * cfg.d_v
        else:
            step = N * cfg.dim + N * H * (cfg.d_nope + cfg.d_rope + cfg.d_v + cfg.d_c + cfg.d_rope + cfg.d_c)
        assert O.memory_bytes(1, dense=dense, **kw) - O.memory_bytes(0, dense=dense, **kw) == \
            cache + step * cfg.elt_bytes + 777
