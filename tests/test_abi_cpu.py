"""C-ABI checks that need no GPU: the library loads, exports every symbol its header declares, and
rejects bad arguments on the host before anything is launched."""
import ctypes
import os
import re

import pytest

from rank_latent_kv_vmla_b200.config import TINY, WAN, VMLA_F32
from rank_latent_kv_vmla_b200 import vmla as V

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "vmla.h")
FAKE = 0x10000          # a 16-byte aligned non-null address: never dereferenced on these paths


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"VMLA_API[^;(]*?\b(vmla_\w+)\s*\(", text)))


def test_header_symbols_exported():
    names = _declared()
    assert len(names) >= 17
    for n in names:
        assert hasattr(V.LIB, n), n
        assert n in V.EXPORTED
    assert V.LIB.vmla_abi_version() == 1


def test_status_strings():
    assert V.LIB.vmla_status_string(0) == b"ok"
    assert V.LIB.vmla_status_string(5) == b"device wait timed out"


def test_cache_bytes_arithmetic():
    # 448 B vs 6144 B per token per layer (bf16), 7.29% of the dense layout
    tok = WAN.window_tokens
    assert V.latent_cache_bytes(WAN, 1) == tok * 224 * 2
    assert V.dense_cache_bytes(WAN, 1) == tok * 3072 * 2
    assert V.latent_cache_bytes(WAN, 8) == 8 * 14_676_480
    assert abs(V.latent_cache_bytes(WAN, 1) / V.dense_cache_bytes(WAN, 1) - 224 / 3072) < 1e-12
    assert V.latent_cache_bytes(TINY, 1) == TINY.window_tokens * (TINY.d_c + TINY.d_rope) * 4


def _cache(frames_written=0, batch=1, c=FAKE, k=FAKE):
    return V.CCache(c, k, batch, 0, frames_written)


def _status(fn, *args):
    st = fn(*args)
    return st, V.LIB.vmla_last_error_detail().decode()


def test_bad_configs_rejected():
    for bad in (TINY.replace(d_rope=7, rope_pairs_w=0), TINY.replace(rope_pairs_t=3),
                TINY.replace(chunk_frames=4), TINY.replace(dim=0), TINY.replace(dtype=7),
                TINY.replace(rope_theta=1.0)):
        cc = V.c_config(bad)
        st, detail = _status(V.LIB.vmla_compress_append, ctypes.byref(cc), FAKE, FAKE, 0,
                             ctypes.byref(_cache()), None)
        assert st == V.VMLA_ERR_INVALID_ARG, (bad, detail)
    st, _ = _status(V.LIB.vmla_compress_append, None, FAKE, FAKE, 0, ctypes.byref(_cache()), None)
    assert st == V.VMLA_ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected():
    cc = V.c_config(TINY)
    st, d = _status(V.LIB.vmla_compress_append, ctypes.byref(cc), None, FAKE, 0, ctypes.byref(_cache()), None)
    assert st == V.VMLA_ERR_INVALID_ARG and "x" in d
    st, d = _status(V.LIB.vmla_compress_append, ctypes.byref(cc), FAKE + 4, FAKE, 0, ctypes.byref(_cache()), None)
    assert st == V.VMLA_ERR_MISALIGNED
    st, d = _status(V.LIB.vmla_value_up, ctypes.byref(cc), 1, 16, FAKE, FAKE + 2, FAKE, None)
    assert st == V.VMLA_ERR_MISALIGNED and "w_uv" in d


def test_append_must_follow_frames_written():
    cc = V.c_config(TINY)
    cache = _cache(frames_written=2)
    st, d = _status(V.LIB.vmla_compress_append, ctypes.byref(cc), FAKE, FAKE, 1, ctypes.byref(cache), None)
    assert st == V.VMLA_ERR_INVALID_ARG and "follow" in d
    assert cache.frames_written == 2


@pytest.mark.parametrize("fw,first,nchunks,ok", [
    (0, 0, 1, False),     # empty cache (kv_len = 0)
    (1, 0, 1, True),
    (1, 1, 1, False),     # query frames not appended yet
    (3, 0, 3, True),      # multi-chunk, everything still in the window (W = 3)
    (4, 3, 1, True),      # window full, newest chunk
    (4, 2, 1, False),     # an older chunk after eviction
    (4, 2, 2, False),     # multi-chunk after eviction
    (3, -1, 1, False),
    (3, 2, 0, False),
])
def test_window_rules(fw, first, nchunks, ok):
    cc = V.c_config(TINY)
    st, d = _status(V.LIB.vmla_check_attention_window, ctypes.byref(cc), fw, first, nchunks)
    assert (st == V.VMLA_OK) == ok, d
    if not ok:
        assert st == V.VMLA_ERR_INVALID_ARG
        # the attention entry points apply the same rule before launching anything
        cache = _cache(frames_written=fw)
        st2, _ = _status(V.LIB.vmla_latent_attention, ctypes.byref(cc), FAKE, ctypes.byref(cache), first,
                         nchunks, FAKE, None, None)
        assert st2 == V.VMLA_ERR_INVALID_ARG
        st3, _ = _status(V.LIB.vmla_dense_mha, ctypes.byref(cc), FAKE,
                         ctypes.byref(V.CDenseCache(FAKE, FAKE, 1, 0, fw)), first, nchunks, FAKE, None, None)
        assert st3 == V.VMLA_ERR_INVALID_ARG


def test_lse_alignment_checked():
    cc = V.c_config(TINY)
    st, _ = _status(V.LIB.vmla_latent_attention, ctypes.byref(cc), FAKE, ctypes.byref(_cache(1)), 0, 1,
                    FAKE, FAKE + 4, None)
    assert st == V.VMLA_ERR_MISALIGNED


def test_device_status_needs_output_pointer():
    assert V.LIB.vmla_device_status(None, None) == V.VMLA_ERR_INVALID_ARG


def test_wait_timeout_setting():
    old = V.set_wait_timeout_ms(0)
    assert old == 1000
    assert V.set_wait_timeout_ms(250) == 1000
    assert V.set_wait_timeout_ms(old) == 250


def test_rewrite_rejects_before_any_append():
    cc = V.c_config(TINY)
    st, detail = _status(V.LIB.vmla_compress_rewrite, ctypes.byref(cc), FAKE, FAKE,
                         ctypes.byref(_cache(frames_written=0)), None)
    assert st == V.VMLA_ERR_INVALID_ARG and "no chunk to rewrite" in detail
    dc = V.CDenseCache(FAKE, FAKE, 1, 0, 0)
    st, detail = _status(V.LIB.vmla_dense_rewrite, ctypes.byref(cc), FAKE, FAKE, ctypes.byref(dc), None)
    assert st == V.VMLA_ERR_INVALID_ARG and "no chunk to rewrite" in detail
    st, _ = _status(V.LIB.vmla_compress_rewrite, ctypes.byref(cc), 0, FAKE,
                    ctypes.byref(_cache(frames_written=1)), None)
    assert st == V.VMLA_ERR_INVALID_ARG                      # NULL x
    st, _ = _status(V.LIB.vmla_compress_rewrite, ctypes.byref(cc), FAKE + 8, FAKE,
                    ctypes.byref(_cache(frames_written=1)), None)
    assert st == V.VMLA_ERR_MISALIGNED


@pytest.mark.parametrize("cfg", [WAN, WAN.replace(d_c=64), TINY], ids=["wan", "wan_dc64", "tiny"])
def test_plan_capacity_matches_oracle(cfg):
    from oracle import vmla_oracle as O
    elt = 2 if cfg.dtype != VMLA_F32 else 4
    for dense, fused in ((False, False), (True, False), (False, True)):
        for n_layers, budget, fixed, extra in ((30, 180 * 10**9, 0, 0), (30, 180 * 10**9, 2_600_000_000, 300_000_000),
                                               (1, 10**6, 0, 0), (4, 5 * 10**8, 10**7, 12345), (30, 10**9, 2 * 10**9, 0)):
            got = V.plan_capacity(cfg, n_layers, budget, dense=dense, fused=fused, fixed_bytes=fixed,
                                  extra_bytes_per_seq=extra)
            want = O.batch_capacity(budget, n_layers=n_layers, window_tokens=cfg.window_tokens, elt_bytes=elt,
                                    fixed_bytes=fixed, extra_bytes_per_seq=extra, dim=cfg.dim,
                                    n_heads=cfg.n_heads, d_nope=cfg.d_nope, d_rope=cfg.d_rope, d_c=cfg.d_c,
                                    d_v=cfg.d_v, tokens_per_chunk=cfg.chunk_tokens, dense=dense, fused=fused)
            assert got["max_batch"] == want, (dense, fused, n_layers, budget, fixed, extra)
    one = V.plan_capacity(cfg, 30, 10**12)
    assert one["cache_bytes_per_seq"] == 30 * V.latent_cache_bytes(cfg, 1)
    assert V.plan_capacity(cfg, 30, 10**12, dense=True)["cache_bytes_per_seq"] == 30 * V.dense_cache_bytes(cfg, 1)


def test_plan_capacity_rejects_bad_arguments():
    cc = V.c_config(WAN)
    out = V.CCapacity()
    for args in ((0, 0, 10, 0, 0), (30, 0, -1, 0, 0), (30, 0, 10, -5, 0), (30, 1, 10, 0, -1), (30, 3, 10, 0, 0),
                 (30, -1, 10, 0, 0)):
        st, _ = _status(V.LIB.vmla_plan_capacity, ctypes.byref(cc), *args, ctypes.byref(out))
        assert st == V.VMLA_ERR_INVALID_ARG
    st, _ = _status(V.LIB.vmla_plan_capacity, ctypes.byref(cc), 30, 0, 10, 0, 0, None)
    assert st == V.VMLA_ERR_INVALID_ARG


def test_fused_attention_rejects_unsupported_shapes():
    """The fused call refuses, before launching, the fp32 path and shapes outside its layout."""
    cache = _cache(frames_written=TINY.chunk_frames)
    for bad, why in ((TINY, "bf16"), (WAN.replace(d_c=96), "d_c"), (WAN.replace(d_nope=88, rope_pairs_t=6), "d_nope"),
                     (WAN.replace(d_v=160), "d_v")):
        cc = V.c_config(bad)
        c = _cache(frames_written=bad.chunk_frames)
        st, detail = _status(V.LIB.vmla_latent_attention_fused, ctypes.byref(cc), FAKE, FAKE, FAKE, FAKE,
                             ctypes.byref(c), 0, 1, FAKE, None, None)
        assert st == V.VMLA_ERR_UNSUPPORTED, (why, st, detail)
    cc = V.c_config(WAN)
    st, _ = _status(V.LIB.vmla_latent_attention_fused, ctypes.byref(cc), FAKE, FAKE, FAKE, FAKE,
                    ctypes.byref(_cache(frames_written=0)), 0, 1, FAKE, None, None)
    assert st == V.VMLA_ERR_INVALID_ARG                       # nothing appended yet
    st, _ = _status(V.LIB.vmla_latent_attention_fused, ctypes.byref(cc), FAKE + 8, FAKE, FAKE, FAKE,
                    ctypes.byref(_cache(frames_written=3)), 0, 1, FAKE, None, None)
    assert st == V.VMLA_ERR_MISALIGNED


def test_executor_workspace_and_rejections():
    """Workspace arithmetic (two slots of x, q_nope, q_rope, out, each 256-byte rounded) and the
    argument checks that run before any CUDA call."""
    cc = V.c_config(WAN)
    n = WAN.chunk_tokens
    per = [n * WAN.dim * 2, n * 12 * 96 * 2, n * 12 * 32 * 2, n * 12 * 128 * 2]
    slot = sum((b + 255) // 256 * 256 for b in per)
    assert V.LIB.vmla_executor_workspace_bytes(ctypes.byref(cc), 1) == 2 * slot
    assert V.LIB.vmla_executor_workspace_bytes(ctypes.byref(cc), 0) == -1
    h = ctypes.c_void_p()
    st, _ = _status(V.LIB.vmla_executor_create, ctypes.byref(V.c_config(TINY)), 1, 0x100000, 1 << 30, None,
                    ctypes.byref(h))
    assert st == V.VMLA_ERR_UNSUPPORTED and not h.value
    st, _ = _status(V.LIB.vmla_executor_create, ctypes.byref(cc), 1, 0x100000 + 16, 1 << 30, None, ctypes.byref(h))
    assert st == V.VMLA_ERR_MISALIGNED
    st, _ = _status(V.LIB.vmla_executor_create, ctypes.byref(cc), 1, 0x100000, 1024, None, ctypes.byref(h))
    assert st == V.VMLA_ERR_INVALID_ARG
    assert V.LIB.vmla_executor_wait(None) == V.VMLA_ERR_INVALID_ARG
    assert V.LIB.vmla_executor_destroy(None) == V.VMLA_OK


def test_binding_rejects_host_tensors_and_bad_shapes():
    """The Python binding checks device, dtype, contiguity and shape before calling the library."""
    import torch
    cfg = WAN
    x = torch.zeros((1, cfg.chunk_tokens, cfg.dim), dtype=torch.bfloat16)           # a host tensor
    w = torch.zeros((cfg.d_c + cfg.d_rope, cfg.dim), dtype=torch.bfloat16)
    cache = V.LatentCache(cfg, 1, device="cpu")
    with pytest.raises(ValueError, match="CUDA tensor"):
        V.compress_append(cfg, x, w, cache)
    with pytest.raises(ValueError, match="CUDA tensor"):
        V.compress_rewrite(cfg, x, w, cache)
    with pytest.raises(ValueError):
        V.absorb_q(cfg, torch.zeros((1, 7, cfg.n_heads, cfg.d_nope), dtype=torch.bfloat16),
                   torch.zeros((1, 7, cfg.n_heads, cfg.d_rope), dtype=torch.bfloat16),
                   torch.zeros((cfg.n_heads, cfg.d_nope, cfg.d_c), dtype=torch.bfloat16), 0)   # 7 tokens
    with pytest.raises(ValueError):
        V.latent_attention_fused(cfg, torch.zeros((1, 7, cfg.n_heads, cfg.d_nope), dtype=torch.bfloat16),
                                 torch.zeros((1, 7, cfg.n_heads, cfg.d_rope), dtype=torch.bfloat16), w, w, cache, 0)
    assert V.latent_cache_bytes(cfg, 1) == cache.nbytes()


def test_status_codes_match_header():
    text = open(HEADER).read()
    for name, value in (("VMLA_OK", 0), ("VMLA_ERR_INVALID_ARG", 1), ("VMLA_ERR_UNSUPPORTED", 2),
                        ("VMLA_ERR_MISALIGNED", 3), ("VMLA_ERR_CUDA", 4), ("VMLA_ERR_TIMEOUT", 5)):
        assert re.search(r"\b%s\s*=\s*%d\b" % (name, value), text), name
        assert getattr(V, name) == value
    for name, value in (("VMLA_PATH_LATENT", 0), ("VMLA_PATH_DENSE", 1), ("VMLA_PATH_LATENT_FUSED", 2)):
        assert re.search(r"\b%s\s*=\s*%d\b" % (name, value), text), name


def test_cache_checkpoint_round_trip(tmp_path):
    """save / load restore the ring planes bit for bit (NaN-poisoned rows included) and frames_written;
    a checkpoint of another configuration or kind is refused."""
    import torch
    cfg = TINY
    cache = V.LatentCache(cfg, 2, device="cpu", fill=float("nan"))
    g = torch.Generator().manual_seed(3)
    cache.c[:, :20] = torch.randn((2, 20, cfg.d_c), generator=g)
    cache.k_r[:, :20] = torch.randn((2, 20, cfg.d_rope), generator=g)
    cache.struct.frames_written = 7
    path = tmp_path / "layer0.pt"
    cache.save(path)
    back = V.LatentCache.load(path, cfg, device="cpu")
    assert back.frames_written == 7 and back.batch == 2
    assert torch.equal(back.c.view(torch.int32), cache.c.view(torch.int32))
    assert torch.equal(back.k_r.view(torch.int32), cache.k_r.view(torch.int32))
    assert back.struct.c == back.c.data_ptr()
    with pytest.raises(ValueError, match="configuration"):
        V.LatentCache.load(path, cfg.replace(window_frames=4), device="cpu")
    with pytest.raises(ValueError, match="latent cache"):
        V.DenseCache.load(path, cfg, device="cpu")
    dense = V.DenseCache(cfg, 1, device="cpu", fill=0.5)
    dense.struct.frames_written = 3
    dense.save(tmp_path / "dense.pt")
    dback = V.DenseCache.load(tmp_path / "dense.pt", cfg, device="cpu")
    assert dback.frames_written == 3 and torch.equal(dback.k, dense.k) and torch.equal(dback.v, dense.v)


@pytest.mark.parametrize("cfg,ok", [
    (WAN, True),
    (WAN.replace(d_c=128), True),
    (WAN.replace(d_c=256), True),
    (WAN.replace(d_c=64), True),
    (WAN.replace(d_c=96), False),        # the fused kernel needs d_c in {64, 128, 192, 256}
    (WAN.replace(d_nope=104, rope_pairs_t=6), False),   # d_nope not a multiple of 16
    (TINY, False),                       # fp32 runs on the SIMT path only
])
def test_fused_support_query(cfg, ok):
    """vmla_check_fused is host-only and agrees with what vmla_latent_attention_fused accepts."""
    cc = V.c_config(cfg)
    st, d = _status(V.LIB.vmla_check_fused, ctypes.byref(cc))
    assert (st == V.VMLA_OK) == ok, d
    assert V.fused_supported(cfg) == ok
    if not ok:
        assert st == V.VMLA_ERR_UNSUPPORTED and d
        cache = _cache(frames_written=cfg.window_frames)
        st2, _ = _status(V.LIB.vmla_latent_attention_fused, ctypes.byref(cc), FAKE, FAKE, FAKE, FAKE,
                         ctypes.byref(cache), cfg.window_frames - cfg.chunk_frames, 1, FAKE, None, None)
        assert st2 == V.VMLA_ERR_UNSUPPORTED


_MIDLIKE = WAN.replace(grid_h=6, grid_w=10, chunk_frames=2, window_frames=5)   # 120-token chunks, bf16


@pytest.mark.parametrize("begin,n", [
    (0, 0),                 # empty range
    (-8, 16),               # negative start
    (64, 64),               # past the chunk's 120 tokens
])
def test_row_range_compress_rejects_bad_ranges(begin, n):
    """vmla_compress_append_rows validates the token range, the replica list and every replica's
    frames_written on the host, and launches nothing for a rejected call (FAKE device pointers are
    never dereferenced)."""
    cfg = _MIDLIKE
    cc = V.c_config(cfg)
    reps = (V.CCache * 2)(_cache(), _cache())
    st, d = _status(V.LIB.vmla_compress_append_rows, ctypes.byref(cc), FAKE, FAKE, 0, begin, n, reps, 2, None)
    assert st == V.VMLA_ERR_INVALID_ARG and "token range" in d, d


def test_row_range_compress_rejects_bad_replicas():
    cfg = _MIDLIKE
    cc = V.c_config(cfg)
    call = lambda reps, k, ff=0: _status(V.LIB.vmla_compress_append_rows, ctypes.byref(cc), FAKE, FAKE, ff, 0, 8,
                                         reps, k, None)
    reps = (V.CCache * 9)(*[_cache() for _ in range(9)])
    assert call(reps, 0)[0] == V.VMLA_ERR_INVALID_ARG                 # no replica
    assert call(reps, 9)[0] == V.VMLA_ERR_INVALID_ARG                 # more than the kernel's 8 destinations
    assert call(None, 1)[0] == V.VMLA_ERR_INVALID_ARG
    bad = (V.CCache * 2)(_cache(), _cache(c=None))
    st, d = call(bad, 2)
    assert st == V.VMLA_ERR_INVALID_ARG and "NULL" in d, d
    bad = (V.CCache * 2)(_cache(), _cache(batch=2))
    st, d = call(bad, 2)
    assert st == V.VMLA_ERR_INVALID_ARG and "batch" in d, d
    bad = (V.CCache * 2)(_cache(), _cache(frames_written=2))
    st, d = call(bad, 2)
    assert st == V.VMLA_ERR_INVALID_ARG and "frames_written" in d, d
    bad = (V.CCache * 2)(_cache(), _cache(c=FAKE + 8))
    assert call(bad, 2)[0] == V.VMLA_ERR_MISALIGNED
    st, d = _status(V.LIB.vmla_compress_append_rows, ctypes.byref(V.c_config(TINY)), FAKE, FAKE, 0, 0, 8,
                    (V.CCache * 1)(_cache()), 1, None)
    assert st == V.VMLA_ERR_UNSUPPORTED                                # fp32 has no row-range path


@pytest.mark.parametrize("begin,n", [(0, 0), (-1, 8), (100, 40), (0, 121)])
def test_row_range_fused_rejects_bad_ranges(begin, n):
    """vmla_latent_attention_fused_rows: the token range must lie inside the call's query tokens."""
    cfg = _MIDLIKE
    cc = V.c_config(cfg)
    cache = _cache(frames_written=cfg.window_frames)
    f0 = cfg.window_frames - cfg.chunk_frames
    st, d = _status(V.LIB.vmla_latent_attention_fused_rows, ctypes.byref(cc), FAKE, FAKE, FAKE, FAKE,
                    ctypes.byref(cache), f0, 1, begin, n, FAKE, None, None)
    assert st == V.VMLA_ERR_INVALID_ARG and "token range" in d, d


def test_ipc_calls_reject_bad_arguments():
    """The CUDA IPC entry points validate their arguments before touching the driver: NULL handles or
    pointers and releasing a pointer that vmla_ipc_import never returned are errors with a detail;
    exporting an address that is not device memory fails cleanly (here: no GPU at all)."""
    h = V.CIpcHandle()
    st, d = _status(V.LIB.vmla_ipc_export, None, ctypes.byref(h))
    assert st == V.VMLA_ERR_INVALID_ARG and "NULL" in d, d
    st, d = _status(V.LIB.vmla_ipc_export, FAKE, None)
    assert st == V.VMLA_ERR_INVALID_ARG, d
    p = ctypes.c_void_p(0)
    st, d = _status(V.LIB.vmla_ipc_import, None, ctypes.byref(p))
    assert st == V.VMLA_ERR_INVALID_ARG, d
    st, d = _status(V.LIB.vmla_ipc_release, FAKE)
    assert st == V.VMLA_ERR_INVALID_ARG and "vmla_ipc_import" in d, d
    st, d = _status(V.LIB.vmla_ipc_export, FAKE, ctypes.byref(h))
    assert st != V.VMLA_OK, d

