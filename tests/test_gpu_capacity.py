"""The capacity planner's per-sequence bytes against what a streaming layer step really allocates on
the device: n_layers latent (or dense) caches plus one layer step's inputs and outputs."""
import pytest
import torch

import synthetic
from parity import MID

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from rank_latent_kv_vmla_b200 import vmla
    return vmla


def _held_bytes(V, cfg, batch, n_layers, dense, fused=False):
    """Device bytes held by n_layers caches and one layer step of ``batch`` sequences."""
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    x, qn, qr = (t.to(DEV) for t in synthetic.draw_chunk(cfg, batch, 5))
    if dense:
        caches = [V.DenseCache(cfg, batch, device=DEV) for _ in range(n_layers)]
        w_kv = torch.zeros((cfg.n_heads * (cfg.d_h + cfg.d_v), cfg.dim), dtype=x.dtype, device=DEV)
        V.dense_append(cfg, x, w_kv, caches[0])
        q = V.rope_q(cfg, qn, qr, 0)
        del qn, qr                                   # the dense step keeps x, q and out
        out = V.dense_mha(cfg, q, caches[0], 0)
        held = [x, q, out, caches]
    else:
        caches = [V.LatentCache(cfg, batch, device=DEV) for _ in range(n_layers)]
        w, w_uk, w_uv = (t.to(DEV) for t in synthetic.draw_weights(cfg, 6))
        weights = sum(t.numel() * t.element_size() for t in (w, w_uk, w_uv))
        V.compress_append(cfg, x, w, caches[0])
        if fused:
            out = V.latent_attention_fused(cfg, qn, qr, w_uk, w_uv, caches[0], 0)
            held = [x, qn, qr, out, caches]
        else:
            q_abs = V.absorb_q(cfg, qn, qr, w_uk, 0)
            o_lat = V.latent_attention(cfg, q_abs, caches[0], 0)
            out = V.value_up(cfg, o_lat, w_uv)
            held = [x, qn, qr, q_abs, o_lat, out, caches]
        base += weights
    torch.cuda.synchronize()
    if dense:
        base += w_kv.numel() * w_kv.element_size()
    return torch.cuda.memory_allocated() - base, held


@pytest.mark.parametrize("dense,fused", [(False, False), (True, False), (False, True)],
                         ids=["latent", "dense", "latent_fused"])
def test_planner_bytes_per_sequence_match_device_allocation(V, dense, fused):
    cfg, n_layers = MID, 3
    a, held_a = _held_bytes(V, cfg, 2, n_layers, dense, fused)
    del held_a
    torch.cuda.empty_cache()
    b, held_b = _held_bytes(V, cfg, 3, n_layers, dense, fused)
    del held_b
    plan = V.plan_capacity(cfg, n_layers, 10**12, dense=dense, fused=fused)
    per_seq = plan["cache_bytes_per_seq"] + plan["buffer_bytes_per_seq"]
    # the caching allocator rounds each block up to 512 bytes
    assert abs((b - a) - per_seq) <= 512 * 16, (b - a, per_seq)
    assert abs(b - 3 * per_seq) <= 512 * 16 * 3, (b, 3 * per_seq)
