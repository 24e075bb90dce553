"""Checkpoint / resume of the streaming state: a rollout saved after chunk k and restored into a fresh
cache continues with bit-identical outputs and cache planes (latent layer, fused path and three-call
path, and the dense comparison layer)."""
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


def _bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("fused", [True, False])
def test_latent_rollout_resumes_bit_identically(V, tmp_path, fused):
    cfg, B, n, split = MID, 2, 6, 3
    w, wuk, wuv = (t.to(DEV) for t in synthetic.draw_weights(cfg, 8))
    chunks = [tuple(t.to(DEV) for t in synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(7, 0, k))) for k in range(n)]
    straight = V.LatentCache(cfg, B, device=DEV, fill=float("nan"))
    ref = [V.layer_step(cfg, *chunks[k], w, wuk, wuv, straight, fused=fused).clone() for k in range(n)]
    part = V.LatentCache(cfg, B, device=DEV, fill=float("nan"))
    for k in range(split):
        V.layer_step(cfg, *chunks[k], w, wuk, wuv, part, fused=fused)
    torch.cuda.synchronize()
    part.save(tmp_path / "layer.pt")
    del part
    resumed = V.LatentCache.load(tmp_path / "layer.pt", cfg, device=DEV)
    assert resumed.frames_written == split * cfg.chunk_frames
    for k in range(split, n):
        o = V.layer_step(cfg, *chunks[k], w, wuk, wuv, resumed, fused=fused)
        torch.cuda.synchronize()
        assert torch.equal(_bits(o), _bits(ref[k])), k
    assert torch.equal(_bits(resumed.c), _bits(straight.c)) and torch.equal(_bits(resumed.k_r), _bits(straight.k_r))
    assert V.device_status() == 0


def test_dense_rollout_resumes_bit_identically(V, tmp_path):
    cfg, B, n, split = MID, 1, 5, 2
    w_kv = synthetic.draw_dense_weights(cfg, 9).to(DEV)
    chunks = [tuple(t.to(DEV) for t in synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(9, 0, k))) for k in range(n)]

    def step(cache, x, qn, qr):
        f0 = cache.frames_written
        V.dense_append(cfg, x, w_kv, cache)
        return V.dense_mha(cfg, V.rope_q(cfg, qn, qr, f0), cache, f0)

    straight = V.DenseCache(cfg, B, device=DEV)
    ref = [step(straight, *chunks[k]).clone() for k in range(n)]
    part = V.DenseCache(cfg, B, device=DEV)
    for k in range(split):
        step(part, *chunks[k])
    torch.cuda.synchronize()
    part.save(tmp_path / "dense.pt")
    resumed = V.DenseCache.load(tmp_path / "dense.pt", cfg, device=DEV)
    for k in range(split, n):
        o = step(resumed, *chunks[k])
        torch.cuda.synchronize()
        assert torch.equal(_bits(o), _bits(ref[k])), k
