"""Seeded synthetic inputs for the VideoMLA latent-attention layer.

This module only draws random numbers: it holds none of the method's arithmetic, and both the float64
oracle (through the tests) and the CUDA path consume exactly the tensors it returns.

Recipe (fixed order, one CPU ``torch.Generator`` per call, seeded by the caller):
  1. W^KV_down [d_c, D] and W^KR [d_rope, D], stacked as one [d_c + d_rope, D] matrix;
  2. W^K_up [n_h, d_nope, d_c];  3. W^V_up [n_h, d_v, d_c];
  4. the token features x of every chunk, chunk by chunk, each [B, F*T_f, D];
  5. q^nope [B, Nq, n_h, d_nope] and q^rope [B, Nq, n_h, d_rope] of the query chunk(s).
Every weight is N(0, 1/fan_in) with fan_in = its last dimension; x and q are N(0, 1) (q has the
distribution that W_q x would have with W_q ~ N(0, 1/D)), optionally multiplied by ``q_gain`` to make
the softmax peaked.  Values are drawn in fp32 and rounded (round-to-nearest-even) to the storage dtype,
so the oracle and the GPU see identical bits.
"""
from __future__ import annotations

import dataclasses
from typing import List

import torch

from rank_latent_kv_vmla_b200.config import VMLA_BF16, VmlaConfig


def storage_dtype(cfg: VmlaConfig) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == VMLA_BF16 else torch.float32


@dataclasses.dataclass
class LayerInputs:
    w_dkv_kr: torch.Tensor          # [d_c + d_rope, D]
    w_uk: torch.Tensor              # [n_h, d_nope, d_c]
    w_uv: torch.Tensor              # [n_h, d_v, d_c]
    x_chunks: List[torch.Tensor]    # each [B, F*T_f, D]
    q_nope: torch.Tensor            # [B, Nq, n_h, d_nope]
    q_rope: torch.Tensor            # [B, Nq, n_h, d_rope]


def _randn(g: torch.Generator, shape, std: float, dt: torch.dtype) -> torch.Tensor:
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dt)


def draw_layer(cfg: VmlaConfig, batch: int, seed: int, n_chunks: int, n_query_chunks: int = 1,
               q_gain: float = 1.0) -> LayerInputs:
    """Draw one layer's weights, ``n_chunks`` chunks of token features and one query set.

    The query set covers ``n_query_chunks`` consecutive chunks (Nq = n_query_chunks * F * T_f).
    """
    g = torch.Generator().manual_seed(int(seed))
    dt = storage_dtype(cfg)
    D, H = cfg.dim, cfg.n_heads
    w_dkv_kr = _randn(g, (cfg.d_c + cfg.d_rope, D), D ** -0.5, dt)
    w_uk = _randn(g, (H, cfg.d_nope, cfg.d_c), cfg.d_c ** -0.5, dt)
    w_uv = _randn(g, (H, cfg.d_v, cfg.d_c), cfg.d_c ** -0.5, dt)
    x_chunks = [_randn(g, (batch, cfg.chunk_tokens, D), 1.0, dt) for _ in range(n_chunks)]
    nq = n_query_chunks * cfg.chunk_tokens
    q_nope = _randn(g, (batch, nq, H, cfg.d_nope), q_gain, dt)
    q_rope = _randn(g, (batch, nq, H, cfg.d_rope), q_gain, dt)
    return LayerInputs(w_dkv_kr, w_uk, w_uv, x_chunks, q_nope, q_rope)


def draw_dense_weights(cfg: VmlaConfig, seed: int) -> torch.Tensor:
    """Independent dense per-head K/V projection [n_h*(d_h + d_v), D] for the dense comparison layer:
    rows h*d_h .. (h+1)*d_h-1 are head h's key rows (the last d_rope of them are rotated by 3D-RoPE),
    followed by the n_h*d_v value rows."""
    g = torch.Generator().manual_seed(int(seed))
    rows = cfg.n_heads * (cfg.d_h + cfg.d_v)
    return _randn(g, (rows, cfg.dim), cfg.dim ** -0.5, storage_dtype(cfg))


def draw_queries(cfg: VmlaConfig, batch: int, seed: int, n_query_chunks: int = 1, q_gain: float = 1.0):
    """A fresh query set q^nope [B, Nq, n_h, d_nope], q^rope [B, Nq, n_h, d_rope], N(0, q_gain^2)."""
    g = torch.Generator().manual_seed(int(seed))
    dt = storage_dtype(cfg)
    nq = n_query_chunks * cfg.chunk_tokens
    q_nope = _randn(g, (batch, nq, cfg.n_heads, cfg.d_nope), q_gain, dt)
    q_rope = _randn(g, (batch, nq, cfg.n_heads, cfg.d_rope), q_gain, dt)
    return q_nope, q_rope


def draw_weights(cfg: VmlaConfig, seed: int):
    """One layer's weights only, in the same order and distributions as draw_layer:
    (W^KV_down || W^KR [d_c + d_rope, D], W^K_up [n_h, d_nope, d_c], W^V_up [n_h, d_v, d_c])."""
    g = torch.Generator().manual_seed(int(seed))
    dt = storage_dtype(cfg)
    D, H = cfg.dim, cfg.n_heads
    w_dkv_kr = _randn(g, (cfg.d_c + cfg.d_rope, D), D ** -0.5, dt)
    w_uk = _randn(g, (H, cfg.d_nope, cfg.d_c), cfg.d_c ** -0.5, dt)
    w_uv = _randn(g, (H, cfg.d_v, cfg.d_c), cfg.d_c ** -0.5, dt)
    return w_dkv_kr, w_uk, w_uv


def rollout_seed(base: int, layer: int, chunk: int) -> int:
    """Seed of the inputs of (layer, chunk) in a streaming rollout; the layer's weights use chunk -1."""
    return int(base) + 1_000_003 * (layer + 1) + 7919 * (chunk + 1)


def draw_chunk(cfg: VmlaConfig, batch: int, seed: int, q_gain: float = 1.0):
    """One streaming chunk's inputs: x [B, F*T_f, D], q^nope [B, F*T_f, n_h, d_nope],
    q^rope [B, F*T_f, n_h, d_rope] (N(0, 1); q scaled by q_gain)."""
    g = torch.Generator().manual_seed(int(seed))
    dt = storage_dtype(cfg)
    n = cfg.chunk_tokens
    x = _randn(g, (batch, n, cfg.dim), 1.0, dt)
    q_nope = _randn(g, (batch, n, cfg.n_heads, cfg.d_nope), q_gain, dt)
    q_rope = _randn(g, (batch, n, cfg.n_heads, cfg.d_rope), q_gain, dt)
    return x, q_nope, q_rope
