"""Layer configuration for VideoMLA latent-KV attention, mirroring ``vmla_config`` in ``include/vmla.h``.

Symbols follow VideoMLA (gist.science technical summary, Method items 1-4): ``d_c`` is the size of the
shared content latent c^KV_t, ``d_rope`` the size of the head-shared positional key k^R_t, ``d_nope`` the
per-head content part of the query/key, ``n_heads`` = n_h.  The frame grid, chunk and window sizes and the
3D-RoPE pair split are workload parameters of a Wan-1.3B-shaped layer (the pages fix only d_c = 192,
d_rope = 32, n_h = 12, d_h = 128).
"""
from __future__ import annotations

import dataclasses
import math

VMLA_BF16 = 0
VMLA_F32 = 1


@dataclasses.dataclass(frozen=True)
class VmlaConfig:
    dim: int                # model width D of the token features x_t
    n_heads: int            # n_h
    d_nope: int             # content part of the per-head query/key
    d_rope: int             # positional part (the size of k^R_t)
    d_c: int                # latent size (the size of c^KV_t)
    d_v: int                # per-head value size
    grid_h: int             # latent-frame grid height (tokens)
    grid_w: int             # latent-frame grid width (tokens)
    chunk_frames: int       # latent frames generated per autoregressive chunk
    window_frames: int      # sliding-window length in latent frames (includes the current chunk)
    rope_pairs_t: int       # rotary pairs driven by the frame index
    rope_pairs_h: int       # rotary pairs driven by the row index
    rope_pairs_w: int       # rotary pairs driven by the column index
    rope_theta: float = 10000.0
    softmax_scale: float = 0.0   # 0 selects 1/sqrt(d_nope + d_rope)
    dtype: int = VMLA_BF16

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def chunk_tokens(self) -> int:
        return self.chunk_frames * self.tokens_per_frame

    @property
    def window_tokens(self) -> int:
        return self.window_frames * self.tokens_per_frame

    @property
    def d_qk(self) -> int:
        """Width of one absorbed query row / one cached key row: d_c + d_rope."""
        return self.d_c + self.d_rope

    @property
    def d_h(self) -> int:
        return self.d_nope + self.d_rope

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale > 0 else 1.0 / math.sqrt(self.d_nope + self.d_rope)

    @property
    def elt_bytes(self) -> int:
        return 2 if self.dtype == VMLA_BF16 else 4

    def latent_scalars_per_token(self) -> int:
        """Cached scalars per token per layer in the latent layout: d_c + d_rope."""
        return self.d_c + self.d_rope

    def dense_scalars_per_token(self) -> int:
        """Cached scalars per token per layer in the dense per-head layout: K and V for every head."""
        return self.n_heads * (self.d_h + self.d_v)

    def replace(self, **kw) -> "VmlaConfig":
        return dataclasses.replace(self, **kw)


# Tiny case checked whole against the oracle: fp32 storage and arithmetic.
TINY = VmlaConfig(dim=64, n_heads=2, d_nope=24, d_rope=8, d_c=16, d_v=32, grid_h=4, grid_w=4,
                  chunk_frames=1, window_frames=3, rope_pairs_t=2, rope_pairs_h=1, rope_pairs_w=1,
                  dtype=VMLA_F32)

# One Wan-1.3B-shaped attention layer: 30x52 latent grid, 3-frame chunks, 21-frame window.
WAN = VmlaConfig(dim=1536, n_heads=12, d_nope=96, d_rope=32, d_c=192, d_v=128, grid_h=30, grid_w=52,
                 chunk_frames=3, window_frames=21, rope_pairs_t=6, rope_pairs_h=5, rope_pairs_w=5,
                 dtype=VMLA_BF16)

PRESETS = {"tiny": TINY, "wan": WAN}
