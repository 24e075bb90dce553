"""Python binding of libvmla (ctypes).  Argument marshalling only: every step runs in the library's
CUDA kernels; PyTorch supplies device memory and the current CUDA stream.

Importing this module loads ``libvmla.so`` from the package directory (or the library named by the
VMLA_LIBRARY environment variable, e.g. the bounds-checked ``libvmla_checked.so``) and raises if it is
missing: there is no fallback implementation.

Besides the per-call functions the module offers LatentCache / DenseCache (ring planes with
checkpoint save / load), Executor (layer steps with host buffers, copies overlapped with the
kernels), plan_capacity, and the row-range and IPC calls used by ``sharding``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .config import VMLA_BF16, VMLA_F32, VmlaConfig

# VMLA_LIBRARY selects another build of the library (e.g. the bounds-checked libvmla_checked.so)
_LIB_PATH = os.environ.get("VMLA_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvmla.so")

VMLA_OK, VMLA_ERR_INVALID_ARG, VMLA_ERR_UNSUPPORTED, VMLA_ERR_MISALIGNED, VMLA_ERR_CUDA, \
    VMLA_ERR_TIMEOUT = range(6)

EXPORTED = ("vmla_compress_append", "vmla_absorb_q", "vmla_latent_attention", "vmla_value_up",
            "vmla_rope_q", "vmla_dense_append", "vmla_dense_mha", "vmla_device_status",
            "vmla_check_attention_window", "vmla_check_fused", "vmla_set_wait_timeout_ms",
            "vmla_debug_drop_kv_tile",
            "vmla_latent_cache_bytes", "vmla_dense_cache_bytes", "vmla_launch_count",
            "vmla_status_string", "vmla_last_error_detail", "vmla_abi_version",
            "vmla_compress_rewrite", "vmla_dense_rewrite", "vmla_plan_capacity",
            "vmla_latent_attention_fused", "vmla_executor_workspace_bytes", "vmla_executor_create",
            "vmla_executor_submit", "vmla_executor_wait", "vmla_executor_destroy",
            "vmla_compress_append_rows", "vmla_latent_attention_fused_rows", "vmla_ipc_export",
            "vmla_ipc_import", "vmla_ipc_release", "vmla_debug_shrink_extents", "vmla_debug_exp2_poly")


class VmlaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"vmla status {status}: {detail}")
        self.status = status
        self.detail = detail


class CConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("dim", "n_heads", "d_nope", "d_rope", "d_c", "d_v",
                                                "grid_h", "grid_w", "chunk_frames", "window_frames",
                                                "rope_pairs_t", "rope_pairs_h", "rope_pairs_w")] + \
               [("rope_theta", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("dtype", ctypes.c_int32)]


class CCache(ctypes.Structure):
    _fields_ = [("c", ctypes.c_void_p), ("k_r", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("frames_written", ctypes.c_int64)]


class CCapacity(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("max_batch", "cache_bytes_per_seq",
                                                "buffer_bytes_per_seq", "weight_bytes")]


class CIpcHandle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64), ("offset", ctypes.c_int64)]


class CDenseCache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("frames_written", ctypes.c_int64)]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libvmla.so is not built ({_LIB_PATH}); run "
                          "`python -m rank_latent_kv_vmla_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I32, I64, VP = ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
    cfgp = P(CConfig)
    sig = {
        "vmla_compress_append": [cfgp, VP, VP, I64, P(CCache), VP],
        "vmla_absorb_q": [cfgp, I32, I32, VP, VP, VP, I64, VP, VP],
        "vmla_latent_attention": [cfgp, VP, P(CCache), I64, I32, VP, VP, VP],
        "vmla_value_up": [cfgp, I32, I64, VP, VP, VP, VP],
        "vmla_rope_q": [cfgp, I32, I32, VP, VP, I64, VP, VP],
        "vmla_dense_append": [cfgp, VP, VP, I64, P(CDenseCache), VP],
        "vmla_dense_mha": [cfgp, VP, P(CDenseCache), I64, I32, VP, VP, VP],
        "vmla_device_status": [VP, P(I32)],
        "vmla_check_attention_window": [cfgp, I64, I64, I32],
        "vmla_check_fused": [cfgp],
        "vmla_compress_rewrite": [cfgp, VP, VP, P(CCache), VP],
        "vmla_dense_rewrite": [cfgp, VP, VP, P(CDenseCache), VP],
        "vmla_plan_capacity": [cfgp, I32, I32, I64, I64, I64, P(CCapacity)],
        "vmla_latent_attention_fused": [cfgp, VP, VP, VP, VP, P(CCache), I64, I32, VP, VP, VP],
        "vmla_executor_create": [cfgp, I32, VP, I64, VP, P(VP)],
        "vmla_compress_append_rows": [cfgp, VP, VP, I64, I64, I64, P(CCache), I32, VP],
        "vmla_latent_attention_fused_rows": [cfgp, VP, VP, VP, VP, P(CCache), I64, I32, I64, I64, VP, VP, VP],
        "vmla_ipc_export": [VP, P(CIpcHandle)],
        "vmla_ipc_import": [P(CIpcHandle), P(VP)],
        "vmla_ipc_release": [VP],
        "vmla_executor_submit": [VP, P(CCache), VP, VP, VP, VP, VP, VP, VP],
        "vmla_executor_wait": [VP],
        "vmla_executor_destroy": [VP],
        "vmla_debug_exp2_poly": [VP, VP, I64, VP],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    for name in ("vmla_latent_cache_bytes", "vmla_dense_cache_bytes"):
        getattr(lib, name).argtypes = [cfgp, I32]
        getattr(lib, name).restype = I64
    lib.vmla_executor_workspace_bytes.argtypes = [cfgp, I32]
    lib.vmla_executor_workspace_bytes.restype = I64
    lib.vmla_launch_count.argtypes = []
    lib.vmla_launch_count.restype = I64
    lib.vmla_status_string.argtypes = [ctypes.c_int]
    lib.vmla_status_string.restype = ctypes.c_char_p
    lib.vmla_last_error_detail.argtypes = []
    lib.vmla_last_error_detail.restype = ctypes.c_char_p
    lib.vmla_debug_drop_kv_tile.argtypes = [I32]
    lib.vmla_debug_drop_kv_tile.restype = None
    lib.vmla_debug_shrink_extents.argtypes = [I64]
    lib.vmla_debug_shrink_extents.restype = I32
    lib.vmla_set_wait_timeout_ms.argtypes = [I32]
    lib.vmla_set_wait_timeout_ms.restype = I32
    lib.vmla_abi_version.argtypes = []
    lib.vmla_abi_version.restype = I32
    return lib


LIB = _load()


def lib_path() -> str:
    return _LIB_PATH


def c_config(cfg: VmlaConfig) -> CConfig:
    return CConfig(cfg.dim, cfg.n_heads, cfg.d_nope, cfg.d_rope, cfg.d_c, cfg.d_v, cfg.grid_h,
                   cfg.grid_w, cfg.chunk_frames, cfg.window_frames, cfg.rope_pairs_t,
                   cfg.rope_pairs_h, cfg.rope_pairs_w, cfg.rope_theta, cfg.softmax_scale, cfg.dtype)


def check(status: int):
    if status != VMLA_OK:
        raise VmlaError(status, LIB.vmla_last_error_detail().decode())


def _dtype(cfg: VmlaConfig) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == VMLA_BF16 else torch.float32


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _arg(t: torch.Tensor, cfg: VmlaConfig, shape, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != _dtype(cfg):
        raise ValueError(f"{name} must be {_dtype(cfg)}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _cache_key(cfg: VmlaConfig) -> dict:
    """The configuration fields a saved cache must match to be restored."""
    return {n: getattr(cfg, n) for n in ("n_heads", "d_nope", "d_rope", "d_c", "d_v", "grid_h", "grid_w",
                                          "chunk_frames", "window_frames", "dtype")}


def _save_planes(path, kind: str, cfg: VmlaConfig, batch: int, frames_written: int, planes: dict) -> None:
    torch.save({"kind": kind, "config": _cache_key(cfg), "batch": batch, "frames_written": frames_written,
                "planes": {k: v.detach().to("cpu") for k, v in planes.items()}}, path)


def _load_planes(path, kind: str, cfg: VmlaConfig) -> dict:
    state = torch.load(path, map_location="cpu", weights_only=True)
    if state.get("kind") != kind:
        raise ValueError(f"{path} holds a {state.get('kind')} cache, not a {kind} cache")
    if state["config"] != _cache_key(cfg):
        raise ValueError(f"{path} was saved with configuration {state['config']}, not {_cache_key(cfg)}")
    return state


class LatentCache:
    """One layer's latent cache: c [B, W*T_f, d_c] and k_r [B, W*T_f, d_rope] plus frames_written."""

    def __init__(self, cfg: VmlaConfig, batch: int, device="cuda", fill: Optional[float] = None):
        rows = cfg.window_tokens
        dt = _dtype(cfg)
        self.cfg = cfg
        self.c = torch.empty((batch, rows, cfg.d_c), dtype=dt, device=device)
        self.k_r = torch.empty((batch, rows, cfg.d_rope), dtype=dt, device=device)
        if fill is not None:
            self.c.fill_(fill)
            self.k_r.fill_(fill)
        self.struct = CCache(self.c.data_ptr(), self.k_r.data_ptr(), batch, 0, 0)

    @property
    def batch(self) -> int:
        return self.struct.batch

    @property
    def frames_written(self) -> int:
        return self.struct.frames_written

    def nbytes(self) -> int:
        return self.c.numel() * self.c.element_size() + self.k_r.numel() * self.k_r.element_size()

    def save(self, path) -> None:
        """Checkpoint: the ring planes and frames_written (the whole state of the layer's cache)."""
        _save_planes(path, "latent", self.cfg, self.batch, self.frames_written, {"c": self.c, "k_r": self.k_r})

    @classmethod
    def load(cls, path, cfg: VmlaConfig, device="cuda") -> "LatentCache":
        """Restore a checkpoint written by save(); streaming continues exactly where it stopped."""
        state = _load_planes(path, "latent", cfg)
        cache = cls(cfg, state["batch"], device=device)
        cache.c.copy_(state["planes"]["c"])
        cache.k_r.copy_(state["planes"]["k_r"])
        cache.struct.frames_written = state["frames_written"]
        return cache


class DenseCache:
    """Dense per-head cache of the comparison layer: k [B, W*T_f, H, d_h], v [B, W*T_f, H, d_v]."""

    def __init__(self, cfg: VmlaConfig, batch: int, device="cuda", fill: Optional[float] = None):
        rows = cfg.window_tokens
        dt = _dtype(cfg)
        self.cfg = cfg
        self.k = torch.empty((batch, rows, cfg.n_heads, cfg.d_h), dtype=dt, device=device)
        self.v = torch.empty((batch, rows, cfg.n_heads, cfg.d_v), dtype=dt, device=device)
        if fill is not None:
            self.k.fill_(fill)
            self.v.fill_(fill)
        self.struct = CDenseCache(self.k.data_ptr(), self.v.data_ptr(), batch, 0, 0)

    @property
    def frames_written(self) -> int:
        return self.struct.frames_written

    def nbytes(self) -> int:
        return self.k.numel() * self.k.element_size() + self.v.numel() * self.v.element_size()

    def save(self, path) -> None:
        _save_planes(path, "dense", self.cfg, self.struct.batch, self.frames_written, {"k": self.k, "v": self.v})

    @classmethod
    def load(cls, path, cfg: VmlaConfig, device="cuda") -> "DenseCache":
        state = _load_planes(path, "dense", cfg)
        cache = cls(cfg, state["batch"], device=device)
        cache.k.copy_(state["planes"]["k"])
        cache.v.copy_(state["planes"]["v"])
        cache.struct.frames_written = state["frames_written"]
        return cache


def compress_append(cfg: VmlaConfig, x: torch.Tensor, w_dkv_kr: torch.Tensor, cache: LatentCache,
                    first_frame: Optional[int] = None) -> None:
    """Append one chunk x [B, F*T_f, D] to ``cache`` (first_frame defaults to cache.frames_written)."""
    B = cache.batch
    ff = cache.frames_written if first_frame is None else first_frame
    cc = c_config(cfg)
    check(LIB.vmla_compress_append(ctypes.byref(cc), _arg(x, cfg, (B, cfg.chunk_tokens, cfg.dim), "x"),
                                   _arg(w_dkv_kr, cfg, (cfg.d_c + cfg.d_rope, cfg.dim), "w_dkv_kr"),
                                   ff, ctypes.byref(cache.struct), _stream(x)))


def compress_rewrite(cfg: VmlaConfig, x: torch.Tensor, w_dkv_kr: torch.Tensor,
                     cache: LatentCache) -> None:
    """Recompute the newest chunk's cache rows in place from x [B, F*T_f, D] (one denoising step of a
    few-step chunk); frames_written is unchanged."""
    B = cache.batch
    cc = c_config(cfg)
    check(LIB.vmla_compress_rewrite(ctypes.byref(cc), _arg(x, cfg, (B, cfg.chunk_tokens, cfg.dim), "x"),
                                    _arg(w_dkv_kr, cfg, (cfg.d_c + cfg.d_rope, cfg.dim), "w_dkv_kr"),
                                    ctypes.byref(cache.struct), _stream(x)))


def absorb_q(cfg: VmlaConfig, q_nope: torch.Tensor, q_rope: torch.Tensor, w_uk: torch.Tensor,
             first_frame: int, n_query_chunks: int = 1, out: Optional[torch.Tensor] = None):
    B, nq = q_nope.shape[0], q_nope.shape[1]
    H = cfg.n_heads
    if out is None:
        out = torch.empty((B, nq, H, cfg.d_qk), dtype=_dtype(cfg), device=q_nope.device)
    if nq != n_query_chunks * cfg.chunk_tokens:
        raise ValueError("q_nope covers %d tokens, expected %d" % (nq, n_query_chunks * cfg.chunk_tokens))
    cc = c_config(cfg)
    check(LIB.vmla_absorb_q(ctypes.byref(cc), B, n_query_chunks,
                            _arg(q_nope, cfg, (B, nq, H, cfg.d_nope), "q_nope"),
                            _arg(q_rope, cfg, (B, nq, H, cfg.d_rope), "q_rope"),
                            _arg(w_uk, cfg, (H, cfg.d_nope, cfg.d_c), "w_uk"), first_frame,
                            _arg(out, cfg, (B, nq, H, cfg.d_qk), "q_abs"), _stream(q_nope)))
    return out


def latent_attention(cfg: VmlaConfig, q_abs: torch.Tensor, cache: LatentCache, first_frame: int,
                     n_query_chunks: int = 1, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, want_lse: bool = False):
    B, nq, H = q_abs.shape[0], q_abs.shape[1], cfg.n_heads
    if out is None:
        out = torch.empty((B, nq, H, cfg.d_c), dtype=_dtype(cfg), device=q_abs.device)
    if lse is None and want_lse:
        lse = torch.empty((B, nq, H), dtype=torch.float32, device=q_abs.device)
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, nq, H)
                            or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 [B, Nq, H] tensor")
    if B != cache.batch:
        raise ValueError("q_abs batch does not match the cache")
    cc = c_config(cfg)
    check(LIB.vmla_latent_attention(ctypes.byref(cc), _arg(q_abs, cfg, (B, nq, H, cfg.d_qk), "q_abs"),
                                    ctypes.byref(cache.struct), first_frame, n_query_chunks,
                                    _arg(out, cfg, (B, nq, H, cfg.d_c), "out_latent"),
                                    lse.data_ptr() if lse is not None else None, _stream(q_abs)))
    return (out, lse) if (lse is not None) else out


def latent_attention_fused(cfg: VmlaConfig, q_nope: torch.Tensor, q_rope: torch.Tensor, w_uk: torch.Tensor,
                           w_uv: torch.Tensor, cache: LatentCache, first_frame: int, n_query_chunks: int = 1,
                           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                           want_lse: bool = False):
    """Absorbed query + latent attention + value up-projection in one launch:
    q^nope [B, Nq, H, d_nope], q^rope [B, Nq, H, d_rope] -> o [B, Nq, H, d_v] (and lse [B, Nq, H])."""
    B, nq, H = cache.batch, q_nope.shape[1], cfg.n_heads
    if out is None:
        out = torch.empty((B, nq, H, cfg.d_v), dtype=_dtype(cfg), device=q_nope.device)
    if lse is None and want_lse:
        lse = torch.empty((B, nq, H), dtype=torch.float32, device=q_nope.device)
    if nq != n_query_chunks * cfg.chunk_tokens:
        raise ValueError("q_nope covers %d tokens, expected %d" % (nq, n_query_chunks * cfg.chunk_tokens))
    cc = c_config(cfg)
    check(LIB.vmla_latent_attention_fused(
        ctypes.byref(cc), _arg(q_nope, cfg, (B, nq, H, cfg.d_nope), "q_nope"),
        _arg(q_rope, cfg, (B, nq, H, cfg.d_rope), "q_rope"), _arg(w_uk, cfg, (H, cfg.d_nope, cfg.d_c), "w_uk"),
        _arg(w_uv, cfg, (H, cfg.d_v, cfg.d_c), "w_uv"), ctypes.byref(cache.struct), first_frame, n_query_chunks,
        _arg(out, cfg, (B, nq, H, cfg.d_v), "out"), lse.data_ptr() if lse is not None else None,
        _stream(q_nope)))
    return (out, lse) if (lse is not None) else out


def value_up(cfg: VmlaConfig, o_latent: torch.Tensor, w_uv: torch.Tensor,
             out: Optional[torch.Tensor] = None):
    B, n, H = o_latent.shape[0], o_latent.shape[1], cfg.n_heads
    if out is None:
        out = torch.empty((B, n, H, cfg.d_v), dtype=_dtype(cfg), device=o_latent.device)
    cc = c_config(cfg)
    check(LIB.vmla_value_up(ctypes.byref(cc), B, n, _arg(o_latent, cfg, (B, n, H, cfg.d_c), "out_latent"),
                            _arg(w_uv, cfg, (H, cfg.d_v, cfg.d_c), "w_uv"),
                            _arg(out, cfg, (B, n, H, cfg.d_v), "out"), _stream(o_latent)))
    return out


def rope_q(cfg: VmlaConfig, q_nope: torch.Tensor, q_rope: torch.Tensor, first_frame: int,
           n_query_chunks: int = 1, out: Optional[torch.Tensor] = None):
    B, nq, H = q_nope.shape[0], q_nope.shape[1], cfg.n_heads
    if out is None:
        out = torch.empty((B, nq, H, cfg.d_h), dtype=_dtype(cfg), device=q_nope.device)
    cc = c_config(cfg)
    check(LIB.vmla_rope_q(ctypes.byref(cc), B, n_query_chunks,
                          _arg(q_nope, cfg, (B, nq, H, cfg.d_nope), "q_nope"),
                          _arg(q_rope, cfg, (B, nq, H, cfg.d_rope), "q_rope"), first_frame,
                          _arg(out, cfg, (B, nq, H, cfg.d_h), "q"), _stream(q_nope)))
    return out


def dense_append(cfg: VmlaConfig, x: torch.Tensor, w_kv: torch.Tensor, cache: DenseCache,
                 first_frame: Optional[int] = None) -> None:
    B = cache.struct.batch
    ff = cache.frames_written if first_frame is None else first_frame
    cc = c_config(cfg)
    check(LIB.vmla_dense_append(ctypes.byref(cc), _arg(x, cfg, (B, cfg.chunk_tokens, cfg.dim), "x"),
                                _arg(w_kv, cfg, (cfg.n_heads * (cfg.d_h + cfg.d_v), cfg.dim), "w_kv"),
                                ff, ctypes.byref(cache.struct), _stream(x)))


def dense_rewrite(cfg: VmlaConfig, x: torch.Tensor, w_kv: torch.Tensor, cache: DenseCache) -> None:
    """Dense counterpart of compress_rewrite."""
    B = cache.struct.batch
    cc = c_config(cfg)
    check(LIB.vmla_dense_rewrite(ctypes.byref(cc), _arg(x, cfg, (B, cfg.chunk_tokens, cfg.dim), "x"),
                                 _arg(w_kv, cfg, (cfg.n_heads * (cfg.d_h + cfg.d_v), cfg.dim), "w_kv"),
                                 ctypes.byref(cache.struct), _stream(x)))


def dense_mha(cfg: VmlaConfig, q: torch.Tensor, cache: DenseCache, first_frame: int,
              n_query_chunks: int = 1, out: Optional[torch.Tensor] = None,
              lse: Optional[torch.Tensor] = None, want_lse: bool = False):
    B, nq, H = q.shape[0], q.shape[1], cfg.n_heads
    if out is None:
        out = torch.empty((B, nq, H, cfg.d_v), dtype=_dtype(cfg), device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, nq, H), dtype=torch.float32, device=q.device)
    cc = c_config(cfg)
    check(LIB.vmla_dense_mha(ctypes.byref(cc), _arg(q, cfg, (B, nq, H, cfg.d_h), "q"),
                             ctypes.byref(cache.struct), first_frame, n_query_chunks,
                             _arg(out, cfg, (B, nq, H, cfg.d_v), "out"),
                             lse.data_ptr() if lse is not None else None, _stream(q)))
    return (out, lse) if (lse is not None) else out


def device_status(stream: Optional[int] = None) -> int:
    """Synchronise the stream and return (and clear) the device status word (0 = no wait ran out)."""
    code = ctypes.c_int32(0)
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    st = LIB.vmla_device_status(s, ctypes.byref(code))
    if st not in (VMLA_OK, VMLA_ERR_TIMEOUT):
        check(st)
    return code.value


def check_attention_window(cfg: VmlaConfig, frames_written: int, first_frame: int,
                           n_query_chunks: int = 1) -> None:
    """Raise VmlaError unless an attention call with these frames would pass the window rule."""
    cc = c_config(cfg)
    check(LIB.vmla_check_attention_window(ctypes.byref(cc), frames_written, first_frame, n_query_chunks))


def fused_supported(cfg: VmlaConfig) -> bool:
    """Whether latent_attention_fused supports this configuration (host-only library check)."""
    cc = c_config(cfg)
    st = LIB.vmla_check_fused(ctypes.byref(cc))
    if st == VMLA_ERR_UNSUPPORTED:
        return False
    check(st)
    return True


def set_wait_timeout_ms(ms: int) -> int:
    """Bound (ms) of every device-side wait of later launches; returns the previous bound."""
    return int(LIB.vmla_set_wait_timeout_ms(int(ms)))


def debug_drop_kv_tile(tile: int) -> None:
    """Test hook: the next bf16 latent attention launch skips loading KV tile ``tile`` (its wait runs
    out and vmla_device_status reports it); tile < 0 clears the request."""
    LIB.vmla_debug_drop_kv_tile(int(tile))


def debug_exp2_poly(x: torch.Tensor) -> torch.Tensor:
    """Test hook: the FMA-pipe 2^x of the attention kernels' softmax, applied to a float32 CUDA tensor."""
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    check(LIB.vmla_debug_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(), _stream(x)))
    return y


def launch_count() -> int:
    return int(LIB.vmla_launch_count())


def latent_cache_bytes(cfg: VmlaConfig, batch: int) -> int:
    cc = c_config(cfg)
    return int(LIB.vmla_latent_cache_bytes(ctypes.byref(cc), batch))


def dense_cache_bytes(cfg: VmlaConfig, batch: int) -> int:
    cc = c_config(cfg)
    return int(LIB.vmla_dense_cache_bytes(ctypes.byref(cc), batch))


def plan_capacity(cfg: VmlaConfig, n_layers: int, budget_bytes: int, *, dense: bool = False,
                  fused: bool = False, fixed_bytes: int = 0, extra_bytes_per_seq: int = 0) -> dict:
    """Largest batch of sequences whose n_layers caches, one layer step's tensors and the given extra
    bytes fit ``budget_bytes`` (host-only; see vmla_plan_capacity).  dense: the dense MHA path;
    fused: the latent path through vmla_latent_attention_fused."""
    cc = c_config(cfg)
    out = CCapacity()
    path = 1 if dense else (2 if fused else 0)
    check(LIB.vmla_plan_capacity(ctypes.byref(cc), n_layers, path, int(budget_bytes),
                                 int(fixed_bytes), int(extra_bytes_per_seq), ctypes.byref(out)))
    return {n: int(getattr(out, n)) for n, _ in CCapacity._fields_}


def compress_append_rows(cfg: VmlaConfig, x_rows: torch.Tensor, w_dkv_kr: torch.Tensor, first_frame: int,
                         token_begin: int, replicas, batch: int) -> None:
    """Compress tokens token_begin .. token_begin + n - 1 of the chunk (x_rows [B, n, D]) into the ring of
    every replica (a sequence of CCache structs, possibly holding peer pointers).  frames_written of the
    replicas is not advanced."""
    n = x_rows.shape[1]
    cc = c_config(cfg)
    arr = (CCache * len(replicas))(*replicas)
    check(LIB.vmla_compress_append_rows(ctypes.byref(cc), _arg(x_rows, cfg, (batch, n, cfg.dim), "x_rows"),
                                        _arg(w_dkv_kr, cfg, (cfg.d_c + cfg.d_rope, cfg.dim), "w_dkv_kr"),
                                        first_frame, token_begin, n, arr, len(replicas), _stream(x_rows)))


def latent_attention_fused_rows(cfg: VmlaConfig, q_nope: torch.Tensor, q_rope: torch.Tensor, w_uk: torch.Tensor,
                                w_uv: torch.Tensor, cache: LatentCache, first_frame: int, token_begin: int,
                                n_query_chunks: int = 1, out: Optional[torch.Tensor] = None,
                                lse: Optional[torch.Tensor] = None, want_lse: bool = False):
    """The fused attention for query tokens token_begin .. token_begin + n - 1 of the call only:
    q^nope [B, n, H, d_nope], q^rope [B, n, H, d_rope] -> o [B, n, H, d_v] (and lse [B, n, H])."""
    B, n, H = cache.batch, q_nope.shape[1], cfg.n_heads
    if out is None:
        out = torch.empty((B, n, H, cfg.d_v), dtype=_dtype(cfg), device=q_nope.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n, H), dtype=torch.float32, device=q_nope.device)
    cc = c_config(cfg)
    check(LIB.vmla_latent_attention_fused_rows(
        ctypes.byref(cc), _arg(q_nope, cfg, (B, n, H, cfg.d_nope), "q_nope"),
        _arg(q_rope, cfg, (B, n, H, cfg.d_rope), "q_rope"), _arg(w_uk, cfg, (H, cfg.d_nope, cfg.d_c), "w_uk"),
        _arg(w_uv, cfg, (H, cfg.d_v, cfg.d_c), "w_uv"), ctypes.byref(cache.struct), first_frame, n_query_chunks,
        token_begin, n, _arg(out, cfg, (B, n, H, cfg.d_v), "out"), lse.data_ptr() if lse is not None else None,
        _stream(q_nope)))
    return (out, lse) if (lse is not None) else out


def ipc_export(t: torch.Tensor) -> bytes:
    """Serialisable handle (72 bytes) of the device buffer holding tensor t."""
    h = CIpcHandle()
    check(LIB.vmla_ipc_export(t.data_ptr(), ctypes.byref(h)))
    return bytes(ctypes.string_at(ctypes.addressof(h), ctypes.sizeof(h)))


def ipc_import(handle: bytes) -> int:
    """Map another process's buffer (a handle from ipc_export) into this one; returns the device pointer."""
    h = CIpcHandle.from_buffer_copy(handle)
    p = ctypes.c_void_p()
    check(LIB.vmla_ipc_import(ctypes.byref(h), ctypes.byref(p)))
    return int(p.value)


def ipc_release(ptr: int) -> None:
    check(LIB.vmla_ipc_release(ptr))


class Executor:
    """Streaming executor of the C library: layer steps with inputs and outputs in (pinned) host memory,
    the copies of neighbouring steps overlapping each step's kernels.  The device workspace is allocated
    here with PyTorch; kernels run on the current stream at creation."""

    def __init__(self, cfg: VmlaConfig, batch: int, device="cuda"):
        self.cfg, self.batch = cfg, batch
        cc = c_config(cfg)
        nbytes = int(LIB.vmla_executor_workspace_bytes(ctypes.byref(cc), batch))
        if nbytes < 0:
            raise VmlaError(VMLA_ERR_INVALID_ARG, "bad executor arguments")
        self.workspace = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.workspace.data_ptr()
        aligned = (base + 255) // 256 * 256
        self._stream = torch.cuda.current_stream(self.workspace.device)
        handle = ctypes.c_void_p()
        check(LIB.vmla_executor_create(ctypes.byref(cc), batch, aligned, nbytes, self._stream.cuda_stream,
                                       ctypes.byref(handle)))
        self._h = handle
        self._keep = []

    def submit(self, cache: LatentCache, w_dkv_kr, w_uk, w_uv, x_host, q_nope_host, q_rope_host, out_host):
        cfg = self.cfg
        for t, name in ((x_host, "x_host"), (q_nope_host, "q_nope_host"), (q_rope_host, "q_rope_host"),
                        (out_host, "out_host")):
            if t.is_cuda or not t.is_contiguous() or t.dtype != _dtype(cfg):
                raise ValueError(f"{name} must be a contiguous host tensor of {_dtype(cfg)}")
        B, n, H = self.batch, cfg.chunk_tokens, cfg.n_heads
        shapes = ((x_host, (B, n, cfg.dim)), (q_nope_host, (B, n, H, cfg.d_nope)),
                  (q_rope_host, (B, n, H, cfg.d_rope)), (out_host, (B, n, H, cfg.d_v)))
        for t, shp in shapes:
            if tuple(t.shape) != shp:
                raise ValueError(f"host tensor has shape {tuple(t.shape)}, expected {shp}")
        check(LIB.vmla_executor_submit(self._h, ctypes.byref(cache.struct),
                                       _arg(w_dkv_kr, cfg, (cfg.d_c + cfg.d_rope, cfg.dim), "w_dkv_kr"),
                                       _arg(w_uk, cfg, (H, cfg.d_nope, cfg.d_c), "w_uk"),
                                       _arg(w_uv, cfg, (H, cfg.d_v, cfg.d_c), "w_uv"),
                                       x_host.data_ptr(), q_nope_host.data_ptr(), q_rope_host.data_ptr(),
                                       out_host.data_ptr()))
        self._keep.append((x_host, q_nope_host, q_rope_host, out_host))

    def wait(self) -> None:
        st = LIB.vmla_executor_wait(self._h)
        self._keep.clear()
        check(st)

    def close(self) -> None:
        if self._h is not None:
            LIB.vmla_executor_destroy(self._h)
            self._h = None
            self._keep.clear()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def layer_step(cfg: VmlaConfig, x: torch.Tensor, q_nope: torch.Tensor, q_rope: torch.Tensor,
               w_dkv_kr: torch.Tensor, w_uk: torch.Tensor, w_uv: torch.Tensor, cache: LatentCache,
               bufs: Optional[dict] = None, fused: Optional[bool] = None) -> torch.Tensor:
    """One streaming step of one layer: append the chunk x, then attend with its queries and project
    the values up.  Returns o [B, F*T_f, H, d_v].  ``bufs`` (optional) holds reusable outputs under the
    keys q_abs, o_latent, o.  ``fused`` selects the single-launch absorb + attention + value-up kernel
    (default: for bf16 configs whose shapes it supports) or the three separate calls."""
    bufs = bufs if bufs is not None else {}
    if fused is None:
        fused = fused_supported(cfg)
    f0 = cache.frames_written
    compress_append(cfg, x, w_dkv_kr, cache, f0)
    if fused:
        return latent_attention_fused(cfg, q_nope, q_rope, w_uk, w_uv, cache, f0, out=bufs.get("o"))
    q_abs = absorb_q(cfg, q_nope, q_rope, w_uk, f0, 1, out=bufs.get("q_abs"))
    o_lat = latent_attention(cfg, q_abs, cache, f0, 1, out=bufs.get("o_latent"))
    return value_up(cfg, o_lat, w_uv, out=bufs.get("o"))


__all__ = ["LIB", "VmlaError", "LatentCache", "DenseCache", "compress_append", "absorb_q",
           "latent_attention", "value_up", "rope_q", "dense_append", "dense_mha", "device_status",
           "launch_count", "latent_cache_bytes", "dense_cache_bytes", "layer_step", "c_config",
           "compress_rewrite", "dense_rewrite", "plan_capacity", "CCapacity", "latent_attention_fused", "Executor",
           "compress_append_rows", "latent_attention_fused_rows", "ipc_export", "ipc_import", "ipc_release",
           "CIpcHandle", "check_attention_window", "fused_supported",
           "CConfig", "CCache", "CDenseCache", "EXPORTED", "VMLA_F32", "VMLA_BF16"]
