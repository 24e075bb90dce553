"""Float64 CPU oracle for VideoMLA latent-KV attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs
of ``bench.py`` may import this module.  It shares no code with the CUDA library: it is a plain, slow,
obviously correct restatement of what the method computes, in float64, with NumPy matrix products as
the only library primitive.  Every function names the passage it follows.

Sources (page title, section):
  [ABS]   "VideoMLA: Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video Diffusion",
          abstract (chatpaper.ai page, English and Spanish text).
  [TS-P]  same title, gist.science technical summary, "Problem definition" section.
  [TS-M1] .. [TS-M4]  same summary, "Method: VideoMLA" items 1-4 (shared latent, on-demand
          reconstruction, decoupled 3D-RoPE, memory reduction).
  [TS-R]  same summary, "Results" section, "Scalability" item (batch size at a fixed memory budget).

Readings where the pages are silent (each one is listed with its reason in the design notes):
  * the head-shared key k^R_t is projected from x_t by its own matrix W^KR (not from c_t);
  * 3D-RoPE acts on interleaved pairs (u[2k], u[2k+1]); the first P_t pairs turn with the absolute
    latent-frame index f, the next P_h with the row i, the last P_w with the column j; within an axis of
    P_a pairs, pair m turns at omega = theta^(-m/P_a); the rotation is (a cos - b sin, a sin + b cos);
  * tokens of a frame are in raster order (n = i*grid_w + j), positions start at 0;
  * the window counts frames and includes the current chunk: query chunk k of a call sees key frames
    [max(0, hi_k - W), hi_k) with hi_k the end frame of its chunk (bidirectional inside a chunk,
    causal across chunks);
  * softmax scale 1/sqrt(d_nope + d_rope); d_v = d_h;
  * few-step generation: a chunk is denoised over several steps and its own keys and values are
    recomputed from each step's features, replacing the chunk's entries in place (older frames kept);
  * batch capacity: the bytes that grow with the batch are every layer's cache plus one layer step's
    tensors (reused across layers) plus caller-given activations; weights are fixed.

Parity status: every function here is pinned by tests/test_oracle_pins.py (closed-form cache
arithmetic printed on the pages, RoPE invariants and the textbook complex-number 1-D RoPE, brute-force
loops on tiny inputs, and torch's float64 scaled_dot_product_attention for the MLA == MHA identity).
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------------------------------
# Cache arithmetic  [TS-M4], [TS-P]
# ---------------------------------------------------------------------------------------------------
def dense_scalars_per_token(n_heads: int, d_h: int) -> int:
    """Dense per-head layout: every cached token stores K and V for every head, 2 * n_h * d_h scalars
    [TS-M4]."""
    return 2 * n_heads * d_h


def latent_scalars_per_token(d_c: int, d_rope: int) -> int:
    """Latent layout: the pair (c^KV_t, k^R_t), d_c + d_rope scalars [TS-M3, TS-M4]."""
    return d_c + d_rope


def memory_reduction(n_heads: int, d_h: int, d_c: int, d_rope: int) -> float:
    """Fraction of per-token KV memory removed at every cached layer [ABS], [TS-M4]."""
    return 1.0 - latent_scalars_per_token(d_c, d_rope) / dense_scalars_per_token(n_heads, d_h)


# ---------------------------------------------------------------------------------------------------
# Positions and 3D-RoPE  [TS-M3]
# ---------------------------------------------------------------------------------------------------
def token_positions(first_frame: int, n_tokens: int, grid_h: int, grid_w: int) -> np.ndarray:
    """(f, i, j) of the tokens of consecutive latent frames starting at ``first_frame``; tokens of a
    frame in raster order.  Returns int64 [n_tokens, 3]."""
    per_frame = grid_h * grid_w
    n = np.arange(n_tokens, dtype=np.int64)
    f = first_frame + n // per_frame
    r = n % per_frame
    return np.stack([f, r // grid_w, r % grid_w], axis=-1)


def rope3d_angles(pos: np.ndarray, pairs: tuple, theta: float) -> np.ndarray:
    """Rotation angle of every rotary pair: pair m of the block that belongs to axis a (a = frame,
    row, column, in that order) turns by pos[a] * theta^(-m / P_a).  Returns [..., sum(pairs)]."""
    cols = []
    for axis, n_pairs in enumerate(pairs):
        for m in range(n_pairs):
            omega = float(theta) ** (-m / n_pairs)
            cols.append(pos[..., axis].astype(F64) * omega)
    return np.stack(cols, axis=-1)


def rope3d(u: np.ndarray, pos: np.ndarray, pairs: tuple, theta: float) -> np.ndarray:
    """Rotate the interleaved pairs (u[2k], u[2k+1]) of ``u`` [..., d_rope] by the 3D-RoPE angles of
    ``pos`` [..., 3] (broadcast against u's leading dims)."""
    alpha = rope3d_angles(pos, pairs, theta)
    u = np.asarray(u, F64)
    a = u[..., 0::2]
    b = u[..., 1::2]
    cos, sin = np.cos(alpha), np.sin(alpha)
    rotated = np.stack([a * cos - b * sin, a * sin + b * cos], axis=-1)   # [..., pairs, 2]
    return rotated.reshape(rotated.shape[:-2] + (2 * rotated.shape[-2],))


# ---------------------------------------------------------------------------------------------------
# Cache write  [TS-M1], [TS-M3], sliding window [ABS], [TS-P]
# ---------------------------------------------------------------------------------------------------
def compress(x: np.ndarray, w_dkv_kr: np.ndarray, d_c: int, pos: np.ndarray, pairs: tuple,
             theta: float):
    """c^KV_t = W^KV_down x_t and k^R_t = RoPE3D(W^KR x_t) for tokens x [..., T, D]; ``w_dkv_kr`` holds
    W^KV_down (first d_c rows) and W^KR (last d_rope rows).  Returns (c [..., T, d_c],
    k_r [..., T, d_rope])."""
    x = np.asarray(x, dtype=F64)
    w = np.asarray(w_dkv_kr, dtype=F64)
    c = x @ w[:d_c].T
    k_r = rope3d(x @ w[d_c:].T, pos, pairs, theta)
    return c, k_r


def frame_of_slot(slot: int, frames_written: int, window_frames: int) -> int:
    """Latent frame held by ring slot ``slot`` after ``frames_written`` frames were appended to a ring
    of ``window_frames`` frame slots (frame f goes to slot f mod W, evicting frame f - W); -1 if the
    slot was never written."""
    if frames_written <= 0:
        return -1
    last = frames_written - 1
    f = last - ((last - slot) % window_frames)
    return f if f >= 0 else -1


def ring_from_history(hist: np.ndarray, frames_written: int, window_frames: int,
                      tokens_per_frame: int, first_frame: int = 0) -> tuple:
    """Expected ring-buffer plane from the history ``hist`` of one batch element, which holds frames
    first_frame .. frames_written-1 in order ([(frames_written - first_frame)*T_f, d]): slot s holds frame
    frame_of_slot(s); frames before first_frame were never written.  Returns (plane [W*T_f, d] with NaN
    in unwritten slots, written-row mask [W*T_f])."""
    d = hist.shape[-1]
    plane = np.full((window_frames * tokens_per_frame, d), np.nan, dtype=F64)
    written = np.zeros(window_frames * tokens_per_frame, dtype=bool)
    for s in range(window_frames):
        f = frame_of_slot(s, frames_written, window_frames)
        if f < first_frame:
            continue
        r = f - first_frame
        plane[s * tokens_per_frame:(s + 1) * tokens_per_frame] = \
            hist[r * tokens_per_frame:(r + 1) * tokens_per_frame]
        written[s * tokens_per_frame:(s + 1) * tokens_per_frame] = True
    return plane, written


# ---------------------------------------------------------------------------------------------------
# Queries, reconstruction, absorption  [TS-M2], [TS-M3]
# ---------------------------------------------------------------------------------------------------
def rotate_query(q_rope: np.ndarray, pos: np.ndarray, pairs: tuple, theta: float) -> np.ndarray:
    """q^R_{n,h} = RoPE3D(q^rope_{n,h}) at the query token's own (f, i, j); q_rope [..., T, H, d_rope],
    pos [T, 3]."""
    return rope3d(np.asarray(q_rope, F64), pos[:, None, :], pairs, theta)


def reconstruct_kv(c: np.ndarray, k_r: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray):
    """On-demand per-head keys and values from the shared latent [TS-M2]:
    k_{t,h} = [W^K_up,h c_t ; k^R_t] (d_nope + d_rope), v_{t,h} = W^V_up,h c_t (d_v).
    c [T, d_c], k_r [T, d_rope], w_uk [H, d_nope, d_c], w_uv [H, d_v, d_c] -> k [T, H, d_h], v [T, H, d_v]."""
    c = np.asarray(c, F64)
    k_r = np.asarray(k_r, F64)
    n_heads = w_uk.shape[0]
    k = np.empty((c.shape[0], n_heads, w_uk.shape[1] + k_r.shape[-1]), dtype=F64)
    v = np.empty((c.shape[0], n_heads, w_uv.shape[1]), dtype=F64)
    for h in range(n_heads):
        k[:, h, :w_uk.shape[1]] = c @ np.asarray(w_uk[h], F64).T
        k[:, h, w_uk.shape[1]:] = k_r
        v[:, h, :] = c @ np.asarray(w_uv[h], F64).T
    return k, v


def absorbed_query(q_nope: np.ndarray, q_rope_rot: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """Absorbed query row [q~_h ; q^R_h] with q~_h = (W^K_up,h)^T q^nope_h, so that
    q~_h . c_t = q^nope_h . (W^K_up,h c_t).  q_nope [T, H, d_nope], q_rope_rot [T, H, d_rope]
    -> [T, H, d_c + d_rope]."""
    q_tilde = np.einsum('hnc,thn->thc', np.asarray(w_uk, F64), np.asarray(q_nope, F64))
    return np.concatenate([q_tilde, np.asarray(q_rope_rot, F64)], axis=-1)


# ---------------------------------------------------------------------------------------------------
# Visibility (sliding window + block-causal chunks)  [ABS], [TS-P]
# ---------------------------------------------------------------------------------------------------
def query_chunk_end(first_frame: int, n_tokens: int, chunk_frames: int, tokens_per_frame: int):
    """End frame hi_n (exclusive) of the chunk of each query token of a call whose first query frame
    is ``first_frame``."""
    n = np.arange(n_tokens, dtype=np.int64)
    chunk = n // (chunk_frames * tokens_per_frame)
    return first_frame + (chunk + 1) * chunk_frames


def visible(query_hi: np.ndarray, key_frames: np.ndarray, window_frames: int) -> np.ndarray:
    """mask[n, t]: key of frame key_frames[t] is visible to query n iff
    max(0, hi_n - W) <= frame < hi_n."""
    lo = np.maximum(0, query_hi - window_frames)[:, None]
    hi = query_hi[:, None]
    kf = key_frames[None, :]
    return (kf >= lo) & (kf < hi)


# ---------------------------------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------------------------------
def _masked_softmax(s: np.ndarray, mask: np.ndarray):
    """Naive softmax over the last axis restricted to ``mask``; also returns log-sum-exp."""
    s = np.where(mask, s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.where(mask, np.exp(s - m), 0.0)
    z = np.sum(e, axis=-1, keepdims=True)
    return e / z, (np.log(z) + m)[..., 0]


def mha(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray, scale: float):
    """Textbook per-head softmax attention.  q [N, H, d], k [T, H, d], v [T, H, d_v], mask [N, T]
    -> (o [N, H, d_v], lse [N, H], p [N, H, T])."""
    q, k, v = np.asarray(q, F64), np.asarray(k, F64), np.asarray(v, F64)
    s = np.stack([q[:, h, :] @ k[:, h, :].T for h in range(q.shape[1])], axis=1) * scale
    p, lse = _masked_softmax(s, mask[:, None, :])
    o = np.stack([p[:, h, :] @ v[:, h, :] for h in range(q.shape[1])], axis=1)
    return o, lse, p


def latent_attention(q_abs: np.ndarray, c: np.ndarray, k_r: np.ndarray, mask: np.ndarray,
                     scale: float):
    """Attention in the absorbed form, written as its plain definition: per (n, h) the score of key t is
    scale * (q~_{n,h} . c_t + q^R_{n,h} . k^R_t); the output is the latent sum o~_{n,h} = sum_t p_t c_t.
    q_abs [N, H, d_c + d_rope], c [T, d_c], k_r [T, d_rope], mask [N, T]
    -> (o_latent [N, H, d_c], lse [N, H])."""
    q_abs = np.asarray(q_abs, F64)
    c, k_r = np.asarray(c, F64), np.asarray(k_r, F64)
    d_c = c.shape[-1]
    s = (q_abs[..., :d_c] @ c.T + q_abs[..., d_c:] @ k_r.T) * scale        # [N, H, T]
    p, lse = _masked_softmax(s, mask[:, None, :])
    return p @ c, lse


def value_up(o_latent: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """o_{n,h} = W^V_up,h o~_{n,h}: the value up-projection applied once to the attention-weighted latent
    [TS-M2].  o_latent [N, H, d_c], w_uv [H, d_v, d_c] -> [N, H, d_v]."""
    return np.einsum('hvc,nhc->nhv', np.asarray(w_uv, F64), np.asarray(o_latent, F64))


# ---------------------------------------------------------------------------------------------------
# A whole layer call, non-absorbed (the reference for end-to-end parity)
# ---------------------------------------------------------------------------------------------------
class History:
    """Full, never-evicted history of one layer's cache for one batch element: c^KV and k^R of every
    appended token, in frame order.  The sliding window is taken by slicing (frames), never by a ring."""

    def __init__(self, d_c: int, d_rope: int):
        self.c = np.zeros((0, d_c), dtype=F64)
        self.k_r = np.zeros((0, d_rope), dtype=F64)
        self.frames = np.zeros((0,), dtype=np.int64)

    def append(self, c: np.ndarray, k_r: np.ndarray, frames: np.ndarray):
        self.c = np.concatenate([self.c, c])
        self.k_r = np.concatenate([self.k_r, k_r])
        self.frames = np.concatenate([self.frames, frames])

    def rewrite_newest(self, c: np.ndarray, k_r: np.ndarray, frames: np.ndarray):
        """One denoising step of a few-step chunk: the newest tokens (whose frames must be ``frames``)
        get the entries computed from this step's features; every older entry is kept.  [TS-P] names
        Self-Forcing-style training; recomputing the chunk in place is the reading."""
        n = len(frames)
        if n == 0 or n > len(self.frames) or not np.array_equal(self.frames[-n:], frames):
            raise ValueError("rewrite must cover exactly the newest tokens")
        self.c = np.concatenate([self.c[:-n], c])
        self.k_r = np.concatenate([self.k_r[:-n], k_r])


def build_history(x_chunks, w_dkv_kr, b: int, *, d_c, d_rope, chunk_frames, grid_h, grid_w, pairs,
                  theta) -> History:
    """Append the chunks x_chunks[k][b] (frames k*F .. (k+1)*F-1) to a fresh history of batch
    element ``b``."""
    hist = History(d_c, d_rope)
    per_chunk = chunk_frames * grid_h * grid_w
    for k, x in enumerate(x_chunks):
        pos = token_positions(k * chunk_frames, per_chunk, grid_h, grid_w)
        c, k_r = compress(np.asarray(x[b], F64), w_dkv_kr, d_c, pos, pairs, theta)
        hist.append(c, k_r, pos[:, 0])
    return hist


def layer_reference(hist: History, q_nope, q_rope, w_uk, w_uv, *, first_frame, query_rows,
                    chunk_frames, window_frames, grid_h, grid_w, pairs, theta, scale):
    """Non-absorbed reference of one attention call for one batch element: per-head K/V are
    materialised from the latent [TS-M2], queries are [q^nope ; RoPE3D(q^rope)], and naive softmax
    attention runs under the window / block-causal mask.

    ``q_nope`` [Nq, H, d_nope] and ``q_rope`` [Nq, H, d_rope] hold the whole query set of the call; only
    the rows listed in ``query_rows`` are evaluated.  Returns a dict with o [R, H, d_v], o_latent
    [R, H, d_c], lse [R, H], q_abs [R, H, d_c + d_rope]."""
    per_frame = grid_h * grid_w
    nq = q_nope.shape[0]
    rows = np.asarray(query_rows, dtype=np.int64)
    pos = token_positions(first_frame, nq, grid_h, grid_w)[rows]
    hi = query_chunk_end(first_frame, nq, chunk_frames, per_frame)[rows]
    q_r = rotate_query(np.asarray(q_rope, F64)[rows], pos, pairs, theta)
    q = np.concatenate([np.asarray(q_nope, F64)[rows], q_r], axis=-1)
    mask = visible(hi, hist.frames, window_frames)
    k, v = reconstruct_kv(hist.c, hist.k_r, w_uk, w_uv)
    o, lse, p = mha(q, k, v, mask, scale)
    o_latent = p @ hist.c
    q_abs = absorbed_query(np.asarray(q_nope, F64)[rows], q_r, w_uk)
    return {"o": o, "o_latent": o_latent, "lse": lse, "q_abs": q_abs, "mask": mask}


# ---------------------------------------------------------------------------------------------------
# Batch capacity at a fixed memory budget  [TS-R], [TS-M4]
# ---------------------------------------------------------------------------------------------------
def step_tensors(batch: int, *, dim, n_heads, d_nope, d_rope, d_c, d_v, tokens_per_chunk, dense,
                 fused=False):
    """Shapes of the tensors one layer step holds for ``batch`` sequences (reused by every layer):
    the chunk features and, latent path, q^nope, q^rope, the absorbed query, the latent output and the
    output (the fused latent step keeps the absorbed query and the latent output on chip); dense path,
    the query and the output."""
    B, N, H = batch, tokens_per_chunk, n_heads
    if dense:
        return {"x": (B, N, dim), "q": (B, N, H, d_nope + d_rope), "out": (B, N, H, d_v)}
    t = {"x": (B, N, dim), "q_nope": (B, N, H, d_nope), "q_rope": (B, N, H, d_rope), "out": (B, N, H, d_v)}
    if not fused:
        t.update({"q_abs": (B, N, H, d_c + d_rope), "out_latent": (B, N, H, d_c)})
    return t


def layer_weights(*, dim, n_heads, d_nope, d_rope, d_c, d_v, dense):
    """Shapes of one layer's attention-path weights: W^KV_down with W^KR stacked, W^K_up and W^V_up
    per head [TS-M1, TS-M2, TS-M3]; dense: per-head K and V projections."""
    if dense:
        return {"w_kv": (n_heads * (d_nope + d_rope + d_v), dim)}
    return {"w_dkv_kr": (d_c + d_rope, dim), "w_uk": (n_heads, d_nope, d_c), "w_uv": (n_heads, d_v, d_c)}


def memory_bytes(batch: int, *, n_layers, window_tokens, elt_bytes, fixed_bytes, extra_bytes_per_seq,
                 dense, fused=False, **shape) -> int:
    """Every byte held at once for ``batch`` sequences: each layer's cache (per token the dense
    2*n_h*d_h or the latent d_c + d_rope scalars [TS-M4]), each layer's weights, one layer step's tensors,
    the caller's fixed bytes and its per-sequence extra bytes."""
    if dense:
        per_token = shape["n_heads"] * (shape["d_nope"] + shape["d_rope"] + shape["d_v"])
    else:
        per_token = latent_scalars_per_token(shape["d_c"], shape["d_rope"])
    scalars = n_layers * batch * window_tokens * per_token
    scalars += n_layers * sum(int(np.prod(v)) for v in layer_weights(dense=dense, **{
        k: shape[k] for k in ("dim", "n_heads", "d_nope", "d_rope", "d_c", "d_v")}).values())
    scalars += sum(int(np.prod(v)) for v in step_tensors(batch, dense=dense, fused=fused, **shape).values())
    return scalars * elt_bytes + fixed_bytes + batch * extra_bytes_per_seq


def batch_capacity(budget_bytes: int, **kw) -> int:
    """Largest batch whose memory_bytes fits ``budget_bytes`` (0 if none): memory grows with the batch,
    so double until it no longer fits, then bisect [TS-R]."""
    if memory_bytes(0, **kw) > budget_bytes:
        return 0
    hi = 1
    while memory_bytes(hi, **kw) <= budget_bytes:
        hi *= 2
    lo = hi // 2                                     # fits; hi does not
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if memory_bytes(mid, **kw) <= budget_bytes:
            lo = mid
        else:
            hi = mid
    return lo
