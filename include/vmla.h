/*
 * vmla.h - C ABI of the VideoMLA latent-KV attention library (libvmla.so, sm_100a).
 *
 * VideoMLA ("VideoMLA: Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video Diffusion",
 * gist.science technical summary, Method items 1-4) caches, for every token t of a sliding window of
 * latent frames, only the pair (c^KV_t, k^R_t): a content latent c^KV_t = W^KV_down x_t shared by all
 * heads (d_c scalars) and one head-shared positional key k^R_t rotated by 3D-RoPE (d_rope scalars).
 * Per-head content keys and values are never stored; this library never materialises them either:
 * the key up-projection is absorbed into the query, q~_h = (W^K_up,h)^T q^nope_h, so the score of key
 * t is  scale * (q~_h . c_t + q^R_h . k^R_t),  and the value up-projection W^V_up,h is applied once to
 * the attention-weighted latent sum.
 *
 * Conventions shared by every call
 *  - Ownership: every tensor argument is a caller-owned DEVICE buffer; the library allocates no device
 *    memory and keeps no pointer after a call returns.  Host structs (vmla_config, vmla_cache) are
 *    read during the call; vmla_cache.frames_written is updated by the append calls.
 *  - Execution: work is enqueued on the caller's CUDA stream (`stream` is a cudaStream_t; NULL is the
 *    legacy default stream) and the call returns without synchronising.
 *  - Layout: row-major, last dimension contiguous, no padding between rows.  Every base pointer must be
 *    16-byte aligned (VMLA_ERR_MISALIGNED otherwise).
 *  - Element type: cfg->dtype selects VMLA_BF16 (bf16 storage, fp32 accumulation, tensor-core kernels)
 *    or VMLA_F32 (fp32 storage and arithmetic, CUDA-core kernels).  The lse outputs are always fp32.
 *  - Errors: arguments are validated on the host before anything is launched; on error nothing is
 *    enqueued and a status is returned.  vmla_last_error_detail() gives a text for the calling thread.
 *    Device-side waits are bounded: a wait that runs out sets a device status word and the kernel
 *    returns; vmla_device_status() reads (and clears) it.
 *
 * Frame geometry: a latent frame is a grid_h x grid_w grid of tokens (T_f = grid_h*grid_w) in raster
 * order; a chunk is chunk_frames (F) frames; the window holds window_frames (W) frames including the
 * current chunk.  Frame f lives in ring slot f mod W, rows [(f mod W)*T_f, (f mod W + 1)*T_f) of the
 * cache planes; appending frame f evicts frame f - W.
 */
#ifndef VMLA_H_
#define VMLA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VMLA_ABI_VERSION 1

#if defined(__GNUC__)
#define VMLA_API __attribute__((visibility("default")))
#else
#define VMLA_API
#endif

typedef enum {
  VMLA_OK = 0,
  VMLA_ERR_INVALID_ARG = 1,   /* a null pointer, a bad size, a frame index that does not follow */
  VMLA_ERR_UNSUPPORTED = 2,   /* sizes the kernels of this dtype do not handle */
  VMLA_ERR_MISALIGNED = 3,    /* a base pointer that is not 16-byte aligned */
  VMLA_ERR_CUDA = 4,          /* a CUDA runtime/driver error (detail has the CUDA error text) */
  VMLA_ERR_TIMEOUT = 5        /* a bounded device-side wait ran out (from vmla_device_status) */
} vmla_status;

typedef enum { VMLA_BF16 = 0, VMLA_F32 = 1 } vmla_dtype;

/* Layer geometry.  d_h = d_nope + d_rope is the per-head query/key width of the equivalent dense
 * layer; d_v is the per-head value width.  rope_pairs_t + rope_pairs_h + rope_pairs_w must equal
 * d_rope / 2 (3D-RoPE pair split over frame, row and column).  softmax_scale <= 0 selects
 * 1 / sqrt(d_nope + d_rope). */
typedef struct {
  int32_t dim, n_heads, d_nope, d_rope, d_c, d_v;
  int32_t grid_h, grid_w, chunk_frames, window_frames;
  int32_t rope_pairs_t, rope_pairs_h, rope_pairs_w;
  float rope_theta;
  float softmax_scale;
  int32_t dtype; /* vmla_dtype */
} vmla_config;

/* The latent cache of one layer: two planes of window_frames*T_f rows per batch element,
 *   c   [batch, W*T_f, d_c]     the content latents c^KV_t,
 *   k_r [batch, W*T_f, d_rope]  the rotated positional keys k^R_t.
 * frames_written counts the frames appended so far (owned by the caller, advanced by
 * vmla_compress_append).  Rows of slots that were never written are never read. */
typedef struct {
  void* c;
  void* k_r;
  int32_t batch;
  int32_t reserved;
  int64_t frames_written;
} vmla_cache;

/* The dense per-head cache of the comparison layer: k [batch, W*T_f, n_heads, d_h] and
 * v [batch, W*T_f, n_heads, d_v], same ring and frame rules as vmla_cache. */
typedef struct {
  void* k;
  void* v;
  int32_t batch;
  int32_t reserved;
  int64_t frames_written;
} vmla_dense_cache;

/* Compress one chunk into the latent cache (VideoMLA, Method item 1 "shared low-rank content latent"
 * and item 3 "decoupled 3D-RoPE"; sliding window: abstract and Problem definition).
 *   x        [batch, F*T_f, dim]          token features of frames first_frame .. first_frame+F-1
 *   w_dkv_kr [d_c + d_rope, dim]          rows 0..d_c-1 = W^KV_down, rows d_c.. = W^KR
 * For every token: c = W^KV_down x, k^R = RoPE3D(W^KR x) at the token's (frame, row, column), both
 * rounded to the storage type and written to its ring row.  first_frame must equal
 * cache->frames_written; on success cache->frames_written += F. */
VMLA_API vmla_status vmla_compress_append(const vmla_config* cfg, const void* x, const void* w_dkv_kr,
                                 int64_t first_frame, vmla_cache* cache, void* stream);

/* One sequence on several GPUs (query-row sharding, replicated cache; the technical summary's Problem
 * definition: a fixed-size sliding window per sequence): every GPU holds a full replica of the latent
 * cache and compresses only a token range of each chunk.  This call compresses tokens token_begin ..
 * token_begin+n_tokens-1 of the chunk of frames first_frame .. first_frame+F-1 and stores each token's
 * c and k^R rows into the rings of all n_replicas caches (1..8).  Replica planes on other GPUs are
 * reached through peer mappings (vmla_ipc_import) with plain stores, so the compute and the exchange of
 * the new latents are one kernel; the caller orders that kernel before any reader on another GPU (for
 * example with a collective on the same stream) and then advances frames_written of every replica by
 * F itself: this call does not.
 *   x_rows [batch, n_tokens, dim]; w_dkv_kr as in vmla_compress_append; replicas[r].frames_written
 *   must all equal first_frame.  bf16 only. */
VMLA_API vmla_status vmla_compress_append_rows(const vmla_config* cfg, const void* x_rows, const void* w_dkv_kr,
                                               int64_t first_frame, int64_t token_begin, int64_t n_tokens,
                                               const vmla_cache* replicas, int32_t n_replicas, void* stream);

/* Peer mappings of device buffers across processes (CUDA IPC).  vmla_ipc_export describes the buffer
 * holding dev_ptr (allocation handle + offset of dev_ptr in it); vmla_ipc_import maps it into this
 * process (another GPU's memory, reached over NVLink) and returns the matching pointer;
 * vmla_ipc_release unmaps it.  The exporter keeps its buffer alive until every importer released it.
 * The buffer must come from cudaMalloc (PyTorch's default caching allocator does); memory from the
 * virtual-memory allocation API (PyTorch's expandable segments) cannot be exported this way and
 * vmla_ipc_export returns VMLA_ERR_CUDA. */
typedef struct {
  unsigned char bytes[64];
  int64_t offset;
} vmla_ipc_handle;
VMLA_API vmla_status vmla_ipc_export(const void* dev_ptr, vmla_ipc_handle* out);
VMLA_API vmla_status vmla_ipc_import(const vmla_ipc_handle* h, void** dev_ptr);
VMLA_API vmla_status vmla_ipc_release(void* dev_ptr);

/* Few-step generation: recompute the newest chunk's cache rows in place.  Streaming video diffusion
 * denoises each chunk over several steps (the technical summary's Problem definition names
 * Self-Forcing-style training); at every step the chunk's own keys come from that step's features,
 * and the last rewrite, with the clean features, is what stays in the window.  This call does what
 * vmla_compress_append does for the frames frames_written-F .. frames_written-1 (same x, w_dkv_kr
 * layouts), without advancing frames_written and without evicting anything: the frames the chunk's
 * first append evicted are outside its window.  Requires frames_written >= F. */
VMLA_API vmla_status vmla_compress_rewrite(const vmla_config* cfg, const void* x, const void* w_dkv_kr,
                                           vmla_cache* cache, void* stream);

/* Absorbed query (VideoMLA, Method item 2 "on-demand reconstruction" with W^K_up folded into the
 * query; item 3 for the rotated part).
 *   q_nope [batch, Nq, n_heads, d_nope], q_rope [batch, Nq, n_heads, d_rope],
 *   w_uk   [n_heads, d_nope, d_c]  (W^K_up,h maps c to the head's content key),
 *   q_abs  [batch, Nq, n_heads, d_c + d_rope]  output rows [q~_h ; RoPE3D(q^rope_h)],
 * with Nq = n_query_chunks*F*T_f tokens of frames first_frame.. (positions of the query tokens). */
VMLA_API vmla_status vmla_absorb_q(const vmla_config* cfg, int32_t batch, int32_t n_query_chunks,
                          const void* q_nope, const void* q_rope, const void* w_uk,
                          int64_t first_frame, void* q_abs, void* stream);

/* Latent attention over the cache (VideoMLA, Method items 2-3; block-causal window: abstract and
 * Problem definition).  Query token n of the call belongs to chunk k = n / (F*T_f) whose frames end at
 * hi_k = first_frame + (k+1)*F; it sees the cached keys of frames [max(0, hi_k - W), hi_k):
 * bidirectional inside its chunk, causal across chunks.  Per (n, h):
 *   s_t = scale*(q~ . c_t + q^R . k^R_t),  p = softmax(s),  out_latent = sum_t p_t c_t,
 *   lse = log(sum_t exp(s_t))  (natural log; lse may be NULL).
 *   q_abs [batch, Nq, n_heads, d_c + d_rope] -> out_latent [batch, Nq, n_heads, d_c], lse [batch, Nq, n_heads].
 * Requires every needed frame to be in the window: hi_last <= frames_written, and if
 * frames_written > W then n_query_chunks == 1 and hi_last == frames_written. */
VMLA_API vmla_status vmla_latent_attention(const vmla_config* cfg, const void* q_abs, const vmla_cache* cache,
                                  int64_t first_frame, int32_t n_query_chunks, void* out_latent,
                                  float* lse, void* stream);

/* The three steps above in one launch: absorbed query, latent attention and value up-projection, with
 * q_abs and the latent output kept on chip (same arithmetic and roundings as vmla_absorb_q ->
 * vmla_latent_attention -> vmla_value_up: q~ and the latent output are rounded to bf16 before their
 * next product).  VideoMLA technical summary, Method item 2 (per-head keys and values rebuilt from the
 * shared latent by W^K_up,h and W^V_up,h) and item 3 (the rotated query part).
 *   q_nope [batch, Nq, n_heads, d_nope], q_rope [batch, Nq, n_heads, d_rope],
 *   w_uk [n_heads, d_nope, d_c], w_uv [n_heads, d_v, d_c]
 *   -> out [batch, Nq, n_heads, d_v], lse [batch, Nq, n_heads] (natural log, or NULL).
 * Same window rules as vmla_latent_attention.  bf16 only; needs d_rope == 32, d_c in {64, 128, 192, 256},
 * d_nope a multiple of 16 in [16, 128] and d_v a multiple of 32 in [32, 128] (VMLA_ERR_UNSUPPORTED
 * otherwise). */
VMLA_API vmla_status vmla_latent_attention_fused(const vmla_config* cfg, const void* q_nope, const void* q_rope,
                                                 const void* w_uk, const void* w_uv, const vmla_cache* cache,
                                                 int64_t first_frame, int32_t n_query_chunks, void* out,
                                                 float* lse, void* stream);

/* vmla_latent_attention_fused for the query tokens token_begin .. token_begin+n_tokens-1 of the call
 * only (a shard of the rows): q_nope [batch, n_tokens, n_heads, d_nope], q_rope [batch, n_tokens,
 * n_heads, d_rope] -> out [batch, n_tokens, n_heads, d_v], lse [batch, n_tokens, n_heads].  Positions and
 * the window rule are those of the tokens' place in the call. */
VMLA_API vmla_status vmla_latent_attention_fused_rows(const vmla_config* cfg, const void* q_nope,
                                                      const void* q_rope, const void* w_uk, const void* w_uv,
                                                      const vmla_cache* cache, int64_t first_frame,
                                                      int32_t n_query_chunks, int64_t token_begin,
                                                      int64_t n_tokens, void* out, float* lse, void* stream);

/* Value up-projection applied once to the attention-weighted latent (VideoMLA, Method item 2):
 *   out[b, n, h, :] = W^V_up,h out_latent[b, n, h, :]
 *   out_latent [batch, n_tokens, n_heads, d_c], w_uv [n_heads, d_v, d_c], out [batch, n_tokens, n_heads, d_v]. */
VMLA_API vmla_status vmla_value_up(const vmla_config* cfg, int32_t batch, int64_t n_tokens,
                          const void* out_latent, const void* w_uv, void* out, void* stream);

/* ---- Dense per-head comparison layer (the layout VideoMLA replaces: Problem definition, and
 *      Method item 4's 2*n_h*d_h scalars per token). ---- */

/* Pack the dense query q [batch, Nq, n_heads, d_h] = [q^nope ; RoPE3D(q^rope)] per head. */
VMLA_API vmla_status vmla_rope_q(const vmla_config* cfg, int32_t batch, int32_t n_query_chunks,
                        const void* q_nope, const void* q_rope, int64_t first_frame, void* q,
                        void* stream);

/* Project one chunk to dense per-head keys and values and append them to the dense ring:
 *   x [batch, F*T_f, dim], w_kv [n_heads*(d_h + d_v), dim]: rows h*d_h .. h*d_h+d_h-1 give head h's key
 *   (its last d_rope entries are rotated by 3D-RoPE), rows n_heads*d_h + h*d_v .. give head h's value.
 * first_frame must equal cache->frames_written; on success cache->frames_written += F. */
VMLA_API vmla_status vmla_dense_append(const vmla_config* cfg, const void* x, const void* w_kv,
                              int64_t first_frame, vmla_dense_cache* cache, void* stream);

/* Dense counterpart of vmla_compress_rewrite: recompute the newest chunk's keys and values in place
 * (frames frames_written-F ..), frames_written unchanged.  Requires frames_written >= F. */
VMLA_API vmla_status vmla_dense_rewrite(const vmla_config* cfg, const void* x, const void* w_kv,
                                        vmla_dense_cache* cache, void* stream);

/* Dense multi-head attention with the same window / block-causal rule as vmla_latent_attention.
 *   q [batch, Nq, n_heads, d_h] -> out [batch, Nq, n_heads, d_v], lse [batch, Nq, n_heads] (or NULL). */
VMLA_API vmla_status vmla_dense_mha(const vmla_config* cfg, const void* q, const vmla_dense_cache* cache,
                           int64_t first_frame, int32_t n_query_chunks, void* out, float* lse,
                           void* stream);

/* ---- Utilities ---- */

/* Host-only check of the window rule of vmla_latent_attention / vmla_dense_mha for a cache holding
 * frames_written frames: VMLA_OK if every frame that query chunks first_frame.. need is still in the
 * window, else VMLA_ERR_INVALID_ARG (with a detail text).  Launches nothing. */
VMLA_API vmla_status vmla_check_attention_window(const vmla_config* cfg, int64_t frames_written,
                                                 int64_t first_frame, int32_t n_query_chunks);

/* Host-only check whether vmla_latent_attention_fused supports this configuration: VMLA_OK, or
 * VMLA_ERR_UNSUPPORTED with the reason in the detail text (VMLA_ERR_INVALID_ARG for an invalid cfg).
 * Launches nothing; callers use it to choose between the fused call and the three separate calls. */
VMLA_API vmla_status vmla_check_fused(const vmla_config* cfg);

/* Synchronise `stream`, then read and clear the device status word of the current device:
 * *code = 0 if no device-side wait ran out since the last call, else a nonzero code naming the wait.
 * The read and the clear are one atomic exchange made by a one-thread kernel on `stream`, so a code
 * that a kernel on another stream raises meanwhile is either returned by this call or kept for the
 * next one, never lost.  Returns VMLA_ERR_TIMEOUT when *code != 0. */
VMLA_API vmla_status vmla_device_status(void* stream, int32_t* code);

/* Bytes of one layer's cache for `batch` sequences at a full window: latent (d_c + d_rope per token)
 * and dense (n_heads*(d_h + d_v) per token), in the storage type of cfg->dtype.  -1 on a bad cfg. */
VMLA_API int64_t vmla_latent_cache_bytes(const vmla_config* cfg, int32_t batch);
VMLA_API int64_t vmla_dense_cache_bytes(const vmla_config* cfg, int32_t batch);

/* Largest batch that fits a fixed memory budget (the technical summary's Results, "Scalability": at a
 * fixed B200 memory budget the latent cache admits a much larger batch than dense MHA).  For a model of
 * n_layers attention layers of this shape, stepped along `path` (a vmla_path):
 *   per sequence  cache   n_layers * W*T_f * (d_c + d_rope)  or  n_layers * W*T_f * n_heads*(d_h + d_v)
 *                 buffers the tensors of one layer step, reused across layers (x [F*T_f, dim] and,
 *                         latent: q_nope, q_rope, q_abs, out_latent, out; latent fused: q_nope,
 *                         q_rope, out; dense: q, out)
 *                 + extra_bytes_per_seq (activations outside this library)
 *   fixed         this library's weights for n_layers layers (latent: w_dkv_kr, w_uk, w_uv; dense:
 *                 w_kv) + fixed_bytes (the rest of the model)
 * all in the storage type of cfg->dtype.  out->max_batch = floor((budget - fixed) / per sequence),
 * 0 when the fixed bytes alone exceed the budget.  Host-only; launches nothing. */
typedef enum {
  VMLA_PATH_LATENT = 0,        /* compress, absorb, latent attention, value up-projection */
  VMLA_PATH_DENSE = 1,         /* dense projection, rope, dense MHA */
  VMLA_PATH_LATENT_FUSED = 2   /* compress, vmla_latent_attention_fused */
} vmla_path;
typedef struct {
  int64_t max_batch;
  int64_t cache_bytes_per_seq;   /* all layers' cache of one sequence */
  int64_t buffer_bytes_per_seq;  /* one layer step's tensors for one sequence */
  int64_t weight_bytes;          /* this library's weights, all layers */
} vmla_capacity;
VMLA_API vmla_status vmla_plan_capacity(const vmla_config* cfg, int32_t n_layers, int32_t path,
                                        int64_t budget_bytes, int64_t fixed_bytes,
                                        int64_t extra_bytes_per_seq, vmla_capacity* out);

/* ---- Streaming executor: layer steps whose inputs and outputs are in host memory ----
 * Each submitted step copies x [batch, F*T_f, dim], q_nope [batch, F*T_f, n_heads, d_nope] and
 * q_rope [batch, F*T_f, n_heads, d_rope] from the host, runs vmla_compress_append and
 * vmla_latent_attention_fused on `cache` with the given weights (device pointers, layouts as in those
 * calls), and copies o [batch, F*T_f, n_heads, d_v] back to out_host.  Two staging slots in the
 * caller's device workspace let the copies of the neighbouring steps overlap this step's kernels: the
 * host -> device copies run on one internal stream, the device -> host copies on another, the kernels
 * on the stream given at creation; events order the three.  Steps may use different caches and
 * weights (one executor can serve every layer).
 * Ownership: the workspace (>= vmla_executor_workspace_bytes(), 256-byte aligned) and every buffer
 * stay the caller's; the executor owns only its two streams and six events.  Host buffers should be
 * page-locked (pageable memory makes the copies synchronous); an input buffer may be reused, and
 * out_host read, only after vmla_executor_wait().  cache->frames_written advances at submit.
 * bf16 only (VMLA_ERR_UNSUPPORTED otherwise); errors of the inner calls are returned as they are.
 * A submit refused on the host (null or misaligned pointers, an unsupported shape) enqueues nothing and
 * leaves the cache and the executor as they were; only a CUDA error after the step's compress was
 * enqueued leaves frames_written advanced (the chunk's rows are then in the ring). */
typedef struct vmla_executor vmla_executor;
VMLA_API int64_t vmla_executor_workspace_bytes(const vmla_config* cfg, int32_t batch);   /* -1 on bad args */
VMLA_API vmla_status vmla_executor_create(const vmla_config* cfg, int32_t batch, void* workspace,
                                          int64_t workspace_bytes, void* stream, vmla_executor** out);
VMLA_API vmla_status vmla_executor_submit(vmla_executor* ex, vmla_cache* cache, const void* w_dkv_kr,
                                          const void* w_uk, const void* w_uv, const void* x_host,
                                          const void* q_nope_host, const void* q_rope_host, void* out_host);
/* Blocks until every submitted step's output is in host memory; then as vmla_device_status(). */
VMLA_API vmla_status vmla_executor_wait(vmla_executor* ex);
VMLA_API vmla_status vmla_executor_destroy(vmla_executor* ex);   /* waits for pending copies first */

/* Set the bound of every device-side wait of later launches to `ms` milliseconds (default 1000) and
 * return the previous bound; ms <= 0 only returns the current bound.  A wait that runs out makes the
 * kernel stop, record a nonzero code for vmla_device_status() and return. */
VMLA_API int32_t vmla_set_wait_timeout_ms(int32_t ms);

/* Test hook for the bounded-wait path: the next bf16 attention launch (vmla_latent_attention, one of
 * the fused calls or vmla_dense_mha) does not load KV tile `tile` (keys tile*128 .. tile*128+127) of
 * any query tile, so the wait for it runs out, the kernel winds down without writing its outputs and
 * vmla_device_status() reports a nonzero code.
 * tile < 0 clears a pending request.  Nothing is faulted; later launches are unaffected. */
VMLA_API void vmla_debug_drop_kv_tile(int32_t tile);

/* Test hook of checked builds (built with VMLA_CHECKED=1, e.g. `build.py --checked`), whose kernels
 * test every computed global store against its buffer's extent and, instead of storing outside it,
 * record code 90 + site in the device status word: later launches record their buffers `bytes`
 * shorter than they are, so that correct stores at the buffers' ends are reported (and skipped).
 * 0 clears it.  Returns 1 in a checked build, 0 otherwise (where the hook has no effect). */
VMLA_API int32_t vmla_debug_shrink_extents(int64_t bytes);

/* Test hook of the exponential that the bf16 attention kernels compute on the FMA pipe for part of
 * their softmax terms (the rest use the MUFU ex2 unit).  Its method: x = n + f with n the nearest
 * integer, 2^f from a cubic fitted for least maximum relative error on [-1/2, 1/2] (Lawson's
 * iteration), n added to the exponent field; arguments below -125 are clamped to -125.  Claimed
 * accuracy: relative error <= 7.5e-5 for -125 <= x <= 120, and 2^-125 within that error for x < -125,
 * -inf and NaN.  y[i] = that 2^x of x[i], i < n: x and y are device buffers of n floats; the kernel
 * runs on `stream`.  n == 0 does nothing; VMLA_ERR_INVALID_ARG on n < 0 or NULL pointers with n > 0. */
VMLA_API vmla_status vmla_debug_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/* Number of kernels the library has launched in this process (all entry points, all devices). */
VMLA_API int64_t vmla_launch_count(void);

VMLA_API const char* vmla_status_string(vmla_status s);
VMLA_API const char* vmla_last_error_detail(void);
VMLA_API int32_t vmla_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VMLA_H_ */
