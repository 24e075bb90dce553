// Host side of libvmla: argument validation, frame/ring bookkeeping, 3D-RoPE tables and kernel
// dispatch for the C ABI declared in include/vmla.h.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "vmla_internal.cuh"
#include "tc_kernels.cuh"

namespace vmla {

namespace {
thread_local std::string g_detail;
std::atomic<int64_t> g_launches{0};

__device__ int g_device_status;
__device__ int g_status_taken;   // the value vmla_device_status last swapped out of g_device_status

// Read and clear the status word in one atomic step, so that a code a kernel on another stream raises
// at any moment is either returned now or kept for the next read.
__global__ void take_status_kernel() { g_status_taken = atomicExch(&g_device_status, 0); }
std::mutex g_take_mu;

constexpr int kMaxDevices = 64;
int* g_status_addr[kMaxDevices];
std::mutex g_status_mu;

vmla_status fail(vmla_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_detail = buf;
  return s;
}

vmla_status cuda_fail(cudaError_t e, const char* what) {
  return fail(VMLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define VMLA_CHECK_PTR(p)                                                                          \
  do {                                                                                             \
    if ((p) == nullptr) return fail(VMLA_ERR_INVALID_ARG, "%s is NULL", #p);                      \
    if (!aligned16(p)) return fail(VMLA_ERR_MISALIGNED, "%s is not 16-byte aligned", #p);         \
  } while (0)

vmla_status check_config(const vmla_config* cfg) {
  if (!cfg) return fail(VMLA_ERR_INVALID_ARG, "cfg is NULL");
  const vmla_config& c = *cfg;
  if (c.dim <= 0 || c.n_heads <= 0 || c.d_nope <= 0 || c.d_rope <= 0 || c.d_c <= 0 || c.d_v <= 0)
    return fail(VMLA_ERR_INVALID_ARG, "all of dim, n_heads, d_nope, d_rope, d_c, d_v must be > 0");
  if (c.grid_h <= 0 || c.grid_w <= 0 || c.chunk_frames <= 0 || c.window_frames <= 0)
    return fail(VMLA_ERR_INVALID_ARG, "grid_h, grid_w, chunk_frames and window_frames must be > 0");
  if (c.chunk_frames > c.window_frames)
    return fail(VMLA_ERR_INVALID_ARG, "chunk_frames (%d) exceeds window_frames (%d)", c.chunk_frames,
                c.window_frames);
  if (c.d_rope % 2 || c.d_c % 2 || c.d_nope % 2 || c.d_v % 2)
    return fail(VMLA_ERR_INVALID_ARG, "d_rope, d_c, d_nope and d_v must be even");
  if (c.rope_pairs_t < 0 || c.rope_pairs_h < 0 || c.rope_pairs_w < 0 ||
      c.rope_pairs_t + c.rope_pairs_h + c.rope_pairs_w != c.d_rope / 2)
    return fail(VMLA_ERR_INVALID_ARG, "rope pair split %d+%d+%d does not equal d_rope/2 = %d",
                c.rope_pairs_t, c.rope_pairs_h, c.rope_pairs_w, c.d_rope / 2);
  if (c.d_rope / 2 > kMaxRopePairs)
    return fail(VMLA_ERR_UNSUPPORTED, "d_rope/2 = %d exceeds %d rotary pairs", c.d_rope / 2,
                kMaxRopePairs);
  if (!(c.rope_theta > 1.f)) return fail(VMLA_ERR_INVALID_ARG, "rope_theta must be > 1");
  if (c.dtype != VMLA_BF16 && c.dtype != VMLA_F32)
    return fail(VMLA_ERR_INVALID_ARG, "unknown dtype %d", c.dtype);
  return VMLA_OK;
}

RopeTable make_rope_table(const vmla_config& c) {
  RopeTable rt{};
  const int per_axis[3] = {c.rope_pairs_t, c.rope_pairs_h, c.rope_pairs_w};
  int p = 0;
  for (int ax = 0; ax < 3; ++ax)
    for (int m = 0; m < per_axis[ax]; ++m, ++p) {
      rt.axis[p] = ax;
      rt.inv_freq[p] = std::pow((double)c.rope_theta, -(double)m / (double)per_axis[ax]);
    }
  rt.n_pairs = p;
  return rt;
}

FrameGeom make_geom(const vmla_config& c, int64_t first_frame) {
  FrameGeom g;
  g.first_frame = first_frame;
  g.tokens_per_frame = c.grid_h * c.grid_w;
  g.grid_w = c.grid_w;
  g.chunk_frames = c.chunk_frames;
  g.window_frames = c.window_frames;
  return g;
}

float softmax_scale(const vmla_config& c) {
  return c.softmax_scale > 0.f ? c.softmax_scale : 1.0f / std::sqrt((float)(c.d_nope + c.d_rope));
}

// Frames needed by an attention call must all be in the window (see include/vmla.h).
vmla_status check_window(const vmla_config& c, int64_t frames_written, int64_t first_frame,
                         int n_query_chunks) {
  if (n_query_chunks <= 0) return fail(VMLA_ERR_INVALID_ARG, "n_query_chunks must be >= 1");
  if (first_frame < 0) return fail(VMLA_ERR_INVALID_ARG, "first_frame must be >= 0");
  if (frames_written <= 0) return fail(VMLA_ERR_INVALID_ARG, "the cache is empty (kv_len = 0)");
  const int64_t hi_last = first_frame + (int64_t)n_query_chunks * c.chunk_frames;
  if (hi_last > frames_written)
    return fail(VMLA_ERR_INVALID_ARG,
                "query frames end at %lld but only %lld frames were appended (append first)",
                (long long)hi_last, (long long)frames_written);
  if (frames_written > c.window_frames && (n_query_chunks != 1 || hi_last != frames_written))
    return fail(VMLA_ERR_INVALID_ARG,
                "frames needed by this call were evicted: with %lld > W = %d frames written only the "
                "newest chunk can attend",
                (long long)frames_written, c.window_frames);
  return VMLA_OK;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace

void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

vmla_status report(vmla_status s, const char* what) { return fail(s, "%s", what); }

int* device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    g_status_addr[dev] = static_cast<int*>(p);
  }
  return g_status_addr[dev];
}

}  // namespace vmla

using namespace vmla;

extern "C" {

int32_t vmla_abi_version(void) { return VMLA_ABI_VERSION; }

const char* vmla_status_string(vmla_status s) {
  switch (s) {
    case VMLA_OK: return "ok";
    case VMLA_ERR_INVALID_ARG: return "invalid argument";
    case VMLA_ERR_UNSUPPORTED: return "unsupported sizes";
    case VMLA_ERR_MISALIGNED: return "misaligned pointer";
    case VMLA_ERR_CUDA: return "CUDA error";
    case VMLA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* vmla_last_error_detail(void) { return g_detail.c_str(); }

int64_t vmla_launch_count(void) { return g_launches.load(); }

int64_t vmla_latent_cache_bytes(const vmla_config* cfg, int32_t batch) {
  if (check_config(cfg) != VMLA_OK || batch <= 0) return -1;
  const int64_t elt = cfg->dtype == VMLA_BF16 ? 2 : 4;
  return (int64_t)batch * cfg->window_frames * cfg->grid_h * cfg->grid_w * (cfg->d_c + cfg->d_rope) *
         elt;
}

int64_t vmla_dense_cache_bytes(const vmla_config* cfg, int32_t batch) {
  if (check_config(cfg) != VMLA_OK || batch <= 0) return -1;
  const int64_t elt = cfg->dtype == VMLA_BF16 ? 2 : 4;
  return (int64_t)batch * cfg->window_frames * cfg->grid_h * cfg->grid_w * cfg->n_heads *
         (cfg->d_nope + cfg->d_rope + cfg->d_v) * elt;
}

vmla_status vmla_plan_capacity(const vmla_config* cfg, int32_t n_layers, int32_t path,
                               int64_t budget_bytes, int64_t fixed_bytes, int64_t extra_bytes_per_seq,
                               vmla_capacity* out) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (!out) return fail(VMLA_ERR_INVALID_ARG, "out is NULL");
  if (n_layers <= 0) return fail(VMLA_ERR_INVALID_ARG, "n_layers must be >= 1");
  if (path < VMLA_PATH_LATENT || path > VMLA_PATH_LATENT_FUSED)
    return fail(VMLA_ERR_INVALID_ARG, "path must be VMLA_PATH_LATENT, VMLA_PATH_DENSE or VMLA_PATH_LATENT_FUSED");
  const bool dense = path == VMLA_PATH_DENSE;
  if (budget_bytes < 0 || fixed_bytes < 0 || extra_bytes_per_seq < 0)
    return fail(VMLA_ERR_INVALID_ARG, "budget, fixed and extra bytes must be >= 0");
  const int64_t elt = cfg->dtype == VMLA_BF16 ? 2 : 4;
  const int64_t H = cfg->n_heads, D = cfg->dim, dh = cfg->d_nope + cfg->d_rope, dv = cfg->d_v;
  const int64_t nq = (int64_t)cfg->chunk_frames * cfg->grid_h * cfg->grid_w;
  const int64_t nk = (int64_t)cfg->window_frames * cfg->grid_h * cfg->grid_w;
  int64_t cache_tok, buffers, weights;
  if (dense) {
    cache_tok = H * (dh + dv);
    buffers = nq * D + nq * H * dh + nq * H * dv;                               // x, q, out
    weights = H * (dh + dv) * D;                                                // w_kv
  } else {
    const int64_t dc = cfg->d_c, dr = cfg->d_rope;
    cache_tok = dc + dr;
    buffers = nq * D + nq * H * cfg->d_nope + nq * H * dr + nq * H * dv;      // x, q_nope, q_rope, out
    if (path == VMLA_PATH_LATENT) buffers += nq * H * (dc + dr) + nq * H * dc;  // q_abs, out_latent
    weights = (dc + dr) * D + H * cfg->d_nope * dc + H * dv * dc;               // w_dkv_kr, w_uk, w_uv
  }
  out->cache_bytes_per_seq = (int64_t)n_layers * nk * cache_tok * elt;
  out->buffer_bytes_per_seq = buffers * elt;
  out->weight_bytes = (int64_t)n_layers * weights * elt;
  const int64_t per_seq = out->cache_bytes_per_seq + out->buffer_bytes_per_seq + extra_bytes_per_seq;
  const int64_t room = budget_bytes - fixed_bytes - out->weight_bytes;
  out->max_batch = room > 0 ? room / per_seq : 0;
  return VMLA_OK;
}

namespace {

// Compress the chunk of frames first_frame .. first_frame+F-1 into its ring rows (shared by append and
// rewrite; the caller has checked first_frame against the cache).
vmla_status compress_chunk(const vmla_config* cfg, const void* x, const void* w_dkv_kr,
                           int64_t first_frame, vmla_cache* cache, void* stream) {
  const FrameGeom g = make_geom(*cfg, first_frame);
  const RopeTable rt = make_rope_table(*cfg);
  cudaError_t e;
  if (cfg->dtype == VMLA_F32) {
    e = simt_compress_append<float>(*cfg, cache->batch, (const float*)x, (const float*)w_dkv_kr, g,
                                    rt, (float*)cache->c, (float*)cache->k_r, as_stream(stream));
  } else {
    vmla_status s = tc_check_compress(*cfg);
    if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
    e = tc_compress_append(*cfg, cache->batch, x, w_dkv_kr, g, rt, cache->c, cache->k_r,
                           as_stream(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "compress launch");
  return VMLA_OK;
}

vmla_status check_compress_args(const vmla_config* cfg, const void* x, const void* w_dkv_kr,
                                const vmla_cache* cache) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (!cache) return fail(VMLA_ERR_INVALID_ARG, "cache is NULL");
  VMLA_CHECK_PTR(x);
  VMLA_CHECK_PTR(w_dkv_kr);
  VMLA_CHECK_PTR(cache->c);
  VMLA_CHECK_PTR(cache->k_r);
  if (cache->batch <= 0) return fail(VMLA_ERR_INVALID_ARG, "cache->batch must be >= 1");
  return VMLA_OK;
}

}  // namespace

vmla_status vmla_compress_append(const vmla_config* cfg, const void* x, const void* w_dkv_kr,
                                 int64_t first_frame, vmla_cache* cache, void* stream) {
  vmla_status s = check_compress_args(cfg, x, w_dkv_kr, cache);
  if (s != VMLA_OK) return s;
  if (first_frame != cache->frames_written)
    return fail(VMLA_ERR_INVALID_ARG, "first_frame %lld does not follow frames_written %lld",
                (long long)first_frame, (long long)cache->frames_written);
  s = compress_chunk(cfg, x, w_dkv_kr, first_frame, cache, stream);
  if (s != VMLA_OK) return s;
  cache->frames_written += cfg->chunk_frames;
  return VMLA_OK;
}

vmla_status vmla_compress_append_rows(const vmla_config* cfg, const void* x_rows, const void* w_dkv_kr,
                                      int64_t first_frame, int64_t token_begin, int64_t n_tokens,
                                      const vmla_cache* replicas, int32_t n_replicas, void* stream) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  VMLA_CHECK_PTR(x_rows);
  VMLA_CHECK_PTR(w_dkv_kr);
  if (!replicas || n_replicas < 1 || n_replicas > kMaxCacheDst)
    return fail(VMLA_ERR_INVALID_ARG, "n_replicas must be in [1, %d]", kMaxCacheDst);
  if (cfg->dtype != VMLA_BF16) return fail(VMLA_ERR_UNSUPPORTED, "row-range compress runs on the bf16 path only");
  const int64_t ntok_chunk = (int64_t)cfg->chunk_frames * cfg->grid_h * cfg->grid_w;
  if (token_begin < 0 || n_tokens <= 0 || token_begin + n_tokens > ntok_chunk)
    return fail(VMLA_ERR_INVALID_ARG, "token range [%lld, %lld) outside the chunk's %lld tokens",
                (long long)token_begin, (long long)(token_begin + n_tokens), (long long)ntok_chunk);
  CacheDst dst[kMaxCacheDst];
  for (int r = 0; r < n_replicas; ++r) {
    const vmla_cache& c = replicas[r];
    if (!c.c || !c.k_r) return fail(VMLA_ERR_INVALID_ARG, "replica %d has a NULL plane", r);
    if (!aligned16(c.c) || !aligned16(c.k_r)) return fail(VMLA_ERR_MISALIGNED, "replica %d is not 16-byte aligned", r);
    if (c.batch != replicas[0].batch || c.batch <= 0)
      return fail(VMLA_ERR_INVALID_ARG, "replicas must share one batch size >= 1");
    if (c.frames_written != first_frame)
      return fail(VMLA_ERR_INVALID_ARG, "first_frame %lld does not follow replica %d's frames_written %lld",
                  (long long)first_frame, r, (long long)c.frames_written);
    dst[r] = CacheDst{c.c, c.k_r};
  }
  s = tc_check_compress(*cfg);
  if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
  const FrameGeom g = make_geom(*cfg, first_frame);
  const RopeTable rt = make_rope_table(*cfg);
  cudaError_t e = tc_compress_rows(*cfg, replicas[0].batch, token_begin, n_tokens, x_rows, w_dkv_kr, g, rt, dst,
                                   n_replicas, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "compress_append_rows launch");
  return VMLA_OK;
}

vmla_status vmla_compress_rewrite(const vmla_config* cfg, const void* x, const void* w_dkv_kr,
                                  vmla_cache* cache, void* stream) {
  vmla_status s = check_compress_args(cfg, x, w_dkv_kr, cache);
  if (s != VMLA_OK) return s;
  if (cache->frames_written < cfg->chunk_frames)
    return fail(VMLA_ERR_INVALID_ARG, "no chunk to rewrite: frames_written %lld < chunk_frames %d",
                (long long)cache->frames_written, cfg->chunk_frames);
  return compress_chunk(cfg, x, w_dkv_kr, cache->frames_written - cfg->chunk_frames, cache, stream);
}

vmla_status vmla_absorb_q(const vmla_config* cfg, int32_t batch, int32_t n_query_chunks,
                          const void* q_nope, const void* q_rope, const void* w_uk,
                          int64_t first_frame, void* q_abs, void* stream) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (batch <= 0 || n_query_chunks <= 0)
    return fail(VMLA_ERR_INVALID_ARG, "batch and n_query_chunks must be >= 1");
  if (first_frame < 0) return fail(VMLA_ERR_INVALID_ARG, "first_frame must be >= 0");
  VMLA_CHECK_PTR(q_nope);
  VMLA_CHECK_PTR(q_rope);
  VMLA_CHECK_PTR(w_uk);
  VMLA_CHECK_PTR(q_abs);
  const int64_t nq = (int64_t)n_query_chunks * cfg->chunk_frames * cfg->grid_h * cfg->grid_w;
  const FrameGeom g = make_geom(*cfg, first_frame);
  const RopeTable rt = make_rope_table(*cfg);
  cudaError_t e;
  if (cfg->dtype == VMLA_F32) {
    e = simt_absorb_q<float>(*cfg, batch, nq, (const float*)q_nope, (const float*)q_rope,
                             (const float*)w_uk, g, rt, (float*)q_abs, as_stream(stream));
  } else {
    s = tc_check_absorb(*cfg);
    if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
    e = tc_absorb_q(*cfg, batch, nq, q_nope, q_rope, w_uk, g, rt, q_abs, as_stream(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "absorb_q launch");
  return VMLA_OK;
}

vmla_status vmla_latent_attention(const vmla_config* cfg, const void* q_abs, const vmla_cache* cache,
                                  int64_t first_frame, int32_t n_query_chunks, void* out_latent,
                                  float* lse, void* stream) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (!cache) return fail(VMLA_ERR_INVALID_ARG, "cache is NULL");
  VMLA_CHECK_PTR(q_abs);
  VMLA_CHECK_PTR(cache->c);
  VMLA_CHECK_PTR(cache->k_r);
  VMLA_CHECK_PTR(out_latent);
  if (lse && !aligned16(lse)) return fail(VMLA_ERR_MISALIGNED, "lse is not 16-byte aligned");
  if (cache->batch <= 0) return fail(VMLA_ERR_INVALID_ARG, "cache->batch must be >= 1");
  s = check_window(*cfg, cache->frames_written, first_frame, n_query_chunks);
  if (s != VMLA_OK) return s;
  const FrameGeom g = make_geom(*cfg, first_frame);
  const int64_t T_f = (int64_t)cfg->grid_h * cfg->grid_w;
  const int64_t nq = (int64_t)n_query_chunks * cfg->chunk_frames * T_f;
  const int64_t cap = (int64_t)cfg->window_frames * T_f;
  const int64_t valid_rows =
      (cache->frames_written < cfg->window_frames ? cache->frames_written : cfg->window_frames) * T_f;
  cudaError_t e;
  if (cfg->dtype == VMLA_F32) {
    if (cfg->d_c > 256) return fail(VMLA_ERR_UNSUPPORTED, "fp32 path needs d_c <= 256");
    SimtAttnArgs a{};
    a.q = q_abs;
    a.a = cache->c; a.a_tok = cfg->d_c; a.a_head = 0; a.da = cfg->d_c;
    a.b = cache->k_r; a.b_tok = cfg->d_rope; a.b_head = 0; a.db = cfg->d_rope;
    a.v = cache->c; a.v_tok = cfg->d_c; a.v_head = 0; a.dv = cfg->d_c;
    a.cap = cap; a.batch = cache->batch; a.heads = cfg->n_heads; a.nq = nq;
    a.scale = softmax_scale(*cfg); a.g = g; a.out = out_latent; a.lse = lse;
    e = simt_attention<float>(a, as_stream(stream));
  } else {
    s = tc_check_latent_attention(*cfg);
    if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
    e = tc_latent_attention(*cfg, cache->batch, nq, q_abs, cache->c, cache->k_r, cap, valid_rows, g,
                            softmax_scale(*cfg), out_latent, lse, device_status_ptr(),
                            as_stream(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "latent_attention launch");
  return VMLA_OK;
}

vmla_status vmla_latent_attention_fused(const vmla_config* cfg, const void* q_nope, const void* q_rope,
                                        const void* w_uk, const void* w_uv, const vmla_cache* cache,
                                        int64_t first_frame, int32_t n_query_chunks, void* out, float* lse,
                                        void* stream) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (!cache) return fail(VMLA_ERR_INVALID_ARG, "cache is NULL");
  VMLA_CHECK_PTR(q_nope);
  VMLA_CHECK_PTR(q_rope);
  VMLA_CHECK_PTR(w_uk);
  VMLA_CHECK_PTR(w_uv);
  VMLA_CHECK_PTR(cache->c);
  VMLA_CHECK_PTR(cache->k_r);
  VMLA_CHECK_PTR(out);
  if (lse && !aligned16(lse)) return fail(VMLA_ERR_MISALIGNED, "lse is not 16-byte aligned");
  if (cache->batch <= 0) return fail(VMLA_ERR_INVALID_ARG, "cache->batch must be >= 1");
  if (cfg->dtype != VMLA_BF16)
    return fail(VMLA_ERR_UNSUPPORTED, "the fused call runs on the bf16 tensor-core path only");
  s = check_window(*cfg, cache->frames_written, first_frame, n_query_chunks);
  if (s != VMLA_OK) return s;
  s = tc_check_fused_attention(*cfg);
  if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
  const FrameGeom g = make_geom(*cfg, first_frame);
  const RopeTable rt = make_rope_table(*cfg);
  const int64_t T_f = (int64_t)cfg->grid_h * cfg->grid_w;
  const int64_t nq = (int64_t)n_query_chunks * cfg->chunk_frames * T_f;
  const int64_t cap = (int64_t)cfg->window_frames * T_f;
  const int64_t valid_rows =
      (cache->frames_written < cfg->window_frames ? cache->frames_written : cfg->window_frames) * T_f;
  cudaError_t e = tc_latent_attention_fused(*cfg, cache->batch, 0, nq, q_nope, q_rope, w_uk, w_uv, cache->c,
                                            cache->k_r, cap, valid_rows, g, rt, softmax_scale(*cfg), out,
                                            lse, device_status_ptr(), as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "latent_attention_fused launch");
  return VMLA_OK;
}

vmla_status vmla_latent_attention_fused_rows(const vmla_config* cfg, const void* q_nope, const void* q_rope,
                                             const void* w_uk, const void* w_uv, const vmla_cache* cache,
                                             int64_t first_frame, int32_t n_query_chunks, int64_t token_begin,
                                             int64_t n_tokens, void* out, float* lse, void* stream) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (!cache) return fail(VMLA_ERR_INVALID_ARG, "cache is NULL");
  VMLA_CHECK_PTR(q_nope);
  VMLA_CHECK_PTR(q_rope);
  VMLA_CHECK_PTR(w_uk);
  VMLA_CHECK_PTR(w_uv);
  VMLA_CHECK_PTR(cache->c);
  VMLA_CHECK_PTR(cache->k_r);
  VMLA_CHECK_PTR(out);
  if (lse && !aligned16(lse)) return fail(VMLA_ERR_MISALIGNED, "lse is not 16-byte aligned");
  if (cache->batch <= 0) return fail(VMLA_ERR_INVALID_ARG, "cache->batch must be >= 1");
  if (cfg->dtype != VMLA_BF16)
    return fail(VMLA_ERR_UNSUPPORTED, "the fused call runs on the bf16 tensor-core path only");
  s = check_window(*cfg, cache->frames_written, first_frame, n_query_chunks);
  if (s != VMLA_OK) return s;
  const int64_t T_f = (int64_t)cfg->grid_h * cfg->grid_w;
  const int64_t nq_call = (int64_t)n_query_chunks * cfg->chunk_frames * T_f;
  if (token_begin < 0 || n_tokens <= 0 || token_begin + n_tokens > nq_call)
    return fail(VMLA_ERR_INVALID_ARG, "token range [%lld, %lld) outside the call's %lld query tokens",
                (long long)token_begin, (long long)(token_begin + n_tokens), (long long)nq_call);
  s = tc_check_fused_attention(*cfg);
  if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
  const FrameGeom g = make_geom(*cfg, first_frame);
  const RopeTable rt = make_rope_table(*cfg);
  const int64_t cap = (int64_t)cfg->window_frames * T_f;
  const int64_t valid_rows =
      (cache->frames_written < cfg->window_frames ? cache->frames_written : cfg->window_frames) * T_f;
  cudaError_t e = tc_latent_attention_fused(*cfg, cache->batch, token_begin, n_tokens, q_nope, q_rope, w_uk,
                                            w_uv, cache->c, cache->k_r, cap, valid_rows, g, rt,
                                            softmax_scale(*cfg), out, lse, device_status_ptr(),
                                            as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "latent_attention_fused_rows launch");
  return VMLA_OK;
}

vmla_status vmla_value_up(const vmla_config* cfg, int32_t batch, int64_t n_tokens,
                          const void* out_latent, const void* w_uv, void* out, void* stream) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (batch <= 0 || n_tokens <= 0) return fail(VMLA_ERR_INVALID_ARG, "batch and n_tokens must be >= 1");
  VMLA_CHECK_PTR(out_latent);
  VMLA_CHECK_PTR(w_uv);
  VMLA_CHECK_PTR(out);
  cudaError_t e;
  if (cfg->dtype == VMLA_F32) {
    e = simt_value_up<float>(*cfg, batch, n_tokens, (const float*)out_latent, (const float*)w_uv,
                             (float*)out, as_stream(stream));
  } else {
    s = tc_check_value_up(*cfg);
    if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
    e = tc_value_up(*cfg, batch, n_tokens, out_latent, w_uv, out, as_stream(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "value_up launch");
  return VMLA_OK;
}

vmla_status vmla_rope_q(const vmla_config* cfg, int32_t batch, int32_t n_query_chunks,
                        const void* q_nope, const void* q_rope, int64_t first_frame, void* q,
                        void* stream) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (batch <= 0 || n_query_chunks <= 0)
    return fail(VMLA_ERR_INVALID_ARG, "batch and n_query_chunks must be >= 1");
  if (first_frame < 0) return fail(VMLA_ERR_INVALID_ARG, "first_frame must be >= 0");
  VMLA_CHECK_PTR(q_nope);
  VMLA_CHECK_PTR(q_rope);
  VMLA_CHECK_PTR(q);
  const int64_t nq = (int64_t)n_query_chunks * cfg->chunk_frames * cfg->grid_h * cfg->grid_w;
  const FrameGeom g = make_geom(*cfg, first_frame);
  const RopeTable rt = make_rope_table(*cfg);
  cudaError_t e;
  if (cfg->dtype == VMLA_F32)
    e = simt_rope_q<float>(*cfg, batch, nq, (const float*)q_nope, (const float*)q_rope, g, rt,
                           (float*)q, as_stream(stream));
  else
    e = tc_rope_q(*cfg, batch, nq, q_nope, q_rope, g, rt, q, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rope_q launch");
  return VMLA_OK;
}

namespace {

vmla_status check_dense_append_args(const vmla_config* cfg, const void* x, const void* w_kv,
                                    const vmla_dense_cache* cache) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (!cache) return fail(VMLA_ERR_INVALID_ARG, "cache is NULL");
  VMLA_CHECK_PTR(x);
  VMLA_CHECK_PTR(w_kv);
  VMLA_CHECK_PTR(cache->k);
  VMLA_CHECK_PTR(cache->v);
  if (cache->batch <= 0) return fail(VMLA_ERR_INVALID_ARG, "cache->batch must be >= 1");
  return VMLA_OK;
}

vmla_status dense_chunk(const vmla_config* cfg, const void* x, const void* w_kv, int64_t first_frame,
                        vmla_dense_cache* cache, void* stream) {
  const FrameGeom g = make_geom(*cfg, first_frame);
  const RopeTable rt = make_rope_table(*cfg);
  cudaError_t e;
  if (cfg->dtype == VMLA_F32) {
    e = simt_dense_append<float>(*cfg, cache->batch, (const float*)x, (const float*)w_kv, g, rt,
                                 (float*)cache->k, (float*)cache->v, as_stream(stream));
  } else {
    vmla_status s = tc_check_dense_append(*cfg);
    if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
    e = tc_dense_append(*cfg, cache->batch, x, w_kv, g, rt, cache->k, cache->v, as_stream(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "dense projection launch");
  return VMLA_OK;
}

}  // namespace

vmla_status vmla_dense_append(const vmla_config* cfg, const void* x, const void* w_kv,
                              int64_t first_frame, vmla_dense_cache* cache, void* stream) {
  vmla_status s = check_dense_append_args(cfg, x, w_kv, cache);
  if (s != VMLA_OK) return s;
  if (first_frame != cache->frames_written)
    return fail(VMLA_ERR_INVALID_ARG, "first_frame %lld does not follow frames_written %lld",
                (long long)first_frame, (long long)cache->frames_written);
  s = dense_chunk(cfg, x, w_kv, first_frame, cache, stream);
  if (s != VMLA_OK) return s;
  cache->frames_written += cfg->chunk_frames;
  return VMLA_OK;
}

vmla_status vmla_dense_rewrite(const vmla_config* cfg, const void* x, const void* w_kv,
                               vmla_dense_cache* cache, void* stream) {
  vmla_status s = check_dense_append_args(cfg, x, w_kv, cache);
  if (s != VMLA_OK) return s;
  if (cache->frames_written < cfg->chunk_frames)
    return fail(VMLA_ERR_INVALID_ARG, "no chunk to rewrite: frames_written %lld < chunk_frames %d",
                (long long)cache->frames_written, cfg->chunk_frames);
  return dense_chunk(cfg, x, w_kv, cache->frames_written - cfg->chunk_frames, cache, stream);
}

vmla_status vmla_dense_mha(const vmla_config* cfg, const void* q, const vmla_dense_cache* cache,
                           int64_t first_frame, int32_t n_query_chunks, void* out, float* lse,
                           void* stream) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (!cache) return fail(VMLA_ERR_INVALID_ARG, "cache is NULL");
  VMLA_CHECK_PTR(q);
  VMLA_CHECK_PTR(cache->k);
  VMLA_CHECK_PTR(cache->v);
  VMLA_CHECK_PTR(out);
  if (lse && !aligned16(lse)) return fail(VMLA_ERR_MISALIGNED, "lse is not 16-byte aligned");
  if (cache->batch <= 0) return fail(VMLA_ERR_INVALID_ARG, "cache->batch must be >= 1");
  s = check_window(*cfg, cache->frames_written, first_frame, n_query_chunks);
  if (s != VMLA_OK) return s;
  const FrameGeom g = make_geom(*cfg, first_frame);
  const int64_t T_f = (int64_t)cfg->grid_h * cfg->grid_w;
  const int64_t nq = (int64_t)n_query_chunks * cfg->chunk_frames * T_f;
  const int64_t cap = (int64_t)cfg->window_frames * T_f;
  const int64_t valid_rows =
      (cache->frames_written < cfg->window_frames ? cache->frames_written : cfg->window_frames) * T_f;
  const int d_h = cfg->d_nope + cfg->d_rope;
  cudaError_t e;
  if (cfg->dtype == VMLA_F32) {
    if (cfg->d_v > 256) return fail(VMLA_ERR_UNSUPPORTED, "fp32 path needs d_v <= 256");
    SimtAttnArgs a{};
    a.q = q;
    a.a = cache->k; a.a_tok = (int64_t)cfg->n_heads * d_h; a.a_head = d_h; a.da = d_h;
    a.b = nullptr; a.b_tok = 0; a.b_head = 0; a.db = 0;
    a.v = cache->v; a.v_tok = (int64_t)cfg->n_heads * cfg->d_v; a.v_head = cfg->d_v; a.dv = cfg->d_v;
    a.cap = cap; a.batch = cache->batch; a.heads = cfg->n_heads; a.nq = nq;
    a.scale = softmax_scale(*cfg); a.g = g; a.out = out; a.lse = lse;
    e = simt_attention<float>(a, as_stream(stream));
  } else {
    s = tc_check_dense_mha(*cfg);
    if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
    e = tc_dense_mha(*cfg, cache->batch, nq, q, cache->k, cache->v, cap, valid_rows, g,
                     softmax_scale(*cfg), out, lse, device_status_ptr(), as_stream(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "dense_mha launch");
  return VMLA_OK;
}

vmla_status vmla_check_attention_window(const vmla_config* cfg, int64_t frames_written,
                                        int64_t first_frame, int32_t n_query_chunks) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  return check_window(*cfg, frames_written, first_frame, n_query_chunks);
}

vmla_status vmla_check_fused(const vmla_config* cfg) {
  vmla_status s = check_config(cfg);
  if (s != VMLA_OK) return s;
  if (cfg->dtype != VMLA_BF16)
    return fail(VMLA_ERR_UNSUPPORTED, "the fused call runs on the bf16 tensor-core path only");
  s = tc_check_fused_attention(*cfg);
  if (s != VMLA_OK) return fail(s, "%s", tc_last_reason());
  return VMLA_OK;
}

vmla_status vmla_device_status(void* stream, int32_t* code) {
  if (!code) return fail(VMLA_ERR_INVALID_ARG, "code is NULL");
  cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  if (!device_status_ptr()) return fail(VMLA_ERR_CUDA, "cannot resolve the device status word");
  int v = 0;
  {
    std::lock_guard<std::mutex> lk(g_take_mu);      // one swap-and-read at a time per process
    take_status_kernel<<<1, 1, 0, st>>>();
    count_launches(1);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbolAsync(&v, g_status_taken, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  *code = v;
  if (v != 0) return fail(VMLA_ERR_TIMEOUT, "device wait %d ran out", v);
  return VMLA_OK;
}

}  // extern "C"
