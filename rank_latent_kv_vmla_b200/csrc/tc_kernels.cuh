// bf16 path of libvmla: tensor-core kernels (tcgen05 / TMEM / TMA on sm_100a).
#pragma once

#include "tc_common.cuh"
#include "vmla_internal.cuh"

namespace vmla {

// Reason text of the last tc_check_* refusal (thread-local).
const char* tc_last_reason();

// One destination cache (its c and k_r planes) of a compress call.
struct CacheDst {
  void* c;
  void* k_r;
};
constexpr int kMaxCacheDst = 8;

vmla_status tc_check_compress(const vmla_config& cfg);
// Tokens tok0 .. tok0+ntok-1 of the chunk (x [batch, ntok, dim]) into the rings of n_dst caches.
cudaError_t tc_compress_rows(const vmla_config& cfg, int batch, int64_t tok0, int64_t ntok, const void* x,
                             const void* w, const FrameGeom& g, const RopeTable& rt, const CacheDst* dst,
                             int n_dst, cudaStream_t st);
cudaError_t tc_compress_append(const vmla_config& cfg, int batch, const void* x, const void* w,
                               const FrameGeom& g, const RopeTable& rt, void* c, void* k_r,
                               cudaStream_t st);

vmla_status tc_check_absorb(const vmla_config& cfg);
cudaError_t tc_absorb_q(const vmla_config& cfg, int batch, int64_t nq, const void* q_nope,
                        const void* q_rope, const void* w_uk, const FrameGeom& g, const RopeTable& rt,
                        void* q_abs, cudaStream_t st);

vmla_status tc_check_latent_attention(const vmla_config& cfg);
cudaError_t tc_latent_attention(const vmla_config& cfg, int batch, int64_t nq, const void* q_abs,
                                const void* c, const void* k_r, int64_t cap, int64_t valid_rows,
                                const FrameGeom& g, float scale, void* out, float* lse, int* status,
                                cudaStream_t st);

// The same call at d_c = 64 / 128, with the keys of every tile split between two softmax warpgroups.
bool tc_latent_split_supported(const vmla_config& cfg);
cudaError_t tc_latent_attention_split(const vmla_config& cfg, int batch, int64_t nq, const void* q_abs,
                                      const void* c, const void* k_r, int64_t cap, int64_t valid_rows,
                                      const FrameGeom& g, float scale, void* out, float* lse, int* status,
                                      cudaStream_t st);

// The fused call (below) at d_c = 64 / 128 with d_v a multiple of 64, keys split the same way.
bool tc_latent_split_fused_supported(const vmla_config& cfg);
cudaError_t tc_latent_attention_split_fused(const vmla_config& cfg, int batch, int64_t tok0, int64_t nq,
                                            const void* q_nope, const void* q_rope, const void* w_uk,
                                            const void* w_uv, const void* c, const void* k_r, int64_t cap,
                                            int64_t valid_rows, const FrameGeom& g, const RopeTable& rt,
                                            float scale, void* out, float* lse, int* status, cudaStream_t st);

// Absorbed query, latent attention and value up-projection in one kernel (q_abs and the latent
// output stay on chip): q_nope [B, Nq, H, d_nope], q_rope [B, Nq, H, 32] -> out [B, Nq, H, d_v].
vmla_status tc_check_fused_attention(const vmla_config& cfg);
// tok0: the nq query tokens are tokens tok0 .. tok0+nq-1 of the call (positions and the window rule).
cudaError_t tc_latent_attention_fused(const vmla_config& cfg, int batch, int64_t tok0, int64_t nq,
                                      const void* q_nope, const void* q_rope, const void* w_uk, const void* w_uv,
                                      const void* c, const void* k_r, int64_t cap, int64_t valid_rows,
                                      const FrameGeom& g, const RopeTable& rt, float scale, void* out, float* lse,
                                      int* status, cudaStream_t st);

vmla_status tc_check_value_up(const vmla_config& cfg);
cudaError_t tc_value_up(const vmla_config& cfg, int batch, int64_t n_tokens, const void* o_lat,
                        const void* w_uv, void* out, cudaStream_t st);

cudaError_t tc_rope_q(const vmla_config& cfg, int batch, int64_t nq, const void* q_nope,
                      const void* q_rope, const FrameGeom& g, const RopeTable& rt, void* q,
                      cudaStream_t st);

vmla_status tc_check_dense_append(const vmla_config& cfg);
cudaError_t tc_dense_append(const vmla_config& cfg, int batch, const void* x, const void* w_kv,
                            const FrameGeom& g, const RopeTable& rt, void* k, void* v,
                            cudaStream_t st);

vmla_status tc_check_dense_mha(const vmla_config& cfg);
cudaError_t tc_dense_mha(const vmla_config& cfg, int batch, int64_t nq, const void* q, const void* k,
                         const void* v, int64_t cap, int64_t valid_rows, const FrameGeom& g,
                         float scale, void* out, float* lse, int* status, cudaStream_t st);

}  // namespace vmla
