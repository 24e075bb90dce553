// Temporary bf16 entry points routed to the CUDA-core kernels until the tcgen05 kernels land.
#include "tc_kernels.cuh"

namespace vmla {
namespace {
using bf16 = __nv_bfloat16;
}

const char* tc_last_reason() { return ""; }
vmla_status tc_check_compress(const vmla_config&) { return VMLA_OK; }
vmla_status tc_check_absorb(const vmla_config&) { return VMLA_OK; }
vmla_status tc_check_latent_attention(const vmla_config& c) {
  return c.d_c <= 256 ? VMLA_OK : VMLA_ERR_UNSUPPORTED;
}
vmla_status tc_check_value_up(const vmla_config&) { return VMLA_OK; }
vmla_status tc_check_dense_append(const vmla_config&) { return VMLA_OK; }
vmla_status tc_check_dense_mha(const vmla_config& c) {
  return c.d_v <= 256 ? VMLA_OK : VMLA_ERR_UNSUPPORTED;
}

cudaError_t tc_compress_append(const vmla_config& cfg, int batch, const void* x, const void* w,
                               const FrameGeom& g, const RopeTable& rt, void* c, void* k_r,
                               cudaStream_t st) {
  return simt_compress_append<bf16>(cfg, batch, (const bf16*)x, (const bf16*)w, g, rt, (bf16*)c,
                                    (bf16*)k_r, st);
}
cudaError_t tc_absorb_q(const vmla_config& cfg, int batch, int64_t nq, const void* q_nope,
                        const void* q_rope, const void* w_uk, const FrameGeom& g, const RopeTable& rt,
                        void* q_abs, cudaStream_t st) {
  return simt_absorb_q<bf16>(cfg, batch, nq, (const bf16*)q_nope, (const bf16*)q_rope,
                             (const bf16*)w_uk, g, rt, (bf16*)q_abs, st);
}
cudaError_t tc_latent_attention(const vmla_config& cfg, int batch, int64_t nq, const void* q_abs,
                                const void* c, const void* k_r, int64_t cap, int64_t, const FrameGeom& g,
                                float scale, void* out, float* lse, int*, cudaStream_t st) {
  SimtAttnArgs a{};
  a.q = q_abs;
  a.a = c; a.a_tok = cfg.d_c; a.a_head = 0; a.da = cfg.d_c;
  a.b = k_r; a.b_tok = cfg.d_rope; a.b_head = 0; a.db = cfg.d_rope;
  a.v = c; a.v_tok = cfg.d_c; a.v_head = 0; a.dv = cfg.d_c;
  a.cap = cap; a.batch = batch; a.heads = cfg.n_heads; a.nq = nq;
  a.scale = scale; a.g = g; a.out = out; a.lse = lse;
  return simt_attention<bf16>(a, st);
}
cudaError_t tc_value_up(const vmla_config& cfg, int batch, int64_t n_tokens, const void* o_lat,
                        const void* w_uv, void* out, cudaStream_t st) {
  return simt_value_up<bf16>(cfg, batch, n_tokens, (const bf16*)o_lat, (const bf16*)w_uv, (bf16*)out,
                             st);
}
cudaError_t tc_rope_q(const vmla_config& cfg, int batch, int64_t nq, const void* q_nope,
                      const void* q_rope, const FrameGeom& g, const RopeTable& rt, void* q,
                      cudaStream_t st) {
  return simt_rope_q<bf16>(cfg, batch, nq, (const bf16*)q_nope, (const bf16*)q_rope, g, rt, (bf16*)q,
                           st);
}
cudaError_t tc_dense_append(const vmla_config& cfg, int batch, const void* x, const void* w_kv,
                            const FrameGeom& g, const RopeTable& rt, void* k, void* v,
                            cudaStream_t st) {
  return simt_dense_append<bf16>(cfg, batch, (const bf16*)x, (const bf16*)w_kv, g, rt, (bf16*)k,
                                 (bf16*)v, st);
}
cudaError_t tc_dense_mha(const vmla_config& cfg, int batch, int64_t nq, const void* q, const void* k,
                         const void* v, int64_t cap, int64_t, const FrameGeom& g, float scale,
                         void* out, float* lse, int*, cudaStream_t st) {
  const int d_h = cfg.d_nope + cfg.d_rope;
  SimtAttnArgs a{};
  a.q = q;
  a.a = k; a.a_tok = (int64_t)cfg.n_heads * d_h; a.a_head = d_h; a.da = d_h;
  a.v = v; a.v_tok = (int64_t)cfg.n_heads * cfg.d_v; a.v_head = cfg.d_v; a.dv = cfg.d_v;
  a.cap = cap; a.batch = batch; a.heads = cfg.n_heads; a.nq = nq;
  a.scale = scale; a.g = g; a.out = out; a.lse = lse;
  return simt_attention<bf16>(a, st);
}

}  // namespace vmla
