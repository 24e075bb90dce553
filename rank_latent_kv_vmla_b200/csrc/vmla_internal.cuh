// Internal declarations shared by the host entry points and the kernels of libvmla.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vmla.h"

namespace vmla {

constexpr int kMaxRopePairs = 64;

// 3D-RoPE table: pair p turns with axis axis[p] (0 = frame, 1 = row, 2 = column) at inv_freq[p]
// radians per unit of position (theta^(-m/P_a) for the m-th pair of an axis with P_a pairs).
// Computed on the host in double precision.
struct RopeTable {
  double inv_freq[kMaxRopePairs];
  int32_t axis[kMaxRopePairs];
  int32_t n_pairs;
};

// Where the tokens of one call sit in the video: a token n (0-based within its batch element) is
// in frame first_frame + n / T_f at row (n % T_f) / grid_w, column n % grid_w.
struct FrameGeom {
  int64_t first_frame;
  int32_t tokens_per_frame;  // T_f
  int32_t grid_w;
  int32_t chunk_frames;      // F
  int32_t window_frames;     // W
};

// Key visibility of one attention call: query token n of chunk k = n / (F*T_f) sees the cache rows
// [0, key_end(n)) of its batch element, key_end(n) = min(first_frame + (k+1)*F, W) * T_f.
__host__ __device__ inline int64_t key_end_rows(const FrameGeom& g, int64_t n) {
  const int64_t k = n / ((int64_t)g.chunk_frames * g.tokens_per_frame);
  int64_t hi = g.first_frame + (k + 1) * g.chunk_frames;
  if (hi > g.window_frames) hi = g.window_frames;
  return hi * g.tokens_per_frame;
}

// Ring row (within a batch element) of token n of an appended chunk.
__host__ __device__ inline int64_t ring_row(const FrameGeom& g, int64_t n) {
  const int64_t f = g.first_frame + n / g.tokens_per_frame;
  return (f % g.window_frames) * g.tokens_per_frame + n % g.tokens_per_frame;
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <class T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Rotate the pair (a, b) = (u[2p], u[2p+1]) of a token at (f, i, j).  The angle is formed and its sine
// and cosine taken in double precision so that large frame indices keep full fp32 accuracy.
__device__ __forceinline__ void rope_rotate(const RopeTable& rt, int p, int64_t f, int64_t i,
                                            int64_t j, float a, float b, float* ra, float* rb) {
  const int ax = rt.axis[p];
  const double pos = (double)(ax == 0 ? f : (ax == 1 ? i : j));
  double s, c;
  sincos(pos * rt.inv_freq[p], &s, &c);
  const float cf = (float)c, sf = (float)s;
  *ra = a * cf - b * sf;
  *rb = a * sf + b * cf;
}

// Same rotation for bf16 outputs: the angle is formed and reduced to [-pi, pi] in double precision
// (so large frame indices lose nothing), then its sine and cosine are taken in single precision.
__device__ __forceinline__ void rope_rotate_f32(const RopeTable& rt, int p, int64_t f, int64_t i,
                                                int64_t j, float a, float b, float* ra, float* rb) {
  const int ax = rt.axis[p];
  const double pos = (double)(ax == 0 ? f : (ax == 1 ? i : j));
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  double ang = pos * rt.inv_freq[p];
  ang = fma(-two_pi, rint(ang * inv_two_pi), ang);
  float sf, cf;
  sincosf((float)ang, &sf, &cf);
  *ra = a * cf - b * sf;
  *rb = a * sf + b * cf;
}

// Rotation of query pair p for the fused prologue: the angle is formed and reduced to [-pi, pi] in
// double precision (large frame indices lose nothing), then the MUFU sine / cosine (absolute error
// about 1e-6 on that interval, far below the bf16 rounding of the result) keep this once-per-row
// step short.
__device__ __forceinline__ void rope_rotate_mufu(const RopeTable& rt, int p, int64_t f, int64_t i, int64_t j,
                                                 float a, float b, float* ra, float* rb) {
  const int ax = rt.axis[p];
  const double pos = (double)(ax == 0 ? f : (ax == 1 ? i : j));
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  double ang = pos * rt.inv_freq[p];
  ang = fma(-two_pi, rint(ang * inv_two_pi), ang);
  float sf, cf;
  __sincosf((float)ang, &sf, &cf);
  *ra = a * cf - b * sf;
  *rb = a * sf + b * cf;
}

// Device status word (bounded waits that ran out record a nonzero code here).
int* device_status_ptr();   // address of this device's status word (host side), nullptr on error
void count_launches(int n);
vmla_status report(vmla_status s, const char* what);   // sets the thread's error detail, returns s

// ------------------------------------------------------------------------------------------------
// CUDA-core kernels (fp32 path)
// ------------------------------------------------------------------------------------------------
template <class T>
cudaError_t simt_compress_append(const vmla_config& cfg, int batch, const T* x, const T* w,
                                 const FrameGeom& g, const RopeTable& rt, T* c, T* k_r,
                                 cudaStream_t st);
template <class T>
cudaError_t simt_absorb_q(const vmla_config& cfg, int batch, int64_t nq, const T* q_nope,
                          const T* q_rope, const T* w_uk, const FrameGeom& g, const RopeTable& rt,
                          T* q_abs, cudaStream_t st);
template <class T>
cudaError_t simt_value_up(const vmla_config& cfg, int batch, int64_t n_tokens, const T* o_lat,
                          const T* w_uv, T* out, cudaStream_t st);
template <class T>
cudaError_t simt_rope_q(const vmla_config& cfg, int batch, int64_t nq, const T* q_nope,
                        const T* q_rope, const FrameGeom& g, const RopeTable& rt, T* q,
                        cudaStream_t st);
template <class T>
cudaError_t simt_dense_append(const vmla_config& cfg, int batch, const T* x, const T* w_kv,
                              const FrameGeom& g, const RopeTable& rt, T* k, T* v, cudaStream_t st);

// Generic flash attention on CUDA cores.  Keys of row t (batch b, head h) are the concatenation of
// plane A (da values at a + (b*cap + t)*a_tok + h*a_head) and plane B (db values, may be empty);
// values are dv values at v + (b*cap + t)*v_tok + h*v_head.  Queries are [batch, nq, heads, da+db],
// outputs [batch, nq, heads, dv].
struct SimtAttnArgs {
  const void* q;
  const void* a; int64_t a_tok, a_head; int da;
  const void* b; int64_t b_tok, b_head; int db;
  const void* v; int64_t v_tok, v_head; int dv;
  int64_t cap;        // rows per batch element in the cache planes (W*T_f)
  int batch, heads;
  int64_t nq;
  float scale;
  FrameGeom g;
  void* out;
  float* lse;
};
template <class T>
cudaError_t simt_attention(const SimtAttnArgs& a, cudaStream_t st);

}  // namespace vmla
