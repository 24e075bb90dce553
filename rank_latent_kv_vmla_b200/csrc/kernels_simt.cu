// CUDA-core kernels of libvmla: the fp32 path (fp32 storage, fp32 arithmetic).
//
// These kernels compute every step of the VideoMLA latent path (compress + 3D-RoPE + ring append,
// absorbed query, latent attention, value up-projection) and of the dense comparison layer with plain
// FFMA arithmetic.  A tensor-core path cannot meet an fp32 tolerance (tf32 keeps 10 mantissa bits),
// so fp32 stays on the CUDA cores.
#include <float.h>

#include "vmla_internal.cuh"

namespace vmla {
namespace {

// ------------------------------------------------------------------------------------------------
// Row-wise linear map  Y[m, n] = sum_k X[m, k] * W(n, k)  with a per-(row, column pair) epilogue.
// X[m, k] = x[z*x_z + m*ldx + k];  W(n, k) = w[z*w_z + n*ldw_n + k*ldw_k]  (both weight layouts).
// A block covers kTM rows x 256 columns; thread t owns the column pair (2t, 2t+1) of its block.
// ------------------------------------------------------------------------------------------------
constexpr int kTM = 16;
constexpr int kTK = 32;
constexpr int kTN = 256;

template <class T, class Epi>
__global__ void __launch_bounds__(128) linear_kernel(const T* __restrict__ x, int64_t ldx, int64_t x_z,
                                                     const T* __restrict__ w, int64_t ldw_n,
                                                     int64_t ldw_k, int64_t w_z, int64_t M, int N,
                                                     int K, Epi epi) {
  __shared__ float xs[kTM][kTK];
  __shared__ float ws[kTN][kTK + 1];
  const int z = blockIdx.z;
  x += z * x_z;
  w += z * w_z;
  const int64_t m0 = (int64_t)blockIdx.x * kTM;
  const int n0 = blockIdx.y * kTN;
  const int t = threadIdx.x;
  float acc[kTM][2];
#pragma unroll
  for (int r = 0; r < kTM; ++r) acc[r][0] = acc[r][1] = 0.f;

  for (int k0 = 0; k0 < K; k0 += kTK) {
    for (int i = t; i < kTM * kTK; i += blockDim.x) {
      const int r = i / kTK, kk = i % kTK;
      const int64_t m = m0 + r;
      const int k = k0 + kk;
      xs[r][kk] = (m < M && k < K) ? to_f32(x[m * ldx + k]) : 0.f;
    }
    if (ldw_k == 1) {  // W stored [N, K]: read along k
      for (int i = t; i < kTN * kTK; i += blockDim.x) {
        const int nn = i / kTK, kk = i % kTK;
        const int n = n0 + nn, k = k0 + kk;
        ws[nn][kk] = (n < N && k < K) ? to_f32(w[(int64_t)n * ldw_n + k]) : 0.f;
      }
    } else {           // W stored [K, N]: read along n
      for (int i = t; i < kTN * kTK; i += blockDim.x) {
        const int kk = i / kTN, nn = i % kTN;
        const int n = n0 + nn, k = k0 + kk;
        ws[nn][kk] = (n < N && k < K) ? to_f32(w[(int64_t)k * ldw_k + n * ldw_n]) : 0.f;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kTK; ++kk) {
      const float w0 = ws[2 * t][kk], w1 = ws[2 * t + 1][kk];
#pragma unroll
      for (int r = 0; r < kTM; ++r) {
        const float xv = xs[r][kk];
        acc[r][0] = fmaf(xv, w0, acc[r][0]);
        acc[r][1] = fmaf(xv, w1, acc[r][1]);
      }
    }
    __syncthreads();
  }
  const int n = n0 + 2 * t;
  if (n >= N) return;
#pragma unroll
  for (int r = 0; r < kTM; ++r) {
    const int64_t m = m0 + r;
    if (m < M) epi(z, m, n, acc[r][0], acc[r][1]);
  }
}

template <class T, class Epi>
cudaError_t launch_linear(const T* x, int64_t ldx, int64_t x_z, const T* w, int64_t ldw_n,
                          int64_t ldw_k, int64_t w_z, int64_t M, int N, int K, int Z, Epi epi,
                          cudaStream_t st) {
  dim3 grid((unsigned)((M + kTM - 1) / kTM), (unsigned)((N + kTN - 1) / kTN), (unsigned)Z);
  linear_kernel<T, Epi><<<grid, 128, 0, st>>>(x, ldx, x_z, w, ldw_n, ldw_k, w_z, M, N, K, epi);
  count_launches(1);
  return cudaGetLastError();
}

// Epilogue of the compress step: columns [0, d_c) are c^KV, [d_c, d_c + d_rope) are W^KR x, rotated.
template <class T>
struct CompressEpi {
  T* c; T* k_r; int d_c, d_rope; int64_t ntok, cap; FrameGeom g; RopeTable rt;
  __device__ void operator()(int, int64_t m, int n, float v0, float v1) const {
    const int64_t b = m / ntok, tok = m % ntok;
    const int64_t row = b * cap + ring_row(g, tok);
    if (n < d_c) {
      c[row * d_c + n] = from_f32<T>(v0);
      c[row * d_c + n + 1] = from_f32<T>(v1);
    } else {
      const int col = n - d_c;
      const int64_t f = g.first_frame + tok / g.tokens_per_frame;
      const int64_t r = tok % g.tokens_per_frame;
      float ra, rb;
      rope_rotate(rt, col / 2, f, r / g.grid_w, r % g.grid_w, v0, v1, &ra, &rb);
      k_r[row * d_rope + col] = from_f32<T>(ra);
      k_r[row * d_rope + col + 1] = from_f32<T>(rb);
    }
  }
};

// Epilogue writing head z's column pair into rows of [*, heads, ld] at column offset col0.
template <class T>
struct HeadRowsEpi {
  T* out; int heads; int64_t ld; int col0;
  __device__ void operator()(int z, int64_t m, int n, float v0, float v1) const {
    T* p = out + (m * heads + z) * ld + col0 + n;
    p[0] = from_f32<T>(v0);
    p[1] = from_f32<T>(v1);
  }
};

// Epilogue of the dense comparison projection: head keys (last d_rope of each rotated), then values.
template <class T>
struct DenseAppendEpi {
  T* k; T* v; int heads, d_nope, d_h, d_v; int64_t ntok, cap; FrameGeom g; RopeTable rt;
  __device__ void operator()(int, int64_t m, int n, float v0, float v1) const {
    const int64_t b = m / ntok, tok = m % ntok;
    const int64_t row = b * cap + ring_row(g, tok);
    if (n < heads * d_h) {
      const int hh = n / d_h, cc = n % d_h;
      T* p = k + (row * heads + hh) * d_h + cc;
      if (cc < d_nope) {
        p[0] = from_f32<T>(v0);
        p[1] = from_f32<T>(v1);
      } else {
        const int64_t f = g.first_frame + tok / g.tokens_per_frame;
        const int64_t r = tok % g.tokens_per_frame;
        float ra, rb;
        rope_rotate(rt, (cc - d_nope) / 2, f, r / g.grid_w, r % g.grid_w, v0, v1, &ra, &rb);
        p[0] = from_f32<T>(ra);
        p[1] = from_f32<T>(rb);
      }
    } else {
      const int nv = n - heads * d_h;
      const int hh = nv / d_v, cc = nv % d_v;
      T* p = v + (row * heads + hh) * d_v + cc;
      p[0] = from_f32<T>(v0);
      p[1] = from_f32<T>(v1);
    }
  }
};

// q_rope [rows = batch*nq*heads, d_rope] rotated at its token's position into out[row*ld + col0 ..];
// optionally copies q_nope [rows, d_nope] into out[row*ld + 0 ..] first.
template <class T>
__global__ void rope_rows_kernel(const T* __restrict__ q_rope, const T* __restrict__ q_nope,
                                 int64_t rows, int heads, int64_t nq, int d_rope, int d_nope,
                                 T* __restrict__ out, int64_t ld, int col0, FrameGeom g, RopeTable rt) {
  const int per_row = d_rope / 2 + (q_nope ? d_nope : 0);
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * per_row) return;
  const int64_t row = idx / per_row;
  int e = (int)(idx % per_row);
  if (q_nope) {
    if (e < d_nope) {
      out[row * ld + e] = q_nope[row * d_nope + e];
      return;
    }
    e -= d_nope;
  }
  const int64_t tok = (row / heads) % nq;
  const int64_t f = g.first_frame + tok / g.tokens_per_frame;
  const int64_t r = tok % g.tokens_per_frame;
  float ra, rb;
  rope_rotate(rt, e, f, r / g.grid_w, r % g.grid_w, to_f32(q_rope[row * d_rope + 2 * e]),
              to_f32(q_rope[row * d_rope + 2 * e + 1]), &ra, &rb);
  out[row * ld + col0 + 2 * e] = from_f32<T>(ra);
  out[row * ld + col0 + 2 * e + 1] = from_f32<T>(rb);
}

template <class T>
cudaError_t launch_rope_rows(const T* q_rope, const T* q_nope, int64_t rows, int heads, int64_t nq,
                             int d_rope, int d_nope, T* out, int64_t ld, int col0, const FrameGeom& g,
                             const RopeTable& rt, cudaStream_t st) {
  const int per_row = d_rope / 2 + (q_nope ? d_nope : 0);
  const int64_t total = rows * per_row;
  const int bs = 256;
  rope_rows_kernel<T><<<(unsigned)((total + bs - 1) / bs), bs, 0, st>>>(q_rope, q_nope, rows, heads,
                                                                        nq, d_rope, d_nope, out, ld,
                                                                        col0, g, rt);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Flash attention on CUDA cores: one warp per (batch, token, head) query row; keys in groups of 32
// (one per lane) with an online softmax; each lane owns output columns lane, lane+32, ...
// ------------------------------------------------------------------------------------------------
constexpr int kAttnWarps = 4;
constexpr int kMaxDvPerLane = 8;   // dv <= 256

template <class T>
__global__ void __launch_bounds__(kAttnWarps * 32) simt_attention_kernel(SimtAttnArgs a) {
  extern __shared__ float qs_all[];
  const int warp_in_block = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * kAttnWarps + warp_in_block;
  const int64_t rows = (int64_t)a.batch * a.nq * a.heads;
  if (row >= rows) return;
  const int dq = a.da + a.db;
  float* qs = qs_all + warp_in_block * dq;
  const int h = (int)(row % a.heads);
  const int64_t bn = row / a.heads;
  const int64_t n = bn % a.nq;
  const int64_t b = bn / a.nq;
  const T* q = reinterpret_cast<const T*>(a.q) + row * dq;
  for (int d = lane; d < dq; d += 32) qs[d] = to_f32(q[d]);
  __syncwarp();

  const T* A = reinterpret_cast<const T*>(a.a);
  const T* B = reinterpret_cast<const T*>(a.b);
  const T* V = reinterpret_cast<const T*>(a.v);
  const int64_t kend = key_end_rows(a.g, n);
  float m_run = -FLT_MAX, l_run = 0.f;
  float o[kMaxDvPerLane];
#pragma unroll
  for (int i = 0; i < kMaxDvPerLane; ++i) o[i] = 0.f;

  for (int64_t t0 = 0; t0 < kend; t0 += 32) {
    const int64_t t = t0 + lane;
    float s = -FLT_MAX;
    if (t < kend) {
      const T* ka = A + (b * a.cap + t) * a.a_tok + (int64_t)h * a.a_head;
      float acc = 0.f;
      for (int d = 0; d < a.da; ++d) acc = fmaf(qs[d], to_f32(ka[d]), acc);
      if (a.db > 0) {
        const T* kb = B + (b * a.cap + t) * a.b_tok + (int64_t)h * a.b_head;
        for (int d = 0; d < a.db; ++d) acc = fmaf(qs[a.da + d], to_f32(kb[d]), acc);
      }
      s = acc * a.scale;
    }
    float mt = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
    const float m_new = fmaxf(m_run, mt);
    const float alpha = expf(m_run - m_new);
    const float p = (t < kend) ? expf(s - m_new) : 0.f;
    float ps = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l_run = l_run * alpha + ps;
    m_run = m_new;
#pragma unroll
    for (int i = 0; i < kMaxDvPerLane; ++i) o[i] *= alpha;
    const int nvalid = (int)((kend - t0) < 32 ? (kend - t0) : 32);
    for (int j = 0; j < nvalid; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
      const T* vr = V + (b * a.cap + t0 + j) * a.v_tok + (int64_t)h * a.v_head;
#pragma unroll
      for (int i = 0; i < kMaxDvPerLane; ++i) {
        const int d = lane + 32 * i;
        if (d < a.dv) o[i] = fmaf(pj, to_f32(vr[d]), o[i]);
      }
    }
  }
  T* out = reinterpret_cast<T*>(a.out) + row * a.dv;
  const float inv_l = 1.f / l_run;
#pragma unroll
  for (int i = 0; i < kMaxDvPerLane; ++i) {
    const int d = lane + 32 * i;
    if (d < a.dv) out[d] = from_f32<T>(o[i] * inv_l);
  }
  if (a.lse && lane == 0) a.lse[row] = m_run + logf(l_run);
}

}  // namespace

template <class T>
cudaError_t simt_compress_append(const vmla_config& cfg, int batch, const T* x, const T* w,
                                 const FrameGeom& g, const RopeTable& rt, T* c, T* k_r,
                                 cudaStream_t st) {
  const int64_t ntok = (int64_t)cfg.chunk_frames * cfg.grid_h * cfg.grid_w;
  const int64_t cap = (int64_t)cfg.window_frames * cfg.grid_h * cfg.grid_w;
  CompressEpi<T> epi{c, k_r, cfg.d_c, cfg.d_rope, ntok, cap, g, rt};
  return launch_linear<T>(x, cfg.dim, 0, w, cfg.dim, 1, 0, (int64_t)batch * ntok,
                          cfg.d_c + cfg.d_rope, cfg.dim, 1, epi, st);
}

template <class T>
cudaError_t simt_absorb_q(const vmla_config& cfg, int batch, int64_t nq, const T* q_nope,
                          const T* q_rope, const T* w_uk, const FrameGeom& g, const RopeTable& rt,
                          T* q_abs, cudaStream_t st) {
  const int H = cfg.n_heads, dqk = cfg.d_c + cfg.d_rope;
  const int64_t M = (int64_t)batch * nq;
  // q~[m, h, :] = q_nope[m, h, :] . W_uk[h]  (W_uk[h] is [d_nope (K), d_c (N)])
  HeadRowsEpi<T> epi{q_abs, H, dqk, 0};
  cudaError_t e = launch_linear<T>(q_nope, (int64_t)H * cfg.d_nope, cfg.d_nope, w_uk, 1, cfg.d_c,
                                   (int64_t)cfg.d_nope * cfg.d_c, M, cfg.d_c, cfg.d_nope, H, epi, st);
  if (e != cudaSuccess) return e;
  return launch_rope_rows<T>(q_rope, nullptr, M * H, H, nq, cfg.d_rope, 0, q_abs, dqk, cfg.d_c, g, rt,
                             st);
}

template <class T>
cudaError_t simt_value_up(const vmla_config& cfg, int batch, int64_t n_tokens, const T* o_lat,
                          const T* w_uv, T* out, cudaStream_t st) {
  const int H = cfg.n_heads;
  HeadRowsEpi<T> epi{out, H, cfg.d_v, 0};
  return launch_linear<T>(o_lat, (int64_t)H * cfg.d_c, cfg.d_c, w_uv, cfg.d_c, 1,
                          (int64_t)cfg.d_v * cfg.d_c, (int64_t)batch * n_tokens, cfg.d_v, cfg.d_c, H,
                          epi, st);
}

template <class T>
cudaError_t simt_rope_q(const vmla_config& cfg, int batch, int64_t nq, const T* q_nope,
                        const T* q_rope, const FrameGeom& g, const RopeTable& rt, T* q,
                        cudaStream_t st) {
  const int d_h = cfg.d_nope + cfg.d_rope;
  return launch_rope_rows<T>(q_rope, q_nope, (int64_t)batch * nq * cfg.n_heads, cfg.n_heads, nq,
                             cfg.d_rope, cfg.d_nope, q, d_h, cfg.d_nope, g, rt, st);
}

template <class T>
cudaError_t simt_dense_append(const vmla_config& cfg, int batch, const T* x, const T* w_kv,
                              const FrameGeom& g, const RopeTable& rt, T* k, T* v, cudaStream_t st) {
  const int64_t ntok = (int64_t)cfg.chunk_frames * cfg.grid_h * cfg.grid_w;
  const int64_t cap = (int64_t)cfg.window_frames * cfg.grid_h * cfg.grid_w;
  const int d_h = cfg.d_nope + cfg.d_rope;
  DenseAppendEpi<T> epi{k, v, cfg.n_heads, cfg.d_nope, d_h, cfg.d_v, ntok, cap, g, rt};
  return launch_linear<T>(x, cfg.dim, 0, w_kv, cfg.dim, 1, 0, (int64_t)batch * ntok,
                          cfg.n_heads * (d_h + cfg.d_v), cfg.dim, 1, epi, st);
}

template <class T>
cudaError_t simt_attention(const SimtAttnArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.batch * a.nq * a.heads;
  const size_t smem = sizeof(float) * kAttnWarps * (a.da + a.db);
  simt_attention_kernel<T><<<(unsigned)((rows + kAttnWarps - 1) / kAttnWarps), kAttnWarps * 32, smem,
                             st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

#define VMLA_INSTANTIATE(T)                                                                        \
  template cudaError_t simt_compress_append<T>(const vmla_config&, int, const T*, const T*,        \
                                               const FrameGeom&, const RopeTable&, T*, T*,         \
                                               cudaStream_t);                                      \
  template cudaError_t simt_absorb_q<T>(const vmla_config&, int, int64_t, const T*, const T*,      \
                                        const T*, const FrameGeom&, const RopeTable&, T*,          \
                                        cudaStream_t);                                             \
  template cudaError_t simt_value_up<T>(const vmla_config&, int, int64_t, const T*, const T*, T*,  \
                                        cudaStream_t);                                             \
  template cudaError_t simt_rope_q<T>(const vmla_config&, int, int64_t, const T*, const T*,        \
                                      const FrameGeom&, const RopeTable&, T*, cudaStream_t);       \
  template cudaError_t simt_dense_append<T>(const vmla_config&, int, const T*, const T*,           \
                                            const FrameGeom&, const RopeTable&, T*, T*,            \
                                            cudaStream_t);                                         \
  template cudaError_t simt_attention<T>(const SimtAttnArgs&, cudaStream_t);

VMLA_INSTANTIATE(float)
// bf16 element-wise packing of the dense comparison query (no arithmetic beyond the rotation)
template cudaError_t simt_rope_q<__nv_bfloat16>(const vmla_config&, int, int64_t, const __nv_bfloat16*,
                                                const __nv_bfloat16*, const FrameGeom&, const RopeTable&,
                                                __nv_bfloat16*, cudaStream_t);

}  // namespace vmla
