// Pieces shared by the projection kernels (tc_gemm.cu, tc_compress.cu): the per-CTA 3D-RoPE cos/sin
// table of their epilogues and the SM count of the current device.
#pragma once

#include <cuda_runtime.h>

#include "vmla_internal.cuh"

namespace vmla {

// 3D-RoPE of the epilogues through a per-CTA table: cos/sin of every (rotary pair, position along its
// axis) that the call can meet -- the call's frames, every row, every column -- computed once per CTA
// in shared memory (angle reduced in double precision, then sincosf).  Pair p's entries start at
// off[p]; frame positions are stored relative to base_f.  n_entries == 0 (table too large) falls back
// to computing each rotation directly.
constexpr int kRopeTabEntries = 2048;

struct RopeLookup {
  RopeTable rt;
  int off[kMaxRopePairs];
  int64_t base_f;
  int n_entries;
  __device__ void rotate32(const float2* tab, int pair0, int64_t f, int64_t i, int64_t j, float* v) const {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int p = pair0 + q;
      float a, b;
      if (n_entries) {
        const int ax = rt.axis[p];
        const int64_t pos = ax == 0 ? f - base_f : (ax == 1 ? i : j);
        const float2 cs = tab[off[p] + pos];
        a = v[2 * q] * cs.x - v[2 * q + 1] * cs.y;
        b = v[2 * q] * cs.y + v[2 * q + 1] * cs.x;
      } else {
        rope_rotate_f32(rt, p, f, i, j, v[2 * q], v[2 * q + 1], &a, &b);
      }
      v[2 * q] = a;
      v[2 * q + 1] = b;
    }
  }

  // Rotate the two pairs of four consecutive columns starting at rotary pair `pair0`.
  __device__ void rotate4(const float2* tab, int pair0, int64_t f, int64_t i, int64_t j, float* v) const {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int p = pair0 + q;
      float a, b;
      if (n_entries) {
        const int ax = rt.axis[p];
        const int64_t pos = ax == 0 ? f - base_f : (ax == 1 ? i : j);
        const float2 cs = tab[off[p] + pos];
        a = v[2 * q] * cs.x - v[2 * q + 1] * cs.y;
        b = v[2 * q] * cs.y + v[2 * q + 1] * cs.x;
      } else {
        rope_rotate_f32(rt, p, f, i, j, v[2 * q], v[2 * q + 1], &a, &b);
      }
      v[2 * q] = a;
      v[2 * q + 1] = b;
    }
  }

  // fill the table with threads t0 .. t0 + nthreads - 1 (the caller synchronises them afterwards).  The
  // angle is reduced to [-pi, pi] in double precision, then the MUFU sine / cosine (absolute error
  // about 1e-6 there, far below the bf16 rounding of the rotated values) keep the build short.
  __device__ void build(float2* smem_tab, int t0, int nthreads) const {
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
    for (int e = t0; e < n_entries; e += nthreads) {
      int p = 0;
      while (p + 1 < rt.n_pairs && off[p + 1] <= e) ++p;
      const int64_t v = e - off[p];
      const double pos = (double)(rt.axis[p] == 0 ? base_f + v : v);
      double ang = pos * rt.inv_freq[p];
      ang = fma(-two_pi, rint(ang * inv_two_pi), ang);
      float sn, cs;
      __sincosf((float)ang, &sn, &cs);
      smem_tab[e] = make_float2(cs, sn);
    }
  }
};

// Host: table layout for a call whose tokens span `frames` frames starting at g.first_frame.
inline RopeLookup make_rope_lookup(const RopeTable& rt, const FrameGeom& g, int frames,
                                   int max_entries = kRopeTabEntries) {
  RopeLookup L{};
  L.rt = rt;
  L.base_f = g.first_frame;
  const int extent[3] = {frames, g.tokens_per_frame / g.grid_w, g.grid_w};
  int total = 0;
  for (int p = 0; p < rt.n_pairs; ++p) {
    L.off[p] = total;
    total += extent[rt.axis[p]];
  }
  L.n_entries = total <= max_entries ? total : 0;
  return L;
}

inline int num_sms() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cached[dev] = v;
  }
  return cached[dev];
}

}  // namespace vmla
