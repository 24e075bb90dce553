// Projection GEMMs of the VideoMLA path on the sm_100a tensor cores (tcgen05 + TMEM + TMA), each
// with its own fused epilogue:
//   compress_append  [c ; W^KR x] = [W^KV_down ; W^KR] x, 3D-RoPE on the last d_rope columns, bf16
//                    store into the ring rows of the chunk's frames (Method items 1 and 3);
//   absorb_q         q~_h = (W^K_up,h)^T q^nope_h per head (B operand read MN-major from W^K_up as
//                    stored), plus RoPE3D(q^rope_h) written beside it (Method items 2 and 3);
//   value_up         o_h = W^V_up,h o~_h per head (Method item 2);
//   dense_append     the dense comparison layer's per-head K and V projection (RoPE on each head's
//                    last d_rope key columns) into the dense ring.
// One CTA computes one 128-row x BN tile: warp 0 streams A/B k-tiles with TMA into a 4-deep ring,
// warp 1 owns TMEM and issues tcgen05.mma (K = 16 per instruction, fp32 accumulation), warps 2-5 read
// the accumulator rows back (one thread per row) and run the epilogue.
#include <cuda.h>

#include <atomic>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "tc_kernels.cuh"

namespace vmla {
namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int kThreads = 192;
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB

struct GemmShape {
  int64_t M;          // rows of A (all batch elements)
  int N;              // output columns of this GEMM (per head)
  int K;              // reduction length
  int a_head;         // head coordinate of A's map (0 or blockIdx.z)
  uint64_t limit_ns;
  int* status;
};

__device__ __forceinline__ void store32(bf16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = u;
  }
}

__device__ __forceinline__ void rope32(const RopeTable& rt, int pair0, int64_t f, int64_t i, int64_t j,
                                       float* v) {
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    float a, b;
    rope_rotate_f32(rt, pair0 + q, f, i, j, v[2 * q], v[2 * q + 1], &a, &b);
    v[2 * q] = a;
    v[2 * q + 1] = b;
  }
}

// ---- epilogues: called per (row m, 32-column chunk starting at col0) with the fp32 values ----
struct EpiCompress {
  bf16* c; bf16* k_r; int d_c, d_rope; int64_t ntok, cap; FrameGeom g; RopeTable rt;
  __device__ void operator()(int, int64_t m, int col0, float* v) const {
    const int64_t b = m / ntok, tok = m % ntok;
    const int64_t row = b * cap + ring_row(g, tok);
    if (col0 < d_c) {
      store32(c + row * d_c + col0, v);
    } else {
      const int64_t f = g.first_frame + tok / g.tokens_per_frame;
      const int64_t r = tok % g.tokens_per_frame;
      rope32(rt, (col0 - d_c) / 2, f, r / g.grid_w, r % g.grid_w, v);
      store32(k_r + row * d_rope + (col0 - d_c), v);
    }
  }
  __device__ void finish(int, int64_t) const {}
};

struct EpiAbsorb {
  bf16* q_abs; const bf16* q_rope; int heads, d_c, d_rope; int64_t nq; FrameGeom g; RopeTable rt;
  __device__ void operator()(int h, int64_t m, int col0, float* v) const {
    store32(q_abs + (m * heads + h) * (d_c + d_rope) + col0, v);
  }
  // RoPE3D(q^rope) of row m, head h -> q_abs[m, h, d_c : d_c + d_rope]
  __device__ void finish(int h, int64_t m) const {
    const int64_t tok = m % nq;
    const int64_t f = g.first_frame + tok / g.tokens_per_frame;
    const int64_t r = tok % g.tokens_per_frame;
    const bf16* src = q_rope + (m * heads + h) * d_rope;
    for (int c0 = 0; c0 < d_rope; c0 += 32) {
      float v[32];
      const uint4* s4 = reinterpret_cast<const uint4*>(src + c0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 u = s4[q];
        const bf16* e = reinterpret_cast<const bf16*>(&u);
#pragma unroll
        for (int t = 0; t < 8; ++t) v[8 * q + t] = __bfloat162float(e[t]);
      }
      rope32(rt, c0 / 2, f, r / g.grid_w, r % g.grid_w, v);
      store32(q_abs + (m * heads + h) * (d_c + d_rope) + d_c + c0, v);
    }
  }
};

struct EpiValueUp {
  bf16* out; int heads, d_v;
  __device__ void operator()(int h, int64_t m, int col0, float* v) const {
    store32(out + (m * heads + h) * d_v + col0, v);
  }
  __device__ void finish(int, int64_t) const {}
};

struct EpiDense {
  bf16* k; bf16* v; int heads, d_nope, d_h, d_v; int64_t ntok, cap; FrameGeom g; RopeTable rt;
  __device__ void operator()(int, int64_t m, int col0, float* x) const {
    const int64_t b = m / ntok, tok = m % ntok;
    const int64_t row = b * cap + ring_row(g, tok);
    if (col0 < heads * d_h) {
      const int hh = col0 / d_h, cc = col0 % d_h;
      if (cc >= d_nope) {
        const int64_t f = g.first_frame + tok / g.tokens_per_frame;
        const int64_t r = tok % g.tokens_per_frame;
        rope32(rt, (cc - d_nope) / 2, f, r / g.grid_w, r % g.grid_w, x);
      }
      store32(k + (row * heads + hh) * d_h + cc, x);
    } else {
      const int cv = col0 - heads * d_h;
      store32(v + (row * heads + cv / d_v) * d_v + cv % d_v, x);
    }
  }
  __device__ void finish(int, int64_t) const {}
};

template <int BN, bool B_MN_MAJOR, int STAGES>
struct GemmPlan {
  static constexpr int kStages = STAGES;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmemBytes = kStages * kStageBytes + 256 + 1024;
  static constexpr uint32_t kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static_assert(BN % 32 == 0 && BN <= 256, "BN");
  static_assert(!B_MN_MAJOR || BN % 64 == 0, "MN-major B is loaded in 64-column boxes");
};

template <int BN, bool B_MN_MAJOR, int STAGES, class Epi>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
            const GemmShape sh, Epi epi) {
  using PL = GemmPlan<BN, B_MN_MAJOR, STAGES>;
  constexpr int kStages = STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * PL::kStageBytes);
  uint64_t* full = bars;                 // kStages
  uint64_t* empty = bars + kStages;      // kStages
  uint64_t* acc_full = bars + 2 * kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int64_t m0 = (int64_t)blockIdx.x * kBM;
  const int n0 = blockIdx.y * BN;
  const int head = blockIdx.z;
  const int nk = (sh.K + kBK - 1) / kBK;
  int zero_flag = 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      int issued = 0;
      for (int kt = 0; kt < nk; ++kt) {
        const int st = kt % kStages;
        if (kt >= kStages &&
            !mbar_wait(empty + st, ((kt / kStages) - 1) & 1, abort_flag, sh.status, 11, sh.limit_ns))
          break;
        uint8_t* sa = smem + st * PL::kStageBytes;
        uint8_t* sb = sa + kABytes;
        mbar_arrive_expect_tx(full + st, PL::kStageBytes);
        tma_load_4d(sa, &map_a, full + st, kt * kBK, sh.a_head ? head : 0, (int)m0, 0);
        if (B_MN_MAJOR) {
#pragma unroll
          for (int i = 0; i < BN / 64; ++i)
            tma_load_4d(sb + i * (kBK * 128), &map_b, full + st, n0 + 64 * i, kt * kBK, head, 0);
        } else {
          tma_load_4d(sb, &map_b, full + st, kt * kBK, n0, head, 0);
        }
        issued = kt + 1;
      }
      if (*abort_flag)
        for (int kt = (issued > kStages ? issued - kStages : 0); kt < issued; ++kt)
          mbar_wait(full + kt % kStages, (kt / kStages) & 1, &zero_flag, nullptr, 0, sh.limit_ns);
    }
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, 0, B_MN_MAJOR ? 1 : 0);
      bool ok = true;
      for (int kt = 0; kt < nk; ++kt) {
        const int st = kt % kStages;
        if (!mbar_wait(full + st, (kt / kStages) & 1, abort_flag, sh.status, 12, sh.limit_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + st * PL::kStageBytes);
        const uint32_t b = a + kABytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = smem_desc(a + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = B_MN_MAJOR ? smem_desc(b + kk * 2048, kBK * 128, 1024, kSwizzle128B)
                                         : smem_desc(b + kk * 32, 16, 1024, kSwizzle128B);
          mma_ss(tmem, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(empty + st);
      }
      mma_commit(acc_full);
      (void)ok;
      // every MMA of this CTA has completed before TMEM is released
      mbar_wait(acc_full, 0, &zero_flag, nullptr, 0, sh.limit_ns);
    }
  } else {
    // epilogue: warps 2..5, TMEM lane quadrant = warp % 4
    const int quad = warp & 3;
    const int r = quad * 32 + (threadIdx.x & 31);
    const int64_t m = m0 + r;
    const bool got = mbar_wait(acc_full, 0, abort_flag, sh.status, 13, sh.limit_ns);
    if (__all_sync(0xffffffffu, got)) {     // the TMEM loads below are warp-collective
      tc_fence_after();
      const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_base + c0, raw);
        tmem_ld_wait();
        if (m < sh.M && n0 + c0 < sh.N) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
          epi(head, m, n0 + c0, v);
        }
      }
      if (m < sh.M && blockIdx.y == 0) epi.finish(head, m);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kTmemCols);
  }
}

template <int BN, bool B_MN_MAJOR, int STAGES, class Epi>
cudaError_t launch_gemm_st(const CUtensorMap& a, const CUtensorMap& b, const GemmShape& sh, int heads,
                           const Epi& epi, cudaStream_t st) {
  using PL = GemmPlan<BN, B_MN_MAJOR, STAGES>;
  auto kern = gemm_kernel<BN, B_MN_MAJOR, STAGES, Epi>;
  static std::atomic<uint64_t> done{0};
  cudaError_t attr_err = ensure_smem_attr((const void*)kern, PL::kSmemBytes, done);
  if (attr_err != cudaSuccess) return attr_err;
  dim3 grid((unsigned)((sh.M + kBM - 1) / kBM), (unsigned)((sh.N + BN - 1) / BN), (unsigned)heads);
  kern<<<grid, kThreads, PL::kSmemBytes, st>>>(a, b, sh, epi);
  count_launches(1);
  return cudaGetLastError();
}

// Short reductions (K <= 2 k-tiles per stage ring) use a 2-deep ring so that several CTAs share an SM
// and one CTA's epilogue overlaps another's loads; long ones (the D = 1536 projections) a 4-deep ring.
template <int BN, bool B_MN_MAJOR, class Epi>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmShape& sh, int heads,
                        const Epi& epi, cudaStream_t st) {
  if (sh.K <= 4 * kBK) return launch_gemm_st<BN, B_MN_MAJOR, 2>(a, b, sh, heads, epi, st);
  return launch_gemm_st<BN, B_MN_MAJOR, 4>(a, b, sh, heads, epi, st);
}

}  // namespace

static int pick_bn(int N);
static bool bn_supported(int bn, bool mn_major);

vmla_status tc_check_compress(const vmla_config& c) {
  if (c.d_rope != 32 || c.d_c % 32 || c.dim % 8 || !bn_supported(pick_bn(c.d_c + c.d_rope), false)) {
    set_tc_reason("tensor-core compress needs d_rope == 32, d_c % 32 == 0, dim % 8 == 0");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
}

vmla_status tc_check_absorb(const vmla_config& c) {
  if (c.d_rope % 32 || !bn_supported(c.d_c, true) || c.d_nope % 8) {
    set_tc_reason("tensor-core absorb_q needs d_c % 64 == 0, d_c <= 256, d_rope % 32 == 0, d_nope % 8 == 0");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
}

vmla_status tc_check_value_up(const vmla_config& c) {
  if (!bn_supported(c.d_v, false) || c.d_c % 8) {
    set_tc_reason("tensor-core value_up needs d_v in {64, 96, 128, 160, 192, 224, 256}, d_c % 8 == 0");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
}

vmla_status tc_check_dense_append(const vmla_config& c) {
  const int d_h = c.d_nope + c.d_rope;
  if (c.d_nope % 32 || c.d_rope % 32 || c.d_v % 32 || c.dim % 8 || (c.n_heads * (d_h + c.d_v)) % 32 ||
      d_h % 32) {
    set_tc_reason("tensor-core dense_append needs d_nope, d_rope, d_v multiples of 32 and dim % 8 == 0");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
}

// Column tile used for an N-wide projection: the whole N when it fits one tcgen05.mma (N <= 256),
// else 160-column tiles.  Every candidate is a multiple of 32 (epilogue chunks) and of 16 (MMA N).
static int pick_bn(int N) { return N <= 256 ? N : 160; }

template <bool B_MN_MAJOR, class Epi>
static cudaError_t dispatch_bn(int bn, const CUtensorMap& a, const CUtensorMap& b, const GemmShape& sh,
                               int heads, const Epi& epi, cudaStream_t st) {
  switch (bn) {
    case 64: return launch_gemm<64, B_MN_MAJOR>(a, b, sh, heads, epi, st);
    case 128: return launch_gemm<128, B_MN_MAJOR>(a, b, sh, heads, epi, st);
    case 192: return launch_gemm<192, B_MN_MAJOR>(a, b, sh, heads, epi, st);
    case 256: return launch_gemm<256, B_MN_MAJOR>(a, b, sh, heads, epi, st);
    default: break;
  }
  if constexpr (!B_MN_MAJOR) {
    switch (bn) {
      case 96: return launch_gemm<96, false>(a, b, sh, heads, epi, st);
      case 160: return launch_gemm<160, false>(a, b, sh, heads, epi, st);
      case 224: return launch_gemm<224, false>(a, b, sh, heads, epi, st);
      default: break;
    }
  }
  return cudaErrorInvalidValue;
}

static bool bn_supported(int bn, bool mn_major) {
  if (bn == 64 || bn == 128 || bn == 192 || bn == 256) return true;
  return !mn_major && (bn == 96 || bn == 160 || bn == 224);
}

cudaError_t tc_compress_append(const vmla_config& cfg, int batch, const void* x, const void* w,
                               const FrameGeom& g, const RopeTable& rt, void* c, void* k_r,
                               cudaStream_t st) {
  const int64_t ntok = (int64_t)cfg.chunk_frames * cfg.grid_h * cfg.grid_w;
  const int64_t M = batch * ntok;
  const int N = cfg.d_c + cfg.d_rope, K = cfg.dim;
  const int bn = pick_bn(N);
  CUtensorMap ma, mb;
  cudaError_t e;
  // A = x [M, D]; B = [W^KV_down ; W^KR] [N, D], both K-major
  if ((e = make_map_4d(&ma, x, K, 1, M, 1, (int64_t)K * 2, (int64_t)K * 2, M * K * 2, kBK, 1, kBM, 128)) != cudaSuccess)
    return e;
  if ((e = make_map_4d(&mb, w, K, N, 1, 1, (int64_t)K * 2, (int64_t)N * K * 2, (int64_t)N * K * 2, kBK, bn, 1, 128)) != cudaSuccess)
    return e;
  GemmShape sh{M, N, K, 0, wait_limit_ns(), device_status_ptr()};
  EpiCompress epi{(bf16*)c, (bf16*)k_r, cfg.d_c, cfg.d_rope, ntok, (int64_t)cfg.window_frames * cfg.grid_h * cfg.grid_w, g, rt};
  return dispatch_bn<false>(bn, ma, mb, sh, 1, epi, st);
}

cudaError_t tc_absorb_q(const vmla_config& cfg, int batch, int64_t nq, const void* q_nope,
                        const void* q_rope, const void* w_uk, const FrameGeom& g, const RopeTable& rt,
                        void* q_abs, cudaStream_t st) {
  const int H = cfg.n_heads, K = cfg.d_nope, N = cfg.d_c;
  const int64_t M = batch * nq;
  CUtensorMap ma, mb;
  cudaError_t e;
  // A = q_nope [M, H, d_nope] (head h's rows); B = W^K_up [H, d_nope (K), d_c (N)] read MN-major
  if ((e = make_map_4d(&ma, q_nope, K, H, M, 1, (int64_t)K * 2, (int64_t)H * K * 2, M * H * K * 2, kBK, 1, kBM, 128)) != cudaSuccess)
    return e;
  if ((e = make_map_4d(&mb, w_uk, N, K, H, 1, (int64_t)N * 2, (int64_t)K * N * 2, (int64_t)H * K * N * 2, 64, kBK, 1, 128)) != cudaSuccess)
    return e;
  GemmShape sh{M, N, K, 1, wait_limit_ns(), device_status_ptr()};
  EpiAbsorb epi{(bf16*)q_abs, (const bf16*)q_rope, H, cfg.d_c, cfg.d_rope, nq, g, rt};
  return dispatch_bn<true>(N, ma, mb, sh, H, epi, st);
}

cudaError_t tc_value_up(const vmla_config& cfg, int batch, int64_t n_tokens, const void* o_lat,
                        const void* w_uv, void* out, cudaStream_t st) {
  const int H = cfg.n_heads, K = cfg.d_c, N = cfg.d_v;
  const int64_t M = batch * n_tokens;
  CUtensorMap ma, mb;
  cudaError_t e;
  // A = o~ [M, H, d_c] (head h's rows); B = W^V_up [H, d_v (N), d_c (K)], K-major
  if ((e = make_map_4d(&ma, o_lat, K, H, M, 1, (int64_t)K * 2, (int64_t)H * K * 2, M * H * K * 2, kBK, 1, kBM, 128)) != cudaSuccess)
    return e;
  if ((e = make_map_4d(&mb, w_uv, K, N, H, 1, (int64_t)K * 2, (int64_t)N * K * 2, (int64_t)H * N * K * 2, kBK, N, 1, 128)) != cudaSuccess)
    return e;
  GemmShape sh{M, N, K, 1, wait_limit_ns(), device_status_ptr()};
  EpiValueUp epi{(bf16*)out, H, N};
  return dispatch_bn<false>(N, ma, mb, sh, H, epi, st);
}

cudaError_t tc_dense_append(const vmla_config& cfg, int batch, const void* x, const void* w_kv,
                            const FrameGeom& g, const RopeTable& rt, void* k, void* v,
                            cudaStream_t st) {
  const int64_t ntok = (int64_t)cfg.chunk_frames * cfg.grid_h * cfg.grid_w;
  const int64_t M = batch * ntok;
  const int d_h = cfg.d_nope + cfg.d_rope;
  const int N = cfg.n_heads * (d_h + cfg.d_v), K = cfg.dim;
  const int bn = N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64);
  CUtensorMap ma, mb;
  cudaError_t e;
  if ((e = make_map_4d(&ma, x, K, 1, M, 1, (int64_t)K * 2, (int64_t)K * 2, M * K * 2, kBK, 1, kBM, 128)) != cudaSuccess)
    return e;
  if ((e = make_map_4d(&mb, w_kv, K, N, 1, 1, (int64_t)K * 2, (int64_t)N * K * 2, (int64_t)N * K * 2, kBK, bn, 1, 128)) != cudaSuccess)
    return e;
  GemmShape sh{M, N, K, 0, wait_limit_ns(), device_status_ptr()};
  EpiDense epi{(bf16*)k, (bf16*)v, cfg.n_heads, cfg.d_nope, d_h, cfg.d_v, ntok,
               (int64_t)cfg.window_frames * cfg.grid_h * cfg.grid_w, g, rt};
  return dispatch_bn<false>(bn, ma, mb, sh, 1, epi, st);
}

cudaError_t tc_rope_q(const vmla_config& cfg, int batch, int64_t nq, const void* q_nope,
                      const void* q_rope, const FrameGeom& g, const RopeTable& rt, void* q,
                      cudaStream_t st) {
  return simt_rope_q<bf16>(cfg, batch, nq, (const bf16*)q_nope, (const bf16*)q_rope, g, rt, (bf16*)q, st);
}

}  // namespace vmla
