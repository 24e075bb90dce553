// Flash-style attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA) for
//  * the VideoMLA latent cache (absorbed form): one KV "head" shared by every query head, keys
//    [c ; k^R] (d_c + 32 wide) and values c (d_c wide) read from the same shared-memory stage
//    (VideoMLA technical summary, Method items 2-3: per-head keys and values are reconstructed from
//    the shared latent; here the reconstruction is folded into the query and applied after the sum);
//  * the dense per-head comparison layer (d_h = d_v = 128 per head).
//
// One CTA owns one tile of 128 query rows and streams every visible KV tile of 128 keys:
//   warp 4      TMA producer: Q tile once, then KV tiles into an NST-deep shared-memory ring;
//   warp 5      TMEM owner and MMA issuer: S_j = Q K_j^T into one of two TMEM S buffers, then
//               O += P_{j-1} V_{j-1} with P read from TMEM (it overwrites S_{j-1} as bf16);
//   warps 0-3   softmax, one thread per query row (TMEM lane): masked running max with a lazy
//               rescale of O (only when the max grows by more than 2^8), exp2, row sum, P to TMEM;
//               finally O / l to global memory and the log-sum-exp.
// The KV ring is released by tcgen05.commit after the P*V MMAs that last read a stage.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "tc_kernels.cuh"

namespace vmla {
namespace {

using namespace sm100;

constexpr int kThreads = 192;          // 6 warps
constexpr int kBlockM = 128;           // query rows per CTA
constexpr int kBlockN = 128;           // keys per KV tile
constexpr int kBoxBytes = kBlockN * 64 * 2;   // one [128 x 64] bf16 box (16 KB)
constexpr int kRopeBoxBytes = kBlockN * 32 * 2;  // one [128 x 32] bf16 box (8 KB)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;       // O accumulator columns start here (S buffers at 0 and 128)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnParams {
  int rows_per_b;        // query rows per batch element (latent: Nq*H, dense: Nq)
  int tiles_per_group;   // query tiles per (batch[, head]) group
  int heads;             // dense: heads per token (tile groups are (b, h)); latent: n = row / heads
  int dense;             // 1 for the per-head dense layer
  int64_t nq;            // query tokens per batch element
  FrameGeom g;
  float scale_log2;      // softmax_scale * log2(e)
  void* out;
  float* lse;
  int* status;
  uint64_t limit_ns;
  int drop_kv_tile;      // test hook: this KV tile is never loaded (-1: none)
};

// Shared-memory plan of one kernel instance.
template <int KB, int KR, int VB, bool V_ALIAS>
struct Plan {
  static constexpr int kQBytes = KB * kBoxBytes + (KR ? kRopeBoxBytes : 0);
  static constexpr int kKBytes = KB * kBoxBytes + (KR ? kRopeBoxBytes : 0);
  static constexpr int kVBytes = V_ALIAS ? 0 : VB * kBoxBytes;
  static constexpr int kStageBytes = kKBytes + kVBytes;
  static constexpr int kBudget = 232448 - 1024 - 256;
  static constexpr int kStages = ((kBudget - kQBytes) / kStageBytes) >= 4 ? 4 : ((kBudget - kQBytes) / kStageBytes);
  static constexpr int kSmemBytes = kQBytes + kStages * kStageBytes + 256 + 1024;
  static constexpr int kDV = 64 * VB;
  static_assert(kStages >= 2, "shared memory too small for two KV stages");
  static_assert(kTmemO + kDV <= kTmemCols, "TMEM budget");
};

template <int KB, int KR, int VB, bool V_ALIAS>
__global__ void __launch_bounds__(kThreads, 1)
attention_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_qr,
                 const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_kr,
                 const __grid_constant__ CUtensorMap map_v, const AttnParams p) {
  using P = Plan<KB, KR, VB, V_ALIAS>;
  constexpr int NST = P::kStages;
  constexpr int DV = P::kDV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + P::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NST * P::kStageBytes);
  uint64_t* bar_q = bars;                 // 1
  uint64_t* kv_full = bars + 1;           // NST
  uint64_t* kv_empty = bars + 1 + NST;    // NST
  uint64_t* s_full = bars + 1 + 2 * NST;  // 2
  uint64_t* p_ready = s_full + 2;         // 2
  uint64_t* o_bar = p_ready + 2;          // 1
  uint64_t* drain = o_bar + 1;            // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;

  // ---- tile coordinates ----
  const int tile = blockIdx.x;
  const int group = tile / p.tiles_per_group;
  const int row0 = (tile % p.tiles_per_group) * kBlockM;      // first query row of the tile
  const int b = p.dense ? group / p.heads : group;
  const int h = p.dense ? group % p.heads : 0;
  const int tok_div = p.dense ? 1 : p.heads;                   // query row -> token
  const int last_row = min(row0 + kBlockM, p.rows_per_b) - 1;
  const int64_t kend_first = key_end_rows(p.g, row0 / tok_div);
  const int64_t kend_last = key_end_rows(p.g, last_row / tok_div);
  const int n_kv = (int)((kend_last + kBlockN - 1) / kBlockN);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NST; ++s) { mbar_init(kv_full + s, 1); mbar_init(kv_empty + s, 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(s_full + s, 1); mbar_init(p_ready + s, 128); }
    mbar_init(o_bar, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int zero_flag = 0;

  if (warp == 4) {
    // ================= TMA producer =================
    if (elect_one()) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      if (!V_ALIAS) tma_prefetch_desc(&map_v);
      mbar_arrive_expect_tx(bar_q, P::kQBytes);
      for (int i = 0; i < KB; ++i) tma_load_4d(sQ + i * kBoxBytes, &map_q, bar_q, 64 * i, h, row0, b);
      if (KR) tma_load_4d(sQ + KB * kBoxBytes, &map_qr, bar_q, 64 * KB, h, row0, b);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % NST;
        if (j >= NST && !mbar_wait(kv_empty + st, ((j / NST) - 1) & 1, abort_flag, p.status, 1, p.limit_ns))
          break;
        issued = j + 1;
        if (j == p.drop_kv_tile) continue;
        uint8_t* stage = sKV + st * P::kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, P::kStageBytes);
        const int krow = j * kBlockN;
        for (int i = 0; i < KB; ++i) tma_load_4d(stage + i * kBoxBytes, &map_k, kv_full + st, 64 * i, h, krow, b);
        if (KR) tma_load_4d(stage + KB * kBoxBytes, &map_kr, kv_full + st, 0, 0, krow, b);
        if (!V_ALIAS)
          for (int i = 0; i < VB; ++i)
            tma_load_4d(stage + P::kKBytes + i * kBoxBytes, &map_v, kv_full + st, 64 * i, h, krow, b);
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        mbar_wait(bar_q, 0, &zero_flag, nullptr, 0, p.limit_ns);
        for (int j = (issued > NST ? issued - NST : 0); j < issued; ++j)
          if (j != p.drop_kv_tile) mbar_wait(kv_full + j % NST, (j / NST) & 1, &zero_flag, nullptr, 0, p.limit_ns);
      }
    }
  } else if (warp == 5) {
    // ================= MMA issuer =================
    if (elect_one()) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, DV, 0, 1);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t kv_base = smem_u32(sKV);
      bool ok = mbar_wait(bar_q, 0, abort_flag, p.status, 2, p.limit_ns);
      auto issue_pv = [&](int jp) -> bool {
        const int bp = jp & 1;
        if (!mbar_wait(p_ready + bp, (jp >> 1) & 1, abort_flag, p.status, 3, p.limit_ns)) return false;
        tc_fence_after();
        const uint32_t v_base = kv_base + (jp % NST) * P::kStageBytes + (V_ALIAS ? 0 : P::kKBytes);
#pragma unroll
        for (int k = 0; k < kBlockN / 16; ++k) {
          // V tile [128 keys][64*VB] as MN-major operand: 8-key groups 1024 B apart (SBO), 64-column
          // boxes 16 KB apart (LBO); each K step of 16 keys advances 2048 B.
          const uint64_t vdesc = smem_desc(v_base + k * 2048, kBoxBytes, 1024, kSwizzle128B);
          mma_ts(tmem + kTmemO, tmem + bp * 128 + k * 8, vdesc, idesc_pv, (jp > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(kv_empty + (jp % NST));
        mma_commit(o_bar);
        return true;
      };
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j % NST, bj = j & 1;
        if (!mbar_wait(kv_full + st, (j / NST) & 1, abort_flag, p.status, 4, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_base = kv_base + st * P::kStageBytes;
#pragma unroll
        for (int k = 0; k < KB * 4; ++k) {
          const uint32_t off = (k >> 2) * kBoxBytes + (k & 3) * 32;
          mma_ss(tmem + bj * 128, smem_desc(q_base + off, 16, 1024, kSwizzle128B),
                 smem_desc(k_base + off, 16, 1024, kSwizzle128B), idesc_qk, k > 0 ? 1u : 0u);
        }
        if (KR) {
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint32_t off = KB * kBoxBytes + k * 32;
            mma_ss(tmem + bj * 128, smem_desc(q_base + off, 16, 512, kSwizzle64B),
                   smem_desc(k_base + off, 16, 512, kSwizzle64B), idesc_qk, 1u);
          }
        }
        mma_commit(s_full + bj);
        if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && n_kv > 0) issue_pv(n_kv - 1);
      // every MMA of this CTA has completed before TMEM is released
      mma_commit(drain);
      mbar_wait(drain, 0, &zero_flag, nullptr, 0, p.limit_ns);
    }
  } else {
    // ================= softmax + epilogue (warps 0-3, thread = query row = TMEM lane) =================
    const int r = threadIdx.x;                      // 0..127
    const int row = row0 + r;
    const bool row_valid = row < p.rows_per_b;
    const int64_t kend = row_valid ? key_end_rows(p.g, row / tok_div) : kend_last;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    // Wait until P_{k} V_{k} has completed (phase k of o_bar).  Only called from tile j = k + 1,
    // where o_bar is at most one phase away from phase k: s_full[j] completing implies that
    // P_{j-2} V_{j-2} completed (it was issued before S_j), and P_j V_j cannot start before this
    // thread releases P_j, so a parity wait is unambiguous.  Warp-uniform (__all_sync) because the
    // TMEM loads/stores that follow are warp-collective.
    auto wait_pv = [&](int k) -> bool {
      const bool got = mbar_wait(o_bar, k & 1, abort_flag, p.status, 5, p.limit_ns);
      return __all_sync(0xffffffffu, got);
    };
    for (int j = 0; j < n_kv; ++j) {
      const int bj = j & 1;
      const bool got = mbar_wait(s_full + bj, (j >> 1) & 1, abort_flag, p.status, 6, p.limit_ns);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      // S row of this thread (raw scores): four 32-column TMEM loads, one wait
      uint32_t sr[kBlockN];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(tmem + lane_base + bj * 128 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + c * 32));
      tmem_ld_wait();
      const int64_t key0 = (int64_t)j * kBlockN;
      if (key0 + kBlockN > kend_first) {
#pragma unroll
        for (int i = 0; i < kBlockN; ++i)
          if (key0 + i >= kend) sr[i] = __float_as_uint(-INFINITY);
      }
      // row max as a tree of 8 independent chains (the scale is positive, so it is applied after)
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(sr[i]);
#pragma unroll
      for (int i = 8; i < kBlockN; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sr[i]));
#pragma unroll
      for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
      const float m_new = fmaxf(m_ref, mx[0] * p.scale_log2);
      const bool need = m_new > m_ref + kRescaleThreshold;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = fast_exp2(m_ref - m_new);   // 0 on the first tile
        if (j > 0) {
          if (!wait_pv(j - 1)) { ok = false; break; }
          tc_fence_after();
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < DV / 32; ++c) {
            tmem_ld32(tmem + lane_base + kTmemO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_base + kTmemO + c * 32, o);
          }
        }
        l_sum *= alpha;
        m_ref = m_new;
      }
      // p = 2^(s * scale*log2(e) - m) (one FFMA + one MUFU.EX2 per score), row sum in 8 chains,
      // P packed to bf16 pairs over the first 64 columns of this S buffer
      const float neg_m = -m_ref;
      float ls[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ls[i] = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sr[c * 64 + 2 * i]), p.scale_log2, neg_m));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sr[c * 64 + 2 * i + 1]), p.scale_log2, neg_m));
          ls[(2 * i) & 7] += p0;
          ls[(2 * i + 1) & 7] += p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tmem + lane_base + bj * 128 + c * 32, pk);
      }
#pragma unroll
      for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) ls[i] += ls[i + w];
      l_sum += ls[0];
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_ready + bj);
    }
    // `drain` is committed once, after the last P*V, so its single phase marks O complete
    bool fin = ok && mbar_wait(drain, 0, abort_flag, p.status, 7, p.limit_ns);
    fin = __all_sync(0xffffffffu, fin && !*abort_flag);
    if (fin) {
      tc_fence_after();
      const float inv_l = 1.f / l_sum;
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
      int64_t orow;
      if (p.dense) orow = (((int64_t)b * p.nq + row) * p.heads + h);
      else orow = (int64_t)b * p.rows_per_b + row;
      uint32_t o[32];
#pragma unroll
      for (int c = 0; c < DV / 32; ++c) {
        tmem_ld32(tmem + lane_base + kTmemO + c * 32, o);
        tmem_ld_wait();
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(out + orow * DV + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
            dst[q] = v;
          }
        }
      }
      if (row_valid && p.lse) p.lse[orow] = (m_ref + __log2f(l_sum)) * 0.69314718055994530942f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int KB, int KR, int VB, bool V_ALIAS>
std::atomic<uint64_t>& attr_done() {
  static std::atomic<uint64_t> mask{0};
  return mask;
}

template <int KB, int KR, int VB, bool V_ALIAS>
cudaError_t launch_attention(const TmaMaps5& m, const AttnParams& p, int n_tiles, cudaStream_t st) {
  using PL = Plan<KB, KR, VB, V_ALIAS>;
  auto kern = attention_kernel<KB, KR, VB, V_ALIAS>;
  cudaError_t attr_err = ensure_smem_attr((const void*)kern, PL::kSmemBytes, attr_done<KB, KR, VB, V_ALIAS>());
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<n_tiles, kThreads, PL::kSmemBytes, st>>>(m.q, m.qr, m.k, m.kr, m.v, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

vmla_status tc_check_latent_attention(const vmla_config& c) {
  if (c.d_rope != 32) { set_tc_reason("tensor-core latent attention needs d_rope == 32"); return VMLA_ERR_UNSUPPORTED; }
  if (c.d_c % 64 || c.d_c < 64 || c.d_c > 256) {
    set_tc_reason("tensor-core latent attention needs d_c in {64, 128, 192, 256}");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
}

vmla_status tc_check_dense_mha(const vmla_config& c) {
  const int d_h = c.d_nope + c.d_rope;
  if (d_h != 128 || c.d_v != 128) {
    set_tc_reason("tensor-core dense attention needs d_h == d_v == 128");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
}

cudaError_t tc_latent_attention(const vmla_config& cfg, int batch, int64_t nq, const void* q_abs,
                                const void* c, const void* k_r, int64_t cap, int64_t valid_rows,
                                const FrameGeom& g, float scale, void* out, float* lse, int* status,
                                cudaStream_t st) {
  const int H = cfg.n_heads, dqk = cfg.d_c + cfg.d_rope;
  const int64_t rows = nq * H;
  TmaMaps5 m{};
  cudaError_t e;
  // q_abs [B, Nq*H, d_qk] viewed as 4D {d_qk, 1, Nq*H, B}
  if ((e = make_map_4d(&m.q, q_abs, dqk, 1, rows, batch, (int64_t)dqk * 2, (int64_t)dqk * 2,
                       rows * dqk * 2, 64, 1, kBlockM, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.qr, q_abs, dqk, 1, rows, batch, (int64_t)dqk * 2, (int64_t)dqk * 2,
                       rows * dqk * 2, 32, 1, kBlockM, 64)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.k, c, cfg.d_c, 1, valid_rows, batch, (int64_t)cfg.d_c * 2, (int64_t)cfg.d_c * 2,
                       cap * cfg.d_c * 2, 64, 1, kBlockN, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.kr, k_r, 32, 1, valid_rows, batch, 64, 64, cap * 64, 32, 1, kBlockN, 64)) != cudaSuccess)
    return e;
  m.v = m.k;
  AttnParams p{};
  p.rows_per_b = (int)rows;
  p.tiles_per_group = (int)((rows + kBlockM - 1) / kBlockM);
  p.heads = H;
  p.dense = 0;
  p.nq = nq;
  p.g = g;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.limit_ns = wait_limit_ns();
  p.drop_kv_tile = take_drop_kv_tile();
  const int n_tiles = batch * p.tiles_per_group;
  switch (cfg.d_c) {
    case 64: return launch_attention<1, 32, 1, true>(m, p, n_tiles, st);
    case 128: return launch_attention<2, 32, 2, true>(m, p, n_tiles, st);
    case 192: return launch_attention<3, 32, 3, true>(m, p, n_tiles, st);
    default: return launch_attention<4, 32, 4, true>(m, p, n_tiles, st);
  }
}

cudaError_t tc_dense_mha(const vmla_config& cfg, int batch, int64_t nq, const void* q, const void* k,
                         const void* v, int64_t cap, int64_t valid_rows, const FrameGeom& g,
                         float scale, void* out, float* lse, int* status, cudaStream_t st) {
  const int H = cfg.n_heads;
  const int D = 128;
  TmaMaps5 m{};
  cudaError_t e;
  if ((e = make_map_4d(&m.q, q, D, H, nq, batch, D * 2, (int64_t)H * D * 2, nq * H * D * 2, 64, 1, kBlockM,
                       128)) != cudaSuccess) return e;
  m.qr = m.q;
  if ((e = make_map_4d(&m.k, k, D, H, valid_rows, batch, D * 2, (int64_t)H * D * 2, cap * H * D * 2, 64, 1,
                       kBlockN, 128)) != cudaSuccess) return e;
  m.kr = m.k;
  if ((e = make_map_4d(&m.v, v, D, H, valid_rows, batch, D * 2, (int64_t)H * D * 2, cap * H * D * 2, 64, 1,
                       kBlockN, 128)) != cudaSuccess) return e;
  AttnParams p{};
  p.rows_per_b = (int)nq;
  p.tiles_per_group = (int)((nq + kBlockM - 1) / kBlockM);
  p.heads = H;
  p.dense = 1;
  p.nq = nq;
  p.g = g;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.limit_ns = wait_limit_ns();
  p.drop_kv_tile = -1;
  const int n_tiles = batch * H * p.tiles_per_group;
  return launch_attention<2, 0, 2, false>(m, p, n_tiles, st);
}

}  // namespace vmla
