// Dense per-head attention of the comparison layer (d_h = d_v = 128 per head, the block-causal window
// of the VideoMLA technical summary's Problem definition, keys and values stored per head as in its
// Method item 4 baseline) on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// At 512 flops per (query, key, head) the tensor cores finish a 128 x 128 tile of scores in ~1024
// cycles, less than the softmax of the tile takes.  So the keys of every tile are split between two
// softmax warpgroups, each with its own running max, row sum and O accumulator (split-KV inside the CTA,
// no per-tile exchange between the warpgroups); the two partial results are merged once, at the end.
// The exponentials of a tile still share each sub-partition's MUFU and FMA pipes (~1000 of the ~1330
// cycles a half takes, measured), and the tile period is the chain S_j -> softmax -> P_j V_j ->
// S_{j+2} spread over the two S buffers; releasing P in 32-key parts shortens its tail.
//
// One CTA owns one tile of 128 query rows of one (batch, head) and streams every visible KV tile:
//   warp 8      TMA producer: the Q tile once, then K and V tiles of 128 keys into a 3-deep ring;
//   warp 9      TMEM owner and MMA issuer: S_j = Q K_j^T (Q and K from shared memory) into one of two
//               TMEM S buffers, then for each key half w: O_w += P_{j-1,w} V_{j-1,w} (P read from TMEM,
//               where it overwrote the half's own scores as bf16);
//   warps 0-3   keys 0-63 of every tile, warps 4-7 keys 64-127; one thread per query row (= TMEM lane,
//               warps w and w + 4 share the lanes): masked running max with a lazy rescale of O_w (only
//               when the max grows by more than 2^8), exp2 (3/8 by an FMA-pipe polynomial), row
//               sum, P released to the MMA warp in two parts of 32 keys.  Finally the halves swap
//               (max, sum) through shared memory and each warpgroup writes 64 of the 128 output
//               columns of o = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / l, warps 0-3 also the log-sum-exp.
// TMEM: S buffers at columns [0, 128) and [128, 256), O_0 at [256, 384), O_1 at [384, 512).
// Every mbarrier wait is bounded; a wait that runs out records its code (21-27) in the status word and
// every role winds down (copies in flight land, MMAs drain, TMEM is freed).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "tc_kernels.cuh"

namespace vmla {
namespace {

using namespace sm100;

constexpr int kThreads = 320;                 // 10 warps
constexpr int kBlockM = 128;                  // query rows per CTA
constexpr int kHead = 128;                    // d_h = d_v
constexpr int kBN = 128;                      // keys per KV tile
constexpr int kHalf = kBN / 2;                // keys per softmax warpgroup
constexpr int kBox = kBN * 128;               // [128 rows x 64 columns] bf16, 128-byte swizzle
constexpr int kQBytes = 2 * kBlockM * 128;    // Q tile: two 64-column boxes
constexpr int kStageBytes = 4 * kBox;         // K boxes | V boxes
constexpr int kStages = 3;
constexpr int kAuxBytes = 512;                // barriers
constexpr int kSmemBytes = kQBytes + kStages * kStageBytes + kAuxBytes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 2 * kBN;          // O_w at kTmemO + w * kHead
constexpr float kRescaleThreshold = 8.0f;     // log2 units
// Of the 8 score pairs in each 16-key chunk, this many take 2^x from the FMA-pipe polynomial (with two
// softmax warps per SM sub-partition, 3 measured best of 2-4).
#ifndef VMLA_DENSE_EXP2_POLY_PAIRS
#define VMLA_DENSE_EXP2_POLY_PAIRS 3
#endif
constexpr int kPolyPairs = VMLA_DENSE_EXP2_POLY_PAIRS;
// Each key half releases its P to the P V MMAs in this many parts.
#ifndef VMLA_DENSE_P_PARTS
#define VMLA_DENSE_P_PARTS 2
#endif
constexpr int kPParts = VMLA_DENSE_P_PARTS;
constexpr int kStepsPerPart = kHalf / 16 / kPParts;   // 16-key MMA steps per released part
static_assert((kHalf / 16) % kPParts == 0, "P parts");
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kTmemO + 2 * kHead <= kTmemCols, "TMEM budget");

struct DenseParams {
  int rows_per_b;        // query tokens per batch element (Nq)
  int tiles_per_group;   // query tiles per (batch, head)
  int heads;
  int64_t nq;
  FrameGeom g;
  float scale_log2;      // softmax_scale * log2(e)
  void* out;             // [B, Nq, H, 128] bf16
  float* lse;            // [B, Nq, H] or null
  int* status;
  uint64_t limit_ns;
  int drop_kv_tile;      // test hook: this KV tile is never loaded (-1: none)
  Span out_span, lse_span;
};

__global__ void __launch_bounds__(kThreads, 1)
dense_attention_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v, const DenseParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + kStages * kStageBytes);
  uint64_t* bar_q = bars;                    // Q tile landed
  uint64_t* kv_full = bars + 1;              // [kStages]
  uint64_t* kv_empty = kv_full + kStages;    // [kStages]
  uint64_t* s_full = kv_empty + kStages;     // [2 S buffers]
  uint64_t* p_ready = s_full + 2;            // [2 S buffers][2 key halves][kPParts], 128 arrivals each
  uint64_t* pv_done = p_ready + 4 * kPParts; // [2 S buffers][2 key halves]: that half's P V completed
  uint64_t* drain = pv_done + 4;             // every MMA of the CTA completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int tile = blockIdx.x;
  const int group = tile / p.tiles_per_group;
  const int row0 = (tile % p.tiles_per_group) * kBlockM;
  const int b = group / p.heads;
  const int h = group % p.heads;
  const int last_row = min(row0 + kBlockM, p.rows_per_b) - 1;
  const int64_t kend_first = key_end_rows(p.g, row0);
  const int64_t kend_last = key_end_rows(p.g, last_row);
  const int n_kv = (int)((kend_last + kBN - 1) / kBN);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(kv_full + s, 1); mbar_init(kv_empty + s, 1); }
    for (int s = 0; s < 2; ++s) mbar_init(s_full + s, 1);
    for (int i = 0; i < 4 * kPParts; ++i) mbar_init(p_ready + i, 128);
    for (int i = 0; i < 4; ++i) mbar_init(pv_done + i, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int zero_flag = 0;

  if (warp == 8) {
    // ================= TMA producer =================
    if (elect_one()) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      mbar_arrive_expect_tx(bar_q, kQBytes);
      for (int i = 0; i < 2; ++i) tma_load_4d(sQ + i * kBlockM * 128, &map_q, bar_q, 64 * i, h, row0, b);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % kStages;
        // stage st is free once the P V MMAs of load j - kStages have completed
        if (j >= kStages && !mbar_wait(kv_empty + st, ((j / kStages) - 1) & 1, abort_flag, p.status, 21, p.limit_ns))
          break;
        issued = j + 1;
        if (j == p.drop_kv_tile) continue;
        uint8_t* stage = sKV + st * kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, kStageBytes);
        const int krow = j * kBN;
        for (int i = 0; i < 2; ++i) tma_load_4d(stage + i * kBox, &map_k, kv_full + st, 64 * i, h, krow, b);
        for (int i = 0; i < 2; ++i) tma_load_4d(stage + (2 + i) * kBox, &map_v, kv_full + st, 64 * i, h, krow, b);
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        mbar_wait(bar_q, 0, &zero_flag, nullptr, 0, p.limit_ns);
        for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
          if (j != p.drop_kv_tile) mbar_wait(kv_full + j % kStages, (j / kStages) & 1, &zero_flag, nullptr, 0, p.limit_ns);
      }
    }
  } else if (warp == 9) {
    // ================= MMA issuer =================
    if (elect_one()) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, kHead, 0, 1);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t kv_base = smem_u32(sKV);
      bool ok = mbar_wait(bar_q, 0, abort_flag, p.status, 22, p.limit_ns);
      // O_w += P_{jp,w} V_{jp,w} for both key halves, each as soon as its warpgroup released its P
      auto issue_pv = [&](int jp) -> bool {
        const int bp = jp & 1;
        const uint32_t v_base = kv_base + (jp % kStages) * kStageBytes + 2 * kBox;
        for (int w = 0; w < 2; ++w) {
#pragma unroll
          for (int k = 0; k < kHalf / 16; ++k) {
            if (k % kStepsPerPart == 0) {
              if (!mbar_wait(p_ready + (2 * bp + w) * kPParts + k / kStepsPerPart, (jp >> 1) & 1, abort_flag,
                             p.status, 23, p.limit_ns))
                return false;
              tc_fence_after();
            }
            // V tile [128 keys][128 columns] as MN-major operand: 8-key groups 1024 B apart (SBO), the two
            // 64-column boxes kBox apart (LBO); 16 keys are 2048 B.  P of keys 64w + 16k .. + 15 sits in
            // the 8 columns at 64w + 8k of the S buffer.
            const int ks = w * (kHalf / 16) + k;
            const uint64_t vdesc = smem_desc(v_base + ks * 2048, kBox, 1024, kSwizzle128B);
            mma_ts(tmem + kTmemO + w * kHead, tmem + bp * kBN + w * kHalf + k * 8, vdesc, idesc_pv,
                   (jp > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(pv_done + 2 * bp + w);
        }
        mma_commit(kv_empty + (jp % kStages));
        return true;
      };
      if (ok) tc_fence_after();
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j % kStages, bj = j & 1;
        if (!mbar_wait(kv_full + st, (j / kStages) & 1, abort_flag, p.status, 24, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        // S buffer bj last held P_{j-2}, whose P V MMAs were issued before this point (in order)
        const uint32_t k_base = kv_base + st * kStageBytes;
#pragma unroll
        for (int k = 0; k < kHead / 16; ++k) {
          // 16 columns of d_h: box k/4, 32-byte step k%4 inside the 128-byte swizzle atom
          const uint64_t qdesc = smem_desc(q_base + (k >> 2) * kBlockM * 128 + (k & 3) * 32, 16, 1024, kSwizzle128B);
          const uint64_t kdesc = smem_desc(k_base + (k >> 2) * kBox + (k & 3) * 32, 16, 1024, kSwizzle128B);
          mma_ss(tmem + bj * kBN, qdesc, kdesc, idesc_qk, k > 0 ? 1u : 0u);
        }
        mma_commit(s_full + bj);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(n_kv - 1);
      mma_commit(drain);
      mbar_wait(drain, 0, &zero_flag, nullptr, 0, p.limit_ns);
    }
  } else {
    // ====== softmax of one key half (warps 0-3: keys 0-63, warps 4-7: keys 64-127), epilogue ======
    const int wg = warp >> 2;
    const int r = threadIdx.x & 127;                 // query row in the tile = TMEM lane
    const int row = row0 + r;
    const bool row_valid = row < p.rows_per_b;
    const int64_t kend = row_valid ? key_end_rows(p.g, row) : kend_last;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int64_t orow = ((int64_t)b * p.nq + row) * p.heads + h;
    const uint32_t o_own = tmem + lane_base + kTmemO + wg * kHead;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    // P_{k,wg} V_{k,wg} completed: phase k/2 of pv_done[k % 2][wg].  Called from tile k + 1, when that
    // barrier is at most one phase away (S_{k+1} complete implies P_{k-1} V_{k-1} complete; P_{k+2} does
    // not exist yet).
    auto wait_pv = [&](int k) -> bool {
      const bool got = mbar_wait(pv_done + 2 * (k & 1) + wg, (k >> 1) & 1, abort_flag, p.status, 25, p.limit_ns);
      return __all_sync(0xffffffffu, got);
    };
    const float sc = p.scale_log2;
    for (int j = 0; ok && j < n_kv; ++j) {
      const int bj = j & 1;
      const bool got = mbar_wait(s_full + bj, (j >> 1) & 1, abort_flag, p.status, 26, p.limit_ns);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + bj * kBN + wg * kHalf;
      float sr[kHalf];
      tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_ld_wait();
      const int64_t key0 = (int64_t)j * kBN + wg * kHalf;
      if (key0 + kHalf > kend_first) {
#pragma unroll
        for (int i = 0; i < kHalf; ++i)
          if (key0 + i >= kend) sr[i] = -INFINITY;
      }
      // max of the half row: 8 chains of 3-input max, then a tree (the scale is positive, applied after)
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = fmaxf(sr[q], sr[8 + q]);
#pragma unroll
      for (int i = 16; i < kHalf; i += 16)
#pragma unroll
        for (int q = 0; q < 8; ++q) mx[q] = fmax3(mx[q], sr[i + q], sr[i + 8 + q]);
      const float m_tile = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmaxf(fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_new = fmaxf(m_ref, m_tile * sc);
      const bool need = m_new > m_ref + kRescaleThreshold;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = fast_exp2(m_ref - m_new);   // 0 while this half has seen no visible key
        if (j > 0) {
          if (!wait_pv(j - 1)) { ok = false; break; }
          tc_fence_after();
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < kHead / 32; ++c) {
            tmem_ld32(o_own + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(o_own + c * 32, o);
          }
        }
        l_sum *= alpha;
        m_ref = m_new;
      }
      // p = 2^(s * scale*log2(e) - m): one packed FMA per pair, then MUFU.EX2 (or the polynomial); P as
      // bf16 pairs over the first 32 of this half's 64 S columns (already read).  A half that has seen
      // only masked keys keeps m = -inf and takes p = 2^(-inf) = 0 (2^-125 from the polynomial).
      const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
      float ls[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ls[i] = 0.f;
#pragma unroll
      for (int c = 0; c < kHalf / 16; ++c) {
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float x0, x1;
          ffma2(x0, x1, sr[c * 16 + 2 * i], sr[c * 16 + 2 * i + 1], sc, sc, neg_m, neg_m);
          float p0, p1;
          if (i < kPolyPairs) {
            exp2_poly2(p0, p1, x0, x1);
          } else {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          }
          fadd2(ls[(2 * i) & 7], ls[(2 * i + 1) & 7], p0, p1);
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st8(s_addr + c * 8, pk);
        if ((c + 1) % kStepsPerPart == 0 && c + 1 < kHalf / 16) {   // a part of the half: release it
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(p_ready + (2 * bj + wg) * kPParts + c / kStepsPerPart);
        }
      }
      fadd2(ls[0], ls[1], ls[4], ls[5]);
      fadd2(ls[2], ls[3], ls[6], ls[7]);
      fadd2(ls[0], ls[1], ls[2], ls[3]);
      l_sum += ls[0] + ls[1];
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_ready + (2 * bj + wg) * kPParts + kPParts - 1);
    }
    bool fin = ok && mbar_wait(drain, 0, abort_flag, p.status, 27, p.limit_ns);
    fin = __all_sync(0xffffffffu, fin && !*abort_flag);
    // (max, sum) of both halves through the Q buffer (every S = Q K^T MMA has completed).  Every softmax
    // thread passes the barrier once; a run that did not finish cleanly has raised the abort flag
    // before it, so both halves agree on whether to write.
    float* xch = reinterpret_cast<float*>(sQ);       // [2 halves][max, sum][128 rows]
    if (fin) {
      xch[wg * 256 + r] = m_ref;
      xch[wg * 256 + 128 + r] = l_sum;
    }
    named_bar_sync(1, 256);
    fin = fin && !*abort_flag;
    if (fin) {
      tc_fence_after();
      const float m_oth = xch[(wg ^ 1) * 256 + r];
      const float l_oth = xch[(wg ^ 1) * 256 + 128 + r];
      const float m = fmaxf(m_ref, m_oth);            // finite: key 0 is visible to every row
      const float a_own = fast_exp2(m_ref - m), a_oth = fast_exp2(m_oth - m);
      const float l_row = l_sum * a_own + l_oth * a_oth;
      const float inv_l = 1.f / l_row;
      const float f_own = a_own * inv_l, f_oth = a_oth * inv_l;
      const uint32_t o_oth = tmem + lane_base + kTmemO + (wg ^ 1) * kHead;
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
      uint32_t oa[32], ob[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int col = wg * 64 + c * 32;             // this warpgroup's 64 output columns
        tmem_ld32(o_own + col, oa);
        tmem_ld32(o_oth + col, ob);
        tmem_ld_wait();
        if (row_valid && store_ok(p.out_span, out + orow * kHead + col, 64, p.status, 10)) {
          uint4* dst = reinterpret_cast<uint4*>(out + orow * kHead + col);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v[8];
#pragma unroll
            for (int t = 0; t < 8; ++t)
              v[t] = fmaf(__uint_as_float(oa[8 * q + t]), f_own, __uint_as_float(ob[8 * q + t]) * f_oth);
            uint4 u;
            u.x = pack_bf16x2(v[0], v[1]);
            u.y = pack_bf16x2(v[2], v[3]);
            u.z = pack_bf16x2(v[4], v[5]);
            u.w = pack_bf16x2(v[6], v[7]);
            dst[q] = u;
          }
        }
      }
      if (wg == 0 && row_valid && p.lse && store_ok(p.lse_span, p.lse + orow, 4, p.status, 11))
        p.lse[orow] = (m + __log2f(l_row)) * 0.69314718055994530942f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

vmla_status tc_check_dense_mha(const vmla_config& c) {
  const int d_h = c.d_nope + c.d_rope;
  if (d_h != kHead || c.d_v != kHead) {
    set_tc_reason("tensor-core dense attention needs d_h == d_v == 128");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
}

cudaError_t tc_dense_mha(const vmla_config& cfg, int batch, int64_t nq, const void* q, const void* k,
                         const void* v, int64_t cap, int64_t valid_rows, const FrameGeom& g,
                         float scale, void* out, float* lse, int* status, cudaStream_t st) {
  const int H = cfg.n_heads;
  constexpr int D = kHead;
  CUtensorMap map_q, map_k, map_v;
  cudaError_t e;
  // q [B, Nq, H, 128], k / v [B, cap, H, 128] as {128, H, rows, B}: a 128-row box of one head
  if ((e = make_map_4d(&map_q, q, D, H, nq, batch, D * 2, (int64_t)H * D * 2, nq * H * D * 2, 64, 1, kBlockM,
                       128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&map_k, k, D, H, valid_rows, batch, D * 2, (int64_t)H * D * 2, cap * H * D * 2, 64, 1,
                       kBN, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&map_v, v, D, H, valid_rows, batch, D * 2, (int64_t)H * D * 2, cap * H * D * 2, 64, 1,
                       kBN, 128)) != cudaSuccess) return e;
  DenseParams p{};
  p.rows_per_b = (int)nq;
  p.tiles_per_group = (int)((nq + kBlockM - 1) / kBlockM);
  p.heads = H;
  p.nq = nq;
  p.g = g;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.limit_ns = wait_limit_ns();
  p.drop_kv_tile = take_drop_kv_tile();
  p.out_span = make_span(out, checked_extent((int64_t)batch * nq * H * D * 2));
  p.lse_span = make_span(lse, checked_extent((int64_t)batch * nq * H * 4));
  const int n_tiles = batch * H * p.tiles_per_group;
  static std::atomic<uint64_t> done{0};
  if ((e = ensure_smem_attr((const void*)dense_attention_kernel, kSmemBytes, done)) != cudaSuccess) return e;
  dense_attention_kernel<<<n_tiles, kThreads, kSmemBytes, st>>>(map_q, map_k, map_v, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace vmla
