// Projection GEMMs of the VideoMLA path on the sm_100a tensor cores (tcgen05 + TMEM + TMA), each
// with its own fused epilogue:
//   compress_append  [c ; W^KR x] = [W^KV_down ; W^KR] x, 3D-RoPE on the last d_rope columns, bf16
//                    store into the ring rows of the chunk's frames (Method items 1 and 3); also a
//                    token range of the chunk into several replicas of the ring (peer mappings), and
//                    the column tile narrows to 128 / 64 when the row tiles alone leave SMs idle;
//   absorb_q         q~_h = (W^K_up,h)^T q^nope_h per head (B operand read MN-major from W^K_up as
//                    stored), plus RoPE3D(q^rope_h) written beside it (Method items 2 and 3);
//   value_up         o_h = W^V_up,h o~_h per head (Method item 2);
//   dense_append     the dense comparison layer's per-head K and V projection (RoPE on each head's
//                    last d_rope key columns) into the dense ring.
// Persistent kernels: one CTA per SM loops over 128-row x BN output tiles.  Warp 0 streams A/B
// k-tiles with TMA into a shared-memory ring, warp 1 owns TMEM and issues tcgen05.mma (K = 16 per
// instruction, fp32 accumulation) into one of two TMEM accumulators, and warps 2-5 read the other
// accumulator back (one thread per row) and run the epilogue, so a tile's epilogue overlaps the next
// tile's loads and MMAs.  The epilogue warps also build the CTA's 3D-RoPE cos/sin table while the
// first loads and MMAs run.  In checked builds every epilogue store is tested against its buffer.
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
  int a_head;         // whether A's map has a head coordinate (per-head A rows)
  uint64_t limit_ns;
  int* status;
  int heads;          // independent GEMMs (heads) sharing the shapes; set by the launcher
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
RopeLookup make_rope_lookup(const RopeTable& rt, const FrameGeom& g, int frames) {
  RopeLookup L{};
  L.rt = rt;
  L.base_f = g.first_frame;
  const int extent[3] = {frames, g.tokens_per_frame / g.grid_w, g.grid_w};
  int total = 0;
  for (int p = 0; p < rt.n_pairs; ++p) {
    L.off[p] = total;
    total += extent[rt.axis[p]];
  }
  L.n_entries = total <= kRopeTabEntries ? total : 0;
  return L;
}

// ---- epilogues: called per (row m, 32-column chunk starting at col0) with the fp32 values ----
// Row m of the GEMM is token tok0 + m % ntok of batch element m / ntok; its c and k^R rows go to the
// ring of every destination cache (several when replicas of the cache live on other GPUs: plain stores
// through peer mappings, so the exchange of the chunk's latents is done by this epilogue).
struct EpiCompress {
  static constexpr bool kRope = true;
  bf16* c[kMaxCacheDst]; bf16* k_r[kMaxCacheDst]; int n_dst;
  int d_c, d_rope; int64_t ntok, tok0, cap; FrameGeom g; RopeLookup rope;
  Span c_span[kMaxCacheDst], kr_span[kMaxCacheDst]; int* status;
  __device__ void operator()(const float2* tab, int, int64_t m, int col0, float* v) const {
    const int64_t b = m / ntok, tok = tok0 + m % ntok;
    const int64_t row = b * cap + ring_row(g, tok);
    if (col0 < d_c) {
      for (int d = 0; d < n_dst; ++d) {
        bf16* q = c[d] + row * d_c + col0;
        if (store_ok(c_span[d], q, 64, status, 1)) store32(q, v);
      }
    } else {
      const int64_t f = g.first_frame + tok / g.tokens_per_frame;
      const int64_t r = tok % g.tokens_per_frame;
      rope.rotate32(tab, (col0 - d_c) / 2, f, r / g.grid_w, r % g.grid_w, v);
      for (int d = 0; d < n_dst; ++d) {
        bf16* q = k_r[d] + row * d_rope + (col0 - d_c);
        if (store_ok(kr_span[d], q, 64, status, 2)) store32(q, v);
      }
    }
    // stores to other GPUs' memory: make them visible system-wide before this thread goes on
    if (n_dst > 1) __threadfence_system();
  }
  __device__ void finish(const float2*, int, int64_t) const {}
};

struct EpiAbsorb {
  static constexpr bool kRope = true;
  bf16* q_abs; const bf16* q_rope; int heads, d_c, d_rope; int64_t nq; FrameGeom g; RopeLookup rope;
  Span span; int* status;
  __device__ void operator()(const float2* tab, int h, int64_t m, int col0, float* v) const {
    bf16* q = q_abs + (m * heads + h) * (d_c + d_rope) + col0;
    if (store_ok(span, q, 64, status, 3)) store32(q, v);
  }
  // RoPE3D(q^rope) of row m, head h -> q_abs[m, h, d_c : d_c + d_rope]
  __device__ void finish(const float2* tab, int h, int64_t m) const {
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
      rope.rotate32(tab, c0 / 2, f, r / g.grid_w, r % g.grid_w, v);
      bf16* q = q_abs + (m * heads + h) * (d_c + d_rope) + d_c + c0;
      if (store_ok(span, q, 64, status, 3)) store32(q, v);
    }
  }
};

struct EpiValueUp {
  static constexpr bool kRope = false;
  RopeLookup rope;   // unused
  bf16* out; int heads, d_v;
  Span span; int* status;
  __device__ void operator()(const float2* tab, int h, int64_t m, int col0, float* v) const {
    bf16* q = out + (m * heads + h) * d_v + col0;
    if (store_ok(span, q, 64, status, 4)) store32(q, v);
  }
  __device__ void finish(const float2*, int, int64_t) const {}
};

struct EpiDense {
  static constexpr bool kRope = true;
  bf16* k; bf16* v; int heads, d_nope, d_h, d_v; int64_t ntok, cap; FrameGeom g; RopeLookup rope;
  Span k_span, v_span; int* status;
  __device__ void operator()(const float2* tab, int, int64_t m, int col0, float* x) const {
    const int64_t b = m / ntok, tok = m % ntok;
    const int64_t row = b * cap + ring_row(g, tok);
    if (col0 < heads * d_h) {
      const int hh = col0 / d_h, cc = col0 % d_h;
      if (cc >= d_nope) {
        const int64_t f = g.first_frame + tok / g.tokens_per_frame;
        const int64_t r = tok % g.tokens_per_frame;
        rope.rotate32(tab, (cc - d_nope) / 2, f, r / g.grid_w, r % g.grid_w, x);
      }
      bf16* q = k + (row * heads + hh) * d_h + cc;
      if (store_ok(k_span, q, 64, status, 5)) store32(q, x);
    } else {
      const int cv = col0 - heads * d_h;
      bf16* q = v + (row * heads + cv / d_v) * d_v + cv % d_v;
      if (store_ok(v_span, q, 64, status, 6)) store32(q, x);
    }
  }
  __device__ void finish(const float2*, int, int64_t) const {}
};

template <int BN, bool B_MN_MAJOR, bool PAIR>
struct GemmPlan {
  // PAIR: a CTA pair shares one M = 256 MMA per k-step; each CTA loads its 128 rows of A and half of
  // the BN columns of B, so the weight crosses L2 -> SM once per 256 rows instead of once per 128
  static constexpr int kBRows = PAIR ? BN / 2 : BN;
  static constexpr int kBBytes = kBRows * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTileRows = PAIR ? 2 * kBM : kBM;
  static constexpr int kTabBytes = kRopeTabEntries * 8;   // RoPE table (epilogues that rotate)
  static constexpr int kFit = (232448 - 1024 - 256 - kTabBytes) / kStageBytes;
  static constexpr int kStages = kFit >= 6 ? 6 : kFit;
  static constexpr int kSmemBytes = kStages * kStageBytes + 256 + kTabBytes + 1024;
  // one fp32 accumulator of BN columns, double-buffered in TMEM
  static constexpr uint32_t kAccCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static constexpr uint32_t kTmemCols = 2 * kAccCols;
  static_assert(BN % 32 == 0 && BN <= 256, "BN");
  static_assert(!B_MN_MAJOR || BN % 64 == 0, "MN-major B is loaded in 64-column boxes");
  static_assert(!PAIR || (!B_MN_MAJOR && BN % 32 == 0), "paired MMA: K-major B, N/2 a multiple of 16");
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned for the 128-byte swizzle");
  static_assert(kStages >= 2, "shared memory too small for two stages");
};

// Persistent tile loop: tile t -> (head z, column tile nt, row tile mt) with mt fastest (consecutive
// CTAs share the weight tile); CTA c takes tiles c, c + grid, c + 2*grid, ...
struct TileCoord { int mt, nt, z; };
__device__ __forceinline__ TileCoord tile_coord(int t, int n_m, int n_n) {
  TileCoord c;
  c.z = t / (n_m * n_n);
  const int rem = t - c.z * n_m * n_n;
  c.nt = rem / n_m;
  c.mt = rem - c.nt * n_m;
  return c;
}

// PAIR = true: launched in clusters of two CTAs.  Both CTAs walk the same 256-row tiles; CTA rank r
// loads rows r * 128 .. r * 128 + 127 of A and B columns r * BN/2 .. (r + 1) * BN/2 - 1, every copy of
// both completing on the first CTA's `full` barrier, and the first CTA issues tcgen05.mma.cta_group::2
// (M = 256), whose commits arrive on the barriers of both CTAs.  Each CTA's epilogue reads its own
// 128 x BN accumulator and releases it on the first CTA's `acc_empty` (one arrival per warp).
template <int BN, bool B_MN_MAJOR, bool PAIR, class Epi>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
            const GemmShape sh, const Epi epi) {
  using PL = GemmPlan<BN, B_MN_MAJOR, PAIR>;
  constexpr int kStages = PL::kStages;
  constexpr uint16_t kBoth = 3;           // cta mask of a pair's commits
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * PL::kStageBytes);
  uint64_t* full = bars;                  // kStages
  uint64_t* empty = full + kStages;       // kStages
  uint64_t* acc_full = empty + kStages;   // 2: accumulator buffer ready for the epilogue
  uint64_t* acc_empty = acc_full + 2;     // 2: accumulator buffer read back by the epilogue
  uint64_t* drain = acc_empty + 2;        // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float2* rope_tab = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(bars) + 256);

  const int warp = threadIdx.x / 32;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int nk = (sh.K + kBK - 1) / kBK;
  const int n_m = (int)((sh.M + PL::kTileRows - 1) / PL::kTileRows);
  const int n_n = (sh.N + BN - 1) / BN;
  const int n_tiles = n_m * n_n * sh.heads;
  int zero_flag = 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(acc_full + s, 1); mbar_init(acc_empty + s, PAIR ? 8 : 128); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, PL::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, PL::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers are initialised and their TMEM allocated before either CTA touches the other's
  if constexpr (PAIR) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producer (k-iterations counted across tiles) =================
    if (elect_one()) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      int it = 0;
      bool ok = true;
      for (int t = unit; ok && t < n_tiles; t += n_units) {
        const TileCoord tc = tile_coord(t, n_m, n_n);
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int st = it % kStages;
          if (it >= kStages &&
              !mbar_wait(empty + st, ((it / kStages) - 1) & 1, abort_flag, sh.status, 11, sh.limit_ns)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * PL::kStageBytes;
          uint8_t* sb = sa + kABytes;
          if constexpr (PAIR) {
            // the first CTA expects both CTAs' bytes; the peer's copies may land before that arrival
            if (leader) mbar_arrive_expect_tx(full + st, 2 * PL::kStageBytes);
            const uint32_t fb = cluster_addr(smem_u32(full + st), 0);
            tma_load_4d_pair(sa, &map_a, fb, kt * kBK, sh.a_head ? tc.z : 0,
                             tc.mt * PL::kTileRows + (int)rank * kBM, 0);
            tma_load_4d_pair(sb, &map_b, fb, kt * kBK, tc.nt * BN + (int)rank * PL::kBRows, tc.z, 0);
          } else {
            mbar_arrive_expect_tx(full + st, PL::kStageBytes);
            tma_load_4d(sa, &map_a, full + st, kt * kBK, sh.a_head ? tc.z : 0, tc.mt * kBM, 0);
            if (B_MN_MAJOR) {
#pragma unroll
              for (int i = 0; i < BN / 64; ++i)
                tma_load_4d(sb + i * (kBK * 128), &map_b, full + st, tc.nt * BN + 64 * i, kt * kBK, tc.z, 0);
            } else {
              tma_load_4d(sb, &map_b, full + st, kt * kBK, tc.nt * BN, tc.z, 0);
            }
          }
        }
      }
      if (!ok && (!PAIR || leader)) {
        // let the copies already issued land before the CTA exits (a pair's copies all complete on
        // the first CTA's barriers; the peer is held by the closing cluster barrier until then)
        for (int j = (it > kStages ? it - kStages : 0); j < it; ++j)
          mbar_wait(full + j % kStages, (j / kStages) & 1, &zero_flag, nullptr, 0, sh.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (the pair's first CTA issues for both) =================
    if ((!PAIR || leader) && elect_one()) {
      constexpr uint32_t idesc = idesc_bf16_f32(PAIR ? 2 * kBM : kBM, BN, 0, B_MN_MAJOR ? 1 : 0);
      int it = 0, li = 0;
      bool ok = true;
      for (int t = unit; ok && t < n_tiles; t += n_units, ++li) {
        const int ab = li & 1;
        if (li >= 2 && !mbar_wait(acc_empty + ab, ((li >> 1) - 1) & 1, abort_flag, sh.status, 14, sh.limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + ab * PL::kAccCols;
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(full + st, (it / kStages) & 1, abort_flag, sh.status, 12, sh.limit_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + st * PL::kStageBytes);
          const uint32_t b = a + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc(a + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = B_MN_MAJOR ? smem_desc(b + kk * 2048, kBK * 128, 1024, kSwizzle128B)
                                           : smem_desc(b + kk * 32, 16, 1024, kSwizzle128B);
            if constexpr (PAIR)
              mma_ss_pair(acc, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
            else
              mma_ss(acc, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
          }
          if constexpr (PAIR) mma_commit_pair(empty + st, kBoth);
          else mma_commit(empty + st);
        }
        if (ok) {
          if constexpr (PAIR) mma_commit_pair(acc_full + ab, kBoth);
          else mma_commit(acc_full + ab);
        }
      }
      // every MMA of this CTA (of both CTAs, for a pair) has completed before TMEM is released
      if constexpr (PAIR) mma_commit_pair(drain, kBoth);
      else mma_commit(drain);
      mbar_wait(drain, 0, &zero_flag, nullptr, 0, sh.limit_ns);
    }
  } else {
    // ================= epilogue: warps 2..5, TMEM lane quadrant = warp % 4 =================
    // the RoPE table is built by these four warps while the producer and the MMA warp already run
    if constexpr (Epi::kRope) {
      epi.rope.build(rope_tab, threadIdx.x - 64, 128);
      named_bar_sync(1, 128);
    }
    const int quad = warp & 3;
    const int r = quad * 32 + (threadIdx.x & 31);
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    int li = 0;
    for (int t = unit; t < n_tiles; t += n_units, ++li) {
      const TileCoord tc = tile_coord(t, n_m, n_n);
      const int ab = li & 1;
      const bool got = mbar_wait(acc_full + ab, (li >> 1) & 1, abort_flag, sh.status, 13, sh.limit_ns);
      if (!__all_sync(0xffffffffu, got)) break;      // the TMEM loads below are warp-collective
      tc_fence_after();
      const int64_t m = (int64_t)tc.mt * PL::kTileRows + (int)rank * kBM + r;
      const int n0 = tc.nt * BN;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_base + ab * PL::kAccCols + c0, raw);
        tmem_ld_wait();
        if (m < sh.M && n0 + c0 < sh.N) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
          epi(rope_tab, tc.z, m, n0 + c0, v);
        }
      }
      tc_fence_before();
      if constexpr (PAIR) {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) {
          if (leader) mbar_arrive(acc_empty + ab);
          else mbar_arrive_cluster(cluster_addr(smem_u32(acc_empty + ab), 0));
        }
      } else {
        mbar_arrive(acc_empty + ab);
      }
      if (m < sh.M && tc.nt == 0) epi.finish(rope_tab, tc.z, m);
    }
  }
  tc_fence_before();
  __syncthreads();
  // a pair: the first CTA's MMAs (which read the peer's shared memory and write its TMEM) have drained
  // and every remote arrival has been made before either CTA frees TMEM or exits
  if constexpr (PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem, PL::kTmemCols);
    else tmem_dealloc(tmem, PL::kTmemCols);
  }
}

int num_sms() {
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

// One CTA per SM (TMEM holds two accumulators), each looping over its share of the tiles; PAIR: one
// cluster of two CTAs per two SMs, each pair looping over 256-row tiles.
template <int BN, bool B_MN_MAJOR, bool PAIR = false, class Epi>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmShape& sh, int heads,
                        const Epi& epi, cudaStream_t st) {
  using PL = GemmPlan<BN, B_MN_MAJOR, PAIR>;
  auto kern = gemm_kernel<BN, B_MN_MAJOR, PAIR, Epi>;
  static std::atomic<uint64_t> done{0};
  cudaError_t attr_err = ensure_smem_attr((const void*)kern, PL::kSmemBytes, done);
  if (attr_err != cudaSuccess) return attr_err;
  GemmShape s2 = sh;
  s2.heads = heads;
  const int64_t tiles = ((sh.M + PL::kTileRows - 1) / PL::kTileRows) * ((sh.N + BN - 1) / BN) * heads;
  if constexpr (PAIR) {
    const int pairs = (int)(tiles < num_sms() / 2 ? tiles : num_sms() / 2);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = PL::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, b, s2, epi);
    count_launches(1);
    return e != cudaSuccess ? e : cudaGetLastError();
  } else {
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    kern<<<grid, kThreads, PL::kSmemBytes, st>>>(a, b, s2, epi);
    count_launches(1);
    return cudaGetLastError();
  }
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

// Paired-CTA instances (K-major B, all N columns in one tile): N = d_c + d_rope of the compress GEMM.
template <class Epi>
static cudaError_t dispatch_pair(int bn, const CUtensorMap& a, const CUtensorMap& b, const GemmShape& sh,
                                 int heads, const Epi& epi, cudaStream_t st) {
  switch (bn) {
    case 96: return launch_gemm<96, false, true>(a, b, sh, heads, epi, st);
    case 128: return launch_gemm<128, false, true>(a, b, sh, heads, epi, st);
    case 160: return launch_gemm<160, false, true>(a, b, sh, heads, epi, st);
    case 192: return launch_gemm<192, false, true>(a, b, sh, heads, epi, st);
    case 224: return launch_gemm<224, false, true>(a, b, sh, heads, epi, st);
    case 256: return launch_gemm<256, false, true>(a, b, sh, heads, epi, st);
    default: break;
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
  CacheDst d{c, k_r};
  return tc_compress_rows(cfg, batch, 0, (int64_t)cfg.chunk_frames * cfg.grid_h * cfg.grid_w, x, w, g, rt,
                          &d, 1, st);
}

cudaError_t tc_compress_rows(const vmla_config& cfg, int batch, int64_t tok0, int64_t ntok, const void* x,
                             const void* w, const FrameGeom& g, const RopeTable& rt, const CacheDst* dst,
                             int n_dst, cudaStream_t st) {
  if (n_dst < 1 || n_dst > kMaxCacheDst) return cudaErrorInvalidValue;
  const int64_t M = batch * ntok;
  const int N = cfg.d_c + cfg.d_rope, K = cfg.dim;
  // one 224-wide column tile per 128 rows leaves most SMs idle at small batch: narrow the column tile
  // until the tiles cover the SMs (the x tile is then re-read from L2 by each column tile; the RoPE
  // columns d_c .. d_c+31 stay inside one 32-column chunk of one tile because d_c % 32 == 0)
  int bn = pick_bn(N);
  const int64_t m_tiles = (M + kBM - 1) / kBM;
  for (int cand : {128, 64})
    if (m_tiles * ((N + bn - 1) / bn) < num_sms() && cand < bn) bn = cand;
  // once 256-row tiles of all N columns occupy every SM, a CTA pair per tile: each CTA pulls x once and
  // only half of the weight, which every tile re-reads from L2 (measured on B200 at 4 x 4680 tokens:
  // 33.8 vs 35.8 us per launch after an attention launch; at 2 x 4680, with half the SMs idle, the
  // pairs were slower than 128-column tiles on every SM)
  const int64_t pair_tiles = (M + 2 * kBM - 1) / (2 * kBM);
  const bool pair = N <= 256 && N % 32 == 0 && 2 * pair_tiles >= num_sms();
  if (pair) bn = N;
  CUtensorMap ma, mb;
  cudaError_t e;
  // A = x [M, D]; B = [W^KV_down ; W^KR] [N, D], both K-major (a pair's CTAs load N/2 rows of B each)
  if ((e = make_map_4d(&ma, x, K, 1, M, 1, (int64_t)K * 2, (int64_t)K * 2, M * K * 2, kBK, 1, kBM, 128)) != cudaSuccess)
    return e;
  if ((e = make_map_4d(&mb, w, K, N, 1, 1, (int64_t)K * 2, (int64_t)N * K * 2, (int64_t)N * K * 2, kBK,
                       pair ? bn / 2 : bn, 1, 128)) != cudaSuccess)
    return e;
  GemmShape sh{M, N, K, 0, wait_limit_ns(), device_status_ptr()};
  EpiCompress epi{};
  const int64_t cap_rows = (int64_t)batch * cfg.window_frames * cfg.grid_h * cfg.grid_w;
  for (int d = 0; d < n_dst; ++d) {
    epi.c[d] = (bf16*)dst[d].c;
    epi.k_r[d] = (bf16*)dst[d].k_r;
    epi.c_span[d] = make_span(dst[d].c, checked_extent(cap_rows * cfg.d_c * 2));
    epi.kr_span[d] = make_span(dst[d].k_r, checked_extent(cap_rows * cfg.d_rope * 2));
  }
  epi.status = device_status_ptr();
  epi.n_dst = n_dst;
  epi.d_c = cfg.d_c;
  epi.d_rope = cfg.d_rope;
  epi.ntok = ntok;
  epi.tok0 = tok0;
  epi.cap = (int64_t)cfg.window_frames * cfg.grid_h * cfg.grid_w;
  epi.g = g;
  epi.rope = make_rope_lookup(rt, g, cfg.chunk_frames);
  return pair ? dispatch_pair(bn, ma, mb, sh, 1, epi, st) : dispatch_bn<false>(bn, ma, mb, sh, 1, epi, st);
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
  EpiAbsorb epi{(bf16*)q_abs, (const bf16*)q_rope, H, cfg.d_c, cfg.d_rope, nq, g,
                make_rope_lookup(rt, g, (int)(nq / ((int64_t)cfg.grid_h * cfg.grid_w)))};
  epi.span = make_span(q_abs, checked_extent(M * H * (cfg.d_c + cfg.d_rope) * 2));
  epi.status = device_status_ptr();
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
  EpiValueUp epi{RopeLookup{}, (bf16*)out, H, N};
  epi.span = make_span(out, checked_extent(M * H * N * 2));
  epi.status = device_status_ptr();
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
               (int64_t)cfg.window_frames * cfg.grid_h * cfg.grid_w, g, make_rope_lookup(rt, g, cfg.chunk_frames)};
  const int64_t dense_rows = (int64_t)batch * cfg.window_frames * cfg.grid_h * cfg.grid_w * cfg.n_heads;
  epi.k_span = make_span(k, checked_extent(dense_rows * d_h * 2));
  epi.v_span = make_span(v, checked_extent(dense_rows * cfg.d_v * 2));
  epi.status = device_status_ptr();
  return dispatch_bn<false>(bn, ma, mb, sh, 1, epi, st);
}

cudaError_t tc_rope_q(const vmla_config& cfg, int batch, int64_t nq, const void* q_nope,
                      const void* q_rope, const FrameGeom& g, const RopeTable& rt, void* q,
                      cudaStream_t st) {
  return simt_rope_q<bf16>(cfg, batch, nq, (const bf16*)q_nope, (const bf16*)q_rope, g, rt, (bf16*)q, st);
}

}  // namespace vmla
