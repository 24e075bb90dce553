// Compress + 3D-RoPE + ring append on the sm_100a tensor cores (VideoMLA technical summary, Method
// item 1: the shared content latent c^KV_t = W^KV_down x_t; item 3: the head-shared positional key
// k^R_t = RoPE3D(W^KR x_t); sliding window: abstract and Problem definition).
//
// [c ; W^KR x] = [W^KV_down ; W^KR] x is a GEMM with a small N (d_c + d_rope = 224 at the defaults) and
// a long reduction over the model width.  x streams from HBM and is read once per column tile; the
// weight (0.7 MB) is read again, from L2, by every row tile, and at these shapes those L2 reads, not
// HBM, bound the kernel: every SM streams its tiles through TMA at a limited rate, so the kernel is
// organised to put as few bytes as possible through each SM.
//   * A work unit is a 128-token row tile times a column tile: all N columns in one (one tcgen05.mma;
//     two of N/2 above 256), or 128-column tiles when the row tiles alone would leave most SMs idle.
//   * At small batch the reduction is further split across a cluster of two CTAs (split-K): each
//     streams half of the k-steps into its own shared memory and accumulates a partial tile in TMEM;
//     the two partials are summed through distributed shared memory, CTA r of the pair finishing rows
//     [64 r, 64 r + 64).  At 4680 tokens (37 row tiles) that is 37 x 2 column tiles x 2 = 148 CTAs.
//   * Otherwise (S = 1) the CTAs are persistent over the work units, with two TMEM accumulators so that
//     a unit's epilogue overlaps the next unit's loads and MMAs.
//   * x and the weight have separate TMA rings: x comes from HBM and needs a deep ring to have enough
//     bytes in flight; the weight is served by L2, and two or three k-steps of it keep up.
// Roles: warp 0 issues the TMA loads (lane 0 x, lane 1 the weight), warp 1 owns TMEM and issues the
// MMAs, warps 2-5 run the epilogue: rotate the k^R columns (per-CTA cos/sin table), round to bf16 and
// stage the rows in shared memory with each row's ring position, then write them out by whole warps,
// 16 bytes per lane, several rows in flight per warp (a row's c and k^R segments are each contiguous),
// to every destination replica of the cache (several when replicas live on other GPUs: plain stores
// through peer mappings).  Every wait is bounded; a wait that runs out makes the CTA wind down, and the
// cluster barriers are passed on every path, so no CTA of a pair waits for one that left.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "tc_kernels.cuh"
#include "tc_proj_common.cuh"

namespace vmla {
namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int kThreads = 192;
constexpr int kBM = 128;                      // tokens per row tile
constexpr int kBK = 64;                       // model-width columns per k-step (one 128-byte swizzle row)
constexpr int kMaxN = 288;                    // d_c + d_rope
constexpr int kNarrowBN = 128;                // column tile when the columns are split
constexpr int kABytes = kBM * kBK * 2;        // x box: 16 KB
constexpr int kTabEntries = 1024;             // RoPE cos/sin table entries (the Wan grid needs 428)
constexpr int kTabBytes = kTabEntries * 8;
constexpr int kAuxBytes = 256;                // barriers, TMEM address, flags
constexpr int kRowDstBytes = kBM * 8;         // ring row of every staged row
constexpr int kSmemBytes = 232448;            // all of it: the layout is carved at run time
constexpr int kMaxXStages = 8;
constexpr int kMaxWStages = 3;
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = 512;

struct CompressArgs {
  int M;                  // rows of the GEMM: batch * ntok tokens
  int K;                  // model width D
  int N;                  // d_c + d_rope (multiple of 32, <= kMaxN)
  int d_c;                // content columns; columns d_c .. N-1 are the rotated k^R
  int nt;                 // column tiles per row tile (1, or 2 of kNarrowBN columns)
  int bn;                 // columns per column tile (N, or kNarrowBN)
  int ntok, tok0;         // row m is token tok0 + m % ntok of batch element m / ntok
  int tokens_per_frame, grid_w, window_frames;
  int first_slot;         // first_frame mod window_frames
  int64_t first_frame;
  int64_t cap;            // ring rows per batch element (W * T_f)
  int xs, ws, w_bytes, row_stride;       // shared-memory layout: x ring depth, weight ring depth
  RopeLookup rope;
  bf16* c[kMaxCacheDst];
  bf16* k_r[kMaxCacheDst];
  Span c_span[kMaxCacheDst], kr_span[kMaxCacheDst];
  int n_dst;
  int* status;
  uint64_t limit_ns;
};

// Ring row (over all batch elements) and 3D position of GEMM row m; 32-bit arithmetic only.
struct RowPos {
  int64_t ring;
  int64_t f;
  int i, j;
};
__device__ __forceinline__ RowPos row_pos(const CompressArgs& a, int m) {
  const int b = m / a.ntok;
  const int tok = a.tok0 + (m - b * a.ntok);
  const int fi = tok / a.tokens_per_frame;                 // frame within the chunk
  const int r = tok - fi * a.tokens_per_frame;
  int slot = a.first_slot + fi;
  slot -= (slot / a.window_frames) * a.window_frames;
  RowPos p;
  p.ring = (int64_t)b * a.cap + (int64_t)slot * a.tokens_per_frame + r;
  p.f = a.first_frame + fi;
  p.i = r / a.grid_w;
  p.j = r - p.i * a.grid_w;
  return p;
}

// Write staged rows [0, nrows) of `sout` (columns n0 .. n1-1 of the output) to their ring rows
// (rowdst).  A row has (n1 - n0) / 8 16-byte chunks; with G lanes per row (the chunk count rounded up to
// a power of two, at most 32) a warp covers 32 / G rows per store instruction, and each warp loads four
// such row groups from shared memory before storing them, so that several stores are in flight.
__device__ __forceinline__ void store_rows(const CompressArgs& a, const uint8_t* sout, const int64_t* rowdst,
                                           int nrows, int n0, int n1, int epi_warp, int lane) {
  constexpr int U = 4;
  const int ch0 = n0 / 8, nch = (n1 - n0) / 8, nc = a.d_c / 8;
  int g = 1;
  while (g < nch && g < 32) g *= 2;
  const int rows_per_pass = 32 / g;                        // rows one store instruction covers
  const int sub = lane / g, cl = lane % g;                 // this lane's row within the pass, chunk
  const int step = rows_per_pass * U * (kEpiThreads / 32);
  for (int r0 = epi_warp * rows_per_pass * U; r0 < nrows; r0 += step) {
    int64_t row[U];
    int rr[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      rr[u] = r0 + u * rows_per_pass + sub;
      row[u] = rr[u] < nrows ? rowdst[rr[u]] : -1;
    }
    for (int c = cl; c < nch; c += g) {
      const int ch = ch0 + c;                              // absolute 16-byte chunk of the output row
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (row[u] >= 0) v[u] = *reinterpret_cast<const uint4*>(sout + rr[u] * a.row_stride + c * 16);
      const bool is_c = ch < nc;
      const int64_t stride = is_c ? a.d_c : 32;
      for (int d = 0; d < a.n_dst; ++d) {
        bf16* base = is_c ? a.c[d] + ch * 8 : a.k_r[d] + (ch - nc) * 8;
        const Span span = is_c ? a.c_span[d] : a.kr_span[d];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          if (row[u] < 0) continue;
          bf16* q = base + row[u] * stride;
          if (store_ok(span, q, 16, a.status, is_c ? 1 : 2)) *reinterpret_cast<uint4*>(q) = v[u];
        }
      }
    }
  }
  // stores to other GPUs' memory: make them visible system-wide before this thread goes on
  if (a.n_dst > 1) __threadfence_system();
}

template <int S>
__global__ void __launch_bounds__(kThreads, 1)
compress_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                const CompressArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring = smem;                                   // x k-step boxes (HBM: a deep ring)
  uint8_t* wring = xring + a.xs * kABytes;                 // weight k-step boxes (L2: a shallow ring)
  uint8_t* partials = smem;                                // after the MMAs: split-K partials (both rings)
  uint8_t* sout = wring + a.ws * a.w_bytes;                // staged bf16 output rows
  int64_t* rowdst = reinterpret_cast<int64_t*>(sout + kBM * a.row_stride);
  float2* tab = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(rowdst) + kRowDstBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(tab) + kTabBytes);
  uint64_t* x_full = bars;                  // kMaxXStages
  uint64_t* x_empty = x_full + kMaxXStages; // kMaxXStages
  uint64_t* w_full = x_empty + kMaxXStages; // kMaxWStages
  uint64_t* w_empty = w_full + kMaxWStages; // kMaxWStages
  uint64_t* acc_full = w_empty + kMaxWStages;   // 2
  uint64_t* acc_empty = acc_full + 2;      // 2 (kEpiThreads arrivals)
  uint64_t* drain = acc_empty + 2;         // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile uint32_t* ok_flags = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);   // [S]: partial ready

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int xs = a.xs, ws = a.ws;
  const int nk = (a.K + kBK - 1) / kBK;
  const int n_units = ((a.M + kBM - 1) / kBM) * a.nt;      // (row tile, column tile), column tile fastest
  const uint32_t rank = S > 1 ? cluster_ctarank() : 0;
  // S > 1: cluster blockIdx.x / S owns unit blockIdx.x / S and this CTA its k-steps [kb, ke);
  // S == 1: CTA c loops over units c, c + grid, ...
  const int kb = (int)(rank * nk / S), ke = (int)((rank + 1) * nk / S);
  const int u_first = S > 1 ? (int)(blockIdx.x / S) : (int)blockIdx.x;
  const int u_step = S > 1 ? n_units : (int)gridDim.x;
  const bool split_n = a.bn > 256;                         // two MMAs (and weight boxes) of bn/2
  const int n_acc = split_n ? 1 : 2;                       // TMEM accumulators
  int zero_flag = 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < xs; ++s) { mbar_init(x_full + s, 1); mbar_init(x_empty + s, 1); }
    for (int s = 0; s < ws; ++s) { mbar_init(w_full + s, 1); mbar_init(w_empty + s, 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(acc_full + s, 1); mbar_init(acc_empty + s, kEpiThreads); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (S > 1) cluster_sync_all();          // both CTAs of the pair run before any remote access
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producers: lane 0 the x ring, lane 1 the weight ring =================
    // (two threads, so that x loads, which wait on HBM, run as far ahead as the deep ring allows while
    // the weight, which L2 serves quickly, is only a few k-steps ahead)
    if (lane < 2) {
      const bool is_x = lane == 0;
      if (is_x) { tma_prefetch_desc(&map_x); } else { tma_prefetch_desc(&map_w); }
      const int depth = is_x ? xs : ws;
      uint64_t* fullb = is_x ? x_full : w_full;
      uint64_t* emptyb = is_x ? x_empty : w_empty;
      int it = 0;
      bool ok = true;
      for (int u = u_first; ok && u < n_units; u += u_step) {
        const int t = u / a.nt, n0 = (u % a.nt) * a.bn;
        for (int k = kb; k < ke; ++k, ++it) {
          const int st = it % depth;
          if (it >= depth &&
              !mbar_wait(emptyb + st, ((it / depth) - 1) & 1, abort_flag, a.status, is_x ? 21 : 25, a.limit_ns)) {
            ok = false;
            break;
          }
          if (is_x) {
            mbar_arrive_expect_tx(fullb + st, kABytes);
            tma_load_4d(xring + st * kABytes, &map_x, fullb + st, k * kBK, 0, t * kBM, 0);
          } else {
            uint8_t* sb = wring + st * a.w_bytes;
            mbar_arrive_expect_tx(fullb + st, a.bn * kBK * 2);
            if (split_n) {
              tma_load_4d(sb, &map_w, fullb + st, k * kBK, n0, 0, 0);
              tma_load_4d(sb + (a.bn / 2) * 128, &map_w, fullb + st, k * kBK, n0 + a.bn / 2, 0, 0);
            } else {
              tma_load_4d(sb, &map_w, fullb + st, k * kBK, n0, 0, 0);
            }
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA goes on
        for (int j = (it > depth ? it - depth : 0); j < it; ++j)
          mbar_wait(fullb + j % depth, (j / depth) & 1, &zero_flag, nullptr, 0, a.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (elect_one()) {
      const int nmma = split_n ? a.bn / 2 : a.bn;
      const uint32_t idesc = idesc_bf16_f32(kBM, nmma, 0, 0);
      int it = 0, li = 0;
      bool ok = true;
      for (int u = u_first; ok && u < n_units; u += u_step, ++li) {
        const int ab = li % n_acc, use = li / n_acc;
        if (use >= 1 && !mbar_wait(acc_empty + ab, (use - 1) & 1, abort_flag, a.status, 24, a.limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + ab * 256;
        for (int k = kb; k < ke; ++k, ++it) {
          const int sx = it % xs, sw = it % ws;
          if (!mbar_wait(x_full + sx, (it / xs) & 1, abort_flag, a.status, 22, a.limit_ns) ||
              !mbar_wait(w_full + sw, (it / ws) & 1, abort_flag, a.status, 26, a.limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(xring + sx * kABytes);
          const uint32_t sb = smem_u32(wring + sw * a.w_bytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc(sa + kk * 32, 16, 1024, kSwizzle128B);
            const uint32_t acc_flag = (k > kb || kk > 0) ? 1u : 0u;
            mma_ss(acc, ad, smem_desc(sb + kk * 32, 16, 1024, kSwizzle128B), idesc, acc_flag);
            if (split_n)
              mma_ss(acc + nmma, ad, smem_desc(sb + nmma * 128 + kk * 32, 16, 1024, kSwizzle128B), idesc, acc_flag);
          }
          mma_commit(x_empty + sx);
          mma_commit(w_empty + sw);
        }
        if (ok) mma_commit(acc_full + ab);
      }
      // every MMA of this CTA has completed before TMEM is released
      mma_commit(drain);
      mbar_wait(drain, 0, &zero_flag, nullptr, 0, a.limit_ns);
      // S == 1: and the epilogue has read the last units' accumulators (it releases each one on
      // acc_empty); TMEM is not released on the strength of the CTA barrier below alone
      if (S == 1 && ok) {
        for (int q = 0; q < n_acc && q < li; ++q) {
          const int j = li - 1 - q;
          mbar_wait(acc_empty + j % n_acc, (j / n_acc) & 1, &zero_flag, nullptr, 0, a.limit_ns);
        }
      }
    }
  } else {
    // ================= epilogue: warps 2..5, TMEM lane quadrant = warp % 4 =================
    a.rope.build(tab, threadIdx.x - 64, kEpiThreads);
    named_bar_sync(1, kEpiThreads);
    if (S == 1) {
      const int quad = warp & 3;
      const int r = quad * 32 + lane;                  // this thread's row of the tile (= TMEM lane)
      const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
      int li = 0;
      for (int u = u_first; u < n_units; u += u_step, ++li) {
        const int t = u / a.nt, n0 = (u % a.nt) * a.bn;
        const int n1 = n0 + a.bn < a.N ? n0 + a.bn : a.N;
        const int ab = li % n_acc, use = li / n_acc;
        const bool got = mbar_wait(acc_full + ab, use & 1, abort_flag, a.status, 23, a.limit_ns);
        if (!named_bar_and(2, kEpiThreads, got)) break;   // uniform: the barriers below hold all four warps
        tc_fence_after();
        const int m = t * kBM + r;
        const RowPos pos = row_pos(a, m < a.M ? m : a.M - 1);
        rowdst[r] = pos.ring;
        for (int c0 = 0; c0 < n1 - n0; c0 += 64) {
          // two 32-column loads in flight per wait
          uint32_t raw[2][32];
          const bool two = c0 + 32 < n1 - n0;
          tmem_ld32(tmem + lane_base + ab * 256 + c0, raw[0]);
          if (two) tmem_ld32(tmem + lane_base + ab * 256 + c0 + 32, raw[1]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int cc = c0 + 32 * h;
            if (h == 1 && !two) break;
            float v[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(raw[h][q]);
            if (n0 + cc >= a.d_c) a.rope.rotate32(tab, (n0 + cc - a.d_c) / 2, pos.f, pos.i, pos.j, v);
            uint8_t* dst = sout + r * a.row_stride + cc * 2;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 w4;
              w4.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
              w4.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
              w4.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
              w4.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
              *reinterpret_cast<uint4*>(dst + q * 16) = w4;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(acc_empty + ab);                   // the MMAs of a later unit may reuse this accumulator
        named_bar_sync(2, kEpiThreads);                // the tile is staged
        const int rows_left = a.M - t * kBM;
        store_rows(a, sout, rowdst, rows_left < kBM ? rows_left : kBM, n0, n1, warp - 2, lane);
        named_bar_sync(2, kEpiThreads);                // the staging buffer is free again
      }
    }
  }

  if constexpr (S > 1) {
    // ---- split-K: sum the pair's partial tiles through distributed shared memory ----
    // (every thread of both CTAs passes both cluster barriers, whatever happened before)
    constexpr int R = kBM / S;                        // rows each CTA finishes
    const int t = u_first / a.nt, n0 = (u_first % a.nt) * a.bn;
    const int n1 = n0 + a.bn < a.N ? n0 + a.bn : a.N;
    const bool epi = warp >= 2;
    bool mine = false;
    if (epi) {
      const bool got = mbar_wait(acc_full, 0, abort_flag, a.status, 23, a.limit_ns);
      mine = named_bar_and(2, kEpiThreads, got);
      if (threadIdx.x == 64) {
        // tell every CTA of the cluster whether this CTA's partial will be there
        for (uint32_t d = 0; d < (uint32_t)S; ++d)
          asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(map_to_rank(smem_u32((const void*)(ok_flags + rank)), d)),
                       "r"(mine ? 1u : 0u) : "memory");
      }
    }
    cluster_sync_all();                               // #1: both CTAs' MMAs are done, their rings free
    bool all_ok = true;
    for (int s = 0; s < S; ++s) all_ok = all_ok && ok_flags[s] != 0;
    const int nchunk = (n1 - n0) / 4;                 // 16-byte (4 x fp32) column chunks of the unit
    if (epi && all_ok) {
      // warp quadrant q holds rows 32q .. 32q+31, finished by CTA (32q) / R: write them into its slot
      // [this rank][chunk][row within the owner's rows] of that CTA's partial buffer
      const int quad = warp & 3;
      const uint32_t owner = (uint32_t)((quad * 32) / R);
      const int row_local = quad * 32 + lane - (int)owner * R;
      const uint32_t rbase = map_to_rank(smem_u32(partials), owner);
      const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
      tc_fence_after();
      for (int c0 = 0; c0 < n1 - n0; c0 += 32) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_base + c0, raw);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int chunk = c0 / 4 + q;
          if (chunk < nchunk)
            st_cluster_v4(rbase + (uint32_t)((((int)rank * nchunk + chunk) * R + row_local) * 16), raw[4 * q],
                          raw[4 * q + 1], raw[4 * q + 2], raw[4 * q + 3]);
        }
      }
    }
    cluster_sync_all();                               // #2: every partial has landed
    if (epi && all_ok) {
      // this CTA's R rows: thread -> (row, part of the columns); sum the S partials, rotate k^R, bf16
      const int tt = threadIdx.x - 64;
      const int row_local = tt % R, part = tt / R;    // S parts of the unit's chunks
      const int m0 = t * kBM + (int)rank * R;
      const int m = m0 + row_local;
      const RowPos pos = row_pos(a, m < a.M ? m : a.M - 1);
      if (part == 0) rowdst[row_local] = pos.ring;
      const float4* part_buf = reinterpret_cast<const float4*>(partials);
      const int per = (nchunk + S - 1) / S;
      const int c_lo = part * per, c_hi = (part + 1) * per < nchunk ? (part + 1) * per : nchunk;
#pragma unroll 4
      for (int chunk = c_lo; chunk < c_hi; ++chunk) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const float4 p4 = part_buf[(s * nchunk + chunk) * R + row_local];
          v[0] += p4.x; v[1] += p4.y; v[2] += p4.z; v[3] += p4.w;
        }
        const int col = n0 + chunk * 4;
        if (col >= a.d_c) a.rope.rotate4(tab, (col - a.d_c) / 2, pos.f, pos.i, pos.j, v);
        uint2 w2;
        w2.x = pack_bf16x2(v[0], v[1]);
        w2.y = pack_bf16x2(v[2], v[3]);
        *reinterpret_cast<uint2*>(sout + row_local * a.row_stride + chunk * 8) = w2;
      }
      named_bar_sync(2, kEpiThreads);
      const int rows_left = a.M - m0;
      if (rows_left > 0) store_rows(a, sout, rowdst, rows_left < R ? rows_left : R, n0, n1, warp - 2, lane);
    }
  }
  // every role has left its loop (lanes of a warp that took different roles meet first) before TMEM
  // is released
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Largest number of clusters of S CTAs that can run at once with this kernel (0 if unknown), per device.
template <int S>
int max_clusters() {
  static int cached[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (!cached[dev]) {
    cudaLaunchConfig_t lc{};
    lc.gridDim = dim3(S * 148);
    lc.blockDim = dim3(kThreads);
    lc.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, compress_kernel<S>, &lc) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    cached[dev] = n > 0 ? n : -1;
  }
  return cached[dev] > 0 ? cached[dev] : 0;
}

template <int S>
cudaError_t launch_compress(const CUtensorMap& mx, const CUtensorMap& mw, const CompressArgs& a, int grid,
                            cudaStream_t st) {
  cudaLaunchConfig_t lc{};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = kSmemBytes;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  if (S > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
  }
  cudaError_t e = cudaLaunchKernelEx(&lc, compress_kernel<S>, mx, mw, a);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t ensure_compress_attrs() {
  static std::atomic<uint64_t> d1{0}, d2{0};
  cudaError_t e = ensure_smem_attr((const void*)compress_kernel<1>, kSmemBytes, d1);
  if (e == cudaSuccess) e = ensure_smem_attr((const void*)compress_kernel<2>, kSmemBytes, d2);
  return e;
}

}  // namespace

vmla_status tc_check_compress(const vmla_config& c) {
  if (c.d_rope != 32 || c.d_c % 32 || c.d_c < 32 || c.d_c + c.d_rope > kMaxN || c.dim % 8) {
    set_tc_reason("tensor-core compress needs d_rope == 32, d_c a multiple of 32 in [32, 256], dim % 8 == 0");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
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
  if (M <= 0 || M > (int64_t)1 << 30) return cudaErrorInvalidValue;
  const int N = cfg.d_c + cfg.d_rope, K = cfg.dim;
  cudaError_t e = ensure_compress_attrs();
  if (e != cudaSuccess) return e;
  // work decomposition: the row tiles, then (when they leave SMs idle) 128-column tiles and a split of
  // the reduction over a CTA pair, as long as every pair can run at once
  const int n_m = (int)((M + kBM - 1) / kBM);
  const int nk = (K + kBK - 1) / kBK;
  const int sms = num_sms();
  int S = 1, nt = 1;
  if (nk >= 2 && N <= 256) {
    const int pairs = max_clusters<2>();
    if (N > kNarrowBN && 4 * n_m <= sms && 2 * n_m <= pairs) {
      S = 2;
      nt = 2;
    } else if (2 * n_m <= sms && n_m <= pairs) {
      S = 2;
    }
  }
  CompressArgs a{};
  a.M = (int)M;
  a.K = K;
  a.N = N;
  a.d_c = cfg.d_c;
  a.nt = nt;
  a.bn = nt == 1 ? N : kNarrowBN;
  a.ntok = (int)ntok;
  a.tok0 = (int)tok0;
  a.tokens_per_frame = cfg.grid_h * cfg.grid_w;
  a.grid_w = cfg.grid_w;
  a.window_frames = cfg.window_frames;
  a.first_slot = (int)(g.first_frame % cfg.window_frames);
  a.first_frame = g.first_frame;
  a.cap = (int64_t)cfg.window_frames * a.tokens_per_frame;
  // shared memory: x ring | weight ring | staged rows | ring rows | RoPE table | barriers (after 1 KB
  // alignment).  x comes from HBM and needs ~100 KB in flight per SM to stream at the HBM rate, so the
  // x ring gets at least six k-steps where it can; the weight ring (served from L2) two or three.
  a.row_stride = 2 * a.bn + 16;
  a.w_bytes = a.bn * kBK * 2;
  const int fixed = kBM * a.row_stride + kRowDstBytes + kTabBytes + kAuxBytes + 1024;
  a.ws = kMaxWStages;
  while (a.ws > 2 && fixed + a.ws * a.w_bytes + 6 * kABytes > kSmemBytes) --a.ws;
  a.xs = (kSmemBytes - fixed - a.ws * a.w_bytes) / kABytes;
  if (a.xs > kMaxXStages) a.xs = kMaxXStages;
  if (a.xs < 2) return cudaErrorInvalidValue;
  // the pair's partials (S slots of 128/S rows x bn fp32) take the place of both rings
  if (S > 1 && a.bn * 4 * kBM > a.xs * kABytes + a.ws * a.w_bytes) S = 1;
  a.rope = make_rope_lookup(rt, g, cfg.chunk_frames, kTabEntries);
  const int64_t cap_rows = (int64_t)batch * a.cap;
  for (int d = 0; d < n_dst; ++d) {
    a.c[d] = (bf16*)dst[d].c;
    a.k_r[d] = (bf16*)dst[d].k_r;
    a.c_span[d] = make_span(dst[d].c, checked_extent(cap_rows * cfg.d_c * 2));
    a.kr_span[d] = make_span(dst[d].k_r, checked_extent(cap_rows * cfg.d_rope * 2));
  }
  a.n_dst = n_dst;
  a.status = device_status_ptr();
  a.limit_ns = wait_limit_ns();
  // A = x [M, D] and B = [W^KV_down ; W^KR] [N, D], both K-major, 128-byte swizzle; the weight box is
  // one column tile (half of it above 256 columns)
  CUtensorMap mx, mw;
  const int wbox = a.bn > 256 ? a.bn / 2 : a.bn;
  if ((e = make_map_4d(&mx, x, K, 1, M, 1, (int64_t)K * 2, (int64_t)K * 2, M * K * 2, kBK, 1, kBM, 128)) != cudaSuccess)
    return e;
  if ((e = make_map_4d(&mw, w, K, N, 1, 1, (int64_t)K * 2, (int64_t)N * K * 2, (int64_t)N * K * 2, kBK, wbox, 1, 128)) != cudaSuccess)
    return e;
  const int units = n_m * nt;
  if (S == 2) return launch_compress<2>(mx, mw, a, 2 * units, st);
  return launch_compress<1>(mx, mw, a, units < sms ? units : sms, st);
}

}  // namespace vmla
