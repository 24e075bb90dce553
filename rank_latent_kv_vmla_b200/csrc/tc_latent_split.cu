// Latent attention at the lower latent ranks d_c = 64 / 128 on the sm_100a tensor cores, with the keys
// of every tile split between two softmax warpgroups (VideoMLA technical summary, Method items 2-3;
// lower d_c: Results, "Scalability"): the three-call path's vmla_latent_attention and the fused call
// vmla_latent_attention_fused at these ranks.
//
// At d_c <= 128 a score costs 2 (2 d_c + 32) <= 576 MMA flops, so the tensor cores finish a 128 x 128
// tile of scores and its P V well before one warp per SM sub-partition has exponentiated the tile's
// scores: a single softmax warpgroup bounds the kernel.  Here warps 0-3 take keys 0-63 and warps 4-7
// keys 64-127 of every tile, each warpgroup with its own running max, row sum and O accumulator,
// merged once at the end (the layout of the dense comparison kernel, with the latent cache's keys
// [c ; k^R] and values c read from the same shared-memory stage).
//
// One CTA owns 128 query rows and streams every visible KV tile of 128 keys:
//   warp 8      TMA producer: the Q tile once (three-call: q_abs; fused: q^nope and W^K_up,h for the
//               prologue), then the c boxes and the k^R box of each KV tile into a ring of stages (and,
//               fused, W^V_up,h as one more load);
//   warp 9      TMEM owner and MMA issuer: (fused) q~ = q^nope W^K_up,h; S_j = Q K_j^T (K = d_c + 32)
//               into one of two TMEM S buffers; for each key half w: O_w += P_{j-1,w} V_{j-1,w}, V = the
//               c boxes read MN-major; (fused) o = (O / l) W^V_up,h^T at the end;
//   warps 0-7   (fused) RoPE3D(q^rope) and q~ as bf16 into the Q buffer; softmax of one key half (one
//               thread per query row = TMEM lane): masked running max with a lazy rescale of O_w, exp2
//               (a quarter, three eighths in the fused call, by the FMA-pipe polynomial), row sum, P to
//               TMEM in two parts of 32 keys; finally (max, sum) swapped through shared memory, and each warpgroup forms half of the columns of
//               (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / l: stored (three-call) or written as bf16 into the Q
//               buffer for the value up-projection, whose output each warpgroup then stores half of.
// Three-call rows are (token, head) rows of q_abs (every head shares the KV tiles); fused tiles are 128
// tokens of one head.  TMEM: S buffers at columns [0, 128) and [128, 256), O_0 at 256, O_1 at 256 + d_c
// (the prologue's q~ lands in O_0 first; the value up-projection's output in the first S buffer).
// Every mbarrier wait is bounded; a wait that runs out records its code (31-43) in the status word and
// every role winds down (copies in flight land, MMAs drain, TMEM is freed).
#include <cuda.h>

#include <atomic>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "tc_kernels.cuh"

namespace vmla {
namespace {

using namespace sm100;

constexpr int kThreads = 320;                 // 10 warps
constexpr int kBlockM = 128;                  // query rows per CTA
constexpr int kBN = 128;                      // keys per KV tile
constexpr int kHalf = kBN / 2;                // keys per softmax warpgroup
constexpr int kBox = kBN * 128;               // [128 rows x 64 columns] bf16, 128-byte swizzle
constexpr int kRopeBox = kBN * 64;            // [128 rows x 32 columns] bf16, 64-byte swizzle
constexpr int kAuxBytes = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 2 * kBN;
constexpr float kRescaleThreshold = 8.0f;     // log2 units
constexpr int kPParts = 2;                    // each key half releases its P in two parts
constexpr int kStepsPerPart = kHalf / 16 / kPParts;

// KB = d_c / 64 latent boxes
template <int KB, bool FUSED>
struct SplitPlan {
  static constexpr int kDV = 64 * KB;
  // Q buffer: the c boxes (fused: at least the two boxes q^nope is staged in), then the rope box
  static constexpr int kQBoxes = (FUSED && KB < 2) ? 2 : KB;
  static constexpr int kQRopeOff = kQBoxes * kBlockM * 128;
  static constexpr int kQBytes = kQRopeOff + kBlockM * 64;
  static constexpr int kStageBytes = KB * kBox + kRopeBox;     // multiple of 1024
  static constexpr int kRopeOff = KB * kBox;
  static constexpr int kFit = (232448 - 1024 - kAuxBytes - kQBytes) / kStageBytes;
  static constexpr int kStages = kFit >= 6 ? 6 : kFit;
  static constexpr int kSmemBytes = kQBytes + kStages * kStageBytes + kAuxBytes + 1024;
  static_assert(kStages >= 3, "shared memory");
  static_assert(kTmemO + 2 * kDV <= kTmemCols, "TMEM budget");
};

struct SplitParams {
  int rows_per_b;        // query rows per batch element (three-call: Nq * H; fused: Nq tokens)
  int tiles_per_group;   // query tiles per (batch[, head]) group
  int heads;
  int64_t nq;            // query tokens per batch element
  int64_t tok0;          // fused: row r of a tile is token tok0 + r of the call (a token range)
  FrameGeom g;
  float scale_log2;
  void* out;             // three-call: [B, Nq*H, d_c]; fused: [B, Nq, H, d_v]  (bf16)
  float* lse;            // [B, Nq, H] or null
  int* status;
  uint64_t limit_ns;
  int drop_kv_tile;
  // fused only
  const void* q_rope;    // [B, Nq, H, 32] bf16: rotated in the prologue
  int d_nope;            // K of the absorbing MMA (multiple of 16, <= 128)
  int d_v;               // N of the value up-projection (multiple of 64, <= 128)
  RopeTable rt;
  Span out_span, lse_span;
};

template <int KB, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
latent_split_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_qr,
                    const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_kr,
                    const __grid_constant__ CUtensorMap map_wuk, const __grid_constant__ CUtensorMap map_wuv,
                    const SplitParams p) {
  using PL = SplitPlan<KB, FUSED>;
  constexpr int NST = PL::kStages;
  constexpr int DV = PL::kDV;
  // of the 8 score pairs per 16 keys, how many take the FMA-pipe 2^x (measured on B200 at batch 16,
  // d_c = 64 / 128: three pairs 4-5 % faster than two for the fused call, within 1 % either way for
  // the three-call attention; four slower for both)
  constexpr int kPolyPairs = FUSED ? 3 : 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + PL::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NST * PL::kStageBytes);
  uint64_t* bar_q = bars;                    // Q in place (TMA landed, or both warpgroups wrote it)
  uint64_t* kv_full = bars + 1;              // [NST]
  uint64_t* kv_empty = kv_full + NST;        // [NST]
  uint64_t* s_full = kv_empty + NST;         // [2 S buffers]
  uint64_t* p_ready = s_full + 2;            // [2 S buffers][2 key halves][kPParts], 128 arrivals each
  uint64_t* pv_done = p_ready + 4 * kPParts; // [2 S buffers][2 key halves]
  uint64_t* drain = pv_done + 4;             // every MMA of the main loop completed
  uint64_t* bar_pro = drain + 1;             // fused: q^nope and W^K_up,h landed
  uint64_t* qa_full = bar_pro + 1;           // fused: q~ complete in TMEM
  uint64_t* o_ready = qa_full + 1;           // fused: O / l written to the Q buffer (256 arrivals)
  uint64_t* out_full = o_ready + 1;          // fused: the value up-projection complete in TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(out_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int tile = blockIdx.x;
  const int group = tile / p.tiles_per_group;
  const int row0 = (tile % p.tiles_per_group) * kBlockM;
  const int b = FUSED ? group / p.heads : group;
  const int h = FUSED ? group % p.heads : 0;
  const int tok_div = FUSED ? 1 : p.heads;                     // query row -> token
  const int64_t tok_base = FUSED ? p.tok0 : 0;
  const int last_row = min(row0 + kBlockM, p.rows_per_b) - 1;
  const int64_t kend_first = key_end_rows(p.g, tok_base + row0 / tok_div);
  const int64_t kend_last = key_end_rows(p.g, tok_base + last_row / tok_div);
  const int n_kv = (int)((kend_last + kBN - 1) / kBN);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, FUSED ? 256 : 1);
    for (int s = 0; s < NST; ++s) { mbar_init(kv_full + s, 1); mbar_init(kv_empty + s, 1); }
    for (int s = 0; s < 2; ++s) mbar_init(s_full + s, 1);
    for (int i = 0; i < 4 * kPParts; ++i) mbar_init(p_ready + i, 128);
    for (int i = 0; i < 4; ++i) mbar_init(pv_done + i, 1);
    mbar_init(drain, 1);
    mbar_init(bar_pro, 1);
    mbar_init(qa_full, 1);
    mbar_init(o_ready, 256);
    mbar_init(out_full, 1);
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
      tma_prefetch_desc(&map_kr);
      if (!FUSED) {
        mbar_arrive_expect_tx(bar_q, PL::kQBytes);
        for (int i = 0; i < KB; ++i) tma_load_4d(sQ + i * kBlockM * 128, &map_q, bar_q, 64 * i, 0, row0, b);
        tma_load_4d(sQ + PL::kQRopeOff, &map_qr, bar_q, 64 * KB, 0, row0, b);
      } else {
        // prologue operands: the q^nope tile (two 64-column boxes; columns past d_nope read as zeros)
        // into the Q buffer, W^K_up,h (KB boxes of [d_nope rows][64 columns]) into the last stage
        tma_prefetch_desc(&map_wuk);
        tma_prefetch_desc(&map_wuv);
        uint8_t* wst = sKV + (NST - 1) * PL::kStageBytes;
        mbar_arrive_expect_tx(bar_pro, 2 * kBlockM * 128 + KB * p.d_nope * 128);
        for (int i = 0; i < 2; ++i) tma_load_4d(sQ + i * kBlockM * 128, &map_q, bar_pro, 64 * i, h, row0, b);
        for (int i = 0; i < KB; ++i) tma_load_4d(wst + i * p.d_nope * 128, &map_wuk, bar_pro, 64 * i, 0, h, 0);
      }
      // load j goes to stage j % NST once the P V of load j - NST has completed; fused: the last stage
      // first holds W^K_up,h until the prologue MMA has completed
      auto claim = [&](int j) -> bool {
        const int st = j % NST;
        if (j >= NST && !mbar_wait(kv_empty + st, ((j / NST) - 1) & 1, abort_flag, p.status, 31, p.limit_ns))
          return false;
        if (FUSED && j == NST - 1 && !mbar_wait(qa_full, 0, abort_flag, p.status, 38, p.limit_ns)) return false;
        return true;
      };
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        if (!claim(j)) break;
        issued = j + 1;
        if (j == p.drop_kv_tile) continue;
        const int st = j % NST;
        uint8_t* stage = sKV + st * PL::kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, PL::kStageBytes);
        const int krow = j * kBN;
        for (int i = 0; i < KB; ++i) tma_load_4d(stage + i * kBox, &map_k, kv_full + st, 64 * i, 0, krow, b);
        tma_load_4d(stage + PL::kRopeOff, &map_kr, kv_full + st, 0, 0, krow, b);
      }
      if (FUSED && issued == n_kv && claim(n_kv)) {
        // W^V_up,h (KB K-major boxes of [d_v rows][64 columns]) as load n_kv of the ring
        const int st = n_kv % NST;
        uint8_t* stage = sKV + st * PL::kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, KB * p.d_v * 128);
        for (int i = 0; i < KB; ++i) tma_load_4d(stage + i * p.d_v * 128, &map_wuv, kv_full + st, 64 * i, 0, h, 0);
        issued = n_kv + 1;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        mbar_wait(FUSED ? bar_pro : bar_q, 0, &zero_flag, nullptr, 0, p.limit_ns);
        for (int j = (issued > NST ? issued - NST : 0); j < issued; ++j)
          if (j != p.drop_kv_tile) mbar_wait(kv_full + j % NST, (j / NST) & 1, &zero_flag, nullptr, 0, p.limit_ns);
      }
    }
  } else if (warp == 9) {
    // ================= MMA issuer =================
    if (elect_one()) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, DV, 0, 1);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t kv_base = smem_u32(sKV);
      bool ok = true;
      if (FUSED) {
        ok = mbar_wait(bar_pro, 0, abort_flag, p.status, 39, p.limit_ns);
        if (ok) {
          tc_fence_after();
          // q~ = q^nope W^K_up,h into the O_0 columns: A K-major (two 64-column boxes), B MN-major
          // ([d_nope rows][64 columns] boxes d_nope*128 B apart = LBO; a K step of 16 rows is 2048 B)
          const uint32_t w_base = kv_base + (NST - 1) * PL::kStageBytes;
          constexpr uint32_t idesc_qa = idesc_bf16_f32(kBlockM, DV, 0, 1);
          for (int k = 0; k < p.d_nope / 16; ++k) {
            const uint64_t adesc = smem_desc(q_base + (k >> 2) * kBlockM * 128 + (k & 3) * 32, 16, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(w_base + k * 2048, p.d_nope * 128, 1024, kSwizzle128B);
            mma_ss(tmem + kTmemO, adesc, bdesc, idesc_qa, k > 0 ? 1u : 0u);
          }
          mma_commit(qa_full);
        }
      }
      ok = ok && mbar_wait(bar_q, 0, abort_flag, p.status, 32, p.limit_ns);
      // O_w += P_{jp,w} V_{jp,w} for both key halves, each as soon as its warpgroup released its P
      auto issue_pv = [&](int jp) -> bool {
        const int bp = jp & 1;
        const uint32_t v_base = kv_base + (jp % NST) * PL::kStageBytes;
        for (int w = 0; w < 2; ++w) {
#pragma unroll
          for (int k = 0; k < kHalf / 16; ++k) {
            if (k % kStepsPerPart == 0) {
              if (!mbar_wait(p_ready + (2 * bp + w) * kPParts + k / kStepsPerPart, (jp >> 1) & 1, abort_flag,
                             p.status, 33, p.limit_ns))
                return false;
              tc_fence_after();
            }
            // V = the c boxes as an MN-major operand: 8-key groups 1024 B apart (SBO), 64-column boxes
            // kBox apart (LBO); 16 keys are 2048 B.  P of keys 64w + 16k .. + 15 sits in the 8 columns
            // at 64w + 8k of the S buffer.
            const int ks = w * (kHalf / 16) + k;
            const uint64_t vdesc = smem_desc(v_base + ks * 2048, kBox, 1024, kSwizzle128B);
            mma_ts(tmem + kTmemO + w * DV, tmem + bp * kBN + w * kHalf + k * 8, vdesc, idesc_pv,
                   (jp > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(pv_done + 2 * bp + w);
        }
        mma_commit(kv_empty + (jp % NST));
        return true;
      };
      if (ok) tc_fence_after();
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j % NST, bj = j & 1;
        if (!mbar_wait(kv_full + st, (j / NST) & 1, abort_flag, p.status, 34, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        // S buffer bj last held P_{j-2}, whose P V MMAs were issued before this point (in order)
        const uint32_t k_base = kv_base + st * PL::kStageBytes;
#pragma unroll
        for (int k = 0; k < KB * 4; ++k) {
          // 16 columns of c: box k/4, 32-byte step k%4 inside the 128-byte swizzle atom
          const uint64_t qdesc = smem_desc(q_base + (k >> 2) * kBlockM * 128 + (k & 3) * 32, 16, 1024, kSwizzle128B);
          const uint64_t kdesc = smem_desc(k_base + (k >> 2) * kBox + (k & 3) * 32, 16, 1024, kSwizzle128B);
          mma_ss(tmem + bj * kBN, qdesc, kdesc, idesc_qk, k > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          // the 32 rotated columns: 64-byte swizzle, 16 columns = 32 bytes
          const uint64_t qdesc = smem_desc(q_base + PL::kQRopeOff + k * 32, 16, 512, kSwizzle64B);
          const uint64_t kdesc = smem_desc(k_base + PL::kRopeOff + k * 32, 16, 512, kSwizzle64B);
          mma_ss(tmem + bj * kBN, qdesc, kdesc, idesc_qk, 1u);
        }
        mma_commit(s_full + bj);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && n_kv > 0) ok = issue_pv(n_kv - 1);
      // every MMA of the main loop has completed before the softmax warps read the final O (and before
      // TMEM is released)
      mma_commit(drain);
      if (FUSED) {
        if (ok) {
          const int st = n_kv % NST;
          ok = mbar_wait(kv_full + st, (n_kv / NST) & 1, abort_flag, p.status, 40, p.limit_ns) &&
               mbar_wait(o_ready, 0, abort_flag, p.status, 41, p.limit_ns);
          if (ok) {
            tc_fence_after();
            // o = (O / l) W^V_up,h^T into the first S buffer: A = O / l (bf16 K-major boxes in the Q
            // buffer), B = W^V_up,h (K-major boxes of [d_v rows][64 columns])
            const uint32_t wv = kv_base + st * PL::kStageBytes;
            const uint32_t idesc_vu = idesc_bf16_f32(kBlockM, p.d_v, 0, 0);
            for (int k = 0; k < DV / 16; ++k) {
              const uint64_t adesc = smem_desc(q_base + (k >> 2) * kBlockM * 128 + (k & 3) * 32, 16, 1024, kSwizzle128B);
              const uint64_t bdesc = smem_desc(wv + (k >> 2) * p.d_v * 128 + (k & 3) * 32, 16, 1024, kSwizzle128B);
              mma_ss(tmem, adesc, bdesc, idesc_vu, k > 0 ? 1u : 0u);
            }
          }
        }
        mma_commit(out_full);
        mbar_wait(out_full, 0, &zero_flag, nullptr, 0, p.limit_ns);
      } else {
        mbar_wait(drain, 0, &zero_flag, nullptr, 0, p.limit_ns);
      }
    }
  } else {
    // ====== softmax of one key half (warps 0-3: keys 0-63, warps 4-7: keys 64-127), epilogue ======
    const int wg = warp >> 2;
    const int r = threadIdx.x & 127;                 // query row in the tile = TMEM lane
    const int row = row0 + r;
    const bool row_valid = row < p.rows_per_b;
    const int64_t kend = row_valid ? key_end_rows(p.g, tok_base + row / tok_div) : kend_last;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    // this row's index in the rows of out / lse: three-call (b, token*H + head), fused (b, token, h)
    const int64_t orow = FUSED ? (((int64_t)b * p.nq + row) * p.heads + h) : (int64_t)b * p.rows_per_b + row;
    const uint32_t o_own = tmem + lane_base + kTmemO + wg * DV;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    if (FUSED) {
      // the Q row, written as the K-major operand TMA would have produced (16-byte chunk k of a
      // 128-byte row of a c box at chunk k ^ (row % 8); of a 64-byte rope row at chunk k ^ ((row / 2) % 4)).
      // Warpgroup 0 first rotates q^rope into the rope box (the prologue's TMA copies do not touch it)
      // while the q^nope W^K_up,h MMA is in flight; then each warpgroup converts half of q~ to bf16.
      if (wg == 0) {
        float v[32];
        if (row_valid) {
          const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.q_rope) + orow * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 u = src[q];
            const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
            for (int t = 0; t < 8; ++t) v[8 * q + t] = __bfloat162float(e[t]);
          }
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = 0.f;
        }
        const int64_t tok = tok_base + row;
        const int64_t f = p.g.first_frame + tok / p.g.tokens_per_frame;
        const int rr = (int)(tok % p.g.tokens_per_frame);
        const int ri = rr / p.g.grid_w, rj = rr % p.g.grid_w;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float a, bb;
          rope_rotate_mufu(p.rt, q, f, ri, rj, v[2 * q], v[2 * q + 1], &a, &bb);
          v[2 * q] = a;
          v[2 * q + 1] = bb;
        }
        uint8_t* ropep = sQ + PL::kQRopeOff + r * 64;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
          w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
          w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
          w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
          *reinterpret_cast<uint4*>(ropep + ((q ^ ((r >> 1) & 3)) << 4)) = w;
        }
      }
      const bool got = mbar_wait(qa_full, 0, abort_flag, p.status, 42, p.limit_ns);
      ok = __all_sync(0xffffffffu, got);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < DV / 64; ++cc) {
          const int c = wg * (DV / 64) + cc;           // 32-column chunk of q~ (this warpgroup's half)
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + kTmemO + c * 32, v);
          tmem_ld_wait();
          uint8_t* rowp = sQ + (c >> 1) * (kBlockM * 128) + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (c & 1) * 4 + q;
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
            w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
            w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
            w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
            *reinterpret_cast<uint4*>(rowp + ((chunk ^ (r & 7)) << 4)) = w;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar_q);
      }
    }
    // P_{k,wg} V_{k,wg} completed: phase k/2 of pv_done[k % 2][wg].  Called from tile k + 1, when that
    // barrier is at most one phase away (S_{k+1} complete implies P_{k-1} V_{k-1} complete; P_{k+2} does
    // not exist yet).
    auto wait_pv = [&](int k) -> bool {
      const bool got = mbar_wait(pv_done + 2 * (k & 1) + wg, (k >> 1) & 1, abort_flag, p.status, 35, p.limit_ns);
      return __all_sync(0xffffffffu, got);
    };
    const float sc = p.scale_log2;
    for (int j = 0; ok && j < n_kv; ++j) {
      const int bj = j & 1;
      const bool got = mbar_wait(s_full + bj, (j >> 1) & 1, abort_flag, p.status, 36, p.limit_ns);
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
          for (int c = 0; c < DV / 32; ++c) {
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
    bool fin = ok && mbar_wait(drain, 0, abort_flag, p.status, 37, p.limit_ns);
    fin = __all_sync(0xffffffffu, fin && !*abort_flag);
    // (max, sum) of both halves through the rope box of the Q buffer (every S = Q K^T MMA has
    // completed, and the fused value up-projection reads only the c boxes).  Every softmax thread passes
    // the barrier once; a run that did not finish cleanly has raised the abort flag before it, so both
    // halves agree on whether to go on.
    float* xch = reinterpret_cast<float*>(sQ + PL::kQRopeOff);   // [2 halves][max, sum][128 rows]
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
      const uint32_t o_oth = tmem + lane_base + kTmemO + (wg ^ 1) * DV;
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
      uint32_t oa[32], ob[32];
#pragma unroll
      for (int cc = 0; cc < DV / 64; ++cc) {
        const int c = wg * (DV / 64) + cc;             // 32-column chunk (this warpgroup's half)
        tmem_ld32(o_own + c * 32, oa);
        tmem_ld32(o_oth + c * 32, ob);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = fmaf(__uint_as_float(oa[t]), f_own, __uint_as_float(ob[t]) * f_oth);
        if (FUSED) {
          // O / l as bf16 into the Q buffer: the A operand of the value up-projection (the layout of q~)
          uint8_t* rowp = sQ + (c >> 1) * (kBlockM * 128) + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (c & 1) * 4 + q;
            uint4 u;
            u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
            u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
            u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
            u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
            *reinterpret_cast<uint4*>(rowp + ((chunk ^ (r & 7)) << 4)) = u;
          }
        } else if (row_valid && store_ok(p.out_span, out + orow * DV + c * 32, 64, p.status, 12)) {
          uint4* dst = reinterpret_cast<uint4*>(out + orow * DV + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
            u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
            u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
            u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
            dst[q] = u;
          }
        }
      }
      if (wg == 0 && row_valid && p.lse && store_ok(p.lse_span, p.lse + orow, 4, p.status, 13))
        p.lse[orow] = (m + __log2f(l_row)) * 0.69314718055994530942f;
      if (FUSED) {
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(o_ready);
        bool got = mbar_wait(out_full, 0, abort_flag, p.status, 43, p.limit_ns);
        got = __all_sync(0xffffffffu, got && !*abort_flag);
        if (got) {
          tc_fence_after();
          // each warpgroup stores half of the d_v output columns of its rows
          for (int c = wg * (p.d_v / 64); c < (wg + 1) * (p.d_v / 64); ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + c * 32, o);
            tmem_ld_wait();
            if (row_valid && store_ok(p.out_span, out + orow * p.d_v + c * 32, 64, p.status, 14)) {
              uint4* dst = reinterpret_cast<uint4*>(out + orow * p.d_v + c * 32);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 u;
                u.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]), __uint_as_float(o[8 * q + 1]));
                u.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]), __uint_as_float(o[8 * q + 3]));
                u.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]), __uint_as_float(o[8 * q + 5]));
                u.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]), __uint_as_float(o[8 * q + 7]));
                dst[q] = u;
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int KB, bool FUSED>
cudaError_t launch_split(const AttnMaps& m, const SplitParams& p, int n_tiles, cudaStream_t st) {
  using PL = SplitPlan<KB, FUSED>;
  auto kern = latent_split_kernel<KB, FUSED>;
  static std::atomic<uint64_t> done{0};
  cudaError_t e = ensure_smem_attr((const void*)kern, PL::kSmemBytes, done);
  if (e != cudaSuccess) return e;
  kern<<<n_tiles, kThreads, PL::kSmemBytes, st>>>(m.q, m.qr, m.k, m.kr, m.wuk, m.wuv, p);
  count_launches(1);
  return cudaGetLastError();
}

template <int KB>
bool fused_split_fits(int d_nope, int d_v) {
  using PL = SplitPlan<KB, true>;
  return KB * d_nope * 128 <= PL::kStageBytes && KB * d_v * 128 <= PL::kStageBytes;
}

}  // namespace

bool tc_latent_split_supported(const vmla_config& cfg) {
  return cfg.d_rope == 32 && (cfg.d_c == 64 || cfg.d_c == 128);
}

bool tc_latent_split_fused_supported(const vmla_config& cfg) {
  if (!tc_latent_split_supported(cfg) || cfg.d_nope % 16 || cfg.d_nope < 16 || cfg.d_nope > 128 ||
      cfg.d_v % 64 || cfg.d_v < 64 || cfg.d_v > 128)
    return false;
  return cfg.d_c == 64 ? fused_split_fits<1>(cfg.d_nope, cfg.d_v) : fused_split_fits<2>(cfg.d_nope, cfg.d_v);
}

cudaError_t tc_latent_attention_split(const vmla_config& cfg, int batch, int64_t nq, const void* q_abs,
                                      const void* c, const void* k_r, int64_t cap, int64_t valid_rows,
                                      const FrameGeom& g, float scale, void* out, float* lse, int* status,
                                      cudaStream_t st) {
  const int H = cfg.n_heads, dqk = cfg.d_c + cfg.d_rope;
  const int64_t rows = nq * H;
  AttnMaps m{};
  cudaError_t e;
  // q_abs [B, Nq*H, d_qk] as {d_qk, 1, Nq*H, B}; the c plane [B, cap, d_c] and k_r [B, cap, 32] as
  // {cols, 1, valid_rows, B}: boxes of 128 rows (unwritten ring rows are never read)
  if ((e = make_map_4d(&m.q, q_abs, dqk, 1, rows, batch, (int64_t)dqk * 2, (int64_t)dqk * 2, rows * dqk * 2, 64, 1,
                       kBlockM, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.qr, q_abs, dqk, 1, rows, batch, (int64_t)dqk * 2, (int64_t)dqk * 2, rows * dqk * 2, 32, 1,
                       kBlockM, 64)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.k, c, cfg.d_c, 1, valid_rows, batch, (int64_t)cfg.d_c * 2, (int64_t)cfg.d_c * 2,
                       cap * cfg.d_c * 2, 64, 1, kBN, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.kr, k_r, 32, 1, valid_rows, batch, 64, 64, cap * 64, 32, 1, kBN, 64)) != cudaSuccess)
    return e;
  m.wuk = m.k;
  m.wuv = m.k;
  SplitParams p{};
  p.rows_per_b = (int)rows;
  p.tiles_per_group = (int)((rows + kBlockM - 1) / kBlockM);
  p.heads = H;
  p.nq = nq;
  p.g = g;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.limit_ns = wait_limit_ns();
  p.drop_kv_tile = take_drop_kv_tile();
  p.out_span = make_span(out, checked_extent((int64_t)batch * rows * cfg.d_c * 2));
  p.lse_span = make_span(lse, checked_extent((int64_t)batch * rows * 4));
  const int n_tiles = batch * p.tiles_per_group;
  return cfg.d_c == 64 ? launch_split<1, false>(m, p, n_tiles, st) : launch_split<2, false>(m, p, n_tiles, st);
}

cudaError_t tc_latent_attention_split_fused(const vmla_config& cfg, int batch, int64_t tok0, int64_t nq,
                                            const void* q_nope, const void* q_rope, const void* w_uk,
                                            const void* w_uv, const void* c, const void* k_r, int64_t cap,
                                            int64_t valid_rows, const FrameGeom& g, const RopeTable& rt,
                                            float scale, void* out, float* lse, int* status, cudaStream_t st) {
  const int H = cfg.n_heads, dn = cfg.d_nope, dc = cfg.d_c, dv = cfg.d_v;
  AttnMaps m{};
  cudaError_t e;
  // q^nope [B, Nq, H, d_nope] as {d_nope, H, Nq, B}: a 128-token box of one head
  if ((e = make_map_4d(&m.q, q_nope, dn, H, nq, batch, (int64_t)dn * 2, (int64_t)H * dn * 2,
                       nq * H * dn * 2, 64, 1, kBlockM, 128)) != cudaSuccess) return e;
  m.qr = m.q;
  if ((e = make_map_4d(&m.k, c, dc, 1, valid_rows, batch, (int64_t)dc * 2, (int64_t)dc * 2,
                       cap * dc * 2, 64, 1, kBN, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.kr, k_r, 32, 1, valid_rows, batch, 64, 64, cap * 64, 32, 1, kBN, 64)) != cudaSuccess)
    return e;
  // W^K_up [H, d_nope, d_c] as {d_c, d_nope, H, 1}: [d_nope rows][64 columns] boxes (MN-major B)
  if ((e = make_map_4d(&m.wuk, w_uk, dc, dn, H, 1, (int64_t)dc * 2, (int64_t)dn * dc * 2,
                       (int64_t)H * dn * dc * 2, 64, dn, 1, 128)) != cudaSuccess) return e;
  // W^V_up [H, d_v, d_c] as {d_c, d_v, H, 1}: [d_v rows][64 columns] boxes (K-major B)
  if ((e = make_map_4d(&m.wuv, w_uv, dc, dv, H, 1, (int64_t)dc * 2, (int64_t)dv * dc * 2,
                       (int64_t)H * dv * dc * 2, 64, dv, 1, 128)) != cudaSuccess) return e;
  SplitParams p{};
  p.rows_per_b = (int)nq;
  p.tiles_per_group = (int)((nq + kBlockM - 1) / kBlockM);
  p.heads = H;
  p.nq = nq;
  p.tok0 = tok0;
  p.g = g;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.limit_ns = wait_limit_ns();
  p.drop_kv_tile = take_drop_kv_tile();
  p.q_rope = q_rope;
  p.d_nope = dn;
  p.d_v = dv;
  p.rt = rt;
  p.out_span = make_span(out, checked_extent((int64_t)batch * nq * H * dv * 2));
  p.lse_span = make_span(lse, checked_extent((int64_t)batch * nq * H * 4));
  const int n_tiles = batch * H * p.tiles_per_group;
  return dc == 64 ? launch_split<1, true>(m, p, n_tiles, st) : launch_split<2, true>(m, p, n_tiles, st);
}

}  // namespace vmla
