// Flash-style attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA) over the VideoMLA latent
// cache (absorbed form): one KV "head" shared by every query head, keys [c ; k^R] (d_c + 32 wide) and
// values c (d_c wide) read from the same shared-memory stage (VideoMLA technical summary, Method items
// 2-3: per-head keys and values are reconstructed from the shared latent; here the reconstruction is
// folded into the query and applied after the sum).  The dense per-head comparison layer has its own
// kernel (tc_dense.cu).
//
// One CTA owns one tile of 128 query rows and streams every visible KV tile of BN keys:
//   warp 4      TMA producer: KV tiles into an NST-deep shared-memory ring (and the Q tile when Q
//               is kept in shared memory);
//   warp 5      TMEM owner and MMA issuer: S_j = Q K_j^T into one of two TMEM S buffers, then
//               O += P_{j-1} V_{j-1} with P read from TMEM (it overwrites S_{j-1} as bf16);
//   warps 0-3   one thread per query row (= TMEM lane): first the Q row into TMEM (when Q is kept
//               in TMEM), then per tile the softmax: masked running max with a lazy rescale of O (only
//               when the max grows by more than 2^8), exp2 (3/8 of them by an FMA-pipe
//               polynomial), row sum, P to TMEM in four parts of 32 keys, each released to the P V
//               MMAs by its own barrier; finally O / l to global memory and the log-sum-exp.  The softmax is
//               latency-bound with one warp per SM sub-partition, so it uses 3-input max and packed
//               f32x2 FMA / add instructions.
// Q lives in TMEM (S = Q K^T then reads only K from shared memory) where the TMEM budget allows it
// with 128-key tiles: d_c = 64 / 128.  For d_c = 192 / 256 (2 S buffers + O leave
// no room for Q at 128 keys) Q stays in shared memory; a Q-in-TMEM build with 96-key tiles was
// measured slower.  The KV ring is released by tcgen05.commit after the P V MMAs that last read a stage.
//
// The fused latent instance also does the two per-head projections around the attention (the
// technical summary's Method item 2: keys and values are rebuilt from the latent with the per-head
// up-projections).  Its tiles are 128 tokens of one head.  Prologue: q^nope (TMA, into the Q buffer) times
// W^K_up,h (TMA, into the last KV stage) on the tensor cores gives q~ in the TMEM O columns; the
// softmax warps round it to bf16 and write it, with RoPE3D(q^rope), into the Q buffer as the 128-byte /
// 64-byte swizzled K-major operand that TMA would have produced.  Epilogue: O / l (bf16) goes back into
// the Q buffer, W^V_up,h comes through the KV ring as one more "tile", and one MMA chain writes
// o = (O / l) W^V_up,h^T into the first S buffer, from which the softmax warps store it.  q_abs and the
// latent output never touch global memory.
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
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Of the 8 score pairs in each 16-key chunk, this many take 2^x from the FMA-pipe polynomial
// (exp2_poly2) and the rest from MUFU.EX2, which one warp per SM sub-partition would otherwise saturate
// (three: 1-1.8 % faster than two at d_c = 192 in interleaved runs on B200, four no better).
#ifndef VMLA_EXP2_POLY_PAIRS
#define VMLA_EXP2_POLY_PAIRS 3
#endif
constexpr int kPolyPairs = VMLA_EXP2_POLY_PAIRS;
// P of a tile is released to the P V MMAs in this many parts (consecutive key ranges), so that the
// MMAs of the first parts run while the softmax warps still exponentiate the rest.
#ifndef VMLA_P_PARTS
#define VMLA_P_PARTS 4
#endif
constexpr int kPParts = VMLA_P_PARTS;

struct AttnParams {
  const void* q;         // query rows (used when Q is kept in TMEM)
  int rows_per_b;        // query rows per batch element (token-major: Nq*H, head-major: Nq)
  int tiles_per_group;   // query tiles per (batch[, head]) group
  int heads;             // head-major: tile groups are (b, h); token-major: token = row / heads
  int64_t nq;            // query tokens per batch element
  int head_major;        // tiles are 128 tokens of one head (the fused layer)
  int64_t tok0;          // head-major: query row r is token tok0 + r of the call (a token range)
  FrameGeom g;
  float scale_log2;      // softmax_scale * log2(e)
  void* out;
  float* lse;
  int* status;
  uint64_t limit_ns;
  int drop_kv_tile;      // test hook: this KV tile is never loaded (-1: none)
  // fused latent layer only
  const void* q_rope;    // [B, Nq, H, 32] bf16: rotated in the prologue
  int d_nope;            // K of the absorbing MMA (multiple of 16, <= 128)
  int d_v;               // N of the value up-projection MMA (multiple of 32, <= BN)
  RopeTable rt;          // 3D-RoPE pairs of the query rotation
  Span out_span, lse_span;   // extents of out and lse (checked builds)
};

// Compile-time plan of one kernel instance.
//   KB    64-column boxes of the key tile from the c plane
//   KR    width of the rope box (0 or 32, 64-byte swizzle)
//   VB    64-column boxes of the value tile: V = the first VB key boxes (the latent c)
//   BN    keys per KV tile;  NS  TMEM S buffers (the MMA runs NS - 1 tiles ahead of P V)
//   Q_TMEM  whether Q lives in TMEM (the A operand of S = Q K^T) or in shared memory
//   ONES  V is extended by 16 columns of ones in shared memory, so that the P V MMA also produces
//         the row sum of P in O's column DV (the softmax then needs no add chains)
template <int KB, int KR, int VB, int BN, int NS, bool Q_TMEM, bool ONES, bool FUSED>
struct Plan {
  static constexpr int kDQK = 64 * KB + KR;
  static constexpr int kDV = 64 * VB;
  static constexpr int kNPV = kDV + (ONES ? 16 : 0);     // N of the P V MMA
  static constexpr int kBox = BN * 128;                 // [BN x 64] bf16 box, 128-byte swizzle
  static constexpr int kRopeBox = BN * 64;              // [BN x 32] bf16 box, 64-byte swizzle
  // Q buffer: the c boxes, then the rope box; the fused prologue first stages q^nope (two boxes) there
  static constexpr int kQBoxes = (FUSED && KB < 2) ? 2 : KB;
  static constexpr int kQRopeOff = kQBoxes * kBlockM * 128;
  static constexpr int kQBytes = Q_TMEM ? 0 : (kQRopeOff + (KR ? kBlockM * 64 : 0));
  // stage layout: c boxes (K, and V = the first VB of them) | ones box | rope box
  static constexpr int kOnesOff = KB * kBox;
  static constexpr int kRopeOff = kOnesOff + (ONES ? kBox : 0);
  static constexpr int kStageRaw = kRopeOff + (KR ? kRopeBox : 0);
  static constexpr int kStageBytes = (kStageRaw + 1023) / 1024 * 1024;
  static constexpr int kLoadBytes = KB * kBox + (KR ? kRopeBox : 0);
  static constexpr int kAuxBytes = 512;                 // barriers
  static constexpr int kBudget = 232448 - 1024 - kAuxBytes;
  static constexpr int kFit = (kBudget - kQBytes) / kStageBytes;
  static constexpr int kStages = kFit >= 6 ? 6 : kFit;
  static constexpr int kSmemBytes = kQBytes + kStages * kStageBytes + kAuxBytes + 1024;
  // TMEM columns: S buffers [b*BN, (b+1)*BN) for b < NS, O [NS*BN, NS*BN + NPV), Q after O
  static constexpr uint32_t kTmemO = NS * BN;
  static constexpr uint32_t kTmemQ = NS * BN + kNPV;
  static_assert(kStages >= NS, "shared memory too small for the KV ring");
  static_assert(kTmemQ + (Q_TMEM ? kDQK / 2 : 0) <= kTmemCols, "TMEM budget");
  static_assert(BN % 32 == 0 && BN <= 128 && NS >= 2 && NS <= 3, "tile shape");
  static_assert(kDV % 32 == 0 && (kDQK / 2) % 8 == 0, "row chunks");
  static_assert(!ONES || Q_TMEM, "the ones box is filled by the warps that also write Q into TMEM");
  static_assert(kNPV <= 256 && kNPV % 16 == 0, "P V MMA shape");
  // fused: q^nope (two 64-column boxes) and then O / l must fit the Q buffer
  static_assert(!FUSED || (!Q_TMEM && KR == 32 && !ONES &&
                           kQRopeOff >= 2 * kBlockM * 128 && kQRopeOff >= VB * kBlockM * 128),
                "fused layout");
};

template <int KB, int KR, int VB, int BN, int NS, bool Q_TMEM, bool ONES, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
attention_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_qr,
                 const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_kr,
                 const __grid_constant__ CUtensorMap map_wuk,
                 const __grid_constant__ CUtensorMap map_wuv, const AttnParams p) {
  using PL = Plan<KB, KR, VB, BN, NS, Q_TMEM, ONES, FUSED>;
  constexpr int NST = PL::kStages;
  constexpr int DV = PL::kDV;
  constexpr int kStepsPerPart = BN / 16 / kPParts;     // 16-key MMA steps per released part of P
  static_assert((BN / 16) % kPParts == 0, "P parts");
  constexpr int DQK = PL::kDQK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + PL::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NST * PL::kStageBytes);
  uint64_t* bar_q = bars;                 // 1: Q in place (TMA landed, or TMEM rows + ones box written)
  uint64_t* kv_full = bars + 1;           // NST
  uint64_t* kv_empty = kv_full + NST;     // NST
  uint64_t* s_full = kv_empty + NST;      // NS
  uint64_t* p_ready = s_full + NS;        // [NS][kPParts]: P of one part of the tile's keys written
  uint64_t* pv_done = p_ready + kPParts * NS;  // NS: P V of a tile of that S buffer completed
  uint64_t* drain = pv_done + NS;         // 1
  uint64_t* bar_pro = drain + 1;          // fused: q^nope and W^K_up,h landed
  uint64_t* qa_full = bar_pro + 1;        // fused: q~ = q^nope W^K_up,h complete in TMEM
  uint64_t* o_ready = qa_full + 1;        // fused: O / l written to shared memory (128 arrivals)
  uint64_t* out_full = o_ready + 1;       // fused: the value up-projection complete in TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(out_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;

  // ---- tile coordinates ----
  const int tile = blockIdx.x;
  const int group = tile / p.tiles_per_group;
  const int row0 = (tile % p.tiles_per_group) * kBlockM;      // first query row of the tile
  const int b = p.head_major ? group / p.heads : group;
  const int h = p.head_major ? group % p.heads : 0;
  const int tok_div = p.head_major ? 1 : p.heads;              // query row -> token
  const int last_row = min(row0 + kBlockM, p.rows_per_b) - 1;
  const int64_t tok_base = p.head_major ? p.tok0 : 0;
  const int64_t kend_first = key_end_rows(p.g, tok_base + row0 / tok_div);
  const int64_t kend_last = key_end_rows(p.g, tok_base + last_row / tok_div);
  const int n_kv = (int)((kend_last + BN - 1) / BN);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, (Q_TMEM || FUSED) ? 128 : 1);
    for (int s = 0; s < NST; ++s) { mbar_init(kv_full + s, 1); mbar_init(kv_empty + s, 1); }
    for (int s = 0; s < NS; ++s) {
      mbar_init(s_full + s, 1);
      for (int q = 0; q < kPParts; ++q) mbar_init(p_ready + kPParts * s + q, 128);
      mbar_init(pv_done + s, 1);
    }
    mbar_init(drain, 1);
    mbar_init(bar_pro, 1);
    mbar_init(qa_full, 1);
    mbar_init(o_ready, 128);
    mbar_init(out_full, 1);
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
      tma_prefetch_desc(&map_k);
      if (!Q_TMEM && !FUSED) {
        mbar_arrive_expect_tx(bar_q, PL::kQBytes);
        for (int i = 0; i < KB; ++i) tma_load_4d(sQ + i * kBlockM * 128, &map_q, bar_q, 64 * i, h, row0, b);
        if (KR) tma_load_4d(sQ + PL::kQRopeOff, &map_qr, bar_q, 64 * KB, h, row0, b);
      }
      if (FUSED) {
        // prologue operands: the q^nope tile (two 64-column boxes; columns past d_nope read as zeros)
        // into the Q buffer, W^K_up,h (d_c/64 boxes of [d_nope rows][64 columns]) into the last stage
        tma_prefetch_desc(&map_wuk);
        tma_prefetch_desc(&map_wuv);
        uint8_t* wst = sKV + (NST - 1) * PL::kStageBytes;
        mbar_arrive_expect_tx(bar_pro, 2 * kBlockM * 128 + VB * p.d_nope * 128);
        for (int i = 0; i < 2; ++i) tma_load_4d(sQ + i * kBlockM * 128, &map_q, bar_pro, 64 * i, h, row0, b);
        for (int i = 0; i < VB; ++i) tma_load_4d(wst + i * p.d_nope * 128, &map_wuk, bar_pro, 64 * i, 0, h, 0);
      }
      // load j goes to stage j % NST once the P V of load j - NST has completed; in the fused layer the
      // last stage first holds W^K_up,h until the prologue MMA has completed
      auto claim = [&](int j) -> bool {
        const int st = j % NST;
        if (j >= NST && !mbar_wait(kv_empty + st, ((j / NST) - 1) & 1, abort_flag, p.status, 1, p.limit_ns))
          return false;
        if (FUSED && j == NST - 1 && !mbar_wait(qa_full, 0, abort_flag, p.status, 8, p.limit_ns)) return false;
        return true;
      };
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % NST;
        if (!claim(j)) break;
        issued = j + 1;
        if (j == p.drop_kv_tile) continue;
        uint8_t* stage = sKV + st * PL::kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, PL::kLoadBytes);
        const int krow = j * BN;
        for (int i = 0; i < KB; ++i) tma_load_4d(stage + i * PL::kBox, &map_k, kv_full + st, 64 * i, 0, krow, b);
        if (KR) tma_load_4d(stage + PL::kRopeOff, &map_kr, kv_full + st, 0, 0, krow, b);
      }
      if (FUSED && issued == n_kv && claim(n_kv)) {
        // W^V_up,h (d_c/64 K-major boxes of [d_v rows][64 columns]) as load n_kv of the ring
        const int st = n_kv % NST;
        uint8_t* stage = sKV + st * PL::kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, VB * p.d_v * 128);
        for (int i = 0; i < VB; ++i) tma_load_4d(stage + i * p.d_v * 128, &map_wuv, kv_full + st, 64 * i, 0, h, 0);
        issued = n_kv + 1;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        if (!Q_TMEM && !FUSED) mbar_wait(bar_q, 0, &zero_flag, nullptr, 0, p.limit_ns);
        if (FUSED) mbar_wait(bar_pro, 0, &zero_flag, nullptr, 0, p.limit_ns);
        for (int j = (issued > NST ? issued - NST : 0); j < issued; ++j)
          if (j != p.drop_kv_tile) mbar_wait(kv_full + j % NST, (j / NST) & 1, &zero_flag, nullptr, 0, p.limit_ns);
      }
    }
  } else if (warp == 5) {
    // ================= MMA issuer =================
    if (elect_one()) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, PL::kNPV, 0, 1);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t kv_base = smem_u32(sKV);
      bool ok = true;
      if (FUSED) {
        ok = mbar_wait(bar_pro, 0, abort_flag, p.status, 9, p.limit_ns);
        if (ok) {
          tc_fence_after();
          // q~ = q^nope W^K_up,h into the O columns: A K-major (two 64-column boxes), B MN-major
          // ([d_nope rows][64 columns] boxes d_nope*128 B apart = LBO; a K step of 16 rows is 2048 B)
          const uint32_t w_base = kv_base + (NST - 1) * PL::kStageBytes;
          const uint32_t idesc_qa = idesc_bf16_f32(kBlockM, DV, 0, 1);
          for (int k = 0; k < p.d_nope / 16; ++k) {
            const uint64_t adesc = smem_desc(q_base + (k >> 2) * kBlockM * 128 + (k & 3) * 32, 16, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(w_base + k * 2048, p.d_nope * 128, 1024, kSwizzle128B);
            mma_ss(tmem + PL::kTmemO, adesc, bdesc, idesc_qa, k > 0 ? 1u : 0u);
          }
          mma_commit(qa_full);
        }
      }
      ok = ok && mbar_wait(bar_q, 0, abort_flag, p.status, 2, p.limit_ns);
      // P V of tile jp in kPParts parts of the keys: the first parts' MMAs run while the softmax warps
      // still produce the rest of P
      auto issue_pv = [&](int jp) -> bool {
        const int bp = jp % NS;
        const uint32_t v_base = kv_base + (jp % NST) * PL::kStageBytes;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          if (k % kStepsPerPart == 0) {
            if (!mbar_wait(p_ready + kPParts * bp + k / kStepsPerPart, (jp / NS) & 1, abort_flag, p.status, 3,
                           p.limit_ns))
              return false;
            tc_fence_after();
          }
          // V tile [BN keys][NPV] as MN-major operand: 8-key groups 1024 B apart (SBO), 64-column
          // boxes BN*128 B apart (LBO, the ones box being the last); a K step of 16 keys is 2048 B.
          const uint64_t vdesc = smem_desc(v_base + k * 2048, PL::kBox, 1024, kSwizzle128B);
          mma_ts(tmem + PL::kTmemO, tmem + bp * BN + k * 8, vdesc, idesc_pv, (jp > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(kv_empty + (jp % NST));
        mma_commit(pv_done + bp);
        return true;
      };
      if (ok) tc_fence_after();
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j % NST, bj = j % NS;
        if (!mbar_wait(kv_full + st, (j / NST) & 1, abort_flag, p.status, 4, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        // S buffer bj last held P_{j-NS}, whose P V was issued before this point (in order)
        const uint32_t k_base = kv_base + st * PL::kStageBytes;
        const uint32_t s_addr = tmem + bj * BN;
#pragma unroll
        for (int k = 0; k < KB * 4; ++k) {
          // 16 columns of the key tile: box k/4, 32-byte step k%4 inside the 128-byte swizzle atom
          const uint64_t kdesc = smem_desc(k_base + (k >> 2) * PL::kBox + (k & 3) * 32, 16, 1024, kSwizzle128B);
          if (Q_TMEM) {
            mma_ts(s_addr, tmem + PL::kTmemQ + k * 8, kdesc, idesc_qk, k > 0 ? 1u : 0u);
          } else {
            const uint64_t qdesc = smem_desc(q_base + (k >> 2) * kBlockM * 128 + (k & 3) * 32, 16, 1024, kSwizzle128B);
            mma_ss(s_addr, qdesc, kdesc, idesc_qk, k > 0 ? 1u : 0u);
          }
        }
        if (KR) {
#pragma unroll
          for (int k = 0; k < KR / 16; ++k) {
            const uint64_t kdesc = smem_desc(k_base + PL::kRopeOff + k * 32, 16, 512, kSwizzle64B);
            if (Q_TMEM) {
              mma_ts(s_addr, tmem + PL::kTmemQ + KB * 32 + k * 8, kdesc, idesc_qk, 1u);
            } else {
              const uint64_t qdesc = smem_desc(q_base + PL::kQRopeOff + k * 32, 16, 512, kSwizzle64B);
              mma_ss(s_addr, qdesc, kdesc, idesc_qk, 1u);
            }
          }
        }
        mma_commit(s_full + bj);
        if (j >= NS - 1 && !issue_pv(j - (NS - 1))) { ok = false; break; }
      }
      for (int jp = (n_kv > NS - 1 ? n_kv - (NS - 1) : 0); ok && jp < n_kv; ++jp)
        if (!issue_pv(jp)) ok = false;
      // every MMA of this CTA has completed before TMEM is released; the softmax warps also wait
      // on this single-phase barrier for the final O
      mma_commit(drain);
      if (FUSED) {
        if (ok) {
          const int st = n_kv % NST;
          ok = mbar_wait(kv_full + st, (n_kv / NST) & 1, abort_flag, p.status, 10, p.limit_ns) &&
               mbar_wait(o_ready, 0, abort_flag, p.status, 11, p.limit_ns);
          if (ok) {
            tc_fence_after();
            // o = (O / l) W^V_up,h^T into the first S buffer: A = O / l (bf16 K-major boxes in the Q
            // buffer, written after every earlier MMA completed), B = W^V_up,h (K-major boxes)
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
    // ========= query rows, softmax, epilogue (warps 0-3; thread = query row = TMEM lane) =========
    const int r = threadIdx.x;                      // 0..127
    const int row = row0 + r;
    const bool row_valid = row < p.rows_per_b;
    const int64_t kend = row_valid ? key_end_rows(p.g, tok_base + row / tok_div) : kend_last;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int64_t orow;                                   // this row's index in [rows of q / out / lse]
    if (p.head_major) orow = (((int64_t)b * p.nq + row) * p.heads + h);
    else orow = (int64_t)b * p.rows_per_b + row;

    if (Q_TMEM) {
      if (ONES) {
        // 16 columns of ones after V in every stage (bf16 1.0 everywhere in the box, so the swizzle
        // does not matter); made visible to the tensor cores' async proxy before bar_q is released
        constexpr int kWords = NST * PL::kBox / 16;
#pragma unroll 4
        for (int i = r; i < kWords; i += 128) {
          const int st = i / (PL::kBox / 16), w = i % (PL::kBox / 16);
          reinterpret_cast<uint4*>(sKV + st * PL::kStageBytes + PL::kOnesOff)[w] =
              make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        }
        fence_proxy_async_smem();
      }
      // the Q row as 32-bit words (bf16 pairs) into TMEM columns [kTmemQ, kTmemQ + DQK/2): exactly the
      // A-operand layout of a 128-row tcgen05.mma (row = lane, K pairs along columns)
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.q) + orow * DQK);
#pragma unroll
      for (int c0 = 0; c0 < DQK / 2; c0 += 8) {
        uint32_t w[8];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint4 v = row_valid ? src[c0 / 4 + q] : make_uint4(0, 0, 0, 0);
          w[4 * q + 0] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
        }
        tmem_st8(tmem + lane_base + PL::kTmemQ + c0, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_q);
    }

    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    if (FUSED) {
      // the Q row, written as the K-major operand TMA would have produced (16-byte chunk k of a
      // 128-byte row of a c box at chunk k ^ (row % 8); of a 64-byte rope row at chunk k ^ ((row / 2) % 4)).
      // First RoPE3D(q^rope) of the row's token into the rope box, which the prologue's TMA copies do not
      // touch, while the q^nope W^K_up,h MMA is still in flight; then q~ (fp32, O columns) as bf16.
      {
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
      const bool got = mbar_wait(qa_full, 0, abort_flag, p.status, 12, p.limit_ns);
      ok = __all_sync(0xffffffffu, got);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < DV / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + PL::kTmemO + c * 32, v);
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
    // Wait until P_{j-1} V_{j-1} has completed: phase (j-1)/NS of pv_done[(j-1) % NS].  Called from tile
    // j, where that barrier is at most one phase away: s_full[j] completing implies that
    // P_{j-1-NS} V_{j-1-NS} completed (issued before S_j), and P_{j-1+NS} V_{j-1+NS} cannot start
    // before this thread releases its P, so a parity wait is unambiguous.  Warp-uniform (__all_sync)
    // because the TMEM loads/stores that follow are warp-collective.
    auto wait_pv = [&](int k) -> bool {
      const bool got = mbar_wait(pv_done + k % NS, (k / NS) & 1, abort_flag, p.status, 5, p.limit_ns);
      return __all_sync(0xffffffffu, got);
    };
    const float sc = p.scale_log2;
    for (int j = 0; ok && j < n_kv; ++j) {
      const int bj = j % NS;
      const bool got = mbar_wait(s_full + bj, (j / NS) & 1, abort_flag, p.status, 6, p.limit_ns);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      // S row of this thread (raw scores): BN/32 TMEM loads, one wait
      float sr[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld32(tmem + lane_base + bj * BN + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + c * 32));
      tmem_ld_wait();
      const int64_t key0 = (int64_t)j * BN;
      if (key0 + BN > kend_first) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (key0 + i >= kend) sr[i] = -INFINITY;
      }
      // row max: 8 chains of 3-input max, then a tree (the scale is positive, applied after)
      static_assert(BN % 16 == 0 && BN >= 32, "max chains");
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = fmaxf(sr[q], sr[8 + q]);                 // keys 0..15
#pragma unroll
      for (int i = 16; i < BN; i += 16)                                              // keys i..i+15
#pragma unroll
        for (int q = 0; q < 8; ++q) mx[q] = fmax3(mx[q], sr[i + q], sr[i + 8 + q]);
      const float m_tile = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmaxf(fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_new = fmaxf(m_ref, m_tile * sc);
      const bool need = m_new > m_ref + kRescaleThreshold;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = fast_exp2(m_ref - m_new);   // 0 on the first tile
        if (j > 0) {
          if (!wait_pv(j - 1)) { ok = false; break; }
          tc_fence_after();
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < DV / 32; ++c) {
            tmem_ld32(tmem + lane_base + PL::kTmemO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_base + PL::kTmemO + c * 32, o);
          }
          if (ONES) {                                   // the row-sum column rescales with O
            tmem_ld16(tmem + lane_base + PL::kTmemO + DV, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(tmem + lane_base + PL::kTmemO + DV, *reinterpret_cast<uint32_t(*)[16]>(o));
          }
        }
        l_sum *= alpha;
        m_ref = m_new;
      }
      // p = 2^(s * scale*log2(e) - m): one packed FMA per pair of scores, then MUFU.EX2; P packed to
      // bf16 pairs over the first BN/2 columns of this S buffer (row sums: the ones columns of V, or
      // 4 packed chains)
      const float neg_m = -m_ref;
      float ls[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ls[i] = 0.f;
#pragma unroll
      for (int c = 0; c < BN / 16; ++c) {
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
          if (!ONES) fadd2(ls[(2 * i) & 7], ls[(2 * i + 1) & 7], p0, p1);
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st8(tmem + lane_base + bj * BN + c * 8, pk);
        if ((c + 1) % kStepsPerPart == 0 && c + 1 < BN / 16) {   // a part of the keys: release it to P V
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(p_ready + kPParts * bj + c / kStepsPerPart);
        }
      }
      if (!ONES) {
        fadd2(ls[0], ls[1], ls[4], ls[5]);
        fadd2(ls[2], ls[3], ls[6], ls[7]);
        fadd2(ls[0], ls[1], ls[2], ls[3]);
        l_sum += ls[0] + ls[1];
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_ready + kPParts * bj + kPParts - 1);
    }
    bool fin = ok && mbar_wait(drain, 0, abort_flag, p.status, 7, p.limit_ns);
    fin = __all_sync(0xffffffffu, fin && !*abort_flag);
    if (fin) {
      tc_fence_after();
      uint32_t o[32];
      float l_row = l_sum;
      if (ONES) {
        tmem_ld16(tmem + lane_base + PL::kTmemO + DV, o);
        tmem_ld_wait();
        l_row = __uint_as_float(o[0]);
      }
      const float inv_l = 1.f / l_row;
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
      if (FUSED) {
        // O / l rounded to bf16 into the Q buffer (every S = Q K^T MMA has completed): the A operand
        // of the value up-projection, same swizzled K-major layout as q~
#pragma unroll
        for (int c = 0; c < DV / 32; ++c) {
          tmem_ld32(tmem + lane_base + PL::kTmemO + c * 32, o);
          tmem_ld_wait();
          uint8_t* rowp = sQ + (c >> 1) * (kBlockM * 128) + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (c & 1) * 4 + q;
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
            *reinterpret_cast<uint4*>(rowp + ((chunk ^ (r & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(o_ready);
        bool got = mbar_wait(out_full, 0, abort_flag, p.status, 13, p.limit_ns);
        got = __all_sync(0xffffffffu, got && !*abort_flag);
        if (got) {
          tc_fence_after();
          for (int c = 0; c < p.d_v / 32; ++c) {
            tmem_ld32(tmem + lane_base + c * 32, o);
            tmem_ld_wait();
            if (row_valid && store_ok(p.out_span, out + orow * p.d_v + c * 32, 64, p.status, 9)) {
              uint4* dst = reinterpret_cast<uint4*>(out + orow * p.d_v + c * 32);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]), __uint_as_float(o[8 * q + 1]));
                v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]), __uint_as_float(o[8 * q + 3]));
                v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]), __uint_as_float(o[8 * q + 5]));
                v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]), __uint_as_float(o[8 * q + 7]));
                dst[q] = v;
              }
            }
          }
        }
      }
#pragma unroll
      for (int c = 0; c < (FUSED ? 0 : DV / 32); ++c) {
        tmem_ld32(tmem + lane_base + PL::kTmemO + c * 32, o);
        tmem_ld_wait();
        if (row_valid && store_ok(p.out_span, out + orow * DV + c * 32, 64, p.status, 7)) {
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
      if (row_valid && p.lse && store_ok(p.lse_span, p.lse + orow, 4, p.status, 8))
        p.lse[orow] = (m_ref + __log2f(l_row)) * 0.69314718055994530942f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int KB, int KR, int VB, int BN, int NS, bool Q_TMEM, bool ONES, bool FUSED>
cudaError_t launch_attention(const AttnMaps& m, const AttnParams& p, int n_tiles, cudaStream_t st) {
  using PL = Plan<KB, KR, VB, BN, NS, Q_TMEM, ONES, FUSED>;
  auto kern = attention_kernel<KB, KR, VB, BN, NS, Q_TMEM, ONES, FUSED>;
  static std::atomic<uint64_t> done{0};
  cudaError_t attr_err = ensure_smem_attr((const void*)kern, PL::kSmemBytes, done);
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<n_tiles, kThreads, PL::kSmemBytes, st>>>(m.q, m.qr, m.k, m.kr, m.wuk, m.wuv, p);
  count_launches(1);
  return cudaGetLastError();
}

// Instances (measured on B200; the softmax warps bound these kernels, the MMA side alone reaches the
// full tensor rate in every one of them):
//   latent d_c = 192 / 256: Q in shared memory, 128-key tiles, two S buffers (fastest per key);
//   latent d_c = 64 / 128: Q in TMEM, 128-key tiles, two S buffers.
// The three-buffer / 64-key / ones-column variant of the template is correct but slower at these
// shapes (its per-tile fixed costs outweigh the shorter dependency chain).
constexpr int kLatentBN = 128;

}  // namespace

vmla_status tc_check_latent_attention(const vmla_config& c) {
  if (c.d_rope != 32) { set_tc_reason("tensor-core latent attention needs d_rope == 32"); return VMLA_ERR_UNSUPPORTED; }
  if (c.d_c % 64 || c.d_c < 64 || c.d_c > 256) {
    set_tc_reason("tensor-core latent attention needs d_c in {64, 128, 192, 256}");
    return VMLA_ERR_UNSUPPORTED;
  }
  return VMLA_OK;
}

cudaError_t tc_latent_attention(const vmla_config& cfg, int batch, int64_t nq, const void* q_abs,
                                const void* c, const void* k_r, int64_t cap, int64_t valid_rows,
                                const FrameGeom& g, float scale, void* out, float* lse, int* status,
                                cudaStream_t st) {
  // d_c = 64 / 128: the softmax chain, not the tensor cores, bounds a single softmax warpgroup there
  if (tc_latent_split_supported(cfg))
    return tc_latent_attention_split(cfg, batch, nq, q_abs, c, k_r, cap, valid_rows, g, scale, out, lse, status, st);
  const int H = cfg.n_heads, dqk = cfg.d_c + cfg.d_rope;
  const int64_t rows = nq * H;
  const int kv_box_rows = kLatentBN;
  AttnMaps m{};
  cudaError_t e;
  // q_abs [B, Nq*H, d_qk] viewed as 4D {d_qk, 1, Nq*H, B} (only read by TMA when Q stays in smem)
  if ((e = make_map_4d(&m.q, q_abs, dqk, 1, rows, batch, (int64_t)dqk * 2, (int64_t)dqk * 2,
                       rows * dqk * 2, 64, 1, kBlockM, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.qr, q_abs, dqk, 1, rows, batch, (int64_t)dqk * 2, (int64_t)dqk * 2,
                       rows * dqk * 2, 32, 1, kBlockM, 64)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.k, c, cfg.d_c, 1, valid_rows, batch, (int64_t)cfg.d_c * 2, (int64_t)cfg.d_c * 2,
                       cap * cfg.d_c * 2, 64, 1, kv_box_rows, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.kr, k_r, 32, 1, valid_rows, batch, 64, 64, cap * 64, 32, 1, kv_box_rows, 64)) != cudaSuccess)
    return e;
  m.wuk = m.k;
  m.wuv = m.k;
  AttnParams p{};
  p.q = q_abs;
  p.rows_per_b = (int)rows;
  p.tiles_per_group = (int)((rows + kBlockM - 1) / kBlockM);
  p.heads = H;
  p.head_major = 0;
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
  switch (cfg.d_c) {
    case 192: return launch_attention<3, 32, 3, kLatentBN, 2, false, false, false>(m, p, n_tiles, st);
    default: return launch_attention<4, 32, 4, kLatentBN, 2, false, false, false>(m, p, n_tiles, st);
  }
}

namespace {

// Fused instances: Q in shared memory (the prologue writes it there), 128-key tiles, two S buffers.
template <int KB>
using FusedPlan = Plan<KB, 32, KB, kLatentBN, 2, false, false, true>;

template <int KB>
bool fused_fits(int d_nope, int d_v) {
  return KB * d_nope * 128 <= FusedPlan<KB>::kStageBytes && KB * d_v * 128 <= FusedPlan<KB>::kStageBytes;
}

}  // namespace

vmla_status tc_check_fused_attention(const vmla_config& c) {
  if (c.d_rope != 32) { set_tc_reason("fused latent attention needs d_rope == 32"); return VMLA_ERR_UNSUPPORTED; }
  if (c.d_c != 64 && c.d_c != 128 && c.d_c != 192 && c.d_c != 256) {
    set_tc_reason("fused latent attention needs d_c in {64, 128, 192, 256}");
    return VMLA_ERR_UNSUPPORTED;
  }
  if (c.d_nope % 16 || c.d_nope < 16 || c.d_nope > 128) {
    set_tc_reason("fused latent attention needs d_nope a multiple of 16 in [16, 128]");
    return VMLA_ERR_UNSUPPORTED;
  }
  if (c.d_v % 32 || c.d_v < 32 || c.d_v > kLatentBN) {
    set_tc_reason("fused latent attention needs d_v a multiple of 32 in [32, 128]");
    return VMLA_ERR_UNSUPPORTED;
  }
  const bool fits = c.d_c == 64 ? fused_fits<1>(c.d_nope, c.d_v)
                    : c.d_c == 128 ? fused_fits<2>(c.d_nope, c.d_v)
                    : c.d_c == 192 ? fused_fits<3>(c.d_nope, c.d_v) : fused_fits<4>(c.d_nope, c.d_v);
  if (!fits) { set_tc_reason("fused latent attention: up-projection weights exceed a KV stage"); return VMLA_ERR_UNSUPPORTED; }
  return VMLA_OK;
}

cudaError_t tc_latent_attention_fused(const vmla_config& cfg, int batch, int64_t tok0, int64_t nq,
                                      const void* q_nope, const void* q_rope, const void* w_uk, const void* w_uv,
                                      const void* c, const void* k_r, int64_t cap, int64_t valid_rows,
                                      const FrameGeom& g, const RopeTable& rt, float scale, void* out, float* lse,
                                      int* status, cudaStream_t st) {
  // d_c = 64 / 128: the softmax chain bounds a single softmax warpgroup; split each tile's keys
  if (tc_latent_split_fused_supported(cfg))
    return tc_latent_attention_split_fused(cfg, batch, tok0, nq, q_nope, q_rope, w_uk, w_uv, c, k_r, cap,
                                           valid_rows, g, rt, scale, out, lse, status, st);
  const int H = cfg.n_heads, dn = cfg.d_nope, dc = cfg.d_c, dv = cfg.d_v;
  AttnMaps m{};
  cudaError_t e;
  // q^nope [B, Nq, H, d_nope] as {d_nope, H, Nq, B}: a 128-token box of one head
  if ((e = make_map_4d(&m.q, q_nope, dn, H, nq, batch, (int64_t)dn * 2, (int64_t)H * dn * 2,
                       nq * H * dn * 2, 64, 1, kBlockM, 128)) != cudaSuccess) return e;
  m.qr = m.q;
  if ((e = make_map_4d(&m.k, c, dc, 1, valid_rows, batch, (int64_t)dc * 2, (int64_t)dc * 2,
                       cap * dc * 2, 64, 1, kLatentBN, 128)) != cudaSuccess) return e;
  if ((e = make_map_4d(&m.kr, k_r, 32, 1, valid_rows, batch, 64, 64, cap * 64, 32, 1, kLatentBN, 64)) != cudaSuccess)
    return e;
  // W^K_up [H, d_nope, d_c] as {d_c, d_nope, H, 1}: [d_nope rows][64 columns] boxes (MN-major B)
  if ((e = make_map_4d(&m.wuk, w_uk, dc, dn, H, 1, (int64_t)dc * 2, (int64_t)dn * dc * 2,
                       (int64_t)H * dn * dc * 2, 64, dn, 1, 128)) != cudaSuccess) return e;
  // W^V_up [H, d_v, d_c] as {d_c, d_v, H, 1}: [d_v rows][64 columns] boxes (K-major B)
  if ((e = make_map_4d(&m.wuv, w_uv, dc, dv, H, 1, (int64_t)dc * 2, (int64_t)dv * dc * 2,
                       (int64_t)H * dv * dc * 2, 64, dv, 1, 128)) != cudaSuccess) return e;
  AttnParams p{};
  p.q = q_nope;
  p.rows_per_b = (int)nq;
  p.tiles_per_group = (int)((nq + kBlockM - 1) / kBlockM);
  p.heads = H;
  p.head_major = 1;
  p.tok0 = tok0;
  p.nq = nq;
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
  switch (dc) {
    case 64: return launch_attention<1, 32, 1, kLatentBN, 2, false, false, true>(m, p, n_tiles, st);
    case 128: return launch_attention<2, 32, 2, kLatentBN, 2, false, false, true>(m, p, n_tiles, st);
    case 192: return launch_attention<3, 32, 3, kLatentBN, 2, false, false, true>(m, p, n_tiles, st);
    default: return launch_attention<4, 32, 4, kLatentBN, 2, false, false, true>(m, p, n_tiles, st);
  }
}

}  // namespace vmla
