// Block-sparse exact attention forward on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), bf16 inputs, fp32 accumulation.
//
// SLA post ("Selective Linear Attention", list "the idea"): critical blocks go
// through FlashAttention -- exact online-softmax attention -- and negligible
// blocks are skipped.  NABLA post point 4: compute only on the kept blocks.
//
// Work decomposition
//   * A CTA owns a 128-row query tile of one (batch, head): one query block
//     of 128 rows, or two consecutive query blocks of 64 rows.  A small plan
//     kernel merges the tile's critical lists into one ascending list of key
//     blocks with a membership bit per query block; key tiles are 128 keys
//     (one block of 128 or two listed blocks of 64).  A row only attends to
//     keys whose block is in its own query block's list (masked otherwise).
//   * Warp 0 (one lane): TMA producer -- Q once, then K and V per key tile
//     into a 2-stage ring, with the 3D tensor map [B*H, N, d] so rows past N
//     read as zeros.
//   * Warp 1 (one lane): MMA issuer -- S = Q K^T (M=128, N=128, K=d) into a
//     double-buffered TMEM tile, O += P V (M=128, N=d, K=128) into TMEM.
//   * Warps 2-5: one thread per query row -- tcgen05.ld of its S row, masking,
//     online softmax in the exp2 domain with lazy rescaling (the running max
//     is only moved when it grows by more than 2^8, which keeps P <= 256),
//     P as bf16 into a 128B-swizzled shared-memory tile, and the epilogue
//     O / l and LSE.  The row sum l accumulates the bf16-rounded P, the same
//     weights the PV product uses.
// Every mbarrier wait is bounded: on expiry the CTA records SLA_ERR_TIMEOUT
// in the status word, drains, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "tc_common.cuh"

namespace sla {

namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 128;
constexpr int kStages = 3;
constexpr int kSBuf = 3;  // S tiles in TMEM (P of a tile overwrites its S)
// One pair in kPolyEvery of a full tile's exponentials is computed by a cubic
// on the FMA pipe instead of the special-function unit (0: none).
constexpr int kPolyEvery = 3;
constexpr int kSoftmaxWarps = 8;                 // two warpgroups
constexpr int kThreads = 64 + 32 * kSoftmaxWarps;  // TMA warp, MMA warp, softmax
constexpr uint32_t kSmemRequest = 232448;          // 227 KB opt-in maximum
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

// ------------------------------------------------------------------ plan
// One key-tile descriptor packs two 16-bit entries (the second only used for
// key blocks of 64): bit 15 present, bits 13-14 membership (bit 13: query
// block of rows 0-63, bit 14: rows 64-127; both for a 128-row block), bits
// 0-12 key-block index.

constexpr uint32_t kPresent = kPlanPresent;

__device__ __forceinline__ uint32_t entry(int blk, uint32_t flags) {
  return kPresent | (flags << 13) | static_cast<uint32_t>(blk);
}

__global__ void plan_kernel(sla_block_lists rows, int BH, int nqb, int nkb, int nqt, int bq,
                            int bk, int32_t* __restrict__ cnt, uint32_t* __restrict__ tiles) {
  const int tile = blockIdx.x * blockDim.x + threadIdx.x;
  if (tile >= BH * nqt) return;
  const int bh = tile / nqt, qt = tile % nqt;
  const int qa = bq == 128 ? qt : 2 * qt;
  const int qb = (bq == 64 && 2 * qt + 1 < nqb) ? 2 * qt + 1 : -1;
  const uint32_t fa = bq == 128 ? 3u : 1u;
  const int ra = bh * nqb + qa;
  const int na = min(max(rows.crit_cnt[ra], 0), nkb);
  const int32_t* la = rows.crit_idx + i64(ra) * nkb;
  int nb = 0;
  const int32_t* lb = nullptr;
  if (qb >= 0) {
    const int rb = bh * nqb + qb;
    nb = min(max(rows.crit_cnt[rb], 0), nkb);
    lb = rows.crit_idx + i64(rb) * nkb;
  }
  uint32_t* out = tiles + i64(tile) * nkb;
  int ia = 0, ib = 0, nt = 0;
  uint32_t pending = 0;
  const int per_tile = kTileN / bk;  // 1 or 2 entries per key tile
  int in_tile = 0;
  while (ia < na || ib < nb) {
    const int a = ia < na ? la[ia] : 0x7fffffff;
    const int b = ib < nb ? lb[ib] : 0x7fffffff;
    int blk;
    uint32_t f;
    if (a == b) { blk = a; f = fa | 2u; ++ia; ++ib; }
    else if (a < b) { blk = a; f = fa; ++ia; }
    else { blk = b; f = 2u; ++ib; }
    if (blk < 0 || blk >= nkb) continue;  // malformed list entry
    pending |= entry(blk, f) << (16 * in_tile);
    if (++in_tile == per_tile) {
      out[nt++] = pending;
      pending = 0;
      in_tile = 0;
      if (nt == nkb) break;  // only reachable with duplicated list entries
    }
  }
  if (in_tile && nt < nkb) out[nt++] = pending;
  cnt[tile] = nt;
}

// ------------------------------------------------------------------ kernel

}  // namespace

// What the kernel writes once the rows are done.  Sparse-only use writes
// o_s; the fused forward writes `out` (bf16), adding the linear branch of
// the tile's query blocks when `marg_cnt` is set: O_lin = phi(Q) H^M /
// (phi(Q) . z^M) from the gathered summaries, then out = O_s + O_lin W.
struct AttnEpilogue {
  float* o_s;                 // [B*H, N, d] fp32, nullable
  float* lse;                 // [B*H, N] fp32
  __nv_bfloat16* out;         // [B*H, N, d] bf16, nullable
  float* o_lin;               // [B*H, N, d] fp32, nullable (linear branch on)
  const float* zm;            // [B*H*Nqb, 128] z^M (linear branch on)
  const int32_t* marg_cnt;    // [B*H*Nqb] marginal counts; nullptr: branch off
  int nqb;
};

namespace {

template <int D, int BQ, int BK>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmHM,
               const __grid_constant__ CUtensorMap tmW, const int32_t* __restrict__ plan_cnt,
               const uint32_t* __restrict__ plan_tiles, int plan_stride, AttnEpilogue ep,
               int32_t* status, int N, int nqt, float scale_log2, long long timeout_cycles,
               int debug_skip) {
  constexpr int DC = D / 64;                  // 64-element (128 B) chunks along d
  constexpr int DH = D / 2;                   // O columns per softmax half
  constexpr uint32_t kQBytes = DC * 16384;    // Q tile 128 x D bf16
  constexpr uint32_t kKBytes = DC * 16384;    // K (or V) tile 128 x D
  constexpr uint32_t offQ = 0;
  constexpr uint32_t offK = offQ + kQBytes;
  constexpr uint32_t offV = offK + kStages * kKBytes;
  constexpr uint32_t offOL = offK + 2 * kKBytes;       // O_lin (bf16) after the loop: K stage 2
  constexpr uint32_t offRed = offV + kStages * kKBytes;  // [2 parity][2 halves][128] fp32
  constexpr uint32_t offBar = offRed + 2 * 2 * 128 * 4;
  constexpr uint32_t kUsed = offBar + 512;
  constexpr uint32_t idesc_qk = idesc_bf16(128, kTileN, 0, 0);
  constexpr uint32_t idesc_pv = idesc_bf16(128, D, 0, 1);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* base = smem_raw + pad;
  const uint32_t sb = raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + offBar);
  constexpr int kB0 = 1 + 4 * kStages;            // first barrier after the K/V rings
  const uint32_t b_q = smem_u32(&bars[0]);
  auto b_k_full = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_v_full = [&](int s) { return smem_u32(&bars[1 + kStages + s]); };
  auto b_k_empty = [&](int s) { return smem_u32(&bars[1 + 2 * kStages + s]); };
  auto b_v_empty = [&](int s) { return smem_u32(&bars[1 + 3 * kStages + s]); };
  // per S buffer j = t % kSBuf: S(t) in TMEM, P(t) in TMEM (8 warps), P V of
  // tile t done
  auto b_s_full = [&](int j) { return smem_u32(&bars[kB0 + j]); };
  auto b_p_full = [&](int j) { return smem_u32(&bars[kB0 + kSBuf + j]); };
  auto b_pv_done = [&](int j) { return smem_u32(&bars[kB0 + 2 * kSBuf + j]); };
  constexpr int kB1 = kB0 + 3 * kSBuf;
  // partial row maxima exchanged between the two warps holding the same 32
  // rows (one per column half): one barrier per (tile parity, lane quadrant)
  auto b_red = [&](int b, int quad) { return smem_u32(&bars[kB1 + 9 + 4 * b + quad]); };
  const uint32_t b_fin = smem_u32(&bars[kB1 + 0]);
  const uint32_t b_lin = smem_u32(&bars[kB1 + 1]);   // H^M and W tiles landed
  const uint32_t b_phiq = smem_u32(&bars[kB1 + 2]);  // phi(Q) written (8 warps)
  const uint32_t b_den = smem_u32(&bars[kB1 + 3]);   // normaliser halves exchanged (8 warps)
  const uint32_t b_num = smem_u32(&bars[kB1 + 4]);   // phi(Q) H^M in TMEM
  const uint32_t b_olin = smem_u32(&bars[kB1 + 5]);  // O_lin (bf16) in shared memory (8 warps)
  const uint32_t b_lout = smem_u32(&bars[kB1 + 6]);  // O_lin W in TMEM
  // every P V product done (single use).  The producer cannot wait on
  // pv_done for this: the completion before the last one on the same
  // barrier may still be pending, and a parity wait would then take the
  // older phase for the newer one.
  const uint32_t b_pv_last = smem_u32(&bars[kB1 + 7]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[kB1 + 17]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[kB1 + 18]);
  static_assert((kB1 + 19) * 8 <= kUsed - offBar, "barrier block too small");
  float* red = reinterpret_cast<float*>(base + offRed);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x;
  const int bh = tile / nqt, qt = tile % nqt;
  const int T = plan_cnt[tile];
  const uint32_t* ptiles = plan_tiles + i64(tile) * plan_stride;
  // linear branch of this tile's query blocks (A: rows 0-63 or the whole
  // 128-row block, B: rows 64-127 when blocks are 64 rows)
  const int nqb = ep.nqb;
  const int qa = BQ == 128 ? qt : 2 * qt;
  const int qb2 = (BQ == 64 && 2 * qt + 1 < nqb) ? 2 * qt + 1 : -1;
  int nm_a = 0, nm_b = 0;
  if (D == 128 && ep.marg_cnt) {
    nm_a = ep.marg_cnt[bh * nqb + qa];
    if (qb2 >= 0) nm_b = ep.marg_cnt[bh * nqb + qb2];
  }
  const bool lin = nm_a > 0 || nm_b > 0;

  // The dynamic window must hold the 1024-aligned layout; it does whenever
  // the window starts 1024-aligned (then pad == 0).  Refuse otherwise.
  if (pad + kUsed > kSmemRequest) {
    if (threadIdx.x == 0) atomicExch(status, static_cast<int32_t>(SLA_ERR_UNSUPPORTED));
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(b_k_full(s), 1);
      mbar_init(b_v_full(s), 1);
      mbar_init(b_k_empty(s), 1);
      mbar_init(b_v_empty(s), 1);
    }
    for (int j = 0; j < kSBuf; ++j) {
      mbar_init(b_s_full(j), 1);
      mbar_init(b_p_full(j), kSoftmaxWarps);
      mbar_init(b_pv_done(j), 1);
    }
    for (int b = 0; b < 2; ++b)
      for (int q = 0; q < 4; ++q) mbar_init(b_red(b, q), 2);
    mbar_init(b_fin, kSoftmaxWarps);
    mbar_init(b_lin, 1);
    mbar_init(b_phiq, kSoftmaxWarps);
    mbar_init(b_den, kSoftmaxWarps);
    mbar_init(b_num, 1);
    mbar_init(b_olin, kSoftmaxWarps);
    mbar_init(b_lout, 1);
    mbar_init(b_pv_last, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // TMEM: 512 columns (S0 | S1 | S2 | O)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // columns: S of tile t at 128 (t % kSBuf), O at 384.  The bf16 P of tile t
  // (two keys per column) overwrites its own S: the column half h puts its
  // 32 P columns at 64 h, columns that only its own threads read.
  // Addresses are computed, not indexed from an array, so none goes through
  // local memory.
  auto tS = [&](int j) { return tmem + 128u * static_cast<uint32_t>(j); };
  const uint32_t tO = tmem + 384;

  auto give_up = [&]() {
    *abort_flag = 1;
    atomicExch(status, static_cast<int32_t>(SLA_ERR_TIMEOUT));
  };
  // bounded wait: false on timeout or when another role gave up
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    const long long t0 = clock64();
    for (uint32_t it = 0;; ++it) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((it & 255u) == 255u) {
        if (*abort_flag) return false;
        if (clock64() - t0 > timeout_cycles) { give_up(); return false; }
      }
    }
  };

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    // K of tile t+2 may load once S of tile t has been computed; V of tile
    // t+2 once P V of tile t has: the two rings advance independently.
    if (lane == 0 && (T > 0 || lin)) {
      mbar_expect_tx(b_q, kQBytes);
#pragma unroll
      for (int c = 0; c < DC; ++c) tma_load_3d(sb + offQ + c * 16384, &tmQ, c * 64, qt * kTileM, bh, b_q);
      auto load = [&](const CUtensorMap* map, uint32_t dst0, uint32_t bar, uint32_t desc) {
        mbar_expect_tx(bar, kKBytes);
        if (BK == 128) {
          const int blk = desc & 0x1FFF;
#pragma unroll
          for (int c = 0; c < DC; ++c) tma_load_3d(dst0 + c * 16384, map, c * 64, blk * 128, bh, bar);
        } else {
          const int blk0 = desc & 0x1FFF;
          const int blk1 = ((desc >> 16) & kPresent) ? (desc >> 16) & 0x1FFF : blk0;
#pragma unroll
          for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int c = 0; c < DC; ++c)
              tma_load_3d(dst0 + c * 16384 + e * 8192, map, c * 64, (e ? blk1 : blk0) * 64, bh, bar);
        }
      };
      int tk = 0, tv = 0;
      long long t0 = clock64();
      while (tv < T) {
        bool moved = false;
        if (tk < T && (tk < kStages || mbar_try_wait(b_k_empty(tk % kStages), ((tk / kStages) & 1) ^ 1))) {
          if (!(debug_skip && tile == 0 && tk == 0))  // test aid: tile 0's K never arrives
            load(&tmK, sb + offK + (tk % kStages) * kKBytes, b_k_full(tk % kStages), ptiles[tk]);
          ++tk;
          moved = true;
        }
        if (tv < tk && (tv < kStages || mbar_try_wait(b_v_empty(tv % kStages), ((tv / kStages) & 1) ^ 1))) {
          load(&tmV, sb + offV + (tv % kStages) * kKBytes, b_v_full(tv % kStages), ptiles[tv]);
          ++tv;
          moved = true;
        }
        if (moved) {
          t0 = clock64();
        } else {
          if (*abort_flag) break;
          if (clock64() - t0 > timeout_cycles) { give_up(); break; }
        }
      }
      // linear branch: H^M of the tile's query blocks and W go into the K/V
      // stages once the last P V product has read them
      if (lin && tv == T && (T == 0 || wait(b_pv_last, 0))) {
        mbar_expect_tx(b_lin, (nm_a > 0 ? 32768u : 0u) + (nm_b > 0 ? 32768u : 0u) + 32768u);
        if (nm_a > 0) {
          tma_load_2d(sb + offK, &tmHM, 0, (bh * nqb + qa) * 128, b_lin);
          tma_load_2d(sb + offK + 16384, &tmHM, 64, (bh * nqb + qa) * 128, b_lin);
        }
        if (nm_b > 0) {
          tma_load_2d(sb + offK + kKBytes, &tmHM, 0, (bh * nqb + qb2) * 128, b_lin);
          tma_load_2d(sb + offK + kKBytes + 16384, &tmHM, 64, (bh * nqb + qb2) * 128, b_lin);
        }
        tma_load_2d(sb + offV, &tmW, 0, 0, b_lin);
        tma_load_2d(sb + offV + 16384, &tmW, 64, 0, b_lin);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && T > 0) {
      bool ok = wait(b_q, 0);
      // base descriptors, built once; each MMA advances one by a constant
      const uint64_t dQ = sdesc(sb + offQ, 16, 1024);
      const uint64_t dK0 = sdesc(sb + offK, 16, 1024);
      const uint64_t dV0 = sdesc(sb + offV, 16384, 1024);
      auto issue_s = [&](int t) -> bool {
        const int s = t % kStages, j = t % kSBuf;
        if (!wait(b_k_full(s), (t / kStages) & 1)) return false;
        // S(t) takes the buffer of tile t - kSBuf: that tile's softmax is done
        // (its P V was issued after its P arrived, before this call) and the
        // tensor pipe reads that P before this MMA overwrites it (it runs in
        // issue order)
        tc_fence_after();
        const uint64_t dK = sdesc_add(dK0, s * kKBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
          tc_mma(tS(j), sdesc_add(dQ, off), sdesc_add(dK, off), idesc_qk, kk > 0);
        }
        tc_commit(b_s_full(j));
        tc_commit(b_k_empty(s));
        return true;
      };
      auto issue_pv = [&](int t) -> bool {
        const int s = t % kStages, j = t % kSBuf;
        if (!wait(b_p_full(j), (t / kSBuf) & 1)) return false;
        if (!wait(b_v_full(s), (t / kStages) & 1)) return false;
        tc_fence_after();
        const uint64_t dV = sdesc_add(dV0, s * kKBytes);
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk)  // 16 keys = 8 TMEM columns of P
          tc_mma_ts(tO, tS(j) + 64 * (kk / 4) + (kk % 4) * 8, sdesc_add(dV, kk * 2048), idesc_pv,
                    (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(b_v_empty(s));
        tc_commit(b_pv_done(j));
        return true;
      };
      // S(t + 2) is issued before the wait for P(t) (its buffer was last
      // read by P V of tile t - 1, issued in the previous round), so the
      // tensor pipe computes it while the softmax works on tile t, and a
      // softmax warp that finishes a tile finds the next S already done
      if (ok) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int t = 0; ok && t < T; ++t) {
        if (t + 2 < T) ok = issue_s(t + 2);
        if (ok) ok = issue_pv(t);
      }
      if (ok) tc_commit(b_pv_last);
    }
    if (lane == 0 && lin) {
      bool ok = wait(b_lin, 0) && wait(b_phiq, 0);
      if (ok) {
        // num = phi(Q) H^M: M = 128 rows, N = 128 channels, K = 128 (A = phi(Q)
        // K-major in the Q tile, B = H^M rows of channels, MN-major)
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 1);
        for (int q2 = 0; q2 < 2; ++q2) {
          if ((q2 == 0 ? nm_a : nm_b) <= 0) continue;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
            tc_mma(tS(q2), sdesc(sb + offQ + off, 16, 1024),
                   sdesc(sb + offK + q2 * kKBytes + kk * 2048, 16384, 1024), idesc, kk > 0);
          }
        }
        tc_commit(b_num);
        ok = wait(b_olin, 0);
      }
      if (ok) {
        // O_lin W: A = O_lin (bf16, K-major, in K stage 2), B = W (MN-major)
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
          tc_mma(tS(0), sdesc(sb + offOL + off, 16, 1024), sdesc(sb + offV + kk * 2048, 16384, 1024),
                 idesc, kk > 0);
        }
        tc_commit(b_lout);
      }
    }
  } else {
    // ---------------------------------------------------------- softmax
    // Two warpgroups; thread (h, r) owns columns [64h, 64h + 64) of query
    // row r and O columns [h*D/2, (h+1)*D/2).  The two halves of a row
    // exchange their partial maxima through shared memory every tile, so
    // both keep the same running max and rescale decisions.
    const int h = (warp - 2) >> 2;        // column half
    const int quad = warp & 3;            // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;       // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t rflag = BQ == 128 ? 3u : (r < 64 ? 1u : 2u);
    const unsigned full = 0xffffffffu;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    // the plan word of the next tile is fetched a tile ahead: a global load
    // on the path from one tile to the next would stall every warp
    uint32_t desc_next = T > 0 ? ptiles[0] : 0u;
    for (int t = 0; ok && t < T; ++t) {
      const int b = t & 1, j = t % kSBuf;
      const uint32_t desc = desc_next;
      if (t + 1 < T) desc_next = ptiles[t + 1];
      // this thread's 64 keys: entry h of a tile of two 64-blocks, or half h
      // of one 128-block
      const uint32_t ent = BK == 64 ? (desc >> (16 * h)) & 0xFFFFu : desc & 0xFFFFu;
      const int blk = ent & 0x1FFF;
      const bool member = (ent & kPresent) && (((ent >> 13) & 3u) & rflag);
      const int kvalid = member ? max(0, min(64, N - blk * BK - (BK == 128 ? h * 64 : 0))) : 0;
      if (!__all_sync(full, wait(b_s_full(j), (t / kSBuf) & 1))) { ok = false; break; }
      tc_fence_after();
      float s[64];
      tmem_ld32(tS(j) + lane_off + h * 64, s);
      tmem_ld32(tS(j) + lane_off + h * 64 + 32, s + 32);
      tmem_wait_ld();
      reg_fence<64>(s);
      // partial max of the raw scores over this thread's valid keys (four
      // independent three-input chains)
      float mx = -INFINITY;
      if (kvalid == 64) {
        float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          a0 = max3(a0, s[c], s[c + 1]);
          a1 = max3(a1, s[c + 2], s[c + 3]);
          a2 = max3(a2, s[c + 4], s[c + 5]);
          a3 = max3(a3, s[c + 6], s[c + 7]);
        }
        mx = max3(a0, a1, fmaxf(a2, a3));
      } else if (kvalid > 0) {
#pragma unroll
        for (int c = 0; c < 64; ++c) mx = c < kvalid ? fmaxf(mx, s[c]) : mx;
      }
      red[(b * 2 + h) * 128 + r] = mx;
      __syncwarp();
      if (lane == 0) mbar_arrive(b_red(b, quad));
      if (!__all_sync(full, wait(b_red(b, quad), (t >> 1) & 1))) { ok = false; break; }
      const float mo = red[(b * 2 + (h ^ 1)) * 128 + r];
      const float mraw = fmaxf(mx, mo);
      // running max (scaled, log2 domain) with lazy rescale
      bool rescale = false;
      float alpha = 1.f;
      if (mraw > -INFINITY) {
        const float mt = mraw * scale_log2;
        if (m_ref == -INFINITY) {
          m_ref = mt;
        } else if (mt > m_ref + kRescaleLog2) {
          alpha = exp2f(m_ref - mt);
          m_ref = mt;
          l *= alpha;
          rescale = true;
        }
      }
      // P = 2^(s * scale_log2 - m_ref) rounded to bf16.  The row sum uses the
      // rounded weights the MMA sees, so O / l is an exact convex
      // combination of V rows.
      uint32_t pk[32];
      float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0, acc2 = acc0, acc3 = acc0;
      const float2 sc2 = make_float2(scale_log2, scale_log2);
      const float2 nm2 = make_float2(-m_ref, -m_ref);
      if (kvalid == 64) {
        // every kPolyEvery-th pair of exponentials goes to the FMA pipe
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 x = fma2(make_float2(s[2 * i], s[2 * i + 1]), sc2, nm2);
          const float2 e = (kPolyEvery > 0 && i % kPolyEvery == kPolyEvery - 1)
                               ? exp2_poly2(x)
                               : make_float2(fast_exp2(x.x), fast_exp2(x.y));
          pk[i] = pack_bf16x2(e.x, e.y);
        }
      } else if (kvalid > 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 x = fma2(make_float2(s[2 * i], s[2 * i + 1]), sc2, nm2);
          pk[i] = pack_bf16x2(2 * i < kvalid ? fast_exp2(x.x) : 0.f,
                              2 * i + 1 < kvalid ? fast_exp2(x.y) : 0.f);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        acc0 = add2(acc0, make_float2(__uint_as_float(pk[i] << 16), __uint_as_float(pk[i] & 0xFFFF0000u)));
        acc1 = add2(acc1, make_float2(__uint_as_float(pk[i + 1] << 16), __uint_as_float(pk[i + 1] & 0xFFFF0000u)));
        acc2 = add2(acc2, make_float2(__uint_as_float(pk[i + 2] << 16), __uint_as_float(pk[i + 2] & 0xFFFF0000u)));
        acc3 = add2(acc3, make_float2(__uint_as_float(pk[i + 3] << 16), __uint_as_float(pk[i + 3] & 0xFFFF0000u)));
      }
      acc0 = add2(add2(acc0, acc1), add2(acc2, acc3));
      l += acc0.x + acc0.y;
      // P (bf16 pairs) over this half's own S columns: its 64 keys become
      // columns [64h, 64h + 32) of the tile's buffer
      tmem_st32u(tS(j) + lane_off + h * 64, pk);
      // rescale this half of O (warp-wide TMEM access) once the previous
      // P V is complete.  That parity wait cannot mistake an older phase:
      // S(t) has completed and was issued after P V of tile t - 3, so P V of
      // tile t - 4 (the barrier's previous use) is complete.
      if (__any_sync(full, rescale)) {
        if (t >= 1 && !__all_sync(full, wait(b_pv_done((t - 1) % kSBuf), ((t - 1) / kSBuf) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < DH; c += 32) {
          float o[32];
          tmem_ld32(tO + lane_off + h * DH + c, o);
          tmem_wait_ld();
          reg_fence<32>(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + lane_off + h * DH + c, o);
        }
      }
      tmem_wait_st();  // P (and any rescaled O) stored
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_p_full(j));
    }
    // epilogue: total row sum from both halves, O / l, LSE
    const int fb = T & 1;  // red slot last used by tile T-2, read by all
    red[(fb * 2 + h) * 128 + r] = l;
    __syncwarp();
    if (lane == 0) mbar_arrive(b_fin);
    bool fin = ok && __all_sync(full, wait(b_fin, 0));
    const float ltot = fin ? l + red[(fb * 2 + (h ^ 1)) * 128 + r] : 0.f;
    const int row = qt * kTileM + r;
    const i64 orow = (i64(bh) * N + row) * D + h * DH;
    const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
    // all P V products done: O final in TMEM, Q, the K/V stages and the S
    // columns free
    // linear branch: this thread's half row of z^M (channels [64h, 64h + 64)),
    // fetched in one batch while the last P V products finish
    const bool second = BQ == 64 && r >= 64;
    const int nm_r = second ? nm_b : nm_a;
    float4 z4[16];
    if (D == 128 && lin && nm_r > 0) {
      const float4* zp = reinterpret_cast<const float4*>(
          ep.zm + (i64(bh) * nqb + (second ? qb2 : qa)) * 128 + h * 64);
#pragma unroll
      for (int i = 0; i < 16; ++i) z4[i] = __ldg(zp + i);
    }
    if (fin && T > 0)
      fin = __all_sync(full, wait(b_pv_done((T - 1) % kSBuf), ((T - 1) / kSBuf) & 1));
    bool lin_ok = false;
    if (D == 128 && lin && fin) {  // (never taken for d = 64: lin is false)
      // phi(Q) in place (this thread: row r, channels [64h, 64h + 64)), and
      // half of the normaliser phi(q) . z^M from the same rounded values
      float dpart = 0.f, dpart2 = 0.f;
      lin_ok = __all_sync(full, wait(b_q, 0));
      if (lin_ok) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint4* p = reinterpret_cast<uint4*>(base + offQ + h * 16384 + sw128(r, u));
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (row < N && nm_r > 0) {
            val = phi_unit(*p);
            const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.x));
            const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.y));
            const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.z));
            const float2 f3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.w));
            const float4 za = z4[2 * u], zb = z4[2 * u + 1];
            dpart = fmaf(f0.x, za.x, fmaf(f0.y, za.y, fmaf(f1.x, za.z, fmaf(f1.y, za.w, dpart))));
            dpart2 = fmaf(f2.x, zb.x, fmaf(f2.y, zb.y, fmaf(f3.x, zb.z, fmaf(f3.y, zb.w, dpart2))));
          }
          *p = val;
        }
        dpart += dpart2;
        const int db = fb ^ 1;  // slot of tile T-1, read by all before b_fin
        red[(db * 2 + h) * 128 + r] = dpart;
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) { mbar_arrive(b_phiq); mbar_arrive(b_den); }
        lin_ok = __all_sync(full, wait(b_den, 0));
      }
      float den = 0.f;
      if (lin_ok) den = dpart + red[((fb ^ 1) * 2 + (h ^ 1)) * 128 + r];
      if (lin_ok) lin_ok = __all_sync(full, wait(b_num, 0));
      if (lin_ok) {
        // O_lin = phi(Q) H^M / den -> o_lin (fp32, optional) and bf16 into K
        // stage 2 as the A operand of the projection
        tc_fence_after();
        const uint32_t tn = tS(second ? 1 : 0);
        const float dinv = (nm_r > 0 && den > 0.f) ? 1.f / den : 0.f;
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          float v[32];
          tmem_ld32(tn + lane_off + h * 64 + c, v);
          tmem_wait_ld();
          reg_fence<32>(v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = nm_r > 0 ? v[i] * dinv : 0.f;  // TMEM unwritten when no list
          if (ep.o_lin && row < N) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(ep.o_lin + orow + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          }
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(base + offOL + h * 16384 + sw128(r, c / 8 + q4)) =
                make_uint4(pack_bf16x2(v[8 * q4], v[8 * q4 + 1]), pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                           pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]), pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
        }
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_olin);
        lin_ok = __all_sync(full, wait(b_lout, 0));
        if (lin_ok) tc_fence_after();
      }
    } else if (ep.o_lin && row < N) {
      for (int c = 0; c < DH; c += 4)
        *reinterpret_cast<float4*>(ep.o_lin + orow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // final: O / l (+ O_lin W) -> out (bf16) and / or o_s (fp32)
#pragma unroll
    for (int c = 0; c < DH; c += 32) {
      float o[32];
      if (fin && T > 0) {
        tmem_ld32(tO + lane_off + h * DH + c, o);
        tmem_wait_ld();
        reg_fence<32>(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= inv;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      if (row < N && ep.o_s) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(ep.o_s + orow + c + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
      }
      if (ep.out) {
        if (D == 128 && lin_ok) {
          float lo[32];
          tmem_ld32(tS(0) + lane_off + h * DH + c, lo);
          tmem_wait_ld();
          reg_fence<32>(lo);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] += lo[i];
        }
        if (row < N) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(ep.out + orow + c + 8 * q4) =
                make_uint4(pack_bf16x2(o[8 * q4], o[8 * q4 + 1]), pack_bf16x2(o[8 * q4 + 2], o[8 * q4 + 3]),
                           pack_bf16x2(o[8 * q4 + 4], o[8 * q4 + 5]), pack_bf16x2(o[8 * q4 + 6], o[8 * q4 + 7]));
        }
      }
    }
    if (row < N && h == 0)
      ep.lse[i64(bh) * N + row] = ltot > 0.f ? (m_ref + log2f(ltot)) * 0.69314718055994531f : -INFINITY;
  }

  // teardown: on an abort let in-flight copies and MMAs drain (bounded)
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) { __nanosleep(1000); }
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ------------------------------------------------------------------ host

// [B*H, N, d] bf16 viewed as a 3D tensor (d fastest); box of 64 x rows x 1
// with 128-byte swizzle, rows past N read as zeros.
bool make_map(CUtensorMap* m, const void* ptr, const Geom& g, int rows) {
  const uint64_t dims[3] = {static_cast<uint64_t>(g.d), static_cast<uint64_t>(g.N),
                            static_cast<uint64_t>(g.BH)};
  const uint64_t strides[2] = {static_cast<uint64_t>(g.d) * 2, static_cast<uint64_t>(g.N) * g.d * 2};
  const uint32_t box[3] = {64, static_cast<uint32_t>(rows), 1};
  return encode_bf16_map(m, ptr, 3, dims, strides, box);
}

template <int D, int BQ, int BK>
cudaError_t launch_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mhm, const CUtensorMap& mw, const int32_t* cnt,
                     const uint32_t* tiles, const Geom& g, int nqt, const AttnEpilogue& ep,
                     int32_t* status, cudaStream_t s) {
  auto kern = attn_tc_kernel<D, BQ, BK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemRequest));
  if (e != cudaSuccess) return e;
  const float scale_log2 = g.scale * 1.4426950408889634f;
  const bool debug = (g.flags & SLA_FLAG_DEBUG_TIMEOUT) != 0;
  const long long timeout = debug ? (1ll << 24) : (1ll << 31);
  kern<<<g.BH * nqt, kThreads, kSmemRequest, s>>>(mq, mk, mv, mhm, mw, cnt, tiles, g.nkb, ep, status,
                                                  g.N, nqt, scale_log2, timeout, debug ? 1 : 0);
  return cudaGetLastError();
}

struct PlanPtrs {
  int32_t* cnt;
  uint32_t* tiles;
};

PlanPtrs plan_ptrs(const Geom& g, void* scratch) {
  const int nqt = (g.N + kTileM - 1) / kTileM;
  const size_t ntiles = static_cast<size_t>(g.BH) * nqt;
  PlanPtrs p;
  p.cnt = static_cast<int32_t*>(scratch);
  p.tiles = reinterpret_cast<uint32_t*>(static_cast<char*>(scratch) +
                                        ((ntiles * sizeof(int32_t) + 255) & ~size_t(255)));
  return p;
}

}  // namespace

bool attn_tc_supported(const Geom& g) {
  return g.dtype == SLA_BF16 && (g.d == 64 || g.d == 128) && (g.bq == 64 || g.bq == 128) &&
         (g.bk == 64 || g.bk == 128) && tma_available();
}

size_t attn_tc_scratch_bytes(const Geom& g) {
  const size_t nqt = (static_cast<size_t>(g.N) + kTileM - 1) / kTileM;
  const size_t tiles = static_cast<size_t>(g.BH) * nqt;
  return tiles * sizeof(int32_t) + 256 + tiles * g.nkb * sizeof(uint32_t);
}

cudaError_t launch_attn_plan(const Geom& g, const sla_block_lists& rows, void* scratch,
                             cudaStream_t s) {
  const int nqt = (g.N + kTileM - 1) / kTileM;
  const size_t ntiles = static_cast<size_t>(g.BH) * nqt;
  const PlanPtrs pp = plan_ptrs(g, scratch);
  plan_kernel<<<static_cast<unsigned>((ntiles + 127) / 128), 128, 0, s>>>(
      rows, g.BH, g.nqb, g.nkb, nqt, g.bq, g.bk, pp.cnt, pp.tiles);
  return cudaGetLastError();
}

cudaError_t launch_tile_plan(const sla_block_lists& lists, int BH, int nrb, int ncb, int rb,
                             int cb, int32_t* cnt, uint32_t* tiles, cudaStream_t s) {
  const int nt = rb == 128 ? nrb : (nrb + 1) / 2;
  const size_t ntiles = static_cast<size_t>(BH) * nt;
  if (ntiles == 0) return cudaSuccess;
  plan_kernel<<<static_cast<unsigned>((ntiles + 127) / 128), 128, 0, s>>>(lists, BH, nrb, ncb, nt,
                                                                          rb, cb, cnt, tiles);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc_fused(const void* q, const void* k, const void* v, const Geom& g,
                                 void* scratch, const AttnOutputs& o, const LinInputs* lin,
                                 int32_t* status, cudaStream_t s) {
  const int nqt = (g.N + kTileM - 1) / kTileM;
  const PlanPtrs pp = plan_ptrs(g, scratch);
  CUtensorMap mq, mk, mv, mhm, mw;
  if (!make_map(&mq, q, g, kTileM) || !make_map(&mk, k, g, g.bk) || !make_map(&mv, v, g, g.bk))
    return cudaErrorInvalidValue;
  AttnEpilogue ep;
  ep.o_s = o.o_s;
  ep.lse = o.lse;
  ep.out = static_cast<__nv_bfloat16*>(o.out);
  ep.o_lin = o.o_lin;
  ep.zm = nullptr;
  ep.marg_cnt = nullptr;
  ep.nqb = g.nqb;
  mhm = mq;  // unused unless the linear branch is fused
  mw = mq;
  if (lin) {
    if (g.d != 128) return cudaErrorNotSupported;
    const uint64_t dh[2] = {128, static_cast<uint64_t>(g.BH) * g.nqb * 128}, sh[1] = {256};
    const uint64_t dw[2] = {128, 128}, sw[1] = {256};
    const uint32_t box[2] = {64, 128};
    if (!encode_bf16_map(&mhm, lin->hm, 2, dh, sh, box) || !encode_bf16_map(&mw, lin->wb, 2, dw, sw, box))
      return cudaErrorInvalidValue;
    ep.zm = lin->zm;
    ep.marg_cnt = lin->marg_cnt;
  }
#define SLA_TC_CASE(D_, BQ_, BK_)                                                                 \
  if (g.d == D_ && g.bq == BQ_ && g.bk == BK_)                                                    \
    return launch_t<D_, BQ_, BK_>(mq, mk, mv, mhm, mw, pp.cnt, pp.tiles, g, nqt, ep, status, s);
  SLA_TC_CASE(128, 64, 64)
  SLA_TC_CASE(128, 64, 128)
  SLA_TC_CASE(128, 128, 64)
  SLA_TC_CASE(128, 128, 128)
  SLA_TC_CASE(64, 64, 64)
  SLA_TC_CASE(64, 64, 128)
  SLA_TC_CASE(64, 128, 64)
  SLA_TC_CASE(64, 128, 128)
#undef SLA_TC_CASE
  return cudaErrorNotSupported;
}

cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, const Geom& g,
                           const sla_block_lists& rows, float* o_s, float* lse, int32_t* status,
                           void* scratch, cudaStream_t s) {
  cudaError_t e = launch_attn_plan(g, rows, scratch, s);
  if (e != cudaSuccess) return e;
  AttnOutputs o;
  o.o_s = o_s;
  o.lse = lse;
  o.out = nullptr;
  o.o_lin = nullptr;
  return launch_attn_tc_fused(q, k, v, g, scratch, o, nullptr, status, s);
}

}  // namespace sla
