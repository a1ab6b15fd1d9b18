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
//     into two 3-stage rings, with the 3D tensor map [B*H, N, d] so rows past
//     N read as zeros.
//   * Warp 1 (one lane): MMA issuer -- S = Q K^T (M=128, N=128, K=d) into the
//     TMEM buffer of the tile's parity, O_h += P V (M=128, N=d, K=128) with P
//     read from TMEM.
//   * Warps 2-9: two warpgroups that take alternate key tiles.  Warpgroup h
//     owns the tiles of parity h, the S buffer h and the accumulator O_h; a
//     thread holds one 128-key row of S -- tcgen05.ld, masking, online
//     softmax in the exp2 domain, and P as bf16 pairs over its own S columns.
//     No row statistic crosses warps inside the loop; (m_h, l_h, O_h) of the
//     two warpgroups are merged once in the epilogue (O / l, LSE).  The two
//     warps that share a TMEM lane quadrant -- and an SM sub-partition --
//     work on different tiles, so one's exponentials overlap the other's
//     loads and stores.  The running max lags a tile: P uses the max of the
//     earlier tiles while the tile's max accumulates in the same pass, and a
//     growth beyond 2^8 raises it on the next tile (P stays below 2^64
//     meanwhile, far inside the fp32 and bf16 range; a larger jump redoes
//     the tile exactly).
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
constexpr int kSBuf = 2;  // S tiles in TMEM, one per warpgroup (P overwrites its S)
constexpr int kSoftmaxWarps = 8;                 // two warpgroups
constexpr int kThreads = 64 + 32 * kSoftmaxWarps;  // TMA warp, MMA warp, softmax
constexpr uint32_t kSmemRequest = 232448;          // 227 KB opt-in maximum
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kGuardLog2 = 64.0f;  // largest exponent of P the one-pass softmax accepts

// ------------------------------------------------------------------ plan
// One key-tile descriptor packs two 16-bit entries (the second only used for
// key blocks of 64): bit 15 present, bits 13-14 membership (bit 13: query
// block of rows 0-63, bit 14: rows 64-127; both for a 128-row block), bits
// 0-12 key-block index.

constexpr uint32_t kPresent = kPlanPresent;

__device__ __forceinline__ uint32_t entry(int blk, uint32_t flags) {
  return kPresent | (flags << 13) | static_cast<uint32_t>(blk);
}

// One warp per query tile: the tile's query blocks' critical lists are
// scattered into per-warp bitmaps over the key blocks (membership a, b),
// then read back in key order (a warp scan of the words' popcounts gives
// each lane its output slot), so the union comes out ascending with its
// membership flags whatever the lists' order; entries outside [0, nkb) are
// skipped and repeated entries collapse.
constexpr int kPlanWarps = 4;
// (parameter validation caps Nqb and Nkb at kMaxBlocks: the bitmaps below
// hold that many blocks and an entry's index field has 13 bits)
static_assert(kMaxBlocks <= 8192, "plan entries hold 13-bit block indices");

__global__ void __launch_bounds__(32 * kPlanWarps) plan_kernel(sla_block_lists rows, int BH, int nqb,
                                                               int nkb, int nqt, int bq, int bk,
                                                               int32_t* __restrict__ cnt,
                                                               uint32_t* __restrict__ tiles,
                                                               int32_t* __restrict__ zero_words,
                                                               int nzero) {
  // (the status words of the step's later kernels, zeroed here instead of by
  // a memset of their own: no kernel before this one writes them)
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < nzero) zero_words[threadIdx.x] = 0;
  __shared__ uint32_t bits[kPlanWarps][2][kMaxBlocks / 32];
  const unsigned full = 0xffffffffu;
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x * kPlanWarps + w;
  if (tile >= BH * nqt) return;  // whole warps; no block-wide barrier below
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
  const int nw = (nkb + 31) / 32;
  uint32_t* ba = bits[w][0];
  uint32_t* bb = bits[w][1];
  for (int i = lane; i < nw; i += 32) { ba[i] = 0u; bb[i] = 0u; }
  __syncwarp();
  for (int e = lane; e < na; e += 32) {
    const int blk = la[e];
    if (blk >= 0 && blk < nkb) atomicOr(&ba[blk >> 5], 1u << (blk & 31));
  }
  for (int e = lane; e < nb; e += 32) {
    const int blk = lb[e];
    if (blk >= 0 && blk < nkb) atomicOr(&bb[blk >> 5], 1u << (blk & 31));
  }
  __syncwarp();
  const int per_tile = kTileN / bk;  // 1 or 2 entries per key tile
  uint32_t* out = tiles + i64(tile) * nkb;
  uint16_t* out16 = reinterpret_cast<uint16_t*>(out);  // entry r of a packed pair list
  int base = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int i = w0 + lane;
    const uint32_t xa = i < nw ? ba[i] : 0u, xb = i < nw ? bb[i] : 0u;
    uint32_t x = xa | xb;
    const int c = __popc(x);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += y;
    }
    int r = base + incl - c;
    while (x) {
      const int bit = __ffs(x) - 1;
      x &= x - 1u;
      const uint32_t f = (((xa >> bit) & 1u) ? fa : 0u) | (((xb >> bit) & 1u) ? 2u : 0u);
      const uint32_t en = entry(i * 32 + bit, f);
      if (per_tile == 2) out16[r] = static_cast<uint16_t>(en);
      else out[r] = en;
      ++r;
    }
    base += __shfl_sync(full, incl, 31);
  }
  if (lane == 0) {
    if (per_tile == 2 && (base & 1)) out16[base] = 0;  // empty second entry
    cnt[tile] = (base + per_tile - 1) / per_tile;
  }
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
               const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmOut,
               const int32_t* __restrict__ plan_cnt,
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
  // merge area of the epilogue ([m | l | den][2 warpgroups][128] fp32), in V
  // stage 1, free once every P V product is done
  constexpr uint32_t offX = offV + kKBytes;
  constexpr uint32_t offBar = offV + kStages * kKBytes;
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
  // per S buffer h (tiles of parity h): S(t) in TMEM, P(t) in TMEM (the four
  // warps of warpgroup h)
  auto b_s_full = [&](int h) { return smem_u32(&bars[kB0 + h]); };
  auto b_p_full = [&](int h) { return smem_u32(&bars[kB0 + kSBuf + h]); };
  constexpr int kB1 = kB0 + 2 * kSBuf;
  const uint32_t b_fin = smem_u32(&bars[kB1 + 0]);
  const uint32_t b_lin = smem_u32(&bars[kB1 + 1]);   // H^M and W tiles landed
  const uint32_t b_phiq = smem_u32(&bars[kB1 + 2]);  // phi(Q) written (8 warps)
  const uint32_t b_den = smem_u32(&bars[kB1 + 3]);   // normaliser halves exchanged (8 warps)
  const uint32_t b_num = smem_u32(&bars[kB1 + 4]);   // phi(Q) H^M in TMEM
  const uint32_t b_olin = smem_u32(&bars[kB1 + 5]);  // O_lin (bf16) in shared memory (8 warps)
  const uint32_t b_lout = smem_u32(&bars[kB1 + 6]);  // O_lin W in TMEM
  // every P V product done (single use): the producer's linear loads and
  // the epilogue wait on it
  const uint32_t b_pv_last = smem_u32(&bars[kB1 + 7]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[kB1 + 8]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[kB1 + 9]);
  static_assert((kB1 + 10) * 8 <= kUsed - offBar, "barrier block too small");
  float* xch = reinterpret_cast<float*>(base + offX);

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
      mbar_init(b_p_full(j), kSoftmaxWarps / 2);
    }
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
  if (warp == 1) {  // TMEM: 512 columns (S0 | S1 | O_0 | O_1)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // columns: S of tile t at 128 (t % 2), O_h at 256 + 128 h.  The bf16 P of
  // tile t (two keys per column) overwrites the last 64 columns of its own
  // S, which only the warp holding those rows reads.  Addresses are computed,
  // not indexed from an array, so none goes through local memory.
  auto tS = [&](int j) { return tmem + 128u * static_cast<uint32_t>(j); };
  auto tO = [&](int h) { return tmem + 256u + 128u * static_cast<uint32_t>(h); };

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
      // linear branch: with every K/V load issued (a few tiles before the
      // end), H^M and z^M of the tile's query blocks -- written by the
      // gather long before, so in HBM by now -- are prefetched into L2, so
      // that the epilogue does not wait for HBM
      if (lin && tv == T) {
        if (nm_a > 0) {
          tma_prefetch_2d(&tmHM, 0, (bh * nqb + qa) * 128);
          tma_prefetch_2d(&tmHM, 64, (bh * nqb + qa) * 128);
          const float* z = ep.zm + (i64(bh) * nqb + qa) * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) prefetch_l2(z + 32 * i);
        }
        if (nm_b > 0) {
          tma_prefetch_2d(&tmHM, 0, (bh * nqb + qb2) * 128);
          tma_prefetch_2d(&tmHM, 64, (bh * nqb + qb2) * 128);
          const float* z = ep.zm + (i64(bh) * nqb + qb2) * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) prefetch_l2(z + 32 * i);
        }
      }
      // H^M of the tile's query blocks and W go into the K/V stages once
      // the last P V product has read them
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
      // S(t) takes the buffer of tile t - 2, whose P V was issued just before:
      // the tensor pipe runs in issue order, so it reads that P before this
      // MMA overwrites it.  The caller has waited for K(t).
      auto issue_s = [&](int t) {
        const int s = t % kStages, j = t & 1;
        tc_fence_after();
        const uint64_t dK = sdesc_add(dK0, s * kKBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
          tc_mma(tS(j), sdesc_add(dQ, off), sdesc_add(dK, off), idesc_qk, kk > 0);
        }
        tc_commit(b_s_full(j));
        tc_commit(b_k_empty(s));
      };
      // the caller has waited for P(t) and V(t)
      auto issue_pv = [&](int t) {
        const int s = t % kStages, j = t & 1;
        tc_fence_after();
        const uint64_t dV = sdesc_add(dV0, s * kKBytes);
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk)  // 16 keys = 8 TMEM columns of P
          tc_mma_ts(tO(j), tS(j) + 64 + kk * 8, sdesc_add(dV, kk * 2048), idesc_pv, (t > 1 || kk > 0) ? 1u : 0u);
        tc_commit(b_v_empty(s));
      };
      // S of the next tile of the same parity follows each P V product;
      // the other warpgroup's tile keeps the tensor pipe busy meanwhile.
      // The commit of S(t + 2) also tells that warpgroup that P V of tile t
      // is complete (commits track every earlier MMA), which its rescale of
      // O relies on.  The operands of the next two products are waited for
      // before P(t): they are almost always there already, and the wait for
      // the softmax is then the only one between P(t) and the tensor pipe.
      for (int t = 0; ok && t < 2 && t < T; ++t) {
        ok = wait(b_k_full(t), 0);
        if (ok) issue_s(t);
      }
      for (int t = 0; ok && t < T; ++t) {
        ok = wait(b_v_full(t % kStages), (t / kStages) & 1);
        if (ok && t + 2 < T) ok = wait(b_k_full((t + 2) % kStages), ((t + 2) / kStages) & 1);
        if (ok) ok = wait(b_p_full(t & 1), (t >> 1) & 1);
        if (!ok) break;
        issue_pv(t);
        if (t + 2 < T) issue_s(t + 2);
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
    // Warpgroup h takes the key tiles t = h, h + 2, ...; thread (h, r) holds
    // row r of those tiles and keeps its own running max, sum and O_h.
    const int h = (warp - 2) >> 2;        // tile parity = S buffer = O accumulator
    const int quad = warp & 3;            // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;       // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t rflag = BQ == 128 ? 3u : (r < 64 ? 1u : 2u);
    const unsigned full = 0xffffffffu;
    const uint32_t tSh = tS(h) + lane_off, tOh = tO(h) + lane_off;
    // running max (log2 domain), a raise of it due on the next tile, sum
    float m_ref = -INFINITY, pend = -INFINITY, l = 0.f;
    bool ok = true;
    // valid keys of row r among the 64 keys from blk * BK + off of entry ent
    auto nvalid = [&](uint32_t ent, int off) -> int {
      const int blk = ent & 0x1FFF;
      const bool member = (ent & kPresent) && (((ent >> 13) & 3u) & rflag);
      return member ? max(0, min(64, N - blk * BK - off)) : 0;
    };
    // the plan word of the next tile is fetched a tile ahead: a global load
    // on the path from one tile to the next would stall every warp
    uint32_t desc_next = h < T ? ptiles[h] : 0u;
    for (int t = h; ok && t < T; t += 2) {
      const uint32_t use = static_cast<uint32_t>(t) >> 1;  // earlier uses of buffer h
      const uint32_t desc = desc_next;
      if (t + 2 < T) desc_next = ptiles[t + 2];
      // keys [0, 64) and [64, 128) of the tile: the two entries of a pair of
      // 64-blocks, or the two halves of one 128-block
      const int kv0 = nvalid(desc & 0xFFFFu, 0);
      const int kv1 = BK == 64 ? nvalid(desc >> 16, 0) : nvalid(desc & 0xFFFFu, 64);
      if (!__all_sync(full, wait(b_s_full(h), use & 1))) { ok = false; break; }
      tc_fence_after();
      // The row is read in two halves of 64 keys, so that 64 scores are live
      // at a time.  P (key k at column 64 + k / 2) goes over the columns of
      // keys 64-127 once every score of the tile has been read.
      float s[64];
      auto load_half = [&](int e) {
        tmem_ld32(tSh + 64 * e, s);
        tmem_ld32(tSh + 64 * e + 32, s + 32);
        tmem_wait_ld();
        reg_fence<64>(s);
      };
      // O_h *= alpha (warp-wide TMEM access; alpha = 1 on rows that keep
      // their scale).  No wait is needed: S(t) has completed, and its commit
      // followed P V of tile t - 2, the last product into O_h.
      auto rescale_o = [&](float alpha) {
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          float o[32];
          tmem_ld32(tOh + c, o);
          tmem_wait_ld();
          reg_fence<32>(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tOh + c, o);
        }
      };
      // a raise of the running max decided on the previous tile of this
      // warpgroup takes effect now, P V of that tile being complete
      if (__any_sync(full, pend > m_ref)) {
        float alpha = 1.f;
        if (pend > m_ref) {
          alpha = exp2f(m_ref - pend);
          m_ref = pend;
          l *= alpha;
        }
        rescale_o(alpha);
      }
      float2 acc0, acc1, acc2, acc3;
      // exponentials of the loaded half (kv of its 64 keys valid) as bf16
      // pairs into pk[0, 32), the sum of those rounded weights -- the ones
      // P V uses, so O / l is a convex combination of V rows -- into acc;
      // returns the max of the valid raw scores.
      auto half_exp = [&](int kv, uint32_t* pk) -> float {
        const float2 sc2 = make_float2(scale_log2, scale_log2);
        const float2 nm2 = make_float2(-m_ref, -m_ref);
        float mh = -INFINITY;
        if (kv == 64) {
          float a0 = -INFINITY, a1 = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (i & 1) a1 = max3(a1, s[2 * i], s[2 * i + 1]);
            else a0 = max3(a0, s[2 * i], s[2 * i + 1]);
            const float2 x = fma2(make_float2(s[2 * i], s[2 * i + 1]), sc2, nm2);
            const float2 ex = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            pk[i] = pack_bf16x2(ex.x, ex.y);
            if (i % 4 == 0) add_bf16x2_f32(pk[i], acc0.x, acc0.y);
            if (i % 4 == 1) add_bf16x2_f32(pk[i], acc1.x, acc1.y);
            if (i % 4 == 2) add_bf16x2_f32(pk[i], acc2.x, acc2.y);
            if (i % 4 == 3) add_bf16x2_f32(pk[i], acc3.x, acc3.y);
          }
          mh = fmaxf(a0, a1);
        } else if (kv > 0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int k = 2 * i;
            mh = k < kv ? fmaxf(mh, s[k]) : mh;
            mh = k + 1 < kv ? fmaxf(mh, s[k + 1]) : mh;
            const float2 x = fma2(make_float2(s[k], s[k + 1]), sc2, nm2);
            const float2 ex = make_float2(k < kv ? fast_exp2(x.x) : 0.f, k + 1 < kv ? fast_exp2(x.y) : 0.f);
            pk[i] = pack_bf16x2(ex.x, ex.y);
            if (i % 2 == 0) add_bf16x2_f32(pk[i], acc0.x, acc0.y);
            else add_bf16x2_f32(pk[i], acc1.x, acc1.y);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = 0u;
        }
        return mh;
      };
      // max of the valid raw scores of the loaded half
      auto half_max = [&](int kv) -> float {
        float mh = -INFINITY;
        if (kv == 64) {
          float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            a0 = max3(a0, s[c], s[c + 1]);
            a1 = max3(a1, s[c + 2], s[c + 3]);
            a2 = max3(a2, s[c + 4], s[c + 5]);
            a3 = max3(a3, s[c + 6], s[c + 7]);
          }
          mh = max3(a0, a1, fmaxf(a2, a3));
        } else if (kv > 0) {
#pragma unroll
          for (int c = 0; c < 64; ++c) mh = c < kv ? fmaxf(mh, s[c]) : mh;
        }
        return mh;
      };
      // One pass: P with the running max of the earlier tiles while this
      // tile's max accumulates.  Rows whose max grows by more than 2^8 raise
      // the running max on the next tile; P stays below 2^kGuardLog2 (beyond
      // that the tile is redone exactly), far inside the fp32 and bf16
      // range.  The exact pass -- the first tile of a row, or a redo -- takes
      // the tile's max first and raises the running max at once.
      uint32_t pk[64];
      bool exact = __any_sync(full, m_ref == -INFINITY);
      for (int pass = 0; pass < 2; ++pass) {
        if (exact) {
          load_half(0);
          float mx = half_max(kv0);
          load_half(1);
          mx = fmaxf(mx, half_max(kv1));
          bool raise = false;
          float alpha = 1.f;
          if (mx > -INFINITY) {
            const float mt = mx * scale_log2;
            if (m_ref == -INFINITY) {
              m_ref = mt;
            } else if (mt > m_ref + kRescaleLog2) {
              alpha = exp2f(m_ref - mt);
              m_ref = mt;
              l *= alpha;
              raise = true;
            }
          }
          if (__any_sync(full, raise)) rescale_o(alpha);
        }
        acc0 = acc1 = acc2 = acc3 = make_float2(0.f, 0.f);
        load_half(1);
        float mx = half_exp(kv1, pk + 32);
        reg_fence_u<32>(pk + 32);  // keys 64-127 done before keys 0-63 load
        load_half(0);
        mx = fmaxf(mx, half_exp(kv0, pk));
        const float mt = mx * scale_log2;
        if (!exact && __any_sync(full, mt > m_ref + kGuardLog2)) {
          exact = true;
          continue;
        }
        tmem_st16u(tSh + 64, pk);
        tmem_st16u(tSh + 80, pk + 16);
        tmem_st16u(tSh + 96, pk + 32);
        tmem_st16u(tSh + 112, pk + 48);
        if (mt > m_ref + kRescaleLog2) pend = mt;  // (never after an exact pass)
        break;
      }
      acc0 = add2(add2(acc0, acc1), add2(acc2, acc3));
      l += acc0.x + acc0.y;
      tmem_wait_st();  // P (and any rescaled O) stored
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_p_full(h));
    }
    // epilogue.  Once every P V product is done O_0 and O_1 are final in
    // TMEM, and Q, the K/V stages and the S columns are free.
    const int row = qt * kTileM + r;
    const i64 orow = (i64(bh) * N + row) * D + h * DH;
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
    bool fin = ok && (T == 0 || __all_sync(full, wait(b_pv_last, 0)));
    // merge the two warpgroups' (m, l) of row r; thread (h, r) then finishes
    // O columns [h D/2, (h + 1) D/2) from both accumulators
    xch[h * 128 + r] = m_ref;
    xch[256 + h * 128 + r] = l;
    __syncwarp();
    if (lane == 0) mbar_arrive(b_fin);
    fin = fin && __all_sync(full, wait(b_fin, 0));
    const float m_o = fin ? xch[(h ^ 1) * 128 + r] : -INFINITY;
    const float l_o = fin ? xch[256 + (h ^ 1) * 128 + r] : 0.f;
    const float mt = fmaxf(m_ref, m_o);
    const float f_s = m_ref > -INFINITY ? exp2f(m_ref - mt) : 0.f;
    const float f_o = m_o > -INFINITY ? exp2f(m_o - mt) : 0.f;
    const float ltot = fin ? l * f_s + l_o * f_o : 0.f;
    const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
    const float w0 = (h == 0 ? f_s : f_o) * inv, w1 = (h == 0 ? f_o : f_s) * inv;
    bool lin_ok = false;
    if (D == 128 && lin && fin) {  // (never taken for d = 64: lin is false)
      // phi(Q) in place (this thread: row r, channels [64h, 64h + 64)), and
      // half of the normaliser phi(q) . z^M from the same rounded values
      float dpart = 0.f, dpart2 = 0.f;
      lin_ok = __all_sync(full, wait(b_q, 0));
      if (lin_ok) {
        // all eight 16-byte pieces are read before any is written back: a
        // read after a store to the same region would wait for it, and the
        // pieces' exponentials would run one after another
        uint4 qv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) qv[u] = *reinterpret_cast<const uint4*>(base + offQ + h * 16384 + sw128(r, u));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (row < N && nm_r > 0) {
            val = phi_unit(qv[u]);
            const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.x));
            const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.y));
            const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.z));
            const float2 f3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.w));
            const float4 za = z4[2 * u], zb = z4[2 * u + 1];
            dpart = fmaf(f0.x, za.x, fmaf(f0.y, za.y, fmaf(f1.x, za.z, fmaf(f1.y, za.w, dpart))));
            dpart2 = fmaf(f2.x, zb.x, fmaf(f2.y, zb.y, fmaf(f3.x, zb.z, fmaf(f3.y, zb.w, dpart2))));
          }
          qv[u] = val;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4*>(base + offQ + h * 16384 + sw128(r, u)) = qv[u];
        dpart += dpart2;
        xch[512 + h * 128 + r] = dpart;
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) { mbar_arrive(b_phiq); mbar_arrive(b_den); }
        lin_ok = __all_sync(full, wait(b_den, 0));
      }
      float den = 0.f;
      if (lin_ok) den = dpart + xch[512 + (h ^ 1) * 128 + r];
      if (lin_ok) lin_ok = __all_sync(full, wait(b_num, 0));
      if (lin_ok) {
        // O_lin = phi(Q) H^M / den -> o_lin (fp32, optional) and bf16 into K
        // stage 2 as the A operand of the projection
        tc_fence_after();
        const uint32_t tn = tS(second ? 1 : 0);
        const float dinv = (nm_r > 0 && den > 0.f) ? 1.f / den : 0.f;
        float vv[64];  // both 32-column chunks in flight before one wait
        tmem_ld32(tn + lane_off + h * 64, vv);
        tmem_ld32(tn + lane_off + h * 64 + 32, vv + 32);
        tmem_wait_ld();
        reg_fence<64>(vv);
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          float* v = vv + c;
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
      float o[32], lo[32];
      // the projection's columns load with the accumulators, one wait for all
      const bool add_lin = D == 128 && lin_ok && ep.out;
      if (fin && T > 1) {
        float o1[32];
        tmem_ld32(tO(0) + lane_off + h * DH + c, o);
        tmem_ld32(tO(1) + lane_off + h * DH + c, o1);
        if (add_lin) tmem_ld32(tS(0) + lane_off + h * DH + c, lo);
        tmem_wait_ld();
        reg_fence<32>(o);
        reg_fence<32>(o1);
        if (add_lin) reg_fence<32>(lo);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = o[i] * w0 + o1[i] * w1;
      } else if (fin && T > 0) {  // one tile: warpgroup 1 had none
        tmem_ld32(tO(0) + lane_off + h * DH + c, o);
        tmem_wait_ld();
        reg_fence<32>(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= w0;
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
        if (add_lin) {
          if (!(fin && T > 1)) {
            tmem_ld32(tS(0) + lane_off + h * DH + c, lo);
            tmem_wait_ld();
            reg_fence<32>(lo);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] += lo[i];
        }
        // bf16 into the staging tile (K stage 0, free: its last readers,
        // the S and linear-branch MMAs, are done), in the 128-byte swizzled
        // layout of the output's tensor map; rows past N are dropped by the
        // store
        const int ch = h * DH + c;  // first channel of these 32
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *reinterpret_cast<uint4*>(base + offK + (ch / 64) * 16384 + sw128(r, (ch % 64) / 8 + q4)) =
              make_uint4(pack_bf16x2(o[8 * q4], o[8 * q4 + 1]), pack_bf16x2(o[8 * q4 + 2], o[8 * q4 + 3]),
                         pack_bf16x2(o[8 * q4 + 4], o[8 * q4 + 5]), pack_bf16x2(o[8 * q4 + 6], o[8 * q4 + 7]));
      }
    }
    if (ep.out) {
      // one TMA store per 64-channel chunk once all 256 threads have written
      fence_async_smem();
      asm volatile("bar.sync 2, 256;" ::: "memory");  // the softmax warps only
      if (threadIdx.x == 64) {
#pragma unroll
        for (int c = 0; c < DC; ++c) tma_store_3d(&tmOut, sb + offK + c * 16384, c * 64, qt * kTileM, bh);
        tma_store_commit();
        tma_store_wait_read();  // the staging tile is read before the CTA ends
      }
    }
    if (row < N && h == 0)
      ep.lse[i64(bh) * N + row] = ltot > 0.f ? (mt + log2f(ltot)) * 0.69314718055994531f : -INFINITY;
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
                     const CUtensorMap& mhm, const CUtensorMap& mw, const CUtensorMap& mo, const int32_t* cnt,
                     const uint32_t* tiles, const Geom& g, int nqt, const AttnEpilogue& ep,
                     int32_t* status, cudaStream_t s) {
  auto kern = attn_tc_kernel<D, BQ, BK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemRequest));
  if (e != cudaSuccess) return e;
  const float scale_log2 = g.scale * 1.4426950408889634f;
  const int debug_skip = debug_withhold(g, SLA_WITHHOLD_ATTENTION) ? 1 : 0;
  kern<<<g.BH * nqt, kThreads, kSmemRequest, s>>>(mq, mk, mv, mhm, mw, mo, cnt, tiles, g.nkb, ep, status,
                                                  g.N, nqt, scale_log2, wait_limit(g), debug_skip);
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
                             cudaStream_t s, int32_t* zero_words, int nzero) {
  if (nzero > 32 * kPlanWarps) return cudaErrorInvalidValue;
  const int nqt = (g.N + kTileM - 1) / kTileM;
  const size_t ntiles = static_cast<size_t>(g.BH) * nqt;
  const PlanPtrs pp = plan_ptrs(g, scratch);
  plan_kernel<<<static_cast<unsigned>((ntiles + kPlanWarps - 1) / kPlanWarps), 32 * kPlanWarps, 0, s>>>(
      rows, g.BH, g.nqb, g.nkb, nqt, g.bq, g.bk, pp.cnt, pp.tiles, zero_words, nzero);
  return cudaGetLastError();
}

cudaError_t launch_tile_plan(const sla_block_lists& lists, int BH, int nrb, int ncb, int rb,
                             int cb, int32_t* cnt, uint32_t* tiles, cudaStream_t s) {
  const int nt = rb == 128 ? nrb : (nrb + 1) / 2;
  const size_t ntiles = static_cast<size_t>(BH) * nt;
  if (ntiles == 0) return cudaSuccess;
  plan_kernel<<<static_cast<unsigned>((ntiles + kPlanWarps - 1) / kPlanWarps), 32 * kPlanWarps, 0, s>>>(
      lists, BH, nrb, ncb, nt, rb, cb, cnt, tiles, nullptr, 0);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc_fused(const void* q, const void* k, const void* v, const Geom& g,
                                 void* scratch, const AttnOutputs& o, const LinInputs* lin,
                                 int32_t* status, cudaStream_t s) {
  const int nqt = (g.N + kTileM - 1) / kTileM;
  const PlanPtrs pp = plan_ptrs(g, scratch);
  CUtensorMap mq, mk, mv, mhm, mw, mo;
  if (!make_map(&mq, q, g, kTileM) || !make_map(&mk, k, g, g.bk) || !make_map(&mv, v, g, g.bk))
    return cudaErrorInvalidValue;
  mo = mq;  // unused without a bf16 output
  if (o.out && !make_map(&mo, o.out, g, kTileM)) return cudaErrorInvalidValue;
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
    return launch_t<D_, BQ_, BK_>(mq, mk, mv, mhm, mw, mo, pp.cnt, pp.tiles, g, nqt, ep, status, s);
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
