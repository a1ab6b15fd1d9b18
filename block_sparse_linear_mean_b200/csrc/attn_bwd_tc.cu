// Backward of the critical (sparse softmax) branch on the tensor cores
// (sm_100a): tcgen05 MMAs with fp32 accumulators in tensor memory, operands
// staged by TMA.
//
// The SLA post ("fine-tuning") adapts a pretrained model with the hybrid
// attention in place, so the critical branch needs the gradients of block
// sparse softmax attention with the block mask held fixed.  With
// P = exp(s * q k^T - LSE) recomputed from the saved log-sum-exp and
// Delta_t = dO_t . O_s[t]:
//   dS = P o (dO V^T - Delta),  dQ = s dS K,  dK = s dS^T Q,  dV = P^T dO.
//
// Two kernels, no atomics (each output row is owned by one CTA):
//   dq kernel   - one CTA per 128-row query tile, streaming 64-key steps of
//                 the tile's critical key blocks (row lists): S = Q K^T and
//                 dP = dO V^T into TMEM, dS (bf16) written back into the S
//                 columns, dQ += dS K with A read from TMEM.
//   dkdv kernel - one CTA per 128-key tile, streaming 64-query steps of the
//                 query blocks for which the tile's key blocks are critical
//                 (column lists): S^T = K Q^T and dP^T = V dO^T, P^T and
//                 dS^T (bf16) written back into their own columns,
//                 dV += P^T dO and dK += dS^T Q with A read from TMEM.
// S / dP are double-buffered by step parity, so the MMAs of step u+1 run
// while the elementwise warps work on step u.  The critical-block FLOPs are
// 4 * 2 * d per (query, key) pair in the dkdv kernel and 3 * 2 * d in the
// dq kernel (S and dP are recomputed there).
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 MMA issuer (one
// thread), warps 2-9 elementwise: thread (h, r) owns TMEM lane r and the
// step's columns [32h, 32h + 32).  Every wait is bounded; on a timeout the
// status word gets SLA_ERR_TIMEOUT and all roles leave.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace sla {

namespace {

constexpr int kBwdThreads = 320;
constexpr int kBwdStages = 4;
constexpr uint32_t kBwdSmemRequest = 232448;
constexpr uint32_t kBwdTmemCols = 512;

// A 64-row step of a plan word: entry e of a word of two 64-blocks, or half
// e of one 128-block (skipped when it starts at or past N).
struct Step {
  int row0;
  uint32_t flags;
  bool present;
};
template <int BLK>
__device__ __forceinline__ Step step_of(uint32_t desc, int e, int N) {
  Step st;
  const uint32_t ent = BLK == 64 ? (desc >> (16 * e)) & 0xFFFFu : desc & 0xFFFFu;
  st.row0 = static_cast<int>(ent & 0x1FFFu) * BLK + (BLK == 128 ? 64 * e : 0);
  st.present = (ent & kPlanPresent) != 0 && st.row0 < N;
  st.flags = (ent >> 13) & 3u;
  return st;
}

// Steps present in a tile's plan.  Every lane of the warp reads a share of
// the plan words at once: one L2 round trip per 32 words instead of one per
// word before any work starts.  Called by whole warps.
template <int BLK>
__device__ __forceinline__ int plan_steps(const uint32_t* ptiles, int T, int N) {
  int c = 0;
  for (int t = static_cast<int>(threadIdx.x % 32); t < T; t += 32)
    c += 1 + (step_of<BLK>(__ldg(ptiles + t), 1, N).present ? 1 : 0);
  return static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c)));
}

struct BwdShared {
  uint64_t* bars;
  volatile int* abort_flag;
  int32_t* status;
  long long timeout;
};

__device__ __forceinline__ bool bwait(const BwdShared& sh, uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u) {
      if (*sh.abort_flag) return false;
      if (clock64() - t0 > sh.timeout) {
        *sh.abort_flag = 1;
        atomicExch(sh.status, static_cast<int32_t>(SLA_ERR_TIMEOUT));
        return false;
      }
    }
  }
}

__device__ __forceinline__ void teardown(const BwdShared& sh, int warp, uint32_t tmem) {
  tc_fence_before();
  __syncthreads();
  if (*sh.abort_flag) {  // let in-flight copies and MMAs drain (bounded)
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) { __nanosleep(1000); }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwdTmemCols);
  }
}

// ------------------------------------------------------------------ dQ
// Query side of the linear branch, fused into the dq kernel's epilogue
// (d = 128): for the tile's query block(s) i with marginal set M_i,
//   g = dO W^T, den = phi(q) . z^M_i, dnum = g / den, dden = -(g . o) / den,
//   dq += (dnum H^M_i^T + dden z^M_i) o phi'(q),
//   dH^M_i = phi(Q_i)^T dnum,  dz^M_i = sum_t phi(q_t) dden_t.
// marg_cnt == nullptr: no linear branch.
struct LinBwdQ {
  const float* zm;          // [B*H*Nqb, 128] z^M
  const int32_t* marg_cnt;  // [B*H*Nqb]
  const float* o_lin;       // [B*H, N, 128] saved O_lin
  const __nv_bfloat16* q;   // [B*H, N, 128] (for phi')
  __nv_bfloat16* dhm;       // [B*H*Nqb, 128, 128] out
  float* dzm;               // [B*H*Nqb, 128] out
  int nqb;
};

// Key side of the linear branch, fused into the dkdv kernel's epilogue
// (d = 128): for the tile's key block(s) j that are marginal somewhere, with
// dH_j, dz_j the sums of dH^M_i, dz^M_i over the query blocks i that hold j,
//   dv += phi(K_j) dH_j,  dk += (V_j dH_j^T + dz_j) o phi'(k).
// marg_cnt == nullptr: no linear branch.
struct LinBwdK {
  const float* dz;          // [B*H*Nkb, 128] dz_j
  const int32_t* marg_cnt;  // [B*H*Nkb] per key block: query blocks holding it
  const __nv_bfloat16* k;   // [B*H, N, 128] (for phi and phi')
  int nkb;
};

template <int D, int BQ, int BK>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmHM, const __grid_constant__ CUtensorMap tmW,
                      const int32_t* __restrict__ tile_cnt, const uint32_t* __restrict__ tiles,
                      int plan_stride, const float* __restrict__ lse,
                      const float* __restrict__ delta, float* __restrict__ dq, LinBwdQ lq,
                      int32_t* status, int N, int nqt, float scale, float scale_log2,
                      long long timeout, int debug_skip) {
  constexpr int DC = D / 64;
  constexpr uint32_t kTileBytes = DC * 16384;  // 128 rows x D bf16 (Q, dO)
  constexpr uint32_t kHalfBytes = DC * 8192;   // 64 rows x D bf16 (K, V)
  constexpr uint32_t kStageBytes = 2 * kHalfBytes;
  constexpr uint32_t offQ = 0, offdO = kTileBytes, offKV = 2 * kTileBytes;
  constexpr uint32_t offBar = offKV + kBwdStages * kStageBytes;
  constexpr uint32_t offRed = offBar + 512;   // [4][128] fp32 exchange slots
  constexpr uint32_t offDd = offRed + 2048;   // [128] dden per row
  constexpr uint32_t kUsed = offDd + 512;
  constexpr uint32_t idesc_s = idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t idesc_dq = idesc_bf16(128, D, 0, 1);
  // linear epilogue: after the main loop the K/V stages hold W (0), H^M of
  // the tile's first and second query block (1, 2) and the bf16 dnum (3)
  constexpr uint32_t offW = offKV, offHA = offKV + kStageBytes, offHB = offKV + 2 * kStageBytes;
  constexpr uint32_t offDn = offKV + 3 * kStageBytes;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* base = smem_raw + pad;
  const uint32_t sb = raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + offBar);
  const uint32_t b_q = smem_u32(&bars[0]);
  auto b_full = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_empty = [&](int s) { return smem_u32(&bars[1 + kBwdStages + s]); };
  auto b_s = [&](int b) { return smem_u32(&bars[1 + 2 * kBwdStages + b]); };   // S, dP in TMEM
  auto b_ds = [&](int b) { return smem_u32(&bars[3 + 2 * kBwdStages + b]); };  // dS in TMEM
  const uint32_t b_done = smem_u32(&bars[5 + 2 * kBwdStages]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[6 + 2 * kBwdStages]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[7 + 2 * kBwdStages]);
  // linear epilogue (single use each)
  constexpr int kL0 = 8 + 2 * kBwdStages;
  const uint32_t b_lin = smem_u32(&bars[kL0]);       // W, H^M landed
  const uint32_t b_g = smem_u32(&bars[kL0 + 1]);     // g in TMEM
  const uint32_t b_den = smem_u32(&bars[kL0 + 2]);   // den halves exchanged (8 warps)
  const uint32_t b_go = smem_u32(&bars[kL0 + 3]);    // g . o halves exchanged (8 warps)
  const uint32_t b_dn = smem_u32(&bars[kL0 + 4]);    // dnum and phi(Q) in smem (8 warps)
  const uint32_t b_df = smem_u32(&bars[kL0 + 5]);    // df in TMEM
  const uint32_t b_dh1 = smem_u32(&bars[kL0 + 6]);   // dH^M of the first block in TMEM
  const uint32_t b_dfr = smem_u32(&bars[kL0 + 7]);   // df read (8 warps)
  const uint32_t b_dh2 = smem_u32(&bars[kL0 + 8]);   // dH^M of the second block in TMEM
  const uint32_t b_dz = smem_u32(&bars[kL0 + 9]);    // dz^M halves exchanged (8 warps)
  const uint32_t b_qt = smem_u32(&bars[kL0 + 10]);   // Q and dO copied into TMEM (8 warps)
  static_assert((kL0 + 11) * 8 <= 512, "barrier block");
  float* red = reinterpret_cast<float*>(base + offRed);
  float* dd = reinterpret_cast<float*>(base + offDd);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x;
  const int bh = tile / nqt, qt = tile % nqt;
  const int T = tile_cnt[tile];
  const uint32_t* ptiles = tiles + static_cast<i64>(tile) * plan_stride;
  // steps present in the plan (all roles count them the same way)
  const int U = plan_steps<BK>(ptiles, T, N);
  // linear branch of the tile's query blocks (A: rows 0-63 or the whole
  // 128-row block; B: rows 64-127 when blocks are 64 rows)
  const bool lin_on = D == 128 && lq.marg_cnt != nullptr;
  const int qa = BQ == 128 ? qt : 2 * qt;
  const int qb2 = (BQ == 64 && 2 * qt + 1 < lq.nqb) ? 2 * qt + 1 : -1;
  int nm_a = 0, nm_b = 0;
  if (lin_on) {
    nm_a = lq.marg_cnt[bh * lq.nqb + qa];
    if (qb2 >= 0) nm_b = lq.marg_cnt[bh * lq.nqb + qb2];
  }
  const bool lin = nm_a > 0 || nm_b > 0;

  if (pad + kUsed > kBwdSmemRequest) {
    if (threadIdx.x == 0) atomicExch(status, static_cast<int32_t>(SLA_ERR_UNSUPPORTED));
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_s(b), 1);
      mbar_init(b_ds(b), 8);
    }
    mbar_init(b_done, 1);
    mbar_init(b_lin, 1);
    mbar_init(b_g, 1);
    mbar_init(b_den, 8);
    mbar_init(b_go, 8);
    mbar_init(b_dn, 8);
    mbar_init(b_df, 1);
    mbar_init(b_dh1, 1);
    mbar_init(b_dfr, 8);
    mbar_init(b_dh2, 1);
    mbar_init(b_dz, 8);
    mbar_init(b_qt, 8);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kBwdTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // columns: S of steps with parity b at 64 b, dP at 128 + 64 b, dQ at 256;
  // dS (bf16, two keys per column) overwrites the first 16 of each half's
  // 32 S columns
  auto tS = [&](int b) { return tmem + 64u * static_cast<uint32_t>(b); };
  auto tP = [&](int b) { return tmem + 128u + 64u * static_cast<uint32_t>(b); };
  const uint32_t tQ = tmem + 256;
  // during the main loop Q and dO also sit in TMEM (bf16 pairs, row m in
  // lane m) as the A operands of S = Q K^T and dP = dO V^T, so those
  // products read only K and V from shared memory; the linear epilogue
  // reuses these columns afterwards
  const uint32_t tQa = tmem + 384, tdOa = tmem + 448;
  BwdShared sh{bars, abort_flag, status, timeout};

  if (warp == 0) {
    if (lane == 0 && (U > 0 || lin)) {
      mbar_expect_tx(b_q, 2 * kTileBytes);
#pragma unroll
      for (int c = 0; c < DC; ++c) {
        tma_load_3d(sb + offQ + c * 16384, &tmQ, c * 64, qt * 128, bh, b_q);
        tma_load_3d(sb + offdO + c * 16384, &tmdO, c * 64, qt * 128, bh, b_q);
      }
      int u = 0;
      bool ok = true;
      uint32_t desc_next = T > 0 ? ptiles[0] : 0u;  // (a plan word fetched a tile ahead)
      for (int t = 0; ok && t < T; ++t) {
        const uint32_t desc = desc_next;
        if (t + 1 < T) desc_next = ptiles[t + 1];
        for (int e = 0; ok && e < 2; ++e) {
          const Step st = step_of<BK>(desc, e, N);
          if (!st.present) continue;
          const int s = u % kBwdStages;
          if (u >= kBwdStages && !bwait(sh, b_empty(s), ((u / kBwdStages) & 1) ^ 1)) { ok = false; break; }
          const uint32_t dst = sb + offKV + s * kStageBytes;
          if (!(debug_skip && tile == 0 && u == 0)) {  // test aid: tile 0's first step never arrives
            mbar_expect_tx(b_full(s), kStageBytes);
#pragma unroll
            for (int c = 0; c < DC; ++c) {
              tma_load_3d(dst + c * 8192, &tmK, c * 64, st.row0, bh, b_full(s));
              tma_load_3d(dst + kHalfBytes + c * 8192, &tmV, c * 64, st.row0, bh, b_full(s));
            }
          }
          ++u;
        }
      }
      // linear epilogue: W and H^M into the K/V stages once every dQ MMA
      // (the stages' last readers) has completed
      if constexpr (D == 128) {
        if (ok && lin && (U == 0 || bwait(sh, b_done, 0))) {
          mbar_expect_tx(b_lin, 32768u + (nm_a > 0 ? 32768u : 0u) + (nm_b > 0 ? 32768u : 0u));
          tma_load_2d(sb + offW, &tmW, 0, 0, b_lin);
          tma_load_2d(sb + offW + 16384, &tmW, 64, 0, b_lin);
          if (nm_a > 0) {
            const int hr = (bh * lq.nqb + qa) * 128;
            tma_load_2d(sb + offHA, &tmHM, 0, hr, b_lin);
            tma_load_2d(sb + offHA + 16384, &tmHM, 64, hr, b_lin);
          }
          if (nm_b > 0) {
            const int hr = (bh * lq.nqb + qb2) * 128;
            tma_load_2d(sb + offHB, &tmHM, 0, hr, b_lin);
            tma_load_2d(sb + offHB + 16384, &tmHM, 64, hr, b_lin);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && U > 0) {
      bool ok = bwait(sh, b_q, 0);
      // base descriptors, built once and advanced by constant offsets
      const uint64_t dQd = sdesc(sb + offQ, 16, 1024), ddO = sdesc(sb + offdO, 16, 1024);
      const uint64_t dKV = sdesc(sb + offKV, 16, 1024), dKVmn = sdesc(sb + offKV, 8192, 1024);
      auto issue_sdp = [&](int u) -> bool {
        const int s = u % kBwdStages, b = u & 1;
        if (!bwait(sh, b_full(s), (u / kBwdStages) & 1)) return false;
        tc_fence_after();
        const uint64_t dK = sdesc_add(dKV, s * kStageBytes), dV = sdesc_add(dK, kHalfBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // 16 channels = 8 TMEM columns of Q
          const uint32_t ob = (kk / 4) * 8192 + (kk % 4) * 32;
          tc_mma_ts(tS(b), tQa + kk * 8, sdesc_add(dK, ob), idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ob = (kk / 4) * 8192 + (kk % 4) * 32;
          tc_mma_ts(tP(b), tdOa + kk * 8, sdesc_add(dV, ob), idesc_s, kk > 0);
        }
        tc_commit(b_s(b));
        return true;
      };
      auto issue_dq = [&](int u) -> bool {
        const int s = u % kBwdStages, b = u & 1;
        if (!bwait(sh, b_ds(b), (u >> 1) & 1)) return false;
        tc_fence_after();
        const uint64_t dKmn = sdesc_add(dKVmn, s * kStageBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 16 keys = 8 columns of dS
          tc_mma_ts(tQ, tS(b) + 32 * (kk / 2) + (kk % 2) * 8, sdesc_add(dKmn, kk * 2048), idesc_dq,
                    (u > 0 || kk > 0) ? 1u : 0u);
        tc_commit(b_empty(s));
        return true;
      };
      if (ok) ok = bwait(sh, b_qt, 0);  // Q and dO in TMEM
      if (ok) ok = issue_sdp(0);
      for (int u = 0; ok && u < U; ++u) {
        if (u + 1 < U) ok = issue_sdp(u + 1);
        if (ok) ok = issue_dq(u);
      }
      if (ok) tc_commit(b_done);
    }
    if constexpr (D == 128) {
      if (lane == 0 && lin) {
        // g = dO W^T -> columns 384.. (M = 128 rows, N = 128, K = 128)
        bool ok = bwait(sh, b_lin, 0) && bwait(sh, b_q, 0);
        constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t id_mn = idesc_bf16(128, 128, 1, 1);
        const uint64_t ddO = sdesc(sb + offdO, 16, 1024), dW = sdesc(sb + offW, 16, 1024);
        const uint64_t dDn = sdesc(sb + offDn, 16, 1024), dDnmn = sdesc(sb + offDn, 16384, 1024);
        const uint64_t dHA = sdesc(sb + offHA, 16, 1024), dHB = sdesc(sb + offHB, 16, 1024);
        const uint64_t dPhimn = sdesc(sb + offQ, 16384, 1024);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t o = (kk / 4) * 16384 + (kk % 4) * 32;
            tc_mma(tmem + 384, sdesc_add(ddO, o), sdesc_add(dW, o), id_kk, kk > 0);
          }
          tc_commit(b_g);
          ok = bwait(sh, b_dn, 0);
        }
        if (ok) {
          // df = dnum H^M^T (M = rows, N = channels a, K = c): block A into
          // columns 0.., block B into 128..
          tc_fence_after();
          for (int q2 = 0; q2 < 2; ++q2) {
            if ((q2 == 0 ? nm_a : nm_b) <= 0) continue;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t o = (kk / 4) * 16384 + (kk % 4) * 32;
              tc_mma(tmem + 128u * q2, sdesc_add(dDn, o), sdesc_add(q2 == 0 ? dHA : dHB, o), id_kk,
                     kk > 0);
            }
          }
          tc_commit(b_df);
          // dH^M of block A = phi(Q_A)^T dnum_A (M = a, N = c, K = its rows),
          // into columns 384.. (g has been read)
          constexpr int kRowsA = BQ == 128 ? 128 : 64;
          if (nm_a > 0) {
#pragma unroll
            for (int kk = 0; kk < kRowsA / 16; ++kk)
              tc_mma(tmem + 384, sdesc_add(dPhimn, kk * 2048), sdesc_add(dDnmn, kk * 2048), id_mn,
                     kk > 0);
          }
          tc_commit(b_dh1);
          if (BQ == 64 && nm_b > 0) {  // block B's rows 64-127, into columns 0.. once df is read
            ok = bwait(sh, b_dfr, 0);
            if (ok) {
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc_mma(tmem, sdesc_add(dPhimn, 8192 + kk * 2048), sdesc_add(dDnmn, 8192 + kk * 2048),
                       id_mn, kk > 0);
              tc_commit(b_dh2);
            }
          }
        }
      }
    }
  } else {
    const int h = (warp - 2) >> 2;  // key half of each step
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t rflag = BQ == 128 ? 3u : (r < 64 ? 1u : 2u);
    const unsigned full = 0xffffffffu;
    const int row = qt * 128 + r;
    float lse2 = INFINITY, dl = 0.f;
    if (row < N) {
      const float l = lse[static_cast<i64>(bh) * N + row];
      lse2 = l > -INFINITY ? l * 1.4426950408889634f : INFINITY;
      dl = delta[static_cast<i64>(bh) * N + row];
    }
    const float2 c2 = make_float2(scale_log2, scale_log2);
    const float2 nl2 = make_float2(-lse2, -lse2);
    const float2 nd2 = make_float2(-dl, -dl);
    bool ok = true;
    if (U > 0) {
      // Q and dO of row r, channels [h D/2, (h + 1) D/2), into TMEM as bf16
      // pairs (even channel in the low half), from their swizzled tiles
      ok = __all_sync(full, bwait(sh, b_q, 0));
      if (ok) {
        uint32_t pq[D / 4], pd[D / 4];
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
          const int ch = h * (D / 2) + 8 * i;
          const uint32_t off = (ch / 64) * 16384 + sw128(r, (ch % 64) / 8);
          const uint4 vq = *reinterpret_cast<const uint4*>(base + offQ + off);
          const uint4 vd = *reinterpret_cast<const uint4*>(base + offdO + off);
          pq[4 * i] = vq.x; pq[4 * i + 1] = vq.y; pq[4 * i + 2] = vq.z; pq[4 * i + 3] = vq.w;
          pd[4 * i] = vd.x; pd[4 * i + 1] = vd.y; pd[4 * i + 2] = vd.z; pd[4 * i + 3] = vd.w;
        }
        if constexpr (D == 128) {
          tmem_st32u(tQa + lane_off + 32 * h, pq);
          tmem_st32u(tdOa + lane_off + 32 * h, pd);
        } else {
          tmem_st16u(tQa + lane_off + 16 * h, pq);
          tmem_st16u(tdOa + lane_off + 16 * h, pd);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_qt);
    }
    int u = 0;
    uint32_t desc_next = T > 0 ? ptiles[0] : 0u;  // (a plan word fetched a tile ahead)
    for (int t = 0; ok && t < T; ++t) {
      const uint32_t desc = desc_next;
      if (t + 1 < T) desc_next = ptiles[t + 1];
      for (int e = 0; e < 2; ++e) {
        const Step st = step_of<BK>(desc, e, N);
        if (!st.present) continue;
        const int b = u & 1;
        const bool member = (st.flags & rflag) != 0;
        const int kvalid = member ? max(0, min(32, N - st.row0 - 32 * h)) : 0;
        if (!__all_sync(full, bwait(sh, b_s(b), (u >> 1) & 1))) { ok = false; break; }
        tc_fence_after();
        float s[32], dp[32];
        tmem_ld32(tS(b) + lane_off + 32 * h, s);
        tmem_ld32(tP(b) + lane_off + 32 * h, dp);
        tmem_wait_ld();
        reg_fence<32>(s);
        reg_fence<32>(dp);
        uint32_t pk[16];
        if (kvalid > 0) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 x = fma2(make_float2(s[2 * i], s[2 * i + 1]), c2, nl2);
            float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            if (kvalid < 32) {
              p.x = 2 * i < kvalid ? p.x : 0.f;
              p.y = 2 * i + 1 < kvalid ? p.y : 0.f;
            }
            const float2 ds = mul2(p, add2(make_float2(dp[2 * i], dp[2 * i + 1]), nd2));
            pk[i] = pack_bf16x2(ds.x, ds.y);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        }
        tmem_st16u(tS(b) + lane_off + 32 * h, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_ds(b));
        ++u;
      }
    }
    // dQ (scaled) -> global; rows of a tile without steps get zeros
    const bool fin = ok && (U == 0 || __all_sync(full, bwait(sh, b_done, 0)));
    if (fin && U > 0) tc_fence_after();
    constexpr int DH = D / 2;
    const i64 orow = (static_cast<i64>(bh) * N + row) * D + h * DH;
    bool lin_done = false;  // dq written by the linear epilogue
    if constexpr (D == 128) {
      if (lin && fin) {
        // this thread: row r, channels [64h, 64h + 64)
        const bool second = BQ == 64 && r >= 64;
        const int nm_r = second ? nm_b : nm_a;
        float4 z4[16];
        if (nm_r > 0) {
          const float4* zp = reinterpret_cast<const float4*>(
              lq.zm + (static_cast<i64>(bh) * lq.nqb + (second ? qb2 : qa)) * 128 + h * 64);
#pragma unroll
          for (int i = 0; i < 16; ++i) z4[i] = __ldg(zp + i);
        }
        bool lok = __all_sync(full, bwait(sh, b_q, 0));
        // phi(Q) in place, and this half of den = phi(q) . z^M from the same
        // rounded values (as the forward forms it)
        float dpart = 0.f, dpart2 = 0.f;
        if (lok) {
          // all eight pieces read before any is written back (a read after
          // a store to the same tile would wait for it)
          uint4 qv[8];
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) qv[u8] = *reinterpret_cast<const uint4*>(base + offQ + h * 16384 + sw128(r, u8));
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) {
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (row < N && nm_r > 0) {
              val = phi_unit(qv[u8]);
              const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.x));
              const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.y));
              const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.z));
              const float2 f3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&val.w));
              const float4 za = z4[2 * u8], zb = z4[2 * u8 + 1];
              dpart = fmaf(f0.x, za.x, fmaf(f0.y, za.y, fmaf(f1.x, za.z, fmaf(f1.y, za.w, dpart))));
              dpart2 = fmaf(f2.x, zb.x, fmaf(f2.y, zb.y, fmaf(f3.x, zb.z, fmaf(f3.y, zb.w, dpart2))));
            }
            qv[u8] = val;
          }
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) *reinterpret_cast<uint4*>(base + offQ + h * 16384 + sw128(r, u8)) = qv[u8];
          red[h * 128 + r] = dpart + dpart2;
          __syncwarp();
          if (lane == 0) mbar_arrive(b_den);
          lok = __all_sync(full, bwait(sh, b_den, 0));
        }
        const float den = lok ? dpart + dpart2 + red[(h ^ 1) * 128 + r] : 0.f;
        const float dinv = (nm_r > 0 && den > 0.f && row < N) ? 1.f / den : 0.f;
        // g and this half of g . o
        if (lok) lok = __all_sync(full, bwait(sh, b_g, 0));
        float gv[64];
        float go = 0.f;
        if (lok) {
          tc_fence_after();
          tmem_ld32(tmem + 384 + lane_off + h * 64, gv);
          tmem_ld32(tmem + 384 + lane_off + h * 64 + 32, gv + 32);
          tmem_wait_ld();
          reg_fence<64>(gv);
          if (row < N && nm_r > 0) {
            const float4* op = reinterpret_cast<const float4*>(
                lq.o_lin + (static_cast<i64>(bh) * N + row) * 128 + h * 64);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float4 o4 = __ldg(op + i);
              go = fmaf(gv[4 * i], o4.x, fmaf(gv[4 * i + 1], o4.y,
                        fmaf(gv[4 * i + 2], o4.z, fmaf(gv[4 * i + 3], o4.w, go))));
            }
          }
          red[(2 + h) * 128 + r] = go;
          __syncwarp();
          if (lane == 0) mbar_arrive(b_go);
          lok = __all_sync(full, bwait(sh, b_go, 0));
        }
        const float ddn = lok ? -(go + red[(2 + (h ^ 1)) * 128 + r]) * dinv : 0.f;
        if (lok) {
          // dnum = g / den (bf16) into the K-major [row][c] tile
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8)
            *reinterpret_cast<uint4*>(base + offDn + h * 16384 + sw128(r, u8)) = make_uint4(
                pack_bf16x2(gv[8 * u8] * dinv, gv[8 * u8 + 1] * dinv),
                pack_bf16x2(gv[8 * u8 + 2] * dinv, gv[8 * u8 + 3] * dinv),
                pack_bf16x2(gv[8 * u8 + 4] * dinv, gv[8 * u8 + 5] * dinv),
                pack_bf16x2(gv[8 * u8 + 6] * dinv, gv[8 * u8 + 7] * dinv));
          if (h == 0) dd[r] = ddn;
          fence_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_dn);
          lok = __all_sync(full, bwait(sh, b_df, 0));
        }
        if (lok) {
          // dq = s dQ + (df + dden z^M) o phi'(q), written once
          tc_fence_after();
          const uint32_t tdf = tmem + (second ? 128u : 0u);
          const __nv_bfloat16* qrow = lq.q + (static_cast<i64>(bh) * N + row) * 128 + h * 64;
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            float dfv[32], dqv[32];
            if (nm_r > 0) tmem_ld32(tdf + lane_off + h * 64 + c0, dfv);
            if (U > 0) tmem_ld32(tQ + lane_off + h * 64 + c0, dqv);
            tmem_wait_ld();
            reg_fence<32>(dfv);
            reg_fence<32>(dqv);
            if (row < N) {
#pragma unroll
              for (int i8 = 0; i8 < 4; ++i8) {
                const uint4 qu = *reinterpret_cast<const uint4*>(qrow + c0 + 8 * i8);
                const uint32_t qw[4] = {qu.x, qu.y, qu.z, qu.w};
                float ov[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qw[e]));
                  const int c = c0 + 8 * i8 + 2 * e;
                  const float zx = reinterpret_cast<const float*>(&z4[c / 4])[c % 4];
                  const float zy = reinterpret_cast<const float*>(&z4[c / 4])[c % 4 + 1];
                  const float base0 = U > 0 ? scale * dqv[8 * i8 + 2 * e] : 0.f;
                  const float base1 = U > 0 ? scale * dqv[8 * i8 + 2 * e + 1] : 0.f;
                  ov[2 * e] = nm_r > 0 ? base0 + (dfv[8 * i8 + 2 * e] + ddn * zx) * dphi(qf.x) : base0;
                  ov[2 * e + 1] = nm_r > 0 ? base1 + (dfv[8 * i8 + 2 * e + 1] + ddn * zy) * dphi(qf.y) : base1;
                }
                float* dst = dq + orow + c0 + 8 * i8;
                *reinterpret_cast<float4*>(dst) = make_float4(ov[0], ov[1], ov[2], ov[3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(ov[4], ov[5], ov[6], ov[7]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_dfr);
          lin_done = true;
        }
      }
    }
#pragma unroll
    for (int c = 0; !lin_done && c < DH; c += 32) {
      float o[32];
      if (fin && U > 0) {
        tmem_ld32(tQ + lane_off + h * DH + c, o);
        tmem_wait_ld();
        reg_fence<32>(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= scale;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      if (row < N && fin) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(dq + orow + c + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
      }
    }
    if constexpr (D == 128) {
      if (lin_on && fin) {
        // dH^M (bf16) and dz^M of the tile's query blocks; zeros for blocks
        // without marginal sets (the key side's gather reads every block).
        // Accumulator lane = channel a.  64-row blocks: half h writes block h;
        // a 128-row block: half h writes columns [64h, 64h + 64) and sums
        // dz^M over rows [64h, 64h + 64).
        const int a = quad * 32 + lane;
        const int bsel = BQ == 64 ? h : 0;
        const int qblk = bsel == 0 ? qa : qb2;
        const int nmb = bsel == 0 ? nm_a : nm_b;
        const bool have = nmb > 0 && lin_done;
        if (qblk >= 0) {
          __nv_bfloat16* dst = lq.dhm + (static_cast<i64>(bh) * lq.nqb + qblk) * 16384 + a * 128;
          constexpr int kCN = BQ == 64 ? 128 : 64;
          const int clo = BQ == 64 ? 0 : h * 64;
          bool hok = have;
          if (have) hok = __all_sync(full, bwait(sh, bsel == 0 ? b_dh1 : b_dh2, 0));
          if (hok) tc_fence_after();
          const uint32_t tsrc = (bsel == 0 ? tmem + 384 : tmem) + lane_off;
#pragma unroll
          for (int c0 = 0; c0 < kCN; c0 += 32) {
            float v[32];
            if (hok) {
              tmem_ld32(tsrc + clo + c0, v);
              tmem_wait_ld();
              reg_fence<32>(v);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              *reinterpret_cast<uint4*>(dst + clo + c0 + 8 * q4) =
                  make_uint4(pack_bf16x2(v[8 * q4], v[8 * q4 + 1]), pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                             pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]), pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
          }
          // dz^M[a] = sum over the block's rows of phi(Q)[row][a] dden[row]
          float dz = 0.f;
          if (hok) {
            const int r0 = BQ == 64 ? 64 * bsel : 64 * h;
            const uint8_t* chunk = base + offQ + (a >> 6) * 16384;
            for (int rr = r0; rr < r0 + 64; ++rr) {
              const uint16_t bits =
                  *reinterpret_cast<const uint16_t*>(chunk + sw128(rr, (a & 63) >> 3) + (a & 7) * 2);
              dz = fmaf(__uint_as_float(static_cast<uint32_t>(bits) << 16), dd[rr], dz);
            }
          }
          float* zdst = lq.dzm + (static_cast<i64>(bh) * lq.nqb + qblk) * 128 + a;
          if (BQ == 64) {
            *zdst = dz;
          } else {
            red[h * 128 + a] = dz;  // (slot 0-1: den was read before the dnum barrier)
            __syncwarp();
            if (lane == 0) mbar_arrive(b_dz);
            if (__all_sync(full, bwait(sh, b_dz, 0)) && h == 0) *zdst = dz + red[128 + a];
          }
        }
      }
    }
  }
  teardown(sh, warp, tmem);
}

// ------------------------------------------------------------------ dK, dV
template <int D, int BQ, int BK>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                        const __grid_constant__ CUtensorMap tmDH,
                        const int32_t* __restrict__ tile_cnt, const uint32_t* __restrict__ tiles,
                        int plan_stride, const float* __restrict__ lse,
                        const float* __restrict__ delta, float* __restrict__ dk,
                        float* __restrict__ dv, LinBwdK lk, int32_t* status, int N, int nkt,
                        float scale, float scale_log2, long long timeout, int debug_skip) {
  constexpr int DC = D / 64;
  constexpr uint32_t kTileBytes = DC * 16384;  // 128 rows x D bf16 (K, V)
  constexpr uint32_t kHalfBytes = DC * 8192;   // 64 rows x D bf16 (Q, dO)
  // stage: Q, dO, then -LSE*log2(e) and -Delta of the step's 64 queries
  constexpr uint32_t kStageBytes = 2 * kHalfBytes + 1024;
  constexpr uint32_t offK = 0, offV = kTileBytes, offSt = 2 * kTileBytes;
  constexpr uint32_t offBar = offSt + kBwdStages * kStageBytes;
  constexpr uint32_t kUsed = offBar + 256;
  constexpr uint32_t idesc_s = idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t idesc_g = idesc_bf16(128, D, 0, 1);
  // linear epilogue: after the main loop the stages hold dH of the tile's
  // first and second key block (0, 1) and, for 64-row blocks, phi(K) with
  // the other block's rows zeroed (2: first block, 3: second)
  constexpr uint32_t offDHA = offSt, offDHB = offSt + kStageBytes;
  constexpr uint32_t offPhA = offSt + 2 * kStageBytes, offPhB = offSt + 3 * kStageBytes;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* base = smem_raw + pad;
  const uint32_t sb = raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + offBar);
  const uint32_t b_kv = smem_u32(&bars[0]);
  auto b_full = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_empty = [&](int s) { return smem_u32(&bars[1 + kBwdStages + s]); };
  auto b_s = [&](int b) { return smem_u32(&bars[1 + 2 * kBwdStages + b]); };   // S^T, dP^T
  auto b_pd = [&](int b) { return smem_u32(&bars[3 + 2 * kBwdStages + b]); };  // P^T, dS^T
  const uint32_t b_done = smem_u32(&bars[5 + 2 * kBwdStages]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[6 + 2 * kBwdStages]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[7 + 2 * kBwdStages]);
  constexpr int kL0 = 8 + 2 * kBwdStages;
  const uint32_t b_lin = smem_u32(&bars[kL0]);       // dH landed
  const uint32_t b_phk = smem_u32(&bars[kL0 + 1]);   // phi(K) in smem (8 warps)
  const uint32_t b_lkv = smem_u32(&bars[kL0 + 2]);   // linear dV, dphi in TMEM
  static_assert((kL0 + 3) * 8 <= 256, "barrier block");

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x;
  const int bh = tile / nkt, kt = tile % nkt;
  const int T = tile_cnt[tile];
  const uint32_t* ptiles = tiles + static_cast<i64>(tile) * plan_stride;
  const int U = plan_steps<BQ>(ptiles, T, N);
  // linear branch of the tile's key blocks (A: rows 0-63 or the whole
  // 128-row block; B: rows 64-127 when blocks are 64 rows)
  const int ja = BK == 128 ? kt : 2 * kt;
  const int jb = (BK == 64 && 2 * kt + 1 < lk.nkb) ? 2 * kt + 1 : -1;
  int nm_a = 0, nm_b = 0;
  if (D == 128 && lk.marg_cnt != nullptr) {
    nm_a = lk.marg_cnt[bh * lk.nkb + ja];
    if (jb >= 0) nm_b = lk.marg_cnt[bh * lk.nkb + jb];
  }
  const bool lin = nm_a > 0 || nm_b > 0;

  if (pad + kUsed > kBwdSmemRequest) {
    if (threadIdx.x == 0) atomicExch(status, static_cast<int32_t>(SLA_ERR_UNSUPPORTED));
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(b_kv, 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(b_full(s), 2);  // TMA bytes + the producer's LSE / Delta stores
      mbar_init(b_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_s(b), 1);
      mbar_init(b_pd(b), 8);
    }
    mbar_init(b_done, 1);
    mbar_init(b_lin, 1);
    mbar_init(b_phk, 8);
    mbar_init(b_lkv, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kBwdTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // columns: S^T of steps with parity b at 64 b, dP^T at 128 + 64 b, dK at
  // 256, dV at 256 + D; P^T and dS^T (bf16) overwrite the first 16 of each
  // half's 32 S^T and dP^T columns
  auto tS = [&](int b) { return tmem + 64u * static_cast<uint32_t>(b); };
  auto tP = [&](int b) { return tmem + 128u + 64u * static_cast<uint32_t>(b); };
  const uint32_t tK = tmem + 256, tV = tmem + 256 + D;
  BwdShared sh{bars, abort_flag, status, timeout};

  if (warp == 0) {
    // K and V tiles stay resident; the steps stream Q, dO and the per-query
    // -LSE*log2(e), -Delta (q >= N: -inf and 0, so those columns vanish)
    if (U > 0 || lin) {
      if (lane == 0) {
        mbar_expect_tx(b_kv, 2 * kTileBytes);
#pragma unroll
        for (int c = 0; c < DC; ++c) {
          tma_load_3d(sb + offK + c * 16384, &tmK, c * 64, kt * 128, bh, b_kv);
          tma_load_3d(sb + offV + c * 16384, &tmV, c * 64, kt * 128, bh, b_kv);
        }
      }
      int u = 0;
      bool ok = true;
      uint32_t desc_next = T > 0 ? ptiles[0] : 0u;  // (a plan word fetched a tile ahead)
      for (int t = 0; ok && t < T; ++t) {
        const uint32_t desc = desc_next;
        if (t + 1 < T) desc_next = ptiles[t + 1];
        for (int e = 0; e < 2; ++e) {
          const Step st = step_of<BQ>(desc, e, N);
          if (!st.present) continue;
          const int s = u % kBwdStages;
          // this step's -LSE log2(e) and -Delta, loaded before the wait for
          // the stage so that their latency hides behind it
          float na[2], nd[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int q = st.row0 + 32 * j + lane;
            na[j] = -INFINITY;
            nd[j] = 0.f;
            if (q < N) {
              const float l = lse[static_cast<i64>(bh) * N + q];
              na[j] = l > -INFINITY ? -l * 1.4426950408889634f : -INFINITY;
              nd[j] = -delta[static_cast<i64>(bh) * N + q];
            }
          }
          bool got = true;
          if (lane == 0 && u >= kBwdStages) got = bwait(sh, b_empty(s), ((u / kBwdStages) & 1) ^ 1);
          if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
          const uint32_t dst = sb + offSt + s * kStageBytes;
          if (lane == 0 && !(debug_skip && tile == 0 && u == 0)) {  // test aid: tile 0's first step
            mbar_expect_tx(b_full(s), 2 * kHalfBytes);                //   never arrives
#pragma unroll
            for (int c = 0; c < DC; ++c) {
              tma_load_3d(dst + c * 8192, &tmQ, c * 64, st.row0, bh, b_full(s));
              tma_load_3d(dst + kHalfBytes + c * 8192, &tmdO, c * 64, st.row0, bh, b_full(s));
            }
          }
          float* nl = reinterpret_cast<float*>(base + offSt + s * kStageBytes + 2 * kHalfBytes);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            nl[32 * j + lane] = na[j];
            nl[64 + 32 * j + lane] = nd[j];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(b_full(s));
          ++u;
        }
      }
      // linear epilogue: dH of the tile's key blocks into stages 0 and 1
      // once every MMA of the main loop (the stages' last readers) completed
      if constexpr (D == 128) {
        if (lane == 0 && ok && lin && (U == 0 || bwait(sh, b_done, 0))) {
          mbar_expect_tx(b_lin, (nm_a > 0 ? 32768u : 0u) + (nm_b > 0 ? 32768u : 0u));
          if (nm_a > 0) {
            const int hr = (bh * lk.nkb + ja) * 128;
            tma_load_2d(sb + offDHA, &tmDH, 0, hr, b_lin);
            tma_load_2d(sb + offDHA + 16384, &tmDH, 64, hr, b_lin);
          }
          if (nm_b > 0) {
            const int hr = (bh * lk.nkb + jb) * 128;
            tma_load_2d(sb + offDHB, &tmDH, 0, hr, b_lin);
            tma_load_2d(sb + offDHB + 16384, &tmDH, 64, hr, b_lin);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && U > 0) {
      bool ok = bwait(sh, b_kv, 0);
      // base descriptors, built once and advanced by constant offsets
      const uint64_t dKd = sdesc(sb + offK, 16, 1024), dVd = sdesc(sb + offV, 16, 1024);
      const uint64_t dSt = sdesc(sb + offSt, 16, 1024), dStmn = sdesc(sb + offSt, 8192, 1024);
      auto issue_sdp = [&](int u) -> bool {
        const int s = u % kBwdStages, b = u & 1;
        if (!bwait(sh, b_full(s), (u / kBwdStages) & 1)) return false;
        tc_fence_after();
        const uint64_t dQs = sdesc_add(dSt, s * kStageBytes), ddOs = sdesc_add(dQs, kHalfBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = (kk / 4) * 16384 + (kk % 4) * 32;
          const uint32_t ob = (kk / 4) * 8192 + (kk % 4) * 32;
          tc_mma(tS(b), sdesc_add(dKd, oa), sdesc_add(dQs, ob), idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = (kk / 4) * 16384 + (kk % 4) * 32;
          const uint32_t ob = (kk / 4) * 8192 + (kk % 4) * 32;
          tc_mma(tP(b), sdesc_add(dVd, oa), sdesc_add(ddOs, ob), idesc_s, kk > 0);
        }
        tc_commit(b_s(b));
        return true;
      };
      auto issue_grad = [&](int u) -> bool {
        const int s = u % kBwdStages, b = u & 1;
        if (!bwait(sh, b_pd(b), (u >> 1) & 1)) return false;
        tc_fence_after();
        const uint64_t dQmn = sdesc_add(dStmn, s * kStageBytes), ddOmn = sdesc_add(dQmn, kHalfBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dV += P^T dO: 16 queries = 8 columns
          tc_mma_ts(tV, tS(b) + 32 * (kk / 2) + (kk % 2) * 8, sdesc_add(ddOmn, kk * 2048), idesc_g,
                    (u > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dK += dS^T Q
          tc_mma_ts(tK, tP(b) + 32 * (kk / 2) + (kk % 2) * 8, sdesc_add(dQmn, kk * 2048), idesc_g,
                    (u > 0 || kk > 0) ? 1u : 0u);
        tc_commit(b_empty(s));
        return true;
      };
      if (ok) ok = issue_sdp(0);
      for (int u = 0; ok && u < U; ++u) {
        if (u + 1 < U) ok = issue_sdp(u + 1);
        if (ok) ok = issue_grad(u);
      }
      if (ok) tc_commit(b_done);
    }
    if constexpr (D == 128) {
      if (lane == 0 && lin) {
        bool ok = bwait(sh, b_lin, 0) && bwait(sh, b_phk, 0);
        if (ok) {
          tc_fence_after();
          constexpr uint32_t id_dv = idesc_bf16(128, 128, 0, 1);  // A phi(K) K-major, B dH MN-major
          constexpr uint32_t id_dp = idesc_bf16(128, 128, 0, 0);  // A V, B dH rows: both K-major
          const uint64_t dHAmn = sdesc(sb + offDHA, 16384, 1024), dHBmn = sdesc(sb + offDHB, 16384, 1024);
          const uint64_t dHAk = sdesc(sb + offDHA, 16, 1024), dHBk = sdesc(sb + offDHB, 16, 1024);
          const uint64_t dPhA = sdesc(sb + (BK == 128 ? offK : offPhA), 16, 1024);
          const uint64_t dPhB = sdesc(sb + offPhB, 16, 1024);
          const uint64_t dVd = sdesc(sb + offV, 16, 1024);
          // dv += phi(K) dH (M = key rows, N = c, K = a), into the dV
          // accumulator (written fresh when the tile had no critical step)
          bool fresh = U == 0;
          for (int q2 = 0; q2 < 2; ++q2) {
            if ((q2 == 0 ? nm_a : nm_b) <= 0) continue;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc_mma(tV, sdesc_add(q2 == 0 ? dPhA : dPhB, (kk / 4) * 16384 + (kk % 4) * 32),
                     sdesc_add(q2 == 0 ? dHAmn : dHBmn, kk * 2048), id_dv, (fresh && kk == 0) ? 0u : 1u);
            fresh = false;
          }
          // dphi = V dH^T (M = key rows, N = a, K = c): block A into
          // columns 0.., block B into 128..
          for (int q2 = 0; q2 < 2; ++q2) {
            if ((q2 == 0 ? nm_a : nm_b) <= 0) continue;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t o = (kk / 4) * 16384 + (kk % 4) * 32;
              tc_mma(tmem + 128u * q2, sdesc_add(dVd, o), sdesc_add(q2 == 0 ? dHAk : dHBk, o), id_dp,
                     kk > 0);
            }
          }
          tc_commit(b_lkv);
        }
      }
    }
  } else {
    const int h = (warp - 2) >> 2;  // query half of each step
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // key row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t rflag = BK == 128 ? 3u : (r < 64 ? 1u : 2u);
    const unsigned full = 0xffffffffu;
    const int key = kt * 128 + r;
    const float2 c2 = make_float2(scale_log2, scale_log2);
    bool ok = true;
    int u = 0;
    uint32_t desc_next = T > 0 ? ptiles[0] : 0u;  // (a plan word fetched a tile ahead)
    for (int t = 0; ok && t < T; ++t) {
      const uint32_t desc = desc_next;
      if (t + 1 < T) desc_next = ptiles[t + 1];
      for (int e = 0; e < 2; ++e) {
        const Step st = step_of<BQ>(desc, e, N);
        if (!st.present) continue;
        const int b = u & 1, s = u % kBwdStages;
        const bool active = (st.flags & rflag) != 0 && key < N;
        if (!__all_sync(full, bwait(sh, b_s(b), (u >> 1) & 1))) { ok = false; break; }
        tc_fence_after();
        float sv[32], dp[32];
        tmem_ld32(tS(b) + lane_off + 32 * h, sv);
        tmem_ld32(tP(b) + lane_off + 32 * h, dp);
        tmem_wait_ld();
        reg_fence<32>(sv);
        reg_fence<32>(dp);
        const float* nl = reinterpret_cast<const float*>(base + offSt + s * kStageBytes + 2 * kHalfBytes) + 32 * h;
        uint32_t pt[16], dt[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 nl2 = *reinterpret_cast<const float2*>(nl + 2 * i);
          const float2 nd2 = *reinterpret_cast<const float2*>(nl + 64 + 2 * i);
          const float2 x = fma2(make_float2(sv[2 * i], sv[2 * i + 1]), c2, nl2);
          float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          if (!active) p = make_float2(0.f, 0.f);
          // masked query columns (-inf) give 0 through ex2 already; the
          // explicit zero also holds if a score there is not finite
          if (nl2.x == -INFINITY) p.x = 0.f;
          if (nl2.y == -INFINITY) p.y = 0.f;
          pt[i] = pack_bf16x2(p.x, p.y);
          const float2 ds = mul2(p, add2(make_float2(dp[2 * i], dp[2 * i + 1]), nd2));
          dt[i] = pack_bf16x2(ds.x, ds.y);
        }
        tmem_st16u(tS(b) + lane_off + 32 * h, pt);
        tmem_st16u(tP(b) + lane_off + 32 * h, dt);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_pd(b));
        ++u;
      }
    }
    const bool fin = ok && (U == 0 || __all_sync(full, bwait(sh, b_done, 0)));
    if (fin && U > 0) tc_fence_after();
    constexpr int DH = D / 2;
    const i64 orow = (static_cast<i64>(bh) * N + key) * D + h * DH;
    bool lin_done = false;  // dk, dv written by the linear epilogue
    if constexpr (D == 128) {
      if (lin && fin) {
        // this thread: key row r, channels [64h, 64h + 64)
        const bool second = BK == 64 && r >= 64;
        const int nm_r = second ? nm_b : nm_a;
        const int jblk = second ? jb : ja;
        bool lok = __all_sync(full, bwait(sh, b_kv, 0));
        if (lok) {
          // phi(K) (rows past N zero): in place for 128-row blocks; for
          // 64-row blocks into the copy of the row's own block, zeros into
          // the other's
          // (all eight pieces read before any store)
          uint4 kv[8];
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) kv[u8] = *reinterpret_cast<const uint4*>(base + offK + h * 16384 + sw128(r, u8));
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) {
            uint4* pk = reinterpret_cast<uint4*>(base + offK + h * 16384 + sw128(r, u8));
            const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
            const uint4 ph = key < N ? phi_unit(kv[u8]) : zero;
            if (BK == 128) {
              *pk = ph;
            } else {
              *reinterpret_cast<uint4*>(base + offPhA + h * 16384 + sw128(r, u8)) = second ? zero : ph;
              *reinterpret_cast<uint4*>(base + offPhB + h * 16384 + sw128(r, u8)) = second ? ph : zero;
            }
          }
          fence_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_phk);
          lok = __all_sync(full, bwait(sh, b_lkv, 0));
        }
        if (lok) {
          // dk = s dK + (dphi + dz) o phi'(k), dv = dV (the linear part is
          // already in the accumulator)
          tc_fence_after();
          float4 z4[16];
          if (nm_r > 0) {
            const float4* zp = reinterpret_cast<const float4*>(
                lk.dz + (static_cast<i64>(bh) * lk.nkb + jblk) * 128 + h * 64);
#pragma unroll
            for (int i = 0; i < 16; ++i) z4[i] = __ldg(zp + i);
          }
          const __nv_bfloat16* krow = lk.k + (static_cast<i64>(bh) * N + key) * 128 + h * 64;
          const uint32_t tdp = tmem + (second ? 128u : 0u);
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            float kv[32], vv[32], dpv[32];
            if (U > 0) tmem_ld32(tK + lane_off + h * 64 + c0, kv);
            tmem_ld32(tV + lane_off + h * 64 + c0, vv);
            if (nm_r > 0) tmem_ld32(tdp + lane_off + h * 64 + c0, dpv);
            tmem_wait_ld();
            reg_fence<32>(kv);
            reg_fence<32>(vv);
            reg_fence<32>(dpv);
            if (key < N) {
#pragma unroll
              for (int i8 = 0; i8 < 4; ++i8) {
                const uint4 ku = *reinterpret_cast<const uint4*>(krow + c0 + 8 * i8);
                const uint32_t kw[4] = {ku.x, ku.y, ku.z, ku.w};
                float ok8[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw[e]));
                  const int c = c0 + 8 * i8 + 2 * e;
                  const float zx = reinterpret_cast<const float*>(&z4[c / 4])[c % 4];
                  const float zy = reinterpret_cast<const float*>(&z4[c / 4])[c % 4 + 1];
                  const float b0 = U > 0 ? scale * kv[8 * i8 + 2 * e] : 0.f;
                  const float b1 = U > 0 ? scale * kv[8 * i8 + 2 * e + 1] : 0.f;
                  ok8[2 * e] = nm_r > 0 ? b0 + (dpv[8 * i8 + 2 * e] + zx) * dphi(kf.x) : b0;
                  ok8[2 * e + 1] = nm_r > 0 ? b1 + (dpv[8 * i8 + 2 * e + 1] + zy) * dphi(kf.y) : b1;
                }
                float* kd = dk + orow + c0 + 8 * i8;
                *reinterpret_cast<float4*>(kd) = make_float4(ok8[0], ok8[1], ok8[2], ok8[3]);
                *reinterpret_cast<float4*>(kd + 4) = make_float4(ok8[4], ok8[5], ok8[6], ok8[7]);
                float* vd = dv + orow + c0 + 8 * i8;
                *reinterpret_cast<float4*>(vd) = make_float4(vv[8 * i8], vv[8 * i8 + 1], vv[8 * i8 + 2], vv[8 * i8 + 3]);
                *reinterpret_cast<float4*>(vd + 4) =
                    make_float4(vv[8 * i8 + 4], vv[8 * i8 + 5], vv[8 * i8 + 6], vv[8 * i8 + 7]);
              }
            }
          }
          lin_done = true;
        }
      }
    }
#pragma unroll
    for (int which = 0; !lin_done && which < 2; ++which) {
      float* dst = which == 0 ? dk : dv;
      const uint32_t src = which == 0 ? tK : tV;
      const float mul = which == 0 ? scale : 1.f;
#pragma unroll
      for (int c = 0; c < DH; c += 32) {
        float o[32];
        if (fin && U > 0) {
          tmem_ld32(src + lane_off + h * DH + c, o);
          tmem_wait_ld();
          reg_fence<32>(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= mul;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (key < N && fin) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + orow + c + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
        }
      }
    }
  }
  teardown(sh, warp, tmem);
}

// ------------------------------------------------------------------ host

bool make_rows_map(CUtensorMap* m, const void* ptr, const Geom& g, int rows) {
  const uint64_t dims[3] = {static_cast<uint64_t>(g.d), static_cast<uint64_t>(g.N),
                            static_cast<uint64_t>(g.BH)};
  const uint64_t strides[2] = {static_cast<uint64_t>(g.d) * 2, static_cast<uint64_t>(g.N) * g.d * 2};
  const uint32_t box[3] = {64, static_cast<uint32_t>(rows), 1};
  return encode_bf16_map(m, ptr, 3, dims, strides, box);
}

struct BwdPlans {
  int32_t* qcnt;
  uint32_t* qtiles;
  int32_t* kcnt;
  uint32_t* ktiles;
  size_t bytes;
};

BwdPlans bwd_plans(const Geom& g, void* scratch) {
  const size_t nqt = (static_cast<size_t>(g.N) + 127) / 128, nkt = nqt;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  BwdPlans p;
  char* base = static_cast<char*>(scratch);
  size_t off = 0;
  p.qcnt = reinterpret_cast<int32_t*>(base + off); off = al(off + g.BH * nqt * sizeof(int32_t));
  p.qtiles = reinterpret_cast<uint32_t*>(base + off); off = al(off + g.BH * nqt * g.nkb * sizeof(uint32_t));
  p.kcnt = reinterpret_cast<int32_t*>(base + off); off = al(off + g.BH * nkt * sizeof(int32_t));
  p.ktiles = reinterpret_cast<uint32_t*>(base + off); off = al(off + g.BH * nkt * g.nqb * sizeof(uint32_t));
  p.bytes = off;
  return p;
}

template <int D, int BQ, int BK>
cudaError_t launch_dq_t(const CUtensorMap* m128, const CUtensorMap* m64, const CUtensorMap& mhm,
                        const CUtensorMap& mw, const LinBwdQ& lq, const BwdPlans& pl,
                        const float* lse, const float* delta, float* dq, int32_t* status,
                        const Geom& g, cudaStream_t s) {
  const int nt = (g.N + 127) / 128;
  const float scale_log2 = g.scale * 1.4426950408889634f;
  const long long timeout = wait_limit(g);
  const int debug_skip = debug_withhold(g, SLA_WITHHOLD_BWD_DQ) ? 1 : 0;
  // m128 / m64: {q, k, v, dout} maps with 128- and 64-row boxes
  auto kq = attn_bwd_dq_tc_kernel<D, BQ, BK>;
  cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kBwdSmemRequest));
  if (e != cudaSuccess) return e;
  kq<<<g.BH * nt, kBwdThreads, kBwdSmemRequest, s>>>(m128[0], m128[3], m64[1], m64[2], mhm, mw,
                                                     pl.qcnt, pl.qtiles, g.nkb, lse, delta, dq, lq,
                                                     status, g.N, nt, g.scale, scale_log2, timeout,
                                                     debug_skip);
  return cudaGetLastError();
}

template <int D, int BQ, int BK>
cudaError_t launch_dkdv_t(const CUtensorMap* m128, const CUtensorMap* m64, const CUtensorMap& mdh,
                          const LinBwdK& lk, const BwdPlans& pl, const float* lse,
                          const float* delta, float* dk, float* dv, int32_t* status,
                          const Geom& g, cudaStream_t s) {
  const int nt = (g.N + 127) / 128;
  const float scale_log2 = g.scale * 1.4426950408889634f;
  const long long timeout = wait_limit(g);
  const int debug_skip = debug_withhold(g, SLA_WITHHOLD_BWD_DKDV) ? 1 : 0;
  auto kk = attn_bwd_dkdv_tc_kernel<D, BQ, BK>;
  cudaError_t e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kBwdSmemRequest));
  if (e != cudaSuccess) return e;
  kk<<<g.BH * nt, kBwdThreads, kBwdSmemRequest, s>>>(m128[1], m128[2], m64[0], m64[3], mdh, pl.kcnt,
                                                     pl.ktiles, g.nqb, lse, delta, dk, dv, lk, status,
                                                     g.N, nt, g.scale, scale_log2, timeout, debug_skip);
  return cudaGetLastError();
}

bool bwd_maps(const void* q, const void* k, const void* v, const void* dout, const Geom& g,
              CUtensorMap* m128, CUtensorMap* m64) {
  const void* src[4] = {q, k, v, dout};
  for (int i = 0; i < 4; ++i)
    if (!make_rows_map(&m128[i], src[i], g, 128) || !make_rows_map(&m64[i], src[i], g, 64))
      return false;
  return true;
}

}  // namespace

size_t attn_bwd_tc_scratch_bytes(const Geom& g) { return bwd_plans(g, nullptr).bytes; }

cudaError_t launch_attn_bwd_tc_dq(const void* q, const void* k, const void* v, const void* dout,
                                  const float* lse, const float* delta,
                                  const sla_block_lists& rows, const sla_block_lists& cols,
                                  float* dq, const Geom& g, void* scratch, int32_t* status,
                                  cudaStream_t s, const LinBwdIn* lin) {
  if (!attn_tc_supported(g)) return cudaErrorNotSupported;
  if (lin && g.d != 128) return cudaErrorNotSupported;
  const BwdPlans pl = bwd_plans(g, scratch);
  cudaError_t e = launch_tile_plan(rows, g.BH, g.nqb, g.nkb, g.bq, g.bk, pl.qcnt, pl.qtiles, s);
  if (e != cudaSuccess) return e;
  e = launch_tile_plan(cols, g.BH, g.nkb, g.nqb, g.bk, g.bq, pl.kcnt, pl.ktiles, s);
  if (e != cudaSuccess) return e;
  CUtensorMap m128[4], m64[4];
  if (!bwd_maps(q, k, v, dout, g, m128, m64)) return cudaErrorInvalidValue;
  // the linear branch's query side runs in the dq kernel's epilogue
  CUtensorMap mhm = m128[0], mw = m128[0];  // placeholders when it is off
  LinBwdQ lq{};
  lq.nqb = g.nqb;
  if (lin) {
    const uint64_t dhm[2] = {128, static_cast<uint64_t>(g.BH) * g.nqb * 128}, dw2[2] = {128, 128};
    const uint64_t s2[1] = {256};
    const uint32_t box[2] = {64, 128};
    if (!encode_bf16_map(&mhm, lin->hm, 2, dhm, s2, box) || !encode_bf16_map(&mw, lin->wb, 2, dw2, s2, box))
      return cudaErrorInvalidValue;
    lq.zm = lin->zm;
    lq.marg_cnt = lin->marg_cnt;
    lq.o_lin = lin->o_lin;
    lq.q = static_cast<const __nv_bfloat16*>(q);
    lq.dhm = static_cast<__nv_bfloat16*>(lin->dhm);
    lq.dzm = lin->dzm;
  }
#define SLA_DQ_CALL(D_, BQ_, BK_) launch_dq_t<D_, BQ_, BK_>(m128, m64, mhm, mw, lq, pl, lse, delta, dq, status, g, s)
#define SLA_DQ(...) SLA_DQ_CALL(__VA_ARGS__)
  if (g.d == 128 && g.bq == 64 && g.bk == 64) return SLA_DQ(128, 64, 64);
  if (g.d == 128 && g.bq == 64 && g.bk == 128) return SLA_DQ(128, 64, 128);
  if (g.d == 128 && g.bq == 128 && g.bk == 64) return SLA_DQ(128, 128, 64);
  if (g.d == 128 && g.bq == 128 && g.bk == 128) return SLA_DQ(128, 128, 128);
  if (g.d == 64 && g.bq == 64 && g.bk == 64) return SLA_DQ(64, 64, 64);
  if (g.d == 64 && g.bq == 64 && g.bk == 128) return SLA_DQ(64, 64, 128);
  if (g.d == 64 && g.bq == 128 && g.bk == 64) return SLA_DQ(64, 128, 64);
  if (g.d == 64 && g.bq == 128 && g.bk == 128) return SLA_DQ(64, 128, 128);
#undef SLA_DQ
#undef SLA_DQ_CALL
  return cudaErrorNotSupported;
}

cudaError_t launch_attn_bwd_tc_dkdv(const void* q, const void* k, const void* v,
                                    const void* dout, const float* lse, const float* delta,
                                    float* dk, float* dv, const Geom& g, void* scratch,
                                    int32_t* status, cudaStream_t s, const LinBwdKIn* lin) {
  if (!attn_tc_supported(g)) return cudaErrorNotSupported;
  if (lin && g.d != 128) return cudaErrorNotSupported;
  const BwdPlans pl = bwd_plans(g, scratch);  // built by launch_attn_bwd_tc_dq
  CUtensorMap m128[4], m64[4];
  if (!bwd_maps(q, k, v, dout, g, m128, m64)) return cudaErrorInvalidValue;
  // the linear branch's key side runs in the dkdv kernel's epilogue
  CUtensorMap mdh = m128[0];  // placeholder when it is off
  LinBwdK lk{};
  lk.nkb = g.nkb;
  if (lin) {
    const uint64_t ddh[2] = {128, static_cast<uint64_t>(g.BH) * g.nkb * 128}, s2[1] = {256};
    const uint32_t box[2] = {64, 128};
    if (!encode_bf16_map(&mdh, lin->dh, 2, ddh, s2, box)) return cudaErrorInvalidValue;
    lk.dz = lin->dz;
    lk.marg_cnt = lin->marg_cnt;
    lk.k = static_cast<const __nv_bfloat16*>(k);
  }
#define SLA_KV(D_, BQ_, BK_) launch_dkdv_t<D_, BQ_, BK_>(m128, m64, mdh, lk, pl, lse, delta, dk, dv, status, g, s)
  if (g.d == 128 && g.bq == 64 && g.bk == 64) return SLA_KV(128, 64, 64);
  if (g.d == 128 && g.bq == 64 && g.bk == 128) return SLA_KV(128, 64, 128);
  if (g.d == 128 && g.bq == 128 && g.bk == 64) return SLA_KV(128, 128, 64);
  if (g.d == 128 && g.bq == 128 && g.bk == 128) return SLA_KV(128, 128, 128);
  if (g.d == 64 && g.bq == 64 && g.bk == 64) return SLA_KV(64, 64, 64);
  if (g.d == 64 && g.bq == 64 && g.bk == 128) return SLA_KV(64, 64, 128);
  if (g.d == 64 && g.bq == 128 && g.bk == 64) return SLA_KV(64, 128, 64);
  if (g.d == 64 && g.bq == 128 && g.bk == 128) return SLA_KV(64, 128, 128);
#undef SLA_KV
  return cudaErrorNotSupported;
}

}  // namespace sla
