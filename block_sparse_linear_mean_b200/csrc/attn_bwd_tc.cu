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

#include "internal.h"
#include "tc_common.cuh"

namespace sla {

namespace {

constexpr int kBwdThreads = 320;
constexpr int kBwdStages = 4;
constexpr uint32_t kBwdSmemRequest = 232448;
constexpr uint32_t kBwdTmemCols = 512;
// One pair in kBwdPolyEvery of a step's exponentials is computed by the
// FMA-pipe cubic instead of the special-function unit.
constexpr int kBwdPolyEvery = 3;

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
template <int D, int BQ, int BK>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const int32_t* __restrict__ tile_cnt, const uint32_t* __restrict__ tiles,
                      int plan_stride, const float* __restrict__ lse,
                      const float* __restrict__ delta, float* __restrict__ dq, int32_t* status,
                      int N, int nqt, float scale, float scale_log2, long long timeout) {
  constexpr int DC = D / 64;
  constexpr uint32_t kTileBytes = DC * 16384;  // 128 rows x D bf16 (Q, dO)
  constexpr uint32_t kHalfBytes = DC * 8192;   // 64 rows x D bf16 (K, V)
  constexpr uint32_t kStageBytes = 2 * kHalfBytes;
  constexpr uint32_t offQ = 0, offdO = kTileBytes, offKV = 2 * kTileBytes;
  constexpr uint32_t offBar = offKV + kBwdStages * kStageBytes;
  constexpr uint32_t kUsed = offBar + 256;
  constexpr uint32_t idesc_s = idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t idesc_dq = idesc_bf16(128, D, 0, 1);

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
  static_assert((8 + 2 * kBwdStages) * 8 <= 256, "barrier block");

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x;
  const int bh = tile / nqt, qt = tile % nqt;
  const int T = tile_cnt[tile];
  const uint32_t* ptiles = tiles + static_cast<i64>(tile) * plan_stride;
  // steps present in the plan (all roles count them the same way)
  int U = 0;
  for (int t = 0; t < T; ++t) {
    const uint32_t desc = ptiles[t];
    U += 1 + (step_of<BK>(desc, 1, N).present ? 1 : 0);
  }

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
  BwdShared sh{bars, abort_flag, status, timeout};

  if (warp == 0) {
    if (lane == 0 && U > 0) {
      mbar_expect_tx(b_q, 2 * kTileBytes);
#pragma unroll
      for (int c = 0; c < DC; ++c) {
        tma_load_3d(sb + offQ + c * 16384, &tmQ, c * 64, qt * 128, bh, b_q);
        tma_load_3d(sb + offdO + c * 16384, &tmdO, c * 64, qt * 128, bh, b_q);
      }
      int u = 0;
      bool ok = true;
      for (int t = 0; ok && t < T; ++t) {
        const uint32_t desc = ptiles[t];
        for (int e = 0; ok && e < 2; ++e) {
          const Step st = step_of<BK>(desc, e, N);
          if (!st.present) continue;
          const int s = u % kBwdStages;
          if (u >= kBwdStages && !bwait(sh, b_empty(s), ((u / kBwdStages) & 1) ^ 1)) { ok = false; break; }
          const uint32_t dst = sb + offKV + s * kStageBytes;
          mbar_expect_tx(b_full(s), kStageBytes);
#pragma unroll
          for (int c = 0; c < DC; ++c) {
            tma_load_3d(dst + c * 8192, &tmK, c * 64, st.row0, bh, b_full(s));
            tma_load_3d(dst + kHalfBytes + c * 8192, &tmV, c * 64, st.row0, bh, b_full(s));
          }
          ++u;
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
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = (kk / 4) * 16384 + (kk % 4) * 32;
          const uint32_t ob = (kk / 4) * 8192 + (kk % 4) * 32;
          tc_mma(tS(b), sdesc_add(dQd, oa), sdesc_add(dK, ob), idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = (kk / 4) * 16384 + (kk % 4) * 32;
          const uint32_t ob = (kk / 4) * 8192 + (kk % 4) * 32;
          tc_mma(tP(b), sdesc_add(ddO, oa), sdesc_add(dV, ob), idesc_s, kk > 0);
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
      if (ok) ok = issue_sdp(0);
      for (int u = 0; ok && u < U; ++u) {
        if (u + 1 < U) ok = issue_sdp(u + 1);
        if (ok) ok = issue_dq(u);
      }
      if (ok) tc_commit(b_done);
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
    int u = 0;
    for (int t = 0; ok && t < T; ++t) {
      const uint32_t desc = ptiles[t];
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
            float2 p = (kBwdPolyEvery > 0 && i % kBwdPolyEvery == kBwdPolyEvery - 1)
                           ? exp2_poly2(x)
                           : make_float2(fast_exp2(x.x), fast_exp2(x.y));
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
#pragma unroll
    for (int c = 0; c < DH; c += 32) {
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
  }
  teardown(sh, warp, tmem);
}

// ------------------------------------------------------------------ dK, dV
template <int D, int BQ, int BK>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                        const int32_t* __restrict__ tile_cnt, const uint32_t* __restrict__ tiles,
                        int plan_stride, const float* __restrict__ lse,
                        const float* __restrict__ delta, float* __restrict__ dk,
                        float* __restrict__ dv, int32_t* status, int N, int nkt, float scale,
                        float scale_log2, long long timeout) {
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
  static_assert((8 + 2 * kBwdStages) * 8 <= 256, "barrier block");

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x;
  const int bh = tile / nkt, kt = tile % nkt;
  const int T = tile_cnt[tile];
  const uint32_t* ptiles = tiles + static_cast<i64>(tile) * plan_stride;
  int U = 0;
  for (int t = 0; t < T; ++t) U += 1 + (step_of<BQ>(ptiles[t], 1, N).present ? 1 : 0);

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
    if (U > 0) {
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
      for (int t = 0; ok && t < T; ++t) {
        const uint32_t desc = ptiles[t];
        for (int e = 0; e < 2; ++e) {
          const Step st = step_of<BQ>(desc, e, N);
          if (!st.present) continue;
          const int s = u % kBwdStages;
          bool got = true;
          if (lane == 0 && u >= kBwdStages) got = bwait(sh, b_empty(s), ((u / kBwdStages) & 1) ^ 1);
          if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
          const uint32_t dst = sb + offSt + s * kStageBytes;
          if (lane == 0) {
            mbar_expect_tx(b_full(s), 2 * kHalfBytes);
#pragma unroll
            for (int c = 0; c < DC; ++c) {
              tma_load_3d(dst + c * 8192, &tmQ, c * 64, st.row0, bh, b_full(s));
              tma_load_3d(dst + kHalfBytes + c * 8192, &tmdO, c * 64, st.row0, bh, b_full(s));
            }
          }
          float* nl = reinterpret_cast<float*>(base + offSt + s * kStageBytes + 2 * kHalfBytes);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int q = st.row0 + 32 * j + lane;
            float a = -INFINITY, dd = 0.f;
            if (q < N) {
              const float l = lse[static_cast<i64>(bh) * N + q];
              a = l > -INFINITY ? -l * 1.4426950408889634f : -INFINITY;
              dd = -delta[static_cast<i64>(bh) * N + q];
            }
            nl[32 * j + lane] = a;
            nl[64 + 32 * j + lane] = dd;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(b_full(s));
          ++u;
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
    for (int t = 0; ok && t < T; ++t) {
      const uint32_t desc = ptiles[t];
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
          float2 p = (kBwdPolyEvery > 0 && i % kBwdPolyEvery == kBwdPolyEvery - 1)
                         ? exp2_poly2(x)
                         : make_float2(fast_exp2(x.x), fast_exp2(x.y));
          if (!active) p = make_float2(0.f, 0.f);
          // masked query columns (-inf) give exactly 0 through the
          // hardware path; the cubic returns at most 2^-126 there
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
#pragma unroll
    for (int which = 0; which < 2; ++which) {
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
cudaError_t launch_bwd_t(const CUtensorMap* m128, const CUtensorMap* m64, const BwdPlans& pl,
                         const float* lse, const float* delta, float* dq, float* dk, float* dv,
                         int32_t* status, const Geom& g, cudaStream_t s) {
  const int nt = (g.N + 127) / 128;
  const float scale_log2 = g.scale * 1.4426950408889634f;
  const bool debug = (g.flags & SLA_FLAG_DEBUG_TIMEOUT) != 0;
  const long long timeout = debug ? (1ll << 24) : (1ll << 31);
  // m128 / m64: {q, k, v, dout} maps with 128- and 64-row boxes
  auto kq = attn_bwd_dq_tc_kernel<D, BQ, BK>;
  cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kBwdSmemRequest));
  if (e != cudaSuccess) return e;
  kq<<<g.BH * nt, kBwdThreads, kBwdSmemRequest, s>>>(m128[0], m128[3], m64[1], m64[2], pl.qcnt,
                                                     pl.qtiles, g.nkb, lse, delta, dq, status, g.N,
                                                     nt, g.scale, scale_log2, timeout);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto kk = attn_bwd_dkdv_tc_kernel<D, BQ, BK>;
  e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kBwdSmemRequest));
  if (e != cudaSuccess) return e;
  kk<<<g.BH * nt, kBwdThreads, kBwdSmemRequest, s>>>(m128[1], m128[2], m64[0], m64[3], pl.kcnt,
                                                     pl.ktiles, g.nqb, lse, delta, dk, dv, status,
                                                     g.N, nt, g.scale, scale_log2, timeout);
  return cudaGetLastError();
}

}  // namespace

size_t attn_bwd_tc_scratch_bytes(const Geom& g) { return bwd_plans(g, nullptr).bytes; }

cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* dout,
                               const float* lse, const float* delta,
                               const sla_block_lists& rows, const sla_block_lists& cols,
                               float* dq, float* dk, float* dv, const Geom& g, void* scratch,
                               int32_t* status, cudaStream_t s) {
  if (!attn_tc_supported(g)) return cudaErrorNotSupported;
  const BwdPlans pl = bwd_plans(g, scratch);
  cudaError_t e = launch_tile_plan(rows, g.BH, g.nqb, g.nkb, g.bq, g.bk, pl.qcnt, pl.qtiles, s);
  if (e != cudaSuccess) return e;
  e = launch_tile_plan(cols, g.BH, g.nkb, g.nqb, g.bk, g.bq, pl.kcnt, pl.ktiles, s);
  if (e != cudaSuccess) return e;
  CUtensorMap m128[4], m64[4];
  const void* src[4] = {q, k, v, dout};
  for (int i = 0; i < 4; ++i)
    if (!make_rows_map(&m128[i], src[i], g, 128) || !make_rows_map(&m64[i], src[i], g, 64))
      return cudaErrorInvalidValue;
#define SLA_BWD_CASE(D_, BQ_, BK_)                  \
  if (g.d == D_ && g.bq == BQ_ && g.bk == BK_)      \
    return launch_bwd_t<D_, BQ_, BK_>(m128, m64, pl, lse, delta, dq, dk, dv, status, g, s);
  SLA_BWD_CASE(128, 64, 64)
  SLA_BWD_CASE(128, 64, 128)
  SLA_BWD_CASE(128, 128, 64)
  SLA_BWD_CASE(128, 128, 128)
  SLA_BWD_CASE(64, 64, 64)
  SLA_BWD_CASE(64, 64, 128)
  SLA_BWD_CASE(64, 128, 64)
  SLA_BWD_CASE(64, 128, 128)
#undef SLA_BWD_CASE
  return cudaErrorNotSupported;
}

}  // namespace sla
