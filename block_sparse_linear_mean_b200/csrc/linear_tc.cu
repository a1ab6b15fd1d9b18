// Linear attention on marginal blocks, on the 5th-generation tensor cores
// (bf16 inputs, fp32 accumulation, d = 128).
//
// SLA post ("Selective Linear Attention", list "the idea"): intermediate
// (marginal) blocks go through linear attention.  With phi = elu + 1 and the
// d x d projection W of the workload:
//   1. summaries     H_j = phi(K_j)^T V_j,  z_j = sum_t phi(k_t)   (per key block)
//   2. gather-sum    H^M_i = sum_{j in M_i} H_j                     (per query block)
//                    computed as one GEMM per head, Ind @ H, with Ind the 0/1
//                    marginal indicator (exact in bf16), so every H_j tile that
//                    reaches shared memory serves 128 query blocks at once
//   3. apply         O_lin = phi(Q) H^M / (phi(Q) . z^M)
//   4. combine       out = O_s + O_lin W
// phi(K) and phi(Q) are rounded to bf16 once (the MMA operands) and the
// normalisers z^M and phi(Q).z^M are formed from those same rounded values,
// so numerator and denominator see identical weights.  H and H^M are stored
// in bf16; all sums accumulate in fp32 (TMEM or registers).
#include <algorithm>

#include "common.cuh"
#include "tc_common.cuh"

namespace sla {

namespace {

constexpr int kD = 128;
constexpr int kHElems = kD * kD;  // 16384

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

__device__ __forceinline__ float bf16_at(const uint8_t* tile, int row, int col) {
  // element `col` (0..63) of `row` in a 128B-swizzled chunk
  const uint16_t bits = *reinterpret_cast<const uint16_t*>(tile + sw128(row, col >> 3) + (col & 7) * 2);
  return __uint_as_float(static_cast<uint32_t>(bits) << 16);
}

// phi in place over the first ROWS rows of a bf16 tile of 128 channels kept
// as two 128-byte-swizzled chunks of 64 channels (`cstride` bytes apart);
// rows at or past `valid` become zeros.  128 threads, each on ROWS / 8
// pieces of 16 bytes in batches of up to eight, a batch read before any of
// it is written back: a read after a store to the same tile would wait for
// the store, and the pieces' exponentials would run one after another.
template <int ROWS>
__device__ __forceinline__ void phi_tile(uint8_t* tile, uint32_t cstride, int valid, int tid) {
  constexpr int kN = ROWS * 16 / 128, kB = kN < 8 ? kN : 8;  // pieces per thread, per batch
#pragma unroll
  for (int b0 = 0; b0 < kN; b0 += kB) {
    uint4 v[kB];
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int x = tid + 128 * (b0 + i);
      v[i] = *reinterpret_cast<const uint4*>(tile + ((x >> 3) & 1) * cstride + sw128(x >> 4, x & 7));
    }
#pragma unroll
    for (int i = 0; i < kB; ++i)
      v[i] = ((tid + 128 * (b0 + i)) >> 4) < valid ? phi_unit(v[i]) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int x = tid + 128 * (b0 + i);
      *reinterpret_cast<uint4*>(tile + ((x >> 3) & 1) * cstride + sw128(x >> 4, x & 7)) = v[i];
    }
  }
}

// ---------------------------------------------------------------------------
// 1. Summaries: one CTA (128 threads) per (key block, head).
//    TMA K_j, V_j -> phi(K) in place (padding rows zeroed) and z_j ->
//    H_j = phi(K)^T V_j (M = 128 channels a, N = 128 channels c, K = BK
//    tokens; both operands MN-major) -> bf16 -> TMA store.
template <int BK>
__global__ void __launch_bounds__(128) lin_summary_tc_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __grid_constant__ CUtensorMap tmH, float* __restrict__ zsum, int N, int nkb,
    int32_t* status, long long timeout, int debug_skip) {
  constexpr uint32_t kChunk = BK * 128;  // bytes of one 64-column chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const uint32_t sb = smem_u32(base);
  const uint32_t offK = 0, offV = 2 * kChunk;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + 4 * kChunk);
  const uint32_t b_tma = smem_u32(&bars[0]), b_mma = smem_u32(&bars[1]);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(&bars[2]);
  const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid / 32;
  const int valid = min(BK, N - j * BK);
  if (tid == 0) {
    mbar_init(b_tma, 1);
    mbar_init(b_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(tslot), 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // (test aid: the first CTA's tiles never arrive)
  if (tid == 0 && !(debug_skip && blockIdx.x == 0 && blockIdx.y == 0)) {
    mbar_expect_tx(b_tma, 4 * kChunk);
    for (int c = 0; c < 2; ++c) {
      tma_load_3d(sb + offK + c * kChunk, &tmK, c * 64, j * BK, bh, b_tma);
      tma_load_3d(sb + offV + c * kChunk, &tmV, c * 64, j * BK, bh, b_tma);
    }
  }
  bool ok = __syncthreads_and(wait_bounded(b_tma, 0, status, timeout));
  if (ok) {
    phi_tile<BK>(base + offK, kChunk, valid, tid);
    __syncthreads();
    {  // z_j[a] from the rounded phi(K) the MMA uses (four chains, added
       // in a fixed order)
      const int a = tid;
      const uint8_t* ch = base + offK + (a >> 6) * kChunk;
      float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
      int u = 0;
      for (; u + 4 <= valid; u += 4) {
        z0 += bf16_at(ch, u, a & 63);
        z1 += bf16_at(ch, u + 1, a & 63);
        z2 += bf16_at(ch, u + 2, a & 63);
        z3 += bf16_at(ch, u + 3, a & 63);
      }
      for (; u < valid; ++u) z0 += bf16_at(ch, u, a & 63);
      zsum[(i64(bh) * nkb + j) * kD + a] = (z0 + z1) + (z2 + z3);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, 1, 1);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        tc_mma(tmem, sdesc(sb + offK + kk * 2048, kChunk, 1024), sdesc(sb + offV + kk * 2048, kChunk, 1024),
               idesc, kk > 0);
      tc_commit(b_mma);
    }
    ok = __syncthreads_and(wait_bounded(b_mma, 0, status, timeout));
  }
  if (ok) {  // TMEM lane a -> bf16 row a of a 128B-swizzled staging tile (reuses K/V space)
    tc_fence_after();
    const int a = tid;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
    for (int c0 = 0; c0 < kD; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_off + c0, v);
      tmem_wait_ld();
      reg_fence<32>(v);
      uint8_t* ch = base + (c0 >> 6) * 16384;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(ch + sw128(a, ((c0 & 63) >> 3) + q)) =
            make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                       pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
    }
    fence_async_smem();
  }
  __syncthreads();
  if (ok && tid == 0) {
    const int row0 = (bh * nkb + j) * kD;
    tma_store_2d(&tmH, sb, 0, row0);
    tma_store_2d(&tmH, sb + 16384, 64, row0);
    tma_store_commit();
    tma_store_wait_read();  // the staging tile is read before the CTA ends
  }
  tc_fence_before();
  __syncthreads();
  if (!ok) {  // let in-flight copies drain (bounded)
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) __nanosleep(1000);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Persistent summaries for key blocks of 64 tokens: each CTA walks the items
// w = blockIdx.x, blockIdx.x + gridDim.x, ... (item w = key block w % nkb of
// head w / nkb) with two K/V buffers, so the next item's tiles load while
// the current one is processed; after its products a buffer is the staging
// tile of that item's H, and the next load into it waits until the store
// has read it.  Same steps as lin_summary_tc_kernel.
__global__ void __launch_bounds__(128) lin_summary_persist_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __grid_constant__ CUtensorMap tmH, float* __restrict__ zsum, int N, int nkb, int nitems,
    int32_t* status, long long timeout, int debug_skip) {
  constexpr int BK = 64;
  constexpr uint32_t kChunk = BK * 128;  // bytes of one 64-column chunk
  constexpr uint32_t kBuf = 4 * kChunk;  // K (2 chunks) then V (2 chunks); 32 KB = one H tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const uint32_t sb = smem_u32(base);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + 2 * kBuf);
  auto b_tma = [&](int b) { return smem_u32(&bars[b]); };
  const uint32_t b_mma = smem_u32(&bars[2]);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(&bars[3]);
  const int tid = threadIdx.x, warp = tid / 32;
  if (tid == 0) {
    mbar_init(b_tma(0), 1);
    mbar_init(b_tma(1), 1);
    mbar_init(b_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(tslot), 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  auto issue_load = [&](int w, int b) {  // (one thread)
    const int j = w % nkb, bh = w / nkb;
    const uint32_t dst = sb + b * kBuf;
    mbar_expect_tx(b_tma(b), kBuf);
    for (int c = 0; c < 2; ++c) {
      tma_load_3d(dst + c * kChunk, &tmK, c * 64, j * BK, bh, b_tma(b));
      tma_load_3d(dst + 2 * kChunk + c * kChunk, &tmV, c * 64, j * BK, bh, b_tma(b));
    }
  };
  // (test aid: the first CTA's first item never arrives)
  if (tid == 0 && static_cast<int>(blockIdx.x) < nitems && !(debug_skip && blockIdx.x == 0))
    issue_load(blockIdx.x, 0);
  bool ok = true;
  int k = 0;
  for (int w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++k) {
    const int b = k & 1, j = w % nkb, bh = w / nkb;
    const int valid = min(BK, N - j * BK);
    uint8_t* buf = base + b * kBuf;
    const uint32_t sbuf = sb + b * kBuf;
    // next item into the other buffer, once the previous item's H store has
    // read it
    if (tid == 0 && w + static_cast<int>(gridDim.x) < nitems) {
      tma_store_wait_read();
      issue_load(w + gridDim.x, b ^ 1);
    }
    ok = __syncthreads_and(wait_bounded(b_tma(b), (k >> 1) & 1, status, timeout));
    if (!ok) break;
    phi_tile<BK>(buf, kChunk, valid, tid);
    __syncthreads();
    {  // z_j[a] from the rounded phi(K) the MMA uses (four chains, added
       // in a fixed order)
      const int a = tid;
      const uint8_t* ch = buf + (a >> 6) * kChunk;
      float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
      int u = 0;
      for (; u + 4 <= valid; u += 4) {
        z0 += bf16_at(ch, u, a & 63);
        z1 += bf16_at(ch, u + 1, a & 63);
        z2 += bf16_at(ch, u + 2, a & 63);
        z3 += bf16_at(ch, u + 3, a & 63);
      }
      for (; u < valid; ++u) z0 += bf16_at(ch, u, a & 63);
      zsum[(i64(bh) * nkb + j) * kD + a] = (z0 + z1) + (z2 + z3);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, 1, 1);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        tc_mma(tmem, sdesc(sbuf + kk * 2048, kChunk, 1024), sdesc(sbuf + 2 * kChunk + kk * 2048, kChunk, 1024),
               idesc, kk > 0);
      tc_commit(b_mma);
    }
    ok = __syncthreads_and(wait_bounded(b_mma, k & 1, status, timeout));
    if (!ok) break;
    // TMEM lane a -> bf16 row a of a 128B-swizzled staging tile (this buffer)
    tc_fence_after();
    {
      const int a = tid;
      const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_off + c0, v);
        tmem_wait_ld();
        reg_fence<32>(v);
        uint8_t* ch = buf + (c0 >> 6) * 16384;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(ch + sw128(a, ((c0 & 63) >> 3) + q)) =
              make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                         pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // (also: every TMEM read done before the next item's products)
    if (tid == 0) {
      const int row0 = (bh * nkb + j) * kD;
      tma_store_2d(&tmH, sbuf, 0, row0);
      tma_store_2d(&tmH, sbuf + 16384, 64, row0);
      tma_store_commit();
    }
  }
  if (tid == 0) tma_store_wait_all();
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (!ok) {  // let in-flight copies drain (bounded)
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) __nanosleep(1000);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------------------
// 2a. Marginal indicator Ind[bh, i, j] (bf16 0/1, row stride ld) from the
//     CSR marginal lists, and z^M_i = sum of z_j over the list (fp32): one
//     CTA of 128 threads per query-block row.  Warp w sums the list entries
//     e = w mod 4 (each lane four channels, one 16-byte load per entry, so a
//     warp keeps several L2 reads in flight), and the four partial sums are
//     added in a fixed order.  With w given, the first CTAs also write the
//     projection W (fp32) as bf16 into wb for the fused epilogue (a launch
//     of its own would cost more than the conversion).
__global__ void __launch_bounds__(128) indicator_kernel(sla_block_lists rows,
                                                        uint16_t* __restrict__ ind,
                                                        const float* __restrict__ zsum,
                                                        float* __restrict__ zm, int nqb, int nkb,
                                                        int ld, const float* __restrict__ w,
                                                        uint16_t* __restrict__ wb) {
  __shared__ int lst[256];
  __shared__ float4 part[4][32];
  const int row = blockIdx.x, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  constexpr int kWCtas = 16;  // CTAs sharing the conversion of W's kHElems entries
  if (w && row < kWCtas) {
    for (int i = row * 128 + tid; i < kHElems; i += kWCtas * 128) {
      const __nv_bfloat16 b = __float2bfloat16_rn(w[i]);
      wb[i] = *reinterpret_cast<const uint16_t*>(&b);
    }
  }
  const int bh = row / nqb;
  uint4* p = reinterpret_cast<uint4*>(ind + i64(row) * ld);
  for (int x = tid; x < ld / 8; x += blockDim.x) p[x] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  const int cnt = min(max(rows.marg_cnt[row], 0), nkb);
  const int32_t* idx = rows.marg_idx + i64(row) * nkb;
  const float4* z4 = reinterpret_cast<const float4*>(zsum + i64(bh) * nkb * kD) + lane;
  float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
  for (int b0 = 0; b0 < cnt; b0 += 256) {
    const int n = min(256, cnt - b0);
    __syncthreads();
    for (int e = tid; e < n; e += blockDim.x) {
      const int jj = idx[b0 + e];
      lst[e] = (jj >= 0 && jj < nkb) ? jj : -1;
      if (jj >= 0 && jj < nkb) ind[i64(row) * ld + jj] = 0x3F80u;  // bf16 1.0
    }
    __syncthreads();
    int e = warp;
    for (; e + 4 < n; e += 8) {  // two entries per step, independent chains
      const int j0 = lst[e], j1 = lst[e + 4];
      if (j0 >= 0) {
        const float4 v = z4[i64(j0) * (kD / 4)];
        acc0.x += v.x; acc0.y += v.y; acc0.z += v.z; acc0.w += v.w;
      }
      if (j1 >= 0) {
        const float4 v = z4[i64(j1) * (kD / 4)];
        acc1.x += v.x; acc1.y += v.y; acc1.z += v.z; acc1.w += v.w;
      }
    }
    if (e < n && lst[e] >= 0) {
      const float4 v = z4[i64(lst[e]) * (kD / 4)];
      acc0.x += v.x; acc0.y += v.y; acc0.z += v.z; acc0.w += v.w;
    }
  }
  part[warp][lane] = make_float4(acc0.x + acc1.x, acc0.y + acc1.y, acc0.z + acc1.z, acc0.w + acc1.w);
  __syncthreads();
  // channel tid = 4 * lane' + c of part[w][lane']
  const float* pf = reinterpret_cast<const float*>(&part[0][0]);
  zm[i64(row) * kD + tid] = ((pf[tid] + pf[128 + tid]) + pf[256 + tid]) + pf[384 + tid];
}

// 2b. Gather GEMM: HM[bh] (Nqb x 16384) = Ind[bh] (Nqb x ld) @ H[bh] (ld x 16384).
//     Persistent: one CTA per SM walks output tiles of 128 x 256 (consecutive
//     tiles share their H columns, so the CTAs working at one time read each
//     H tile from L2 after the first).  K step 64, 4-stage TMA ring; warp 0
//     loads, warp 1 issues tcgen05.mma (A K-major, B MN-major) into one of
//     two TMEM accumulators, warps 2-5 drain the other, 128 columns at a
//     time, into a swizzled bf16 half tile that TMA stores write out -- a
//     tile's epilogue overlaps the next tile's products.
constexpr int kGStages = 4;
constexpr uint32_t kGA = 16384, kGB = 32768, kGStage = kGA + kGB;
constexpr uint32_t kGStaging = kGStages * kGStage;       // 32 KB bf16 half tile
constexpr uint32_t kGBars = kGStaging + 32768;
constexpr size_t kGSmem = kGBars + 256 + 1024;

__global__ void __launch_bounds__(192, 1) gather_gemm_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const __grid_constant__ CUtensorMap tmC, int ksteps, int tiles_m, int tiles_n, int ntiles,
    int32_t* status, long long timeout, int debug_skip) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const uint32_t sb = smem_u32(base);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kGBars);
  auto b_full = [&](int s) { return smem_u32(&bars[s]); };
  auto b_empty = [&](int s) { return smem_u32(&bars[kGStages + s]); };
  auto b_acc_full = [&](int a) { return smem_u32(&bars[2 * kGStages + a]); };
  auto b_acc_empty = [&](int a) { return smem_u32(&bars[2 * kGStages + 2 + a]); };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(&bars[2 * kGStages + 4]);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) { mbar_init(b_full(s), 1); mbar_init(b_empty(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(b_acc_full(a), 1); mbar_init(b_acc_empty(a), 4); }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tslot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // tile -> (m, n, bh), m fastest
  auto coords = [&](int t, int& m0, int& n0, int& bh) {
    const int per = tiles_m * tiles_n;
    bh = t / per;
    const int r = t - bh * per;
    n0 = (r / tiles_m) * 256;
    m0 = (r % tiles_m) * 128;
  };
  bool ok = true;
  if (warp == 0 && lane == 0) {
    int g = 0;  // K steps loaded so far (ring position)
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      int m0, n0, bh;
      coords(t, m0, n0, bh);
      for (int ks = 0; ks < ksteps && ok; ++ks, ++g) {
        const int s = g % kGStages;
        if (g >= kGStages) ok = wait_bounded(b_empty(s), ((g / kGStages) & 1) ^ 1, status, timeout);
        if (!ok) break;
        if (debug_skip && blockIdx.x == 0 && g == 0) continue;  // test aid: this step never arrives
        const uint32_t st = sb + s * kGStage;
        mbar_expect_tx(b_full(s), kGStage);
        tma_load_3d(st, &tmA, ks * 64, m0, bh, b_full(s));
#pragma unroll
        for (int c = 0; c < 4; ++c) tma_load_3d(st + kGA + c * 8192, &tmB, n0 + c * 64, ks * 64, bh, b_full(s));
      }
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, 256, 0, 1);
    const uint64_t dA = sdesc(sb, 16, 1024), dB = sdesc(sb + kGA, 8192, 1024);  // built once
    int g = 0, it = 0;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
      const int a = it & 1;
      // the epilogue has drained this accumulator (tile it - 2)
      if (it >= 2) ok = wait_bounded(b_acc_empty(a), ((it >> 1) & 1) ^ 1, status, timeout);
      for (int ks = 0; ks < ksteps && ok; ++ks, ++g) {
        const int s = g % kGStages;
        ok = wait_bounded(b_full(s), (g / kGStages) & 1, status, timeout);
        if (!ok) break;
        tc_fence_after();
        const uint32_t so = s * kGStage;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma(tmem + 256 * a, sdesc_add(dA, so + kk * 32), sdesc_add(dB, so + kk * 2048), idesc,
                 (ks > 0 || kk > 0) ? 1u : 0u);
        tc_commit(b_empty(s));
      }
      if (ok) tc_commit(b_acc_full(a));
    }
  } else if (warp >= 2) {
    const int quad = warp & 3, r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    int it = 0;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
      const int a = it & 1;
      int m0, n0, bh;
      coords(t, m0, n0, bh);
      ok = wait_bounded(b_acc_full(a), (it >> 1) & 1, status, timeout);
      tc_fence_after();
      for (int hf = 0; hf < 2; ++hf) {  // (every warp reaches the barrier below)
        // the previous stores have read the staging half tile
        if (threadIdx.x == 64) tma_store_wait_read();
        ok = bar_sync_and(1, 128, ok);  // all four warps take the same branch
        if (!ok) break;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float v[32];
          tmem_ld32(tmem + 256 * a + 128 * hf + lane_off + c0, v);
          tmem_wait_ld();
          reg_fence<32>(v);
          uint8_t* ch = base + kGStaging + (c0 >> 6) * 16384;  // 2 chunks of [128 rows][64 cols]
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(ch + sw128(r, ((c0 & 63) >> 3) + q)) =
                make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                           pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
        }
        if (hf == 1) {  // accumulator free for tile it + 2
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_acc_empty(a));
        }
        fence_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 64) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_store_3d(&tmC, sb + kGStaging + c * 16384, n0 + 128 * hf + c * 64, m0, bh);
          tma_store_commit();
        }
      }
    }
    if (threadIdx.x == 64) tma_store_wait_all();
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (!ok) {
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) __nanosleep(1000);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// 3-4. Apply and combine: one CTA (128 threads) per (query block, head).
//   num^T = H^M^T phi(Q)^T   (M = 128 channels c, N = BQ tokens, K = 128 a)
//   O_lin = num / (phi(q) . z^M)                       (per token column)
//   out_lin^T = W^T O_lin^T  (M = 128 channels, N = BQ, K = 128)
//   out = O_s + out_lin (bf16), o_lin optionally saved (fp32)
template <int BQ>
__global__ void __launch_bounds__(128) lin_apply_tc_kernel(
    const __grid_constant__ CUtensorMap tmHM, const __grid_constant__ CUtensorMap tmQ,
    const __grid_constant__ CUtensorMap tmW, const float* __restrict__ zmar,
    sla_block_lists rows, const float* __restrict__ o_s, __nv_bfloat16* __restrict__ out,
    float* __restrict__ o_lin, int N, int nqb, int nkb, int32_t* status, long long timeout) {
  constexpr uint32_t offHM = 0, offW = 32768, offQ = 65536;
  constexpr uint32_t kQChunk = BQ * 128;
  constexpr uint32_t offOL = offQ + 2 * kQChunk;      // BQ/64 chunks of [128 a][64 t]
  constexpr uint32_t offZ = offOL + (BQ / 64) * 16384;
  constexpr uint32_t offDen = offZ + 512;
  constexpr uint32_t offBar = offDen + BQ * 4;
  constexpr uint32_t kCols = BQ == 64 ? 128 : 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const uint32_t sb = smem_u32(base);
  float* zm = reinterpret_cast<float*>(base + offZ);
  float* den = reinterpret_cast<float*>(base + offDen);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + offBar);
  const uint32_t b_tma = smem_u32(&bars[0]), b_m1 = smem_u32(&bars[1]), b_m2 = smem_u32(&bars[2]);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(&bars[3]);
  const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid / 32;
  const int list_row = bh * nqb + i;
  const int nmarg = min(max(rows.marg_cnt[list_row], 0), nkb);
  const int t0g = i * BQ, valid = min(BQ, N - t0g);
  if (tid == 0) {
    mbar_init(b_tma, 1);
    mbar_init(b_m1, 1);
    mbar_init(b_m2, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(tslot), kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const int c = tid;  // channel owned in the epilogues (TMEM lane)
  bool ok = true;
  if (nmarg > 0) {
    if (tid == 0) {
      mbar_expect_tx(b_tma, 2 * 32768 + 2 * kQChunk);
      const int hrow = list_row * kD;
      tma_load_2d(sb + offHM, &tmHM, 0, hrow, b_tma);
      tma_load_2d(sb + offHM + 16384, &tmHM, 64, hrow, b_tma);
      tma_load_2d(sb + offW, &tmW, 0, 0, b_tma);
      tma_load_2d(sb + offW + 16384, &tmW, 64, 0, b_tma);
      tma_load_3d(sb + offQ, &tmQ, 0, t0g, bh, b_tma);
      tma_load_3d(sb + offQ + kQChunk, &tmQ, 64, t0g, bh, b_tma);
    }
    zm[c] = zmar[i64(list_row) * kD + c];  // z^M, gathered by the indicator kernel
    ok = __syncthreads_and(wait_bounded(b_tma, 0, status, timeout));
    if (ok) {
      phi_tile<BQ>(base + offQ, kQChunk, valid, tid);  // phi(Q) in place, padding rows zero
      __syncthreads();
      for (int t = tid; t < BQ; t += 128) {  // normaliser from the rounded phi(q)
        float s = 0.f;
        for (int a = 0; a < kD; ++a) s += bf16_at(base + offQ + (a >> 6) * kQChunk, t, a & 63) * zm[a];
        den[t] = s;
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16(128, BQ, 1, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma(tmem, sdesc(sb + offHM + kk * 2048, 16384, 1024),
                 sdesc(sb + offQ + (kk >> 2) * kQChunk + (kk & 3) * 32, 16, 1024), idesc, kk > 0);
        tc_commit(b_m1);
      }
      ok = __syncthreads_and(wait_bounded(b_m1, 0, status, timeout));
    }
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int tt = 0; tt < BQ; tt += 32) {
        float v[32];
        tmem_ld32(tmem + lane_off + tt, v);
        tmem_wait_ld();
        reg_fence<32>(v);
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int t = tt + q;
          v[q] = t < valid ? v[q] / den[t] : 0.f;
          if (o_lin && t < valid) o_lin[(i64(bh) * N + t0g + t) * kD + c] = v[q];
        }
        uint8_t* ch = base + offOL + (tt >> 6) * 16384;  // row c of [128 a][64 t]
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(ch + sw128(c, ((tt & 63) >> 3) + q)) =
              make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                         pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16(128, BQ, 1, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma(tmem + BQ, sdesc(sb + offW + kk * 2048, 16384, 1024),
                 sdesc(sb + offOL + kk * 2048, 16384, 1024), idesc, kk > 0);
        tc_commit(b_m2);
      }
      ok = __syncthreads_and(wait_bounded(b_m2, 0, status, timeout));
    }
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int tt = 0; tt < BQ; tt += 32) {
        float v[32];
        tmem_ld32(tmem + BQ + lane_off + tt, v);
        tmem_wait_ld();
        reg_fence<32>(v);
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int t = tt + q;
          if (t < valid) {
            const i64 off = (i64(bh) * N + t0g + t) * kD + c;
            out[off] = __float2bfloat16_rn(o_s[off] + v[q]);
          }
        }
      }
    }
  } else {
    for (int t = 0; t < valid; ++t) {  // no marginal blocks: out = O_s
      const i64 off = (i64(bh) * N + t0g + t) * kD + c;
      out[off] = __float2bfloat16_rn(o_s[off]);
      if (o_lin) o_lin[off] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (!ok) {
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) __nanosleep(1000);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

__global__ void to_bf16_kernel(const float* __restrict__ x, uint16_t* __restrict__ y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const __nv_bfloat16 b = __float2bfloat16_rn(x[i]);
    y[i] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

struct LinWs {
  size_t wb, h, z, zm, ind, hm, total;
  int ld;
};

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

LinWs lin_ws(const Geom& g) {
  LinWs w;
  w.ld = (g.nkb + 63) / 64 * 64;
  size_t off = 0;
  w.wb = off; off = a256(off + size_t(kHElems) * 2);
  w.h = off; off = a256(off + size_t(g.BH) * g.nkb * kHElems * 2);
  w.z = off; off = a256(off + size_t(g.BH) * g.nkb * kD * 4);
  w.zm = off; off = a256(off + size_t(g.BH) * g.nqb * kD * 4);
  w.ind = off; off = a256(off + size_t(g.BH) * g.nqb * w.ld * 2);
  w.hm = off; off = a256(off + size_t(g.BH) * g.nqb * kHElems * 2);
  w.total = off;
  return w;
}

template <typename F>
cudaError_t set_smem(F kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

}  // namespace

static cudaError_t launch_gather(const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mC,
                                 int ld, int nrow, int BH, int32_t* status, const Geom& geo,
                                 cudaStream_t s) {
  cudaError_t e;
  if ((e = set_smem(gather_gemm_kernel, kGSmem)) != cudaSuccess) return e;
  const int tiles_m = (nrow + 127) / 128, tiles_n = kHElems / 256;
  const int ntiles = tiles_m * tiles_n * BH;
  const int grid = std::min(ntiles, sm_count());
  gather_gemm_kernel<<<grid, 192, kGSmem, s>>>(mA, mB, mC, ld / 64, tiles_m, tiles_n, ntiles, status,
                                               wait_limit(geo),
                                               debug_withhold(geo, SLA_WITHHOLD_GATHER) ? 1 : 0);
  return cudaGetLastError();
}

bool lin_tc_supported(const Geom& g) {
  return g.dtype == SLA_BF16 && g.d == kD && !(g.flags & SLA_FLAG_SIMT) && tma_available();
}

size_t lin_tc_scratch_bytes(const Geom& g) { return lin_ws(g).total; }

LinInputs lin_tc_inputs(const Geom& g, void* scratch, const sla_block_lists& rows) {
  const LinWs w = lin_ws(g);
  char* sc = static_cast<char*>(scratch);
  LinInputs in;
  in.hm = sc + w.hm;
  in.wb = sc + w.wb;
  in.zm = reinterpret_cast<const float*>(sc + w.zm);
  in.marg_cnt = rows.marg_cnt;
  return in;
}

static cudaError_t lin_tc_impl(const void* q, const void* k, const void* v, const float* proj,
                               const sla_block_lists& rows, const float* o_s, void* out,
                               float* o_lin, const Geom& g, void* scratch, int32_t* status,
                               cudaStream_t s, bool prepare, bool apply);

cudaError_t launch_list_gather(const sla_block_lists& lists, int BH, int nrow, int ncol,
                               const void* src_h, const float* src_z, void* dst_h, float* dst_z,
                               void* ind, int ld, int32_t* status, const Geom& g,
                               cudaStream_t s) {
  cudaError_t e;
  uint16_t* indp = static_cast<uint16_t*>(ind);
  indicator_kernel<<<BH * nrow, 128, 0, s>>>(lists, indp, src_z, dst_z, nrow, ncol, ld, nullptr, nullptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap mA, mB, mC;
  const uint64_t bh = BH, nr = nrow, nc = ncol, l = ld;
  const uint64_t da[3] = {l, nr, bh}, sa[2] = {l * 2, nr * l * 2};
  const uint32_t ba[3] = {64, 128, 1};
  const uint64_t db[3] = {kHElems, nc, bh}, sbt[2] = {kHElems * 2, nc * kHElems * 2};
  const uint32_t bb[3] = {64, 64, 1};
  const uint64_t dc[3] = {kHElems, nr, bh}, sc2[2] = {kHElems * 2, nr * kHElems * 2};
  const uint32_t bc[3] = {64, 128, 1};
  if (!encode_bf16_map(&mA, indp, 3, da, sa, ba) || !encode_bf16_map(&mB, src_h, 3, db, sbt, bb) ||
      !encode_bf16_map(&mC, dst_h, 3, dc, sc2, bc))
    return cudaErrorInvalidValue;
  return launch_gather(mA, mB, mC, ld, nrow, BH, status, g, s);
}

cudaError_t launch_lin_tc_prepare(const void* k, const void* v, const float* proj,
                                  const sla_block_lists& rows, const Geom& g, void* scratch,
                                  int32_t* status, cudaStream_t s) {
  return lin_tc_impl(nullptr, k, v, proj, rows, nullptr, nullptr, nullptr, g, scratch, status, s,
                     true, false);
}

cudaError_t launch_lin_tc(const void* q, const void* k, const void* v, const float* proj,
                          const sla_block_lists& rows, const float* o_s, void* out,
                          float* o_lin, const Geom& g, void* scratch, int32_t* status,
                          cudaStream_t s) {
  return lin_tc_impl(q, k, v, proj, rows, o_s, out, o_lin, g, scratch, status, s, true, true);
}

static cudaError_t lin_tc_impl(const void* q, const void* k, const void* v, const float* proj,
                               const sla_block_lists& rows, const float* o_s, void* out,
                               float* o_lin, const Geom& g, void* scratch, int32_t* status,
                               cudaStream_t s, bool prepare, bool apply) {
  const LinWs w = lin_ws(g);
  char* sc = static_cast<char*>(scratch);
  uint16_t* wb = reinterpret_cast<uint16_t*>(sc + w.wb);
  uint16_t* hbuf = reinterpret_cast<uint16_t*>(sc + w.h);
  float* zbuf = reinterpret_cast<float*>(sc + w.z);
  float* zmbuf = reinterpret_cast<float*>(sc + w.zm);
  uint16_t* ind = reinterpret_cast<uint16_t*>(sc + w.ind);
  uint16_t* hm = reinterpret_cast<uint16_t*>(sc + w.hm);
  cudaError_t e;
  // tensor maps
  CUtensorMap mK, mV, mQ, mH, mA, mB, mC, mHM, mW;
  const uint64_t BH = g.BH, N = g.N, nkb = g.nkb, nqb = g.nqb, ld = w.ld;
  {
    const uint64_t dims[3] = {kD, N, BH}, str[2] = {kD * 2, N * kD * 2};
    const uint32_t boxk[3] = {64, static_cast<uint32_t>(g.bk), 1};
    const uint32_t boxq[3] = {64, static_cast<uint32_t>(g.bq), 1};
    if (!encode_bf16_map(&mK, k, 3, dims, str, boxk) || !encode_bf16_map(&mV, v, 3, dims, str, boxk) ||
        (apply && !encode_bf16_map(&mQ, q, 3, dims, str, boxq)))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {kD, BH * nkb * kD}, str[1] = {kD * 2};
    const uint32_t box[2] = {64, 128};
    if (!encode_bf16_map(&mH, hbuf, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t da[3] = {ld, nqb, BH}, sa[2] = {ld * 2, nqb * ld * 2};
    const uint32_t ba[3] = {64, 128, 1};
    const uint64_t db[3] = {kHElems, nkb, BH}, sbt[2] = {kHElems * 2, nkb * kHElems * 2};
    const uint32_t bb[3] = {64, 64, 1};
    const uint64_t dc[3] = {kHElems, nqb, BH}, sc2[2] = {kHElems * 2, nqb * kHElems * 2};
    const uint32_t bc[3] = {64, 128, 1};
    if (!encode_bf16_map(&mA, ind, 3, da, sa, ba) || !encode_bf16_map(&mB, hbuf, 3, db, sbt, bb) ||
        !encode_bf16_map(&mC, hm, 3, dc, sc2, bc))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {kD, BH * nqb * kD}, str[1] = {kD * 2};
    const uint32_t box[2] = {64, 128};
    const uint64_t dw[2] = {kD, kD}, sw[1] = {kD * 2};
    if (!encode_bf16_map(&mHM, hm, 2, dims, str, box) || !encode_bf16_map(&mW, wb, 2, dw, sw, box))
      return cudaErrorInvalidValue;
  }
  if (prepare) {
  // 1. summaries
  {
    const int debug_skip = debug_withhold(g, SLA_WITHHOLD_SUMMARIES) ? 1 : 0;
    // at least 48 KB so at most 4 CTAs share an SM: 4 x 128 TMEM columns fit
    const size_t smem = std::max<size_t>(4 * size_t(g.bk) * 128 + 64 + 1024, 48 * 1024);
    dim3 grid(g.nkb, g.BH);
    if (g.bk == 64) {
      // persistent: three CTAs per SM (two 32 KB buffers each; 3 x 128 TMEM
      // columns)
      const size_t psmem = 2 * 32768 + 256 + 1024;
      if ((e = set_smem(lin_summary_persist_kernel, psmem)) != cudaSuccess) return e;
      const int nitems = g.BH * g.nkb;
      const int pgrid = std::min(nitems, 3 * sm_count());
      lin_summary_persist_kernel<<<pgrid, 128, psmem, s>>>(mK, mV, mH, zbuf, g.N, g.nkb, nitems, status,
                                                           wait_limit(g), debug_skip);
    } else {
      if ((e = set_smem(lin_summary_tc_kernel<128>, smem)) != cudaSuccess) return e;
      lin_summary_tc_kernel<128><<<grid, 128, smem, s>>>(mK, mV, mH, zbuf, g.N, g.nkb, status,
                                                         wait_limit(g), debug_skip);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // 2. indicator + gather GEMM
  // (W to bf16 rides along in the first CTAs; 16 CTAs x 128 threads)
  if (g.BH * g.nqb < 16) {
    to_bf16_kernel<<<(kHElems + 255) / 256, 256, 0, s>>>(proj, wb, kHElems);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  indicator_kernel<<<g.BH * g.nqb, 128, 0, s>>>(rows, ind, zbuf, zmbuf, g.nqb, g.nkb, w.ld,
                                                 g.BH * g.nqb >= 16 ? proj : nullptr, wb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_gather(mA, mB, mC, w.ld, g.nqb, g.BH, status, g, s)) != cudaSuccess) return e;
  }  // prepare
  // 3-4. apply + combine
  if (apply) {
    dim3 grid(g.nqb, g.BH);
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(out);
    if (g.bq == 64) {
      const size_t smem = 65536 + 2 * 64 * 128 + 16384 + 512 + 256 + 64 + 1024;
      if ((e = set_smem(lin_apply_tc_kernel<64>, smem)) != cudaSuccess) return e;
      lin_apply_tc_kernel<64><<<grid, 128, smem, s>>>(mHM, mQ, mW, zmbuf, rows, o_s, ob, o_lin, g.N,
                                                      g.nqb, g.nkb, status, wait_limit(g));
    } else {
      const size_t smem = 65536 + 2 * 128 * 128 + 32768 + 512 + 512 + 64 + 1024;
      if ((e = set_smem(lin_apply_tc_kernel<128>, smem)) != cudaSuccess) return e;
      lin_apply_tc_kernel<128><<<grid, 128, smem, s>>>(mHM, mQ, mW, zmbuf, rows, o_s, ob, o_lin, g.N,
                                                       g.nqb, g.nkb, status, wait_limit(g));
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sla
