// Pooled block logits on the tensor cores.
//
// SLA post ("Selective Linear Attention", list "the idea") and NABLA post
// (SberAIScience, points 2-3): the block classifier ranks key blocks by the
// softmax of the pooled scores logits[bh, i, j] = scale * <qbar_i, kbar_j>,
// a batched dense contraction (Nqb x Nkb x d per head).
//
// The means arrive split as m = hi + lo with hi = tf32(m), lo = tf32(m - hi)
// (the pooling kernel writes both), and each product is taken as
//   lo_q . hi_k + hi_q . lo_k + hi_q . hi_k
// with kind::tf32 MMAs accumulating in fp32 tensor memory.  With |m - hi| <=
// 2^-11 |m| and |(m - hi) - lo| <= 2^-22 |m|, the dropped lo . lo term and
// the rounding of lo stay below 3 * 2^-22 (under 2^-20) of |q| |k| per
// channel, about the size of fp32 rounding, so the logits carry fp32
// accuracy.
//
// Persistent kernel, one CTA per SM, 128 x 128 output tiles (query blocks x
// key blocks) walked in (m, n, bh) order:
//   warp 0    TMA producer: per 32-channel chunk, hi and lo tiles of both
//             operands (4 x 16 KB, 128-byte swizzle, K-major) into a
//             3-stage ring
//   warp 1    TMEM owner and MMA issuer: 4 K-steps of 8 channels x 3
//             products per chunk into one of two 128-column accumulators
//   warps 2-5 epilogue: TMEM -> registers -> scale -> each lane stores its
//             row's 32 columns with 16-byte stores (the destination is the
//             L2-resident score slab; any Nkb, ragged tiles masked)
#include <algorithm>

#include "common.cuh"
#include "tc_common.cuh"

namespace sla {

namespace {

constexpr int kLStages = 3;
constexpr uint32_t kLPart = 128 * 128;         // 128 rows x 32 fp32 (128 B)
constexpr uint32_t kLStage = 4 * kLPart;       // A hi, A lo, B hi, B lo
constexpr uint32_t kLBars = kLStages * kLStage;
constexpr size_t kLSmem = kLBars + 256 + 1024;
static_assert(kLSmem <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

__global__ void __launch_bounds__(192, 1) logits_tc_kernel(
    const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmQl,
    const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKl,
    float* __restrict__ logits, int nqb, int nkb, int kchunks, int tiles_m, int tiles_n, int ntiles,
    float scale, int32_t* status, long long timeout, int debug_skip) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const uint32_t sb = smem_u32(base);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kLBars);
  auto b_full = [&](int s) { return smem_u32(&bars[s]); };
  auto b_empty = [&](int s) { return smem_u32(&bars[kLStages + s]); };
  auto b_acc_full = [&](int a) { return smem_u32(&bars[2 * kLStages + a]); };
  auto b_acc_empty = [&](int a) { return smem_u32(&bars[2 * kLStages + 2 + a]); };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(&bars[2 * kLStages + 4]);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kLStages; ++s) { mbar_init(b_full(s), 1); mbar_init(b_empty(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(b_acc_full(a), 1); mbar_init(b_acc_empty(a), 4); }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tslot), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // tile -> (m, n, bh), m fastest
  auto coords = [&](int t, int& m0, int& n0, int& bh) {
    const int per = tiles_m * tiles_n;
    bh = t / per;
    const int r = t - bh * per;
    n0 = (r / tiles_m) * 128;
    m0 = (r % tiles_m) * 128;
  };
  bool ok = true;
  if (warp == 0 && lane == 0) {
    int g = 0;  // chunks loaded so far (ring position)
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      int m0, n0, bh;
      coords(t, m0, n0, bh);
      for (int ks = 0; ks < kchunks && ok; ++ks, ++g) {
        const int s = g % kLStages;
        if (g >= kLStages) ok = wait_bounded(b_empty(s), ((g / kLStages) & 1) ^ 1, status, timeout);
        if (!ok) break;
        if (debug_skip && blockIdx.x == 0 && g == 0) continue;  // test aid: this chunk never arrives
        const uint32_t st = sb + s * kLStage;
        mbar_expect_tx(b_full(s), kLStage);
        tma_load_3d(st, &tmQh, ks * 32, m0, bh, b_full(s));
        tma_load_3d(st + kLPart, &tmQl, ks * 32, m0, bh, b_full(s));
        tma_load_3d(st + 2 * kLPart, &tmKh, ks * 32, n0, bh, b_full(s));
        tma_load_3d(st + 3 * kLPart, &tmKl, ks * 32, n0, bh, b_full(s));
      }
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_tf32(128, 128);
    const uint64_t d0 = sdesc(sb, 16, 1024);  // K-major, 128-byte swizzle
    int g = 0, it = 0;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
      const int a = it & 1;
      // the epilogue has drained this accumulator (tile it - 2)
      if (it >= 2) ok = wait_bounded(b_acc_empty(a), ((it >> 1) & 1) ^ 1, status, timeout);
      for (int ks = 0; ks < kchunks && ok; ++ks, ++g) {
        const int s = g % kLStages;
        ok = wait_bounded(b_full(s), (g / kLStages) & 1, status, timeout);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + 128 * a;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 8 channels (32 bytes) per step
          const uint32_t o = s * kLStage + kk * 32;
          tc_mma_tf32(acc, sdesc_add(d0, o + kLPart), sdesc_add(d0, o + 2 * kLPart), idesc,
                      (ks > 0 || kk > 0) ? 1u : 0u);                                      // lo_q hi_k
          tc_mma_tf32(acc, sdesc_add(d0, o), sdesc_add(d0, o + 3 * kLPart), idesc, 1u);   // hi_q lo_k
          tc_mma_tf32(acc, sdesc_add(d0, o), sdesc_add(d0, o + 2 * kLPart), idesc, 1u);   // hi_q hi_k
        }
        tc_commit(b_empty(s));
      }
      if (ok) tc_commit(b_acc_full(a));
    }
  } else if (warp >= 2) {
    const int quad = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    int it = 0;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
      const int a = it & 1;
      int m0, n0, bh;
      coords(t, m0, n0, bh);
      ok = __all_sync(0xffffffffu, wait_bounded(b_acc_full(a), (it >> 1) & 1, status, timeout));
      if (!ok) break;  // (the whole warp: the loop below synchronises it)
      tc_fence_after();
      const int row0 = m0 + quad * 32;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + 128 * a + lane_off + c0, v);
        tmem_wait_ld();
        reg_fence<32>(v);
        if (c0 == 96) {  // this warp's reads of the accumulator are done
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_acc_empty(a));
        }
        // lane l holds row row0 + l, columns n0 + c0 .. + 31, and stores
        // them itself: the destination is the score slab, which stays in L2,
        // so 16-byte stores of one row per lane cost less than a transpose
        // through shared memory into row-coalesced stores
        const int row = row0 + lane;
        const int ncol = min(32, nkb - (n0 + c0));
        if (row < nqb && ncol > 0) {
          float* dst = logits + (i64(bh) * nqb + row) * nkb + n0 + c0;
          if (ncol == 32 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + e) =
                  make_float4(v[e] * scale, v[e + 1] * scale, v[e + 2] * scale, v[e + 3] * scale);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < ncol) dst[e] = v[e] * scale;
          }
        }
      }
    }
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (!ok) {  // let in-flight copies and products drain (bounded)
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) __nanosleep(1000);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool logits_tc_supported(const Geom& g) {
  return tma_available() && !(g.flags & SLA_FLAG_SIMT) && g.d % 32 == 0;
}

cudaError_t launch_logits_tc(const float* qhi, const float* qlo, const float* khi, const float* klo,
                             float* logits, const Geom& g, int32_t* status, cudaStream_t s) {
  CUtensorMap mQh, mQl, mKh, mKl;
  auto mk = [&](CUtensorMap* m, const float* p, int rows) {
    const uint64_t dims[3] = {uint64_t(g.d), uint64_t(rows), uint64_t(g.BH)};
    const uint64_t strides[2] = {uint64_t(g.d) * 4, uint64_t(rows) * g.d * 4};
    const uint32_t box[3] = {32, 128, 1};
    return encode_f32_map(m, p, 3, dims, strides, box);
  };
  if (!mk(&mQh, qhi, g.nqb) || !mk(&mQl, qlo, g.nqb) || !mk(&mKh, khi, g.nkb) || !mk(&mKl, klo, g.nkb))
    return cudaErrorInvalidValue;
  const int tiles_m = (g.nqb + 127) / 128, tiles_n = (g.nkb + 127) / 128;
  const int ntiles = tiles_m * tiles_n * g.BH;
  cudaError_t e = cudaFuncSetAttribute(logits_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kLSmem));
  if (e != cudaSuccess) return e;
  const int grid = std::min(ntiles, sm_count());
  logits_tc_kernel<<<grid, 192, kLSmem, s>>>(mQh, mQl, mKh, mKl, logits, g.nqb, g.nkb, g.d / 32, tiles_m,
                                             tiles_n, ntiles, g.scale, status, wait_limit(g),
                                             debug_withhold(g, SLA_WITHHOLD_LOGITS) ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace sla
