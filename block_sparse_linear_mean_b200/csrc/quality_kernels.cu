// Mask quality: how much of dense attention a block mask keeps.
//
// Veda article (mlllm.io, section "Контекст" / context): a sparsity mask is
// evaluated by how well it reproduces the structure of dense attention, and the
// reference its predictor is distilled toward is the dense attention
// max-pooled over tiles; the article's users' section reports the
// predictor's recall.  Two measurement kernels (not on the hot path):
//
//   block_importance_kernel  imp[bh, i, j] = max over real query tokens t of
//                            block i and real keys s of block j of the dense
//                            softmax probability P[t, s] (each row's
//                            softmax over all N keys, fp32)
//   mask_recall_kernel       per row with c critical blocks: the reference
//                            set is the c blocks of largest importance (ties
//                            by lower index); counts the reference blocks the
//                            mask marks critical, and the same for the kept
//                            (critical or marginal) set
//
// The importance is dense O(N^2 d) work on the SIMT cores, meant for N up to
// tens of thousands; the recall ranks each row's blocks by counting, O(Nkb^2)
// per row.
#include <float.h>

#include "common.cuh"

namespace sla {

namespace {

constexpr int kQWarps = 4;

template <typename T>
__device__ __forceinline__ float ld_elem(const T* p) {
  if constexpr (sizeof(T) == 2) return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  else return *p;
}

// One CTA (4 warps) per (query block, bh).  The block's query rows sit in
// shared memory (rows padded by one word, so the lanes' rows fall in distinct
// banks); lane l owns rows l, l + 32, ...; warp w walks the key blocks
// j = w, w + 4, ..., staging one key row at a time.  Pass 1 keeps an online
// (max, sum) per row over the warp's keys, merged across the warps in
// shared memory; pass 2 recomputes the scores and takes each key block's
// largest probability, reduced across the warp.
template <typename T>
__global__ void __launch_bounds__(32 * kQWarps) block_importance_kernel(
    const T* __restrict__ q, const T* __restrict__ k, float* __restrict__ imp, int N, int d,
    int bq, int bk, int nqb, int nkb, float scale) {
  extern __shared__ float qsm[];
  const int dp = d + 1;                        // padded row
  float* ks = qsm + bq * dp;                   // [kQWarps][d] staged key rows
  float* st_m = ks + kQWarps * d;              // [kQWarps][bq] partial maxima
  float* st_l = st_m + kQWarps * bq;           // [kQWarps][bq] partial sums
  const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  const int t0 = i * bq, nt = min(bq, N - t0);
  const T* qb = q + (i64(bh) * N + t0) * d;
  const T* kb = k + i64(bh) * N * d;
  for (int x = tid; x < bq * d; x += blockDim.x) {
    const int r = x / d, c = x % d;
    qsm[r * dp + c] = r < nt ? ld_elem(qb + i64(r) * d + c) : 0.f;
  }
  __syncthreads();
  const int qpl = bq / 32;  // rows per lane (2 or 4)
  float m[4], l[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) { m[u] = -FLT_MAX; l[u] = 0.f; }
  float* kw = ks + warp * d;
  auto stage = [&](int s) {  // key row s -> this warp's staging row
    __syncwarp();
    for (int c = lane; c < d; c += 32) kw[c] = ld_elem(kb + i64(s) * d + c);
    __syncwarp();
  };
  auto score = [&](int r) {
    const float* qr = qsm + r * dp;
    float a0 = 0.f, a1 = 0.f;
    for (int c = 0; c < d; c += 2) {
      a0 = fmaf(qr[c], kw[c], a0);
      a1 = fmaf(qr[c + 1], kw[c + 1], a1);
    }
    return (a0 + a1) * scale;
  };
  // pass 1: online max and sum of exp over this warp's keys
  for (int j = warp; j < nkb; j += kQWarps) {
    const int s1 = min((j + 1) * bk, N);
    for (int s = j * bk; s < s1; ++s) {
      stage(s);
      for (int u = 0; u < qpl; ++u) {
        const int r = lane + 32 * u;
        if (r >= nt) continue;
        const float z = score(r);
        if (z > m[u]) {
          l[u] = l[u] * expf(m[u] - z) + 1.f;
          m[u] = z;
        } else {
          l[u] += expf(z - m[u]);
        }
      }
    }
  }
  for (int u = 0; u < qpl; ++u) {
    const int r = lane + 32 * u;
    st_m[warp * bq + r] = m[u];
    st_l[warp * bq + r] = l[u];
  }
  __syncthreads();
  for (int u = 0; u < qpl; ++u) {  // merge the warps' partial (max, sum)
    const int r = lane + 32 * u;
    float mm = -FLT_MAX;
    for (int w = 0; w < kQWarps; ++w) mm = fmaxf(mm, st_m[w * bq + r]);
    float ll = 0.f;
    for (int w = 0; w < kQWarps; ++w) {
      const float lw = st_l[w * bq + r];
      if (lw > 0.f) ll += lw * expf(st_m[w * bq + r] - mm);
    }
    m[u] = mm;
    l[u] = ll > 0.f ? 1.f / ll : 0.f;  // (reciprocal of the row's sum)
  }
  // pass 2: each key block's largest probability over the block's rows
  for (int j = warp; j < nkb; j += kQWarps) {
    const int s1 = min((j + 1) * bk, N);
    float bm = 0.f;
    for (int s = j * bk; s < s1; ++s) {
      stage(s);
      for (int u = 0; u < qpl; ++u) {
        const int r = lane + 32 * u;
        if (r >= nt) continue;
        bm = fmaxf(bm, expf(score(r) - m[u]) * l[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    if (lane == 0) imp[(i64(bh) * nqb + i) * nkb + j] = bm;
  }
}

// One CTA per row: the row's importance values and labels in shared memory;
// each block's rank is the number of blocks ordered before it (larger
// value, or equal value and lower index).
__global__ void __launch_bounds__(128) mask_recall_kernel(const int8_t* __restrict__ mask,
                                                          const float* __restrict__ imp, int nkb,
                                                          int32_t* __restrict__ counts) {
  extern __shared__ float rsm[];
  int8_t* lab = reinterpret_cast<int8_t*>(rsm + nkb);
  __shared__ int red[4][4];
  const int row = blockIdx.x, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const float* ir = imp + i64(row) * nkb;
  const int8_t* mr = mask + i64(row) * nkb;
  int c = 0, ck = 0;
  for (int j = tid; j < nkb; j += blockDim.x) {
    rsm[j] = ir[j];
    lab[j] = mr[j];
    c += mr[j] == 2;
    ck += mr[j] != 0;
  }
  __syncthreads();
  auto block_sum = [&](int v, int slot) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[slot][warp] = v;
    __syncthreads();
    const int t = red[slot][0] + red[slot][1] + red[slot][2] + red[slot][3];
    return t;
  };
  c = block_sum(c, 0);
  ck = block_sum(ck, 1);
  int hc = 0, hk = 0;
  for (int j = tid; j < nkb; j += blockDim.x) {
    const float v = rsm[j];
    int rank = 0;
    for (int jj = 0; jj < nkb; ++jj) {
      const float w = rsm[jj];
      rank += (w > v || (w == v && jj < j)) ? 1 : 0;
    }
    hc += (rank < c && lab[j] == 2) ? 1 : 0;
    hk += (rank < ck && lab[j] != 0) ? 1 : 0;
  }
  hc = block_sum(hc, 2);
  hk = block_sum(hk, 3);
  if (tid == 0) {
    atomicAdd(&counts[0], hc);
    atomicAdd(&counts[1], c);
    atomicAdd(&counts[2], hk);
    atomicAdd(&counts[3], ck);
  }
}

}  // namespace

cudaError_t launch_block_importance(const void* q, const void* k, float* imp, const Geom& g,
                                    cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t(g.bq) * (g.d + 1) + size_t(kQWarps) * g.d +
                                       2 * size_t(kQWarps) * g.bq);
  dim3 grid(g.nqb, g.BH);
  cudaError_t e;
  if (g.dtype == SLA_BF16) {
    auto kern = block_importance_kernel<__nv_bfloat16>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
      return e;
    kern<<<grid, 32 * kQWarps, smem, s>>>(static_cast<const __nv_bfloat16*>(q),
                                         static_cast<const __nv_bfloat16*>(k), imp, g.N, g.d, g.bq,
                                         g.bk, g.nqb, g.nkb, g.scale);
  } else {
    auto kern = block_importance_kernel<float>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
      return e;
    kern<<<grid, 32 * kQWarps, smem, s>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                         imp, g.N, g.d, g.bq, g.bk, g.nqb, g.nkb, g.scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_mask_recall(const int8_t* mask, const float* imp, const Geom& g, int32_t* counts,
                               cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(counts, 0, 4 * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  const size_t smem = size_t(g.nkb) * 5 + 16;
  if ((e = cudaFuncSetAttribute(mask_recall_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem))) != cudaSuccess)
    return e;
  mask_recall_kernel<<<g.BH * g.nqb, 128, smem, s>>>(mask, imp, g.nkb, counts);
  return cudaGetLastError();
}

}  // namespace sla
