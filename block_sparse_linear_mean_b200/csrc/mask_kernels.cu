// Block selection: mean pooling, the pooled block scores on the fp32 FMA
// pipe, and block lists from a given mask (the per-row classifier is in
// mask_select.cu, the tensor-core pooled scores in logits_tc.cu).
//
// SLA post ("Selective Linear Attention", list "the idea"): a fast
// mean-pooling step labels the blocks in advance as critical, marginal or
// negligible.  NABLA post (SberAIScience, points 2-3): Q and K are compressed
// per block, and the blocks kept are the top-ranked ones whose summed softmax
// mass exceeds 1 - thr.
#include <float.h>

#include "common.cuh"
#include "tc_common.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// Pooling: out[bh, b, :] = mean of x[bh, t, :] over the real tokens t of
// block b.  One CTA per (block, bh); 16-byte vector loads along d, a fixed
// reduction order (per-thread running sums, then a fixed tree in shared
// memory), so the result is deterministic.

// Block means of Q (blockIdx.z = 0, blocks of bq tokens) and K (z = 1,
// blocks of bk) in one launch: one CTA per (block, bh); each thread sums a
// 16-byte slice of every lanes-th token (the loads of kU such tokens are
// issued together, then added in token order), then the slices' partial
// sums are added in a fixed order.  With lo arrays given, each mean m is
// written split for the tf32 tensor-core logits: hi = tf32(m) in out and
// lo = tf32(m - hi) in lo (m - hi is exact in fp32).
template <typename T>
__global__ void __launch_bounds__(128) pool_kernel(const T* __restrict__ xq, const T* __restrict__ xk,
                                                   float* __restrict__ outq, float* __restrict__ outk,
                                                   float* __restrict__ loq, float* __restrict__ lok,
                                                   int N, int d, int bq, int bk,
                                                   int32_t* __restrict__ zero_words, int nzero,
                                                   int32_t* __restrict__ zero_one) {
  // words the later kernels of the step count or flag into (the status word
  // block, the near-tie counter), zeroed here instead of by memsets of
  // their own: no kernel before this one writes them
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) {
    if (static_cast<int>(threadIdx.x) < nzero) zero_words[threadIdx.x] = 0;
    if (threadIdx.x == 0 && zero_one) *zero_one = 0;
  }
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
  constexpr int kU = 8;                // loads in flight per thread
  const bool isk = blockIdx.z == 1;
  const int block = isk ? bk : bq, nb = (N + block - 1) / block;
  const int b = blockIdx.x, bh = blockIdx.y;
  if (b >= nb) return;
  const T* x = isk ? xk : xq;
  float* out = isk ? outk : outq;
  float* lo = isk ? lok : loq;
  const int t0 = b * block, t1 = min(t0 + block, N), cnt = t1 - t0;
  const T* base = x + (i64(bh) * N) * d;
  const int vpt = d / VEC;                 // vectors per token
  const int lanes = blockDim.x / vpt;      // tokens read per step
  const int v = threadIdx.x % vpt, tl = threadIdx.x / vpt;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  for (int t = t0 + tl; t < t1; t += kU * lanes) {
    uint4 raw[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int tt = t + u * lanes;
      raw[u] = tt < t1 ? __ldg(reinterpret_cast<const uint4*>(base + i64(tt) * d + v * VEC))
                       : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (t + u * lanes >= t1) break;
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
          acc[2 * q] += f.x;
          acc[2 * q + 1] += f.y;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] += __uint_as_float(w[q]);
      }
    }
  }
  __shared__ float part[128 * 8];  // lanes * d <= 128 * VEC
#pragma unroll
  for (int e = 0; e < VEC; ++e) part[tl * d + v * VEC + e] = acc[e];
  __syncthreads();
  const float inv = 1.0f / static_cast<float>(cnt);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < lanes; ++j) s += part[j * d + c];
    const float m = s * inv;
    const i64 o = (i64(bh) * nb + b) * d + c;
    if (lo) {
      const float hi = to_tf32(m);
      out[o] = hi;
      lo[o] = to_tf32(m - hi);
    } else {
      out[o] = m;
    }
  }
}

cudaError_t launch_pool(const void* q, const void* k, int dtype, float* qbar, float* kbar,
                        float* qlo, float* klo, int BH, int N, int d, int bq, int bk, cudaStream_t s,
                        int32_t* zero_words, int nzero, int32_t* zero_one) {
  if (nzero > 128) return cudaErrorInvalidValue;
  dim3 grid((N + min(bq, bk) - 1) / min(bq, bk), BH, 2);
  if (dtype == SLA_BF16)
    pool_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(q),
                                                    static_cast<const __nv_bfloat16*>(k), qbar, kbar,
                                                    qlo, klo, N, d, bq, bk, zero_words, nzero, zero_one);
  else
    pool_kernel<float><<<grid, 128, 0, s>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                            qbar, kbar, qlo, klo, N, d, bq, bk, zero_words, nzero, zero_one);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Pooled logits: logits[bh, i, j] = scale * <qbar[bh, i], kbar[bh, j]>, a
// small fp32 GEMM (64 x 64 tile per CTA, 8 x 8 per thread, sequential
// accumulation over d so every entry has a fixed summation order).

__global__ void __launch_bounds__(64) logits_kernel(const float* __restrict__ qbar,
                                                    const float* __restrict__ kbar,
                                                    float* __restrict__ logits,
                                                    int nqb, int nkb, int d,
                                                    float scale) {
  // 64 threads per 64 x 64 tile, 8 x 8 entries per thread; pooled rows are
  // staged transposed ([k][row]) 32 channels at a time
  __shared__ __align__(16) float As[32][64 + 4];
  __shared__ __align__(16) float Bs[32][64 + 4];
  const int bh = blockIdx.z, i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const float* A = qbar + i64(bh) * nqb * d;
  const float* Bm = kbar + i64(bh) * nkb * d;
  const int tid = threadIdx.x, tx = tid % 8, ty = tid / 8;
  float acc[8][8] = {};
  for (int kk = 0; kk < d; kk += 32) {
#pragma unroll
    for (int it = 0; it < 8; ++it) {  // 64 rows x 8 float4 per operand
      const int e = it * 64 + tid, r = e / 8, c4 = e % 8;
      const int gi = i0 + r, gj = j0 + r;
      const float4 va = gi < nqb ? *reinterpret_cast<const float4*>(A + i64(gi) * d + kk + 4 * c4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 vb = gj < nkb ? *reinterpret_cast<const float4*>(Bm + i64(gj) * d + kk + 4 * c4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
      As[4 * c4][r] = va.x; As[4 * c4 + 1][r] = va.y; As[4 * c4 + 2][r] = va.z; As[4 * c4 + 3][r] = va.w;
      Bs[4 * c4][r] = vb.x; Bs[4 * c4 + 1][r] = vb.y; Bs[4 * c4 + 2][r] = vb.z; Bs[4 * c4 + 3][r] = vb.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {  // channels in order: a fixed summation order per entry
      const float4 a0 = *reinterpret_cast<const float4*>(&As[c][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[c][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[c][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[c][tx * 8 + 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      // paired fp32 FMAs: the same a * b + acc per entry, two entries per
      // instruction
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float2 am = make_float2(a[m], a[m]);
#pragma unroll
        for (int n = 0; n < 8; n += 2) {
          const float2 r2 = fma2(am, make_float2(b[n], b[n + 1]), make_float2(acc[m][n], acc[m][n + 1]));
          acc[m][n] = r2.x;
          acc[m][n + 1] = r2.y;
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int gi = i0 + ty * 8 + m;
    if (gi >= nqb) continue;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int gj = j0 + tx * 8 + n;
      if (gj < nkb) logits[(i64(bh) * nqb + gi) * nkb + gj] = scale * acc[m][n];
    }
  }
}

cudaError_t launch_logits(const float* qbar, const float* kbar, float* logits,
                          const Geom& g, cudaStream_t s) {
  dim3 grid((g.nkb + 63) / 64, (g.nqb + 63) / 64, g.BH);
  logits_kernel<<<grid, 64, 0, s>>>(qbar, kbar, logits, g.nqb, g.nkb, g.d, g.scale);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Lists from a mask row.

constexpr int kCT = 256;  // threads per CTA of the list-from-mask kernel

// Writes the ascending lists of label-2 and label-1 blocks of one row.
// `lab` (shared) holds n labels; `idx_c`/`idx_m` are the row's list slots.
template <int CT>
__device__ void compact_row(const int8_t* lab, int n, int32_t* idx_c,
                            int32_t* cnt_c, int32_t* idx_m, int32_t* cnt_m,
                            int* wsum) {
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  int base_c = 0, base_m = 0;
  for (int j0 = 0; j0 < n; j0 += CT) {
    const int j = j0 + threadIdx.x;
    const int8_t lb = j < n ? lab[j] : 0;
    const unsigned bc = __ballot_sync(0xffffffffu, lb == 2);
    const unsigned bm = __ballot_sync(0xffffffffu, lb == 1);
    __syncthreads();
    if (l == 0) { wsum[w] = __popc(bc); wsum[8 + w] = __popc(bm); }
    __syncthreads();
    int off_c = base_c, off_m = base_m, tot_c = 0, tot_m = 0;
    for (int i = 0; i < CT / 32; ++i) {
      if (i < w) { off_c += wsum[i]; off_m += wsum[8 + i]; }
      tot_c += wsum[i]; tot_m += wsum[8 + i];
    }
    const unsigned below = (1u << l) - 1u;
    if (lb == 2 && idx_c) idx_c[off_c + __popc(bc & below)] = j;
    if (lb == 1 && idx_m) idx_m[off_m + __popc(bm & below)] = j;
    base_c += tot_c;
    base_m += tot_m;
  }
  if (threadIdx.x == 0) {
    if (cnt_c) *cnt_c = base_c;
    if (cnt_m) *cnt_m = base_m;
  }
}

// ---------------------------------------------------------------------------
// Lists from an existing mask.

__global__ void __launch_bounds__(kCT) rows_from_mask_kernel(const int8_t* __restrict__ mask,
                                                             int nkb,
                                                             sla_block_lists rows) {
  extern __shared__ __align__(16) unsigned char smem[];
  int8_t* lab = reinterpret_cast<int8_t*>(smem);
  __shared__ int wsum[32];
  const int row = blockIdx.x;
  for (int j = threadIdx.x; j < nkb; j += kCT) lab[j] = mask[i64(row) * nkb + j];
  __syncthreads();
  const i64 off = i64(row) * nkb;
  compact_row<kCT>(lab, nkb, rows.crit_idx + off, rows.crit_cnt + row,
              rows.marg_idx + off, rows.marg_cnt + row, wsum);
}

cudaError_t launch_rows_from_mask(const int8_t* mask, const Geom& g,
                                  const sla_block_lists& rows, cudaStream_t s) {
  rows_from_mask_kernel<<<g.BH * g.nqb, kCT, g.nkb, s>>>(mask, g.nkb, rows);
  return cudaGetLastError();
}

// One CTA per (bh, 32 consecutive key blocks): 32-row slabs of those 32
// mask columns go through shared memory (rows padded to 36 bytes, so the
// column reads below hit 32 distinct banks); warp w then appends, for its
// four columns, the slab's critical and marginal rows with two ballots each
// -- lists stay ascending.
__global__ void __launch_bounds__(256) cols_from_mask_kernel(const int8_t* __restrict__ mask, int BH,
                                                            int nqb, int nkb, sla_block_lists cols) {
  __shared__ int8_t tile[32][36];
  const int bh = blockIdx.y, j0 = blockIdx.x * 32;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int8_t* mrow = mask + i64(bh) * nqb * nkb;
  const int lr = tid / 8, lb = (tid % 8) * 4;  // loader: slab row, first of four columns
  int nc[4] = {0, 0, 0, 0}, nm[4] = {0, 0, 0, 0};
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = 0; i0 < nqb; i0 += 32) {
    __syncthreads();
    const int i = i0 + lr;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + lb + q;
      tile[lr][lb + q] = (i < nqb && j < nkb) ? mrow[i64(i) * nkb + j] : int8_t(0);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = warp + 8 * k, j = j0 + c;
      if (j >= nkb) continue;  // warp-uniform
      const int8_t v = tile[lane][c];
      const unsigned bc = __ballot_sync(0xffffffffu, v == 2);
      const unsigned bm = __ballot_sync(0xffffffffu, v == 1);
      const i64 t = i64(bh) * nkb + j;
      if (v == 2) cols.crit_idx[t * nqb + nc[k] + __popc(bc & lt)] = i0 + lane;
      if (v == 1) cols.marg_idx[t * nqb + nm[k] + __popc(bm & lt)] = i0 + lane;
      nc[k] += __popc(bc);
      nm[k] += __popc(bm);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = j0 + warp + 8 * k;
    if (lane == 0 && j < nkb) {
      cols.crit_cnt[i64(bh) * nkb + j] = nc[k];
      cols.marg_cnt[i64(bh) * nkb + j] = nm[k];
    }
  }
}

cudaError_t launch_cols_from_mask(const int8_t* mask, const Geom& g,
                                  const sla_block_lists& cols, cudaStream_t s) {
  dim3 grid((g.nkb + 31) / 32, g.BH);
  cols_from_mask_kernel<<<grid, 256, 0, s>>>(mask, g.BH, g.nqb, g.nkb, cols);
  return cudaGetLastError();
}

}  // namespace sla
