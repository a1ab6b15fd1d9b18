// Block selection: mean pooling, pooled block scores and the per-row
// classifier that emits the block mask and the compact block lists.
//
// SLA post ("Selective Linear Attention", list "the idea"): a fast
// mean-pooling step labels the blocks in advance as critical, marginal or
// negligible.  NABLA post (SberAIScience, points 2-3): Q and K are compressed
// per block, and the blocks kept are the top-ranked ones whose summed softmax
// mass exceeds 1 - thr.
#include <float.h>

#include "common.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// Pooling: out[bh, b, :] = mean of x[bh, t, :] over the real tokens t of
// block b.  One CTA per (block, bh); 16-byte vector loads along d, a fixed
// reduction order (per-thread running sums, then a fixed tree in shared
// memory), so the result is deterministic.

template <typename T>
__global__ void __launch_bounds__(256) pool_kernel(const T* __restrict__ x,
                                                   float* __restrict__ out,
                                                   int N, int d, int block) {
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
  const int b = blockIdx.x, bh = blockIdx.y, nb = gridDim.x;
  const int t0 = b * block, t1 = min(t0 + block, N), cnt = t1 - t0;
  const T* base = x + (i64(bh) * N) * d;
  const int vpt = d / VEC;                 // vectors per token
  const int lanes = blockDim.x / vpt;      // tokens read per step
  const int v = threadIdx.x % vpt, tl = threadIdx.x / vpt;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  for (int t = t0 + tl; t < t1; t += lanes) {
    const T* p = base + i64(t) * d + v * VEC;
#pragma unroll
    for (int e = 0; e < VEC; e += 4) {
      float4 f = load4(p + e);
      acc[e] += f.x; acc[e + 1] += f.y; acc[e + 2] += f.z; acc[e + 3] += f.w;
    }
  }
  __shared__ float part[256 * 8];  // lanes * d <= 256 * VEC
#pragma unroll
  for (int e = 0; e < VEC; ++e) part[tl * d + v * VEC + e] = acc[e];
  __syncthreads();
  const float inv = 1.0f / static_cast<float>(cnt);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < lanes; ++j) s += part[j * d + c];
    out[(i64(bh) * nb + b) * d + c] = s * inv;
  }
}

cudaError_t launch_pool(const void* x, int dtype, float* out, int BH, int N,
                        int d, int block, cudaStream_t s) {
  dim3 grid((N + block - 1) / block, BH);
  if (dtype == SLA_BF16)
    pool_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), out, N, d, block);
  else
    pool_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(x), out,
                                            N, d, block);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Pooled logits: logits[bh, i, j] = scale * <qbar[bh, i], kbar[bh, j]>, a
// small fp32 GEMM (64 x 64 tile per CTA, 4 x 4 per thread, sequential
// accumulation over d so every entry has a fixed summation order).

__global__ void __launch_bounds__(256) logits_kernel(const float* __restrict__ qbar,
                                                     const float* __restrict__ kbar,
                                                     float* __restrict__ logits,
                                                     int nqb, int nkb, int d,
                                                     float scale) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int bh = blockIdx.z, i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const float* A = qbar + i64(bh) * nqb * d;
  const float* Bm = kbar + i64(bh) * nkb * d;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int kk = 0; kk < d; kk += 16) {
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int r = e / 16, c = e % 16;
      const int gi = i0 + r, gj = j0 + r;
      As[c][r] = gi < nqb ? A[i64(gi) * d + kk + c] : 0.f;
      Bs[c][r] = gj < nkb ? Bm[i64(gj) * d + kk + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) a[m] = As[c][ty * 4 + m];
#pragma unroll
      for (int n = 0; n < 4; ++n) b[n] = Bs[c][tx * 4 + n];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < 4; ++n) acc[m][n] = fmaf(a[m], b[n], acc[m][n]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int gi = i0 + ty * 4 + m;
    if (gi >= nqb) continue;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const int gj = j0 + tx * 4 + n;
      if (gj < nkb) logits[(i64(bh) * nqb + gi) * nkb + gj] = scale * acc[m][n];
    }
  }
}

cudaError_t launch_logits(const float* qbar, const float* kbar, float* logits,
                          const Geom& g, cudaStream_t s) {
  dim3 grid((g.nkb + 63) / 64, (g.nqb + 63) / 64, g.BH);
  logits_kernel<<<grid, 256, 0, s>>>(qbar, kbar, logits, g.nqb, g.nkb, g.d,
                                     g.scale);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Block-wide helpers (256 threads).

constexpr int kCT = 256;  // classifier threads per CTA

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kCT / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kCT / 32; ++i) r += red[i];
  return r;
}

__device__ __forceinline__ int block_reduce_sum_int(int v, int* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  int r = 0;
  for (int i = 0; i < kCT / 32; ++i) r += red[i];
  return r;
}

// Writes the ascending lists of label-2 and label-1 blocks of one row.
// `lab` (shared) holds n labels; `idx_c`/`idx_m` are the row's list slots.
__device__ void compact_row(const int8_t* lab, int n, int32_t* idx_c,
                            int32_t* cnt_c, int32_t* idx_m, int32_t* cnt_m,
                            int* wsum) {
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  int base_c = 0, base_m = 0;
  for (int j0 = 0; j0 < n; j0 += kCT) {
    const int j = j0 + threadIdx.x;
    const int8_t lb = j < n ? lab[j] : 0;
    const unsigned bc = __ballot_sync(0xffffffffu, lb == 2);
    const unsigned bm = __ballot_sync(0xffffffffu, lb == 1);
    __syncthreads();
    if (l == 0) { wsum[w] = __popc(bc); wsum[8 + w] = __popc(bm); }
    __syncthreads();
    int off_c = base_c, off_m = base_m, tot_c = 0, tot_m = 0;
    for (int i = 0; i < kCT / 32; ++i) {
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
// Classifier: one CTA per (bh, query block) row.
//   1. P = softmax of the row's logits (fp32, fixed reduction order);
//   2. sort 64-bit keys (P bits << 32 | ~index) descending -- rank order is
//      score descending, block index ascending on equal scores;
//   3. top-k: first n_c ranks critical, next n_m marginal;
//      CDF: tail sums of P over the ranks in exact 2^-62 fixed point (integer
//      adds, order-free), a rank is dropped iff its tail sum (itself and all
//      lower ranks) is below thr; the top rank is always kept;
//   4. write the mask row and the ascending CSR lists; count near-ties.

struct ClassifyArgs {
  int nkb, S, mode, n_c, n_m;
  int from_prob;  // input rows are already softmaxed scores, not logits
  uint64_t thr_fx;
  int8_t* mask;
  sla_block_lists rows;
  float* scores;
  int32_t* tie_count;
};

__device__ __forceinline__ uint64_t to_fixed(float p) {
  return __double2ull_rz(static_cast<double>(p) * kFixedOne);
}

__global__ void __launch_bounds__(kCT) classify_kernel(const float* __restrict__ logits,
                                                       ClassifyArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem);
  int8_t* lab = reinterpret_cast<int8_t*>(keys + a.S);
  __shared__ float redf[32];
  __shared__ int redi[32];
  __shared__ uint64_t seg_suffix[kCT];
  __shared__ uint64_t t_at[2];
  const int row = blockIdx.x;
  const int nkb = a.nkb, S = a.S, tid = threadIdx.x;
  const float* lr = logits + i64(row) * nkb;

  // 1. softmax over the row (skipped for rows given as scores)
  float m = 0.f, inv = 1.f;
  if (!a.from_prob) {
    m = -FLT_MAX;
    for (int j = tid; j < nkb; j += kCT) m = fmaxf(m, lr[j]);
    m = block_reduce_max(m, redf);
    float se = 0.f;
    for (int j = tid; j < nkb; j += kCT) se += expf(lr[j] - m);
    se = block_reduce_sum(se, redf);
    inv = 1.0f / se;
  }
  for (int j = tid; j < S; j += kCT) {
    uint64_t key = 0;
    if (j < nkb) {
      // scores are non-negative, so their bit patterns order like the values
      const float p = a.from_prob ? fmaxf(lr[j], 0.f) : expf(lr[j] - m) * inv;
      if (a.scores) a.scores[i64(row) * nkb + j] = p;
      key = (static_cast<uint64_t>(__float_as_uint(p)) << 32) |
            static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(j));
    }
    keys[j] = key;
  }
  __syncthreads();

  // 2. bitonic sort, descending
  for (int k = 2; k <= S; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = tid; i < S; i += kCT) {
        const int ixj = i ^ jj;
        if (ixj > i) {
          const uint64_t x = keys[i], y = keys[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (x < y) : (x > y)) { keys[i] = y; keys[ixj] = x; }
        }
      }
      __syncthreads();
    }
  }

  // 3. number of critical ranks
  int c = a.n_c;
  const int seg = S / kCT;  // ranks per thread (S >= kCT)
  if (a.mode == SLA_MASK_CDF) {
    uint64_t local = 0;
    for (int r = tid * seg; r < (tid + 1) * seg; ++r)
      if (r < nkb) local += to_fixed(__uint_as_float(static_cast<uint32_t>(keys[r] >> 32)));
    seg_suffix[tid] = local;
    __syncthreads();
    if (tid < 32) {  // suffix sums of the 256 segment totals, one warp
      uint64_t v8[8], tot = 0;
      for (int e = 0; e < 8; ++e) { v8[e] = seg_suffix[tid * 8 + e]; tot += v8[e]; }
      uint64_t incl = tot;  // inclusive suffix over lanes >= tid
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_down_sync(0xffffffffu, incl, o);
        if (tid + o < 32) incl += y;
      }
      uint64_t run = incl - tot;  // lanes > tid
      for (int e = 7; e >= 0; --e) { seg_suffix[tid * 8 + e] = run; run += v8[e]; }
    }
    __syncthreads();
    int kept = 0;
    uint64_t run = seg_suffix[tid];
    for (int r = (tid + 1) * seg - 1; r >= tid * seg; --r) {
      if (r >= nkb) continue;
      run += to_fixed(__uint_as_float(static_cast<uint32_t>(keys[r] >> 32)));
      if (run >= a.thr_fx) ++kept;
    }
    c = block_reduce_sum_int(kept, redi);
    if (c < 1) c = 1;
    // record the two decisive tail sums for the tie report
    if (a.tie_count) {
      run = seg_suffix[tid];
      for (int r = (tid + 1) * seg - 1; r >= tid * seg; --r) {
        if (r >= nkb) continue;
        run += to_fixed(__uint_as_float(static_cast<uint32_t>(keys[r] >> 32)));
        if (r == c - 1) t_at[0] = run;
        if (r == c) t_at[1] = run;
      }
    }
  }
  const int nm = min(a.n_m, nkb - c);
  // labels by rank
  for (int r = tid; r < nkb; r += kCT) {
    const int j = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(keys[r]));
    lab[j] = r < c ? 2 : (r < c + nm ? 1 : 0);
  }
  __syncthreads();

  // tie report: the decisive margins of this row, as seen in fp32 P -- score
  // gaps at a cut relative to the higher score, tail sums against thr in
  // absolute (unit mass) terms
  if (a.tie_count && tid == 0) {
    auto pr = [&](int r) { return __uint_as_float(static_cast<uint32_t>(keys[r] >> 32)); };
    auto close = [&](int r) { return (pr(r) - pr(r + 1)) <= kTieEps * pr(r); };
    bool tie = false;
    if (a.mode == SLA_MASK_TOPK) {
      if (c > 0 && c < nkb) tie |= close(c - 1);
    } else if (a.thr_fx > 0) {
      const double thr = static_cast<double>(a.thr_fx) / kFixedOne;
      if (c > 1) tie |= fabs(static_cast<double>(t_at[0]) / kFixedOne - thr) <= kTieEps;
      if (c < nkb) {
        tie |= fabs(thr - static_cast<double>(t_at[1]) / kFixedOne) <= kTieEps;
        tie |= close(c - 1);
      }
    }
    if (nm > 0 && c + nm < nkb) tie |= close(c + nm - 1);
    if (tie) atomicAdd(a.tie_count, 1);
  }

  // 4. mask row and lists
  for (int j = tid; j < nkb; j += kCT) a.mask[i64(row) * nkb + j] = lab[j];
  const i64 off = i64(row) * nkb;
  compact_row(lab, nkb, a.rows.crit_idx + off, a.rows.crit_cnt + row,
              a.rows.marg_idx + off, a.rows.marg_cnt + row, redi);
}

static int sort_size(int n) {
  int s = kCT;
  while (s < n) s <<= 1;
  return s;
}

cudaError_t launch_classify(const float* logits, const Geom& g, int8_t* mask,
                            const sla_block_lists& rows, float* scores,
                            int32_t* tie_count, cudaStream_t s, bool from_prob) {
  ClassifyArgs a;
  a.from_prob = from_prob ? 1 : 0;
  a.nkb = g.nkb;
  a.S = sort_size(g.nkb);
  a.mode = g.mode;
  a.n_c = g.n_c;
  a.n_m = g.n_m;
  a.thr_fx = g.thr_fx;
  a.mask = mask;
  a.rows = rows;
  a.scores = scores;
  a.tie_count = tie_count;
  const size_t smem = static_cast<size_t>(a.S) * 8 + static_cast<size_t>(a.S);
  cudaError_t e = cudaFuncSetAttribute(classify_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (tie_count) {
    e = cudaMemsetAsync(tie_count, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  classify_kernel<<<g.BH * g.nqb, kCT, smem, s>>>(logits, a);
  return cudaGetLastError();
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
  compact_row(lab, nkb, rows.crit_idx + off, rows.crit_cnt + row,
              rows.marg_idx + off, rows.marg_cnt + row, wsum);
}

cudaError_t launch_rows_from_mask(const int8_t* mask, const Geom& g,
                                  const sla_block_lists& rows, cudaStream_t s) {
  rows_from_mask_kernel<<<g.BH * g.nqb, kCT, g.nkb, s>>>(mask, g.nkb, rows);
  return cudaGetLastError();
}

// One thread per (bh, key block): walk the column top to bottom.  Threads of
// a warp read adjacent bytes of each mask row.
__global__ void cols_from_mask_kernel(const int8_t* __restrict__ mask, int BH,
                                      int nqb, int nkb, sla_block_lists cols) {
  const i64 t = i64(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= i64(BH) * nkb) return;
  const int bh = static_cast<int>(t / nkb), j = static_cast<int>(t % nkb);
  int nc = 0, nm = 0;
  const int8_t* col = mask + i64(bh) * nqb * nkb + j;
  int32_t* ic = cols.crit_idx + t * nqb;
  int32_t* im = cols.marg_idx + t * nqb;
  for (int i = 0; i < nqb; ++i) {
    const int8_t lb = col[i64(i) * nkb];
    if (lb == 2) ic[nc++] = i;
    else if (lb == 1) im[nm++] = i;
  }
  cols.crit_cnt[t] = nc;
  cols.marg_cnt[t] = nm;
}

cudaError_t launch_cols_from_mask(const int8_t* mask, const Geom& g,
                                  const sla_block_lists& cols, cudaStream_t s) {
  const i64 n = i64(g.BH) * g.nkb;
  cols_from_mask_kernel<<<static_cast<unsigned>((n + 127) / 128), 128, 0, s>>>(
      mask, g.BH, g.nqb, g.nkb, cols);
  return cudaGetLastError();
}

}  // namespace sla
