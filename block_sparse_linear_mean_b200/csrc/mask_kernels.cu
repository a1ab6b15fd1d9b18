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
                                                   int N, int d, int bq, int bk) {
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
                        float* qlo, float* klo, int BH, int N, int d, int bq, int bk, cudaStream_t s) {
  dim3 grid((N + min(bq, bk) - 1) / min(bq, bk), BH, 2);
  if (dtype == SLA_BF16)
    pool_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(q),
                                                    static_cast<const __nv_bfloat16*>(k), qbar, kbar,
                                                    qlo, klo, N, d, bq, bk);
  else
    pool_kernel<float><<<grid, 128, 0, s>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                            qbar, kbar, qlo, klo, N, d, bq, bk);
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
// Block-wide helpers (256 threads).

constexpr int kCT = 256;  // threads per CTA of the list-from-mask kernel

template <int CT>
__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < CT / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

template <int CT>
__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < CT / 32; ++i) r += red[i];
  return r;
}

template <int CT>
__device__ __forceinline__ int block_reduce_sum_int(int v, int* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  int r = 0;
  for (int i = 0; i < CT / 32; ++i) r += red[i];
  return r;
}

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
// Classifier: one CTA per (bh, query block) row (64 threads for rows of up to
// 1024 blocks, 256 above); top-k rows of up to 1024 blocks take the one-warp
// variant below (classify_topk_warp_kernel), which makes the same cuts.
//   1. P = softmax of the row's logits (fp32, fixed reduction order), kept as
//      32-bit patterns: scores are non-negative, so the patterns order like
//      the values;
//   2. rank order is score descending, block index ascending on equal
//      scores; no sort is needed, only the scores at the cuts:
//      top-k: radix selection (4 passes of 8-bit digits, per-warp histograms)
//      finds the score v at rank k and how many scores exceed it; among the
//      blocks scoring exactly v the lowest indices fill the remaining slots;
//      CDF: the same passes over exact 2^-62 fixed-point sums (integer adds,
//      order-free) find the score at which the running tail sum -- a block
//      plus every lower-ranked block -- first reaches thr; blocks below it
//      are dropped, the top rank is always kept;
//   3. write the mask row and the ascending CSR lists; count near-ties.

struct ClassifyArgs {
  int nkb, mode, n_c, n_m;
  int from_prob;  // input rows are already softmaxed scores, not logits
  uint64_t thr_fx;
  int8_t* mask;
  sla_block_lists rows;
  float* scores;
  int32_t* tie_count;
};


template <int CT>
struct SelShared {
  uint32_t hist[(CT / 32)][256];
  unsigned long long hsum[(CT / 32)][256];
  uint32_t tot[256];
  unsigned long long tots[256];
  uint32_t res_u[4];
  unsigned long long res_l[4];
};

// Rank-k score (k counted from the top, 0-based) among the n patterns: the
// value v and the number of patterns strictly above it.
template <int CT>
__device__ void select_rank(const uint32_t* pb, int n, int k, SelShared<CT>& sh, uint32_t& v,
                            int& above) {
  const int tid = threadIdx.x, w = tid / 32, lane = tid % 32;
  uint32_t prefix = 0, mask = 0;
  int krem = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < (CT / 32) * 256; b += CT) (&sh.hist[0][0])[b] = 0u;
    __syncthreads();
    if constexpr (CT <= 64) {
      // few histograms: lanes with equal digits add once, through their
      // lowest lane (a row's scores share their leading bits, so plain
      // atomics would collide)
      for (int j0 = 0; j0 < n; j0 += CT) {
        const int j = j0 + tid;
        const uint32_t x = j < n ? pb[j] : 0u;
        const bool in = j < n && (x & mask) == prefix;
        const uint32_t dg = in ? (x >> shift) & 255u : 256u;
        const unsigned peers = __match_any_sync(0xffffffffu, dg);
        if (in && (lane == __ffs(peers) - 1)) atomicAdd(&sh.hist[w][dg], static_cast<uint32_t>(__popc(peers)));
      }
    } else {
      for (int j = tid; j < n; j += CT) {
        const uint32_t x = pb[j];
        if ((x & mask) == prefix) atomicAdd(&sh.hist[w][(x >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    for (int b = tid; b < 256; b += CT) {
      uint32_t t = 0;
#pragma unroll
      for (int ww = 0; ww < (CT / 32); ++ww) t += sh.hist[ww][b];
      sh.tot[b] = t;
    }
    __syncthreads();
    if (w == 0) {  // lanes walk bins from the top, 8 each
      uint32_t c[8], local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = sh.tot[255 - 8 * lane - i]; local += c[i]; }
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - local;
      const bool here = excl <= static_cast<uint32_t>(krem) && static_cast<uint32_t>(krem) < incl;
      if (here) {
        uint32_t acc = excl;
        for (int i = 0; i < 8; ++i) {
          if (static_cast<uint32_t>(krem) < acc + c[i]) {
            sh.res_u[0] = 255 - 8 * lane - i;
            sh.res_u[1] = acc;
            break;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    prefix |= sh.res_u[0] << shift;
    mask |= 255u << shift;
    krem -= static_cast<int>(sh.res_u[1]);
    __syncthreads();
  }
  v = prefix;
  above = k - krem;
}

// CDF cut: the score v* of the lowest-ranked kept block and the fixed-point
// mass strictly below v* ("below"), or found = false when the whole row's
// mass stays under thr.
template <int CT>
__device__ void select_mass(const uint32_t* pb, int n, uint64_t thr, SelShared<CT>& sh, uint32_t& v,
                            uint64_t& below, bool& found) {
  const int tid = threadIdx.x, w = tid / 32, lane = tid % 32;
  uint32_t prefix = 0, mask = 0;
  uint64_t blw = 0;
  found = true;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < (CT / 32) * 256; b += CT) (&sh.hsum[0][0])[b] = 0ull;
    __syncthreads();
    for (int j = tid; j < n; j += CT) {
      const uint32_t x = pb[j];
      if ((x & mask) == prefix)
        atomicAdd(&sh.hsum[w][(x >> shift) & 255u], static_cast<unsigned long long>(to_fixed(x)));
    }
    __syncthreads();
    for (int b = tid; b < 256; b += CT) {
      unsigned long long t = 0;
#pragma unroll
      for (int ww = 0; ww < (CT / 32); ++ww) t += sh.hsum[ww][b];
      sh.tots[b] = t;
    }
    __syncthreads();
    if (w == 0) {  // lanes walk bins from the bottom, 8 each
      unsigned long long c[8], local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = sh.tots[8 * lane + i]; local += c[i]; }
      unsigned long long incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned long long excl = incl - local;
      // first bin whose cumulative mass (with everything below) reaches thr
      const bool here = blw + excl < thr && thr <= blw + incl;
      if (lane == 31 && blw + incl < thr) { sh.res_u[0] = 0xFFFFFFFFu; }
      if (here) {
        unsigned long long acc = excl;
        for (int i = 0; i < 8; ++i) {
          if (thr <= blw + acc + c[i]) {
            sh.res_u[0] = 8 * lane + i;
            sh.res_l[0] = acc;
            break;
          }
          acc += c[i];
        }
      }
      if (thr <= blw && lane == 0) {  // already reached (thr = 0): lowest bin
        for (int i = 0; i < 256; ++i) if (sh.tots[i]) { sh.res_u[0] = i; sh.res_l[0] = 0; break; }
      }
    }
    __syncthreads();
    if (sh.res_u[0] == 0xFFFFFFFFu) { found = false; __syncthreads(); return; }
    prefix |= sh.res_u[0] << shift;
    mask |= 255u << shift;
    blw += sh.res_l[0];
    __syncthreads();
  }
  v = prefix;
  below = blw;
}

// Largest pattern strictly below v (0 if none).
template <int CT>
__device__ uint32_t max_below(const uint32_t* pb, int n, uint32_t v, uint32_t* redu) {
  uint32_t m = 0;
  for (int j = threadIdx.x; j < n; j += CT) {
    const uint32_t x = pb[j];
    if (x < v && x > m) m = x;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __syncthreads();
  if (threadIdx.x % 32 == 0) redu[threadIdx.x / 32] = m;
  __syncthreads();
  uint32_t r = 0;
  for (int i = 0; i < CT / 32; ++i) r = max(r, redu[i]);
  return r;
}

// Label pass: in index order, a block is in the top `take` ranks when its
// pattern exceeds v, or equals v and fewer than `fill` lower-indexed blocks
// also equal v.  `lab` gets `val` for those (and keeps larger labels).
template <int CT>
__device__ void label_top(const uint32_t* pb, int n, uint32_t v, int fill, int8_t* lab,
                          int8_t val, int* wsum) {
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  int base = 0;
  for (int j0 = 0; j0 < n; j0 += CT) {
    const int j = j0 + threadIdx.x;
    const uint32_t x = j < n ? pb[j] : 0u;
    const bool eq = j < n && x == v;
    const unsigned be = __ballot_sync(0xffffffffu, eq);
    __syncthreads();
    if (l == 0) wsum[w] = __popc(be);
    __syncthreads();
    int off = base, tot = 0;
    for (int i = 0; i < CT / 32; ++i) {
      if (i < w) off += wsum[i];
      tot += wsum[i];
    }
    const int rank_eq = off + __popc(be & ((1u << l) - 1u));
    if (j < n && (x > v || (eq && rank_eq < fill)) && lab[j] < val) lab[j] = val;
    base += tot;
  }
  __syncthreads();
}

template <int CT>
__global__ void __launch_bounds__(CT) classify_kernel(const float* __restrict__ logits,
                                                       ClassifyArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int nkb = a.nkb, tid = threadIdx.x;
  uint32_t* pb = reinterpret_cast<uint32_t*>(smem);
  int8_t* lab = reinterpret_cast<int8_t*>(pb + nkb);
  __shared__ SelShared<CT> sh;
  __shared__ float redf[32];
  __shared__ int redi[32];
  __shared__ uint32_t redu[32];
  const int row = blockIdx.x;
  const float* lr = logits + i64(row) * nkb;

  // 1. softmax over the row (skipped for rows given as scores)
  float m = 0.f, inv = 1.f;
  if (!a.from_prob) {
    m = -FLT_MAX;
    for (int j = tid; j < nkb; j += CT) m = fmaxf(m, lr[j]);
    m = block_reduce_max<CT>(m, redf);
    float se = 0.f;
    for (int j = tid; j < nkb; j += CT) se += expf(lr[j] - m);
    se = block_reduce_sum<CT>(se, redf);
    inv = 1.0f / se;
  }
  for (int j = tid; j < nkb; j += CT) {
    const float p = a.from_prob ? fmaxf(lr[j], 0.f) : expf(lr[j] - m) * inv;
    if (a.scores) a.scores[i64(row) * nkb + j] = p;
    pb[j] = __float_as_uint(p);
    lab[j] = 0;
  }
  __syncthreads();

  // 2. cuts
  bool tie = false;
  int c = 0;  // critical (kept) count
  if (a.mode == SLA_MASK_TOPK) {
    c = a.n_c;
    if (c > 0) {
      uint32_t v;
      int above;
      select_rank<CT>(pb, nkb, c - 1, sh, v, above);
      label_top<CT>(pb, nkb, v, c - above, lab, 2, redi);
      if (a.tie_count && c < nkb) {  // gap between ranks c-1 and c
        const uint32_t nxt = max_below<CT>(pb, nkb, v, redu);
        // rank c shares v when v's group is not exhausted by the cut
        int eqcount = 0;
        for (int j = tid; j < nkb; j += CT) eqcount += pb[j] == v;
        eqcount = block_reduce_sum_int<CT>(eqcount, redi);
        const float hi = __uint_as_float(v);
        const float lo = (above + eqcount > c) ? hi : __uint_as_float(nxt);
        tie |= (hi - lo) <= kTieEps * hi;
      }
    }
  } else {
    uint32_t v = 0;
    uint64_t below = 0;
    bool found = false;
    if (a.thr_fx > 0) select_mass<CT>(pb, nkb, a.thr_fx, sh, v, below, found);
    if (a.thr_fx == 0) {
      for (int j = tid; j < nkb; j += CT) lab[j] = 2;  // nothing can be dropped
      c = nkb;
      __syncthreads();
    } else {
      uint32_t vk;
      int fill;
      if (found) {
        // group of blocks scoring exactly v: with r = ceil((thr - below) / fx(v))
        // the r lowest-ranked (highest-index) ones are still below thr when
        // taken alone, the other g - r + 1 are kept
        int g = 0;
        for (int j = tid; j < nkb; j += CT) g += pb[j] == v;
        g = block_reduce_sum_int<CT>(g, redi);
        const uint64_t fx = to_fixed(v);
        const uint64_t r = (a.thr_fx - below + fx - 1) / fx;
        vk = v;
        fill = g - static_cast<int>(r) + 1;
      } else {
        // the row's whole mass stays below thr: only the top rank is kept
        uint32_t mx = 0;
        for (int j = tid; j < nkb; j += CT) mx = max(mx, pb[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        __syncthreads();
        if (tid % 32 == 0) redu[tid / 32] = mx;
        __syncthreads();
        mx = 0;
        for (int i = 0; i < CT / 32; ++i) mx = max(mx, redu[i]);
        vk = mx;
        fill = 1;
      }
      label_top<CT>(pb, nkb, vk, fill, lab, 2, redi);
      int above = 0, eqc = 0;
      for (int j = tid; j < nkb; j += CT) { above += pb[j] > vk; eqc += pb[j] == vk; }
      above = block_reduce_sum_int<CT>(above, redi);
      eqc = block_reduce_sum_int<CT>(eqc, redi);
      c = above + fill;
      if (a.tie_count && found) {
        const double thr = static_cast<double>(a.thr_fx) / kFixedOne;
        const uint64_t fx = to_fixed(vk);
        const uint64_t r = static_cast<uint64_t>(eqc - fill + 1);   // kept block's tail count
        const double t_last = static_cast<double>(below + r * fx) / kFixedOne;
        const double t_next = static_cast<double>(below + (r - 1) * fx) / kFixedOne;
        if (c > 1) tie |= fabs(t_last - thr) <= kTieEps;
        if (c < nkb) {
          tie |= fabs(thr - t_next) <= kTieEps;
          const float hi = __uint_as_float(vk);
          const float lo = r >= 2 ? hi : __uint_as_float(max_below<CT>(pb, nkb, vk, redu));
          tie |= (hi - lo) <= kTieEps * hi;
        }
      }
    }
  }
  // marginal: the next n_m ranks after the c critical ones
  const int nm = min(a.n_m, nkb - c);
  if (nm > 0) {
    uint32_t v;
    int above;
    select_rank<CT>(pb, nkb, c + nm - 1, sh, v, above);
    label_top<CT>(pb, nkb, v, c + nm - above, lab, 1, redi);
    if (a.tie_count && c + nm < nkb) {
      const uint32_t nxt = max_below<CT>(pb, nkb, v, redu);
      int eqcount = 0;
      for (int j = tid; j < nkb; j += CT) eqcount += pb[j] == v;
      eqcount = block_reduce_sum_int<CT>(eqcount, redi);
      const float hi = __uint_as_float(v);
      const float lo = (above + eqcount > c + nm) ? hi : __uint_as_float(nxt);
      tie |= (hi - lo) <= kTieEps * hi;
    }
  }
  if (a.tie_count && tid == 0 && tie) atomicAdd(a.tie_count, 1);
  __syncthreads();

  // 3. mask row and lists
  for (int j = tid; j < nkb; j += CT) a.mask[i64(row) * nkb + j] = lab[j];
  const i64 off = i64(row) * nkb;
  compact_row<CT>(lab, nkb, a.rows.crit_idx + off, a.rows.crit_cnt + row,
              a.rows.marg_idx + off, a.rows.marg_cnt + row, redi);
}

// Top-k classifier with one warp per row (rows of up to 32 * VPL blocks):
// the same cuts as classify_kernel with no block-wide barrier.  Lane l holds
// blocks j = l + 32 i (i < VPL) in registers.  The score at rank k is built
// bit by bit from the top (largest pattern t with at least k + 1 scores >= t;
// the count is a warp reduction); equal scores fill the remaining slots in
// index order, and the lists come out of ballots in index order.
template <int VPL>
__global__ void __launch_bounds__(256) classify_topk_warp_kernel(const float* __restrict__ logits,
                                                                   ClassifyArgs a, int nrows) {
  const int row = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (row >= nrows) return;  // whole warps only; no block-wide barrier below
  const unsigned full = 0xffffffffu;
  const int nkb = a.nkb;
  const float* lr = logits + i64(row) * nkb;
  uint32_t pb[VPL];
  // 1. softmax over the row (fixed order: lane-local in i, then a butterfly)
  float x[VPL];
  float m = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    x[i] = j < nkb ? lr[j] : -FLT_MAX;
    m = fmaxf(m, x[i]);
  }
  float inv = 1.f;
  if (!a.from_prob) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(full, m, o));
    float se = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (lane + 32 * i < nkb) se += expf(x[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) se += __shfl_xor_sync(full, se, o);
    inv = 1.0f / se;
  }
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    const float p = a.from_prob ? fmaxf(x[i], 0.f) : expf(x[i] - m) * inv;
    if (a.scores && j < nkb) a.scores[i64(row) * nkb + j] = p;
    pb[i] = j < nkb ? __float_as_uint(p) : 0u;
  }
  auto valid = [&](int i) { return lane + 32 * i < nkb; };
  auto count_eq = [&](uint32_t t) {
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) c += (valid(i) && pb[i] == t) ? 1u : 0u;
    return static_cast<int>(__reduce_add_sync(full, c));
  };
  // largest pattern strictly below t (0 if none)
  auto max_below = [&](uint32_t t) {
    uint32_t mb = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (valid(i) && pb[i] < t && pb[i] > mb) mb = pb[i];
    return __reduce_max_sync(full, mb);
  };
  // patterns at ranks k1 and k2 (0-based from the top), searched side by
  // side so the two chains of warp reductions overlap, and the counts
  // strictly above them (the thresholds are >= 1 and the empty slots hold
  // 0, so empty slots never count)
  auto select_rank2 = [&](int k1, int k2, uint32_t& v1, int& above1, uint32_t& v2, int& above2) {
    uint32_t t1 = 0, t2 = 0;
    for (int bit = 30; bit >= 0; --bit) {  // scores are >= 0: bit 31 is clear
      const uint32_t c1 = t1 | (1u << bit), c2 = t2 | (1u << bit);
      uint32_t n1 = 0, n2 = 0;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        n1 += pb[i] >= c1 ? 1u : 0u;
        n2 += pb[i] >= c2 ? 1u : 0u;
      }
      n1 = __reduce_add_sync(full, n1);
      n2 = __reduce_add_sync(full, n2);
      if (n1 >= static_cast<uint32_t>(k1 + 1)) t1 = c1;
      if (n2 >= static_cast<uint32_t>(k2 + 1)) t2 = c2;
    }
    v1 = t1;
    v2 = t2;
    uint32_t a1 = 0, a2 = 0;  // (t < 2^31, so t + 1 does not wrap)
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      a1 += pb[i] > t1 ? 1u : 0u;
      a2 += pb[i] > t2 ? 1u : 0u;
    }
    above1 = static_cast<int>(__reduce_add_sync(full, a1));
    above2 = static_cast<int>(__reduce_add_sync(full, a2));
  };
  // labels as bit masks over the slots: bit i of crit / kept = block
  // lane + 32 i is critical / critical or marginal
  static_assert(VPL <= 64, "slot masks hold 64 slots");
  uint64_t crit = 0, kept = 0;
  // blocks above v, and the first `fill` blocks equal to v in index order
  auto label_top = [&](uint32_t v, int fill, uint64_t& bits) {
    int base = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const bool eq = valid(i) && pb[i] == v;
      const unsigned be = __ballot_sync(full, eq);
      const int rank_eq = base + __popc(be & ((1u << lane) - 1u));
      if (valid(i) && (pb[i] > v || (eq && rank_eq < fill))) bits |= 1ull << i;
      base += __popc(be);
    }
  };
  bool tie = false;
  const int c = a.n_c;
  const int nm = min(a.n_m, nkb - c);
  // the critical cut at rank c - 1, the marginal one at rank c + nm - 1
  // (an absent cut repeats the other's search)
  uint32_t v_c, v_m;
  int above_c, above_m;
  select_rank2(c > 0 ? c - 1 : c + nm - 1, nm > 0 ? c + nm - 1 : c - 1, v_c, above_c, v_m, above_m);
  if (c > 0) {
    const uint32_t v = v_c;
    const int above = above_c;
    label_top(v, c - above, crit);
    if (a.tie_count && c < nkb) {  // gap between ranks c-1 and c
      const uint32_t nxt = max_below(v);
      const int eqcount = count_eq(v);
      const float hi = __uint_as_float(v);
      const float lo = (above + eqcount > c) ? hi : __uint_as_float(nxt);
      tie |= (hi - lo) <= kTieEps * hi;
    }
  }
  if (nm > 0) {
    const uint32_t v = v_m;
    const int above = above_m;
    label_top(v, c + nm - above, kept);
    if (a.tie_count && c + nm < nkb) {
      const uint32_t nxt = max_below(v);
      const int eqcount = count_eq(v);
      const float hi = __uint_as_float(v);
      const float lo = (above + eqcount > c + nm) ? hi : __uint_as_float(nxt);
      tie |= (hi - lo) <= kTieEps * hi;
    }
  }
  if (a.tie_count && lane == 0 && tie) atomicAdd(a.tie_count, 1);
  // 3. mask row and the ascending lists
  const i64 off = i64(row) * nkb;
  int nc = 0, nmg = 0;
  kept |= crit;  // (the marginal cut ranks below the critical one)
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    const bool is_c = (crit >> i) & 1ull, is_m = !is_c && ((kept >> i) & 1ull);
    if (valid(i)) a.mask[off + j] = static_cast<int8_t>(is_c ? 2 : (is_m ? 1 : 0));
    const unsigned bc = __ballot_sync(full, is_c);
    const unsigned bm = __ballot_sync(full, is_m);
    const unsigned lt = (1u << lane) - 1u;
    if (is_c) a.rows.crit_idx[off + nc + __popc(bc & lt)] = j;
    if (is_m) a.rows.marg_idx[off + nmg + __popc(bm & lt)] = j;
    nc += __popc(bc);
    nmg += __popc(bm);
  }
  if (lane == 0) {
    a.rows.crit_cnt[row] = nc;
    a.rows.marg_cnt[row] = nmg;
  }
}

cudaError_t launch_classify(const float* logits, const Geom& g, int8_t* mask,
                            const sla_block_lists& rows, float* scores,
                            int32_t* tie_count, cudaStream_t s, bool from_prob) {
  ClassifyArgs a;
  a.from_prob = from_prob ? 1 : 0;
  a.nkb = g.nkb;
  a.mode = g.mode;
  a.n_c = g.n_c;
  a.n_m = g.n_m;
  a.thr_fx = g.thr_fx;
  a.mask = mask;
  a.rows = rows;
  a.scores = scores;
  a.tie_count = tie_count;
  const size_t smem = static_cast<size_t>(g.nkb) * 5 + 16;
  cudaError_t e;
  if (tie_count) {
    e = cudaMemsetAsync(tie_count, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  // top-k rows of up to 1024 blocks: one warp per row (measured faster than
  // the CTA kernel there, slower for rows of 1920 blocks); otherwise small
  // CTAs for short rows and for CDF rows of up to 2048 blocks (cheap
  // barriers, many rows per SM), more threads per row for long top-k rows
  // (measured faster at 1920 blocks)
  const int nrows = g.BH * g.nqb;
  if (g.mode == SLA_MASK_TOPK && g.nkb <= 1024) {
    const int grid = (nrows + 7) / 8;
    if (g.nkb <= 512) classify_topk_warp_kernel<16><<<grid, 256, 0, s>>>(logits, a, nrows);
    else classify_topk_warp_kernel<32><<<grid, 256, 0, s>>>(logits, a, nrows);
  } else if (g.nkb <= 1024 || (g.mode == SLA_MASK_CDF && g.nkb <= 2048)) {
    if ((e = cudaFuncSetAttribute(classify_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
      return e;
    classify_kernel<64><<<g.BH * g.nqb, 64, smem, s>>>(logits, a);
  } else {
    if ((e = cudaFuncSetAttribute(classify_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
      return e;
    classify_kernel<256><<<g.BH * g.nqb, 256, smem, s>>>(logits, a);
  }
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
