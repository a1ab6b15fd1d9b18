// Exact softmax attention restricted to each query block's critical key
// blocks, in fp32 FMA (SIMT).  This is the fp32-mode kernel (accuracy 1e-4
// needs fp32 arithmetic throughout) and the portable path for bf16 inputs.
//
// SLA post ("Selective Linear Attention", list "the idea"): critical blocks go
// through FlashAttention, i.e. exact online-softmax attention; negligible
// blocks are skipped.  NABLA post point 4: compute only the kept blocks.
//
// CTA: 64 query rows of one query block (grid.x = Nqb * Bq/64, grid.y = B*H),
// 8 warps x 8 rows.  Keys stream through shared memory in chunks of 32; lane
// l scores key l of the chunk against the warp's 8 rows, then the online
// softmax update and P @ V run with each lane owning d/32 output channels.
#include <math.h>

#include "common.cuh"

namespace sla {

namespace {

constexpr int kRowsPerCta = 64;
constexpr int kRowsPerWarp = 8;
constexpr int kChunk = 32;

template <typename T, int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    sla_block_lists rows, float* __restrict__ o_s, float* __restrict__ lse,
    int N, int bq, int bk, int nqb, int nkb, float scale) {
  constexpr int KP = D + 4;  // padded key row (float4-aligned, conflict-free)
  constexpr int CPL = D / 32;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;                        // [64][D]
  float* Ks = Qs + kRowsPerCta * D;      // [32][KP]
  float* Vs = Ks + kChunk * KP;          // [32][D]

  const int halves = bq / kRowsPerCta;
  const int qb = blockIdx.x / halves, half = blockIdx.x % halves;
  const int bh = blockIdx.y;
  const int row0 = qb * bq + half * kRowsPerCta;
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const i64 head = i64(bh) * N * D;
  const int list_row = bh * nqb + qb;
  const int ncrit = min(max(rows.crit_cnt[list_row], 0), nkb);
  const int32_t* crit = rows.crit_idx + i64(list_row) * nkb;

  // stage the CTA's query rows (zero beyond N)
  for (int e = threadIdx.x * 4; e < kRowsPerCta * D; e += 256 * 4) {
    const int r = e / D, c = e % D, t = row0 + r;
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < N) f = load4(q + head + i64(t) * D + c);
    *reinterpret_cast<float4*>(Qs + r * D + c) = f;
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][CPL];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[r][c] = 0.f;
  }
  const float* qw = Qs + (w * kRowsPerWarp) * D;

  for (int e = 0; e < ncrit; ++e) {
    const int kb = crit[e];
    if (kb < 0 || kb >= nkb) continue;  // malformed list entry: skip
    const int k0 = kb * bk, k1 = min(k0 + bk, N);
    for (int c0 = k0; c0 < k1; c0 += kChunk) {
      __syncthreads();
      for (int x = threadIdx.x * 4; x < kChunk * D; x += 256 * 4) {
        const int r = x / D, c = x % D, t = c0 + r;
        float4 fk = make_float4(0.f, 0.f, 0.f, 0.f), fv = fk;
        if (t < k1) {
          fk = load4(k + head + i64(t) * D + c);
          fv = load4(v + head + i64(t) * D + c);
        }
        *reinterpret_cast<float4*>(Ks + r * KP + c) = fk;
        *reinterpret_cast<float4*>(Vs + r * D + c) = fv;
      }
      __syncthreads();
      const bool valid = c0 + lane < k1;
      float s[kRowsPerWarp];
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) s[r] = 0.f;
      const float* kr = Ks + lane * KP;
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(kr + c);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const float4 qv = *reinterpret_cast<const float4*>(qw + r * D + c);
          s[r] = fmaf(qv.x, kv.x, s[r]);
          s[r] = fmaf(qv.y, kv.y, s[r]);
          s[r] = fmaf(qv.z, kv.z, s[r]);
          s[r] = fmaf(qv.w, kv.w, s[r]);
        }
      }
      float p[kRowsPerWarp];
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        const float x = valid ? s[r] * scale : -INFINITY;
        const float mn = fmaxf(m[r], warp_max(x));
        const float corr = expf(m[r] - mn);  // m = -inf first: corr = 0
        p[r] = valid ? expf(x - mn) : 0.f;
        l[r] = l[r] * corr + warp_sum(p[r]);
        m[r] = mn;
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[r][c] *= corr;
      }
#pragma unroll 4
      for (int kk = 0; kk < kChunk; ++kk) {
        float vv[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) vv[c] = Vs[kk * D + lane + 32 * c];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const float pk = __shfl_sync(0xffffffffu, p[r], kk);
#pragma unroll
          for (int c = 0; c < CPL; ++c) o[r][c] = fmaf(pk, vv[c], o[r][c]);
        }
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int t = row0 + w * kRowsPerWarp + r;
    if (t >= N || t >= (qb + 1) * bq) continue;
    const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c)
      o_s[head + i64(t) * D + lane + 32 * c] = o[r][c] * inv;
    if (lane == 0) lse[i64(bh) * N + t] = l[r] > 0.f ? m[r] + logf(l[r]) : -INFINITY;
  }
}

template <typename T, int D>
cudaError_t launch_simt_t(const void* q, const void* k, const void* v,
                          const Geom& g, const sla_block_lists& rows,
                          float* o_s, float* lse, cudaStream_t s) {
  const size_t smem =
      sizeof(float) * (kRowsPerCta * D + kChunk * (D + 4) + kChunk * D);
  auto kern = attn_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(g.nqb * (g.bq / kRowsPerCta), g.BH);
  kern<<<grid, 256, smem, s>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                               static_cast<const T*>(v), rows, o_s, lse, g.N,
                               g.bq, g.bk, g.nqb, g.nkb, g.scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const void* q, const void* k, const void* v,
                             const Geom& g, const sla_block_lists& rows,
                             float* o_s, float* lse, cudaStream_t s) {
  if (g.dtype == SLA_BF16) {
    return g.d == 128 ? launch_simt_t<__nv_bfloat16, 128>(q, k, v, g, rows, o_s, lse, s)
                      : launch_simt_t<__nv_bfloat16, 64>(q, k, v, g, rows, o_s, lse, s);
  }
  return g.d == 128 ? launch_simt_t<float, 128>(q, k, v, g, rows, o_s, lse, s)
                    : launch_simt_t<float, 64>(q, k, v, g, rows, o_s, lse, s);
}

}  // namespace sla
