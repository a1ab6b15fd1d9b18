// Linear attention on marginal blocks and the combine step.
//
// SLA post ("Selective Linear Attention", list "the idea"): intermediate
// (marginal) blocks go through linear attention; the linear branch is the
// auxiliary that preserves accuracy (list "results").  The feature map is
// phi = elu + 1 and the linear output is projected by a d x d matrix W:
//     H_j = sum_{t in j} phi(k_t)^T v_t,   z_j = sum_{t in j} phi(k_t)
//     O_lin[t] = phi(q_t) H^M / (phi(q_t) . z^M),  H^M = sum_{j in M_i} H_j
//     out[t]   = O_s[t] + O_lin[t] W
#include "common.cuh"

namespace sla {

namespace {

// ---------------------------------------------------------------------------
// Summaries: one CTA per (key block, bh); 256 threads as a 16 x 16 grid of
// (D/16) x (D/16) micro-tiles of H_j.  Tokens stream through shared memory in
// chunks of 32; accumulation is sequential over tokens (fixed order).

template <typename T, int D>
__global__ void __launch_bounds__(256) lin_summary_kernel(
    const T* __restrict__ k, const T* __restrict__ v, float* __restrict__ hsum,
    float* __restrict__ zsum, int N, int bk, int nkb) {
  constexpr int MT = D / 16;  // micro-tile edge
  __shared__ __align__(16) float fk[32][D];
  __shared__ __align__(16) float vs[32][D];
  const int j = blockIdx.x, bh = blockIdx.y;
  const int t0 = j * bk, t1 = min(t0 + bk, N);
  const i64 head = i64(bh) * N * D;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[MT][MT] = {};
  float zacc = 0.f;
  for (int c0 = t0; c0 < t1; c0 += 32) {
    __syncthreads();
    for (int x = threadIdx.x * 4; x < 32 * D; x += 256 * 4) {
      const int r = x / D, c = x % D, t = c0 + r;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (t < t1) {
        a = load4(k + head + i64(t) * D + c);
        b = load4(v + head + i64(t) * D + c);
        a = make_float4(phi(a.x), phi(a.y), phi(a.z), phi(a.w));
      }
      *reinterpret_cast<float4*>(&fk[r][c]) = a;
      *reinterpret_cast<float4*>(&vs[r][c]) = b;
    }
    __syncthreads();
    const int n = min(32, t1 - c0);
    for (int u = 0; u < n; ++u) {
      float a[MT], b[MT];
#pragma unroll
      for (int e = 0; e < MT; ++e) { a[e] = fk[u][ty * MT + e]; b[e] = vs[u][tx * MT + e]; }
#pragma unroll
      for (int x = 0; x < MT; ++x)
#pragma unroll
        for (int y = 0; y < MT; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
    }
    if (threadIdx.x < D)
      for (int u = 0; u < n; ++u) zacc += fk[u][threadIdx.x];
  }
  float* hj = hsum + (i64(bh) * nkb + j) * D * D;
#pragma unroll
  for (int x = 0; x < MT; ++x)
#pragma unroll
    for (int y = 0; y < MT; y += 4)
      *reinterpret_cast<float4*>(hj + (ty * MT + x) * D + tx * MT + y) =
          make_float4(acc[x][y], acc[x][y + 1], acc[x][y + 2], acc[x][y + 3]);
  if (threadIdx.x < D) zsum[(i64(bh) * nkb + j) * D + threadIdx.x] = zacc;
}

// ---------------------------------------------------------------------------
// Apply + combine: one CTA per (query block, bh).  Gathers H^M and z^M of the
// row's marginal list into shared memory (fixed list order), then for groups
// of 8 tokens: phi(q), the normaliser, O_lin, and out = O_s + O_lin W.

template <typename T, int D>
__global__ void __launch_bounds__(256) lin_apply_kernel(
    const T* __restrict__ q, const float* __restrict__ hsum,
    const float* __restrict__ zsum, sla_block_lists rows,
    const float* __restrict__ o_s, const float* __restrict__ proj,
    T* __restrict__ out, float* __restrict__ o_lin, int N, int bq, int nqb,
    int nkb) {
  extern __shared__ __align__(16) float sm[];
  float* HM = sm;               // [D][D]
  float* W = HM + D * D;        // [D][D]
  float* zm = W + D * D;        // [D]
  float* F = zm + D;            // [8][D]  phi(q)
  float* OL = F + 8 * D;        // [8][D]  O_lin
  float* den = OL + 8 * D;      // [8]
  const int i = blockIdx.x, bh = blockIdx.y;
  const int list_row = bh * nqb + i;
  // without summaries (linear branch off) marginal entries are ignored
  const int nmarg = hsum ? min(max(rows.marg_cnt[list_row], 0), nkb) : 0;
  const int32_t* marg = rows.marg_idx + i64(list_row) * nkb;
  const i64 head = i64(bh) * N * D;
  const int t0 = i * bq, t1 = min(t0 + bq, N);
  const int tid = threadIdx.x;

  for (int x = tid * 4; x < D * D; x += 256 * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = 0; e < nmarg; ++e) {
      if (marg[e] < 0 || marg[e] >= nkb) continue;  // malformed list entry
      const float4 h = *reinterpret_cast<const float4*>(
          hsum + (i64(bh) * nkb + marg[e]) * D * D + x);
      acc.x += h.x; acc.y += h.y; acc.z += h.z; acc.w += h.w;
    }
    *reinterpret_cast<float4*>(HM + x) = acc;
    *reinterpret_cast<float4*>(W + x) = *reinterpret_cast<const float4*>(proj + x);
  }
  if (tid < D) {
    float acc = 0.f;
    for (int e = 0; e < nmarg; ++e)
      if (marg[e] >= 0 && marg[e] < nkb) acc += zsum[(i64(bh) * nkb + marg[e]) * D + tid];
    zm[tid] = acc;
  }
  __syncthreads();

  const int c = tid % D;            // output channel of this thread
  const int tg = tid / D;           // token sub-lane (256 / D of them)
  constexpr int TL = 256 / D;
  for (int g0 = t0; g0 < t1; g0 += 8) {
    const int ng = min(8, t1 - g0);
    if (nmarg > 0) {
      for (int x = tid; x < 8 * D; x += 256) {
        const int r = x / D, cc = x % D;
        F[x] = r < ng ? phi(to_f32(q[head + i64(g0 + r) * D + cc])) : 0.f;
      }
      __syncthreads();
      {  // normalisers: warp r handles token r
        const int w = tid / 32, lane = tid % 32;
        float s = 0.f;
        for (int a = lane; a < D; a += 32) s += F[w * D + a] * zm[a];
        s = warp_sum(s);
        if (lane == 0) den[w] = s;
      }
      __syncthreads();
      for (int r = tg; r < ng; r += TL) {
        float num = 0.f;
        for (int a = 0; a < D; ++a) num = fmaf(F[r * D + a], HM[a * D + c], num);
        OL[r * D + c] = num / den[r];
      }
    } else {
      for (int x = tid; x < 8 * D; x += 256) OL[x] = 0.f;
    }
    __syncthreads();
    for (int r = tg; r < ng; r += TL) {
      const i64 off = head + i64(g0 + r) * D + c;
      float acc = o_s[off];
      if (nmarg > 0)
        for (int a = 0; a < D; ++a) acc = fmaf(OL[r * D + a], W[a * D + c], acc);
      out[off] = from_f32<T>(acc);
      if (o_lin) o_lin[off] = OL[r * D + c];
    }
    __syncthreads();
  }
}

template <typename T, int D>
cudaError_t summary_t(const void* k, const void* v, const Geom& g, float* hsum,
                      float* zsum, cudaStream_t s) {
  dim3 grid(g.nkb, g.BH);
  lin_summary_kernel<T, D><<<grid, 256, 0, s>>>(
      static_cast<const T*>(k), static_cast<const T*>(v), hsum, zsum, g.N, g.bk,
      g.nkb);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t apply_t(const void* q, const float* hsum, const float* zsum,
                    const sla_block_lists& rows, const float* o_s,
                    const float* proj, void* out, float* o_lin, const Geom& g,
                    cudaStream_t s) {
  const size_t smem = sizeof(float) * (2 * D * D + D + 16 * D + 8);
  auto kern = lin_apply_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(g.nqb, g.BH);
  kern<<<grid, 256, smem, s>>>(static_cast<const T*>(q), hsum, zsum, rows, o_s,
                               proj, static_cast<T*>(out), o_lin, g.N, g.bq,
                               g.nqb, g.nkb);
  return cudaGetLastError();
}

// Linear branch off: out = O_s in the output dtype, o_lin = 0 (8 elements
// per thread, 32-byte fp32 reads).
template <typename T>
__global__ void combine_copy_kernel(const float* __restrict__ o_s, T* __restrict__ out,
                                    float* __restrict__ o_lin, i64 n8) {
  const i64 i = i64(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(o_s)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(o_s)[2 * i + 1];
  store4(out + 8 * i, a);
  store4(out + 8 * i + 4, b);
  if (o_lin) {
    reinterpret_cast<float4*>(o_lin)[2 * i] = make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4*>(o_lin)[2 * i + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

}  // namespace

cudaError_t launch_combine_copy(const float* o_s, void* out, float* o_lin, const Geom& g,
                                cudaStream_t s) {
  const i64 n8 = i64(g.BH) * g.N * g.d / 8;
  const unsigned blocks = static_cast<unsigned>((n8 + 255) / 256);
  if (g.dtype == SLA_BF16)
    combine_copy_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(o_s, static_cast<__nv_bfloat16*>(out), o_lin, n8);
  else
    combine_copy_kernel<float><<<blocks, 256, 0, s>>>(o_s, static_cast<float*>(out), o_lin, n8);
  return cudaGetLastError();
}

cudaError_t launch_lin_summary(const void* k, const void* v, const Geom& g,
                               float* hsum, float* zsum, cudaStream_t s) {
  if (g.dtype == SLA_BF16)
    return g.d == 128 ? summary_t<__nv_bfloat16, 128>(k, v, g, hsum, zsum, s)
                      : summary_t<__nv_bfloat16, 64>(k, v, g, hsum, zsum, s);
  return g.d == 128 ? summary_t<float, 128>(k, v, g, hsum, zsum, s)
                    : summary_t<float, 64>(k, v, g, hsum, zsum, s);
}

cudaError_t launch_lin_apply(const void* q, const float* hsum,
                             const float* zsum, const sla_block_lists& rows,
                             const float* o_s, const float* proj, void* out,
                             float* o_lin, const Geom& g, cudaStream_t s) {
  if (g.dtype == SLA_BF16)
    return g.d == 128 ? apply_t<__nv_bfloat16, 128>(q, hsum, zsum, rows, o_s, proj, out, o_lin, g, s)
                      : apply_t<__nv_bfloat16, 64>(q, hsum, zsum, rows, o_s, proj, out, o_lin, g, s);
  return g.d == 128 ? apply_t<float, 128>(q, hsum, zsum, rows, o_s, proj, out, o_lin, g, s)
                    : apply_t<float, 64>(q, hsum, zsum, rows, o_s, proj, out, o_lin, g, s);
}

}  // namespace sla
