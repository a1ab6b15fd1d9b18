// Backward pass for fine-tuning (SLA post, list "results": a short
// fine-tune suffices).  The block mask is held fixed.  With g = dO W^T:
//   critical part (standard softmax-attention gradients, P recomputed from
//   the saved log-sum-exp):  Delta_t = dO_t . O_s[t],
//     dS = P o (dO V^T - Delta),  dQ = s dS K,  dK = s dS^T Q,  dV = P^T dO
//   linear part, for t in query block i with marginal set M_i:
//     f = phi(q_t), den = f . z^M, num = f H^M,
//     df = H^M (g/den) - z^M (g . num)/den^2,  dq_t += df o phi'(q_t)
//     dH^M_i = sum_t f_t (g_t/den_t)^T,  dz^M_i = -sum_t f_t (g_t . num_t)/den_t^2
//     every key block j in M_i receives dH^M_i, dz^M_i; then for u in j:
//     dk_u += (dH_j v_u + dz_j) o phi'(k_u),  dv_u += dH_j^T phi(k_u)
//   dW = sum over batch, heads and tokens of O_lin[t]^T dO[t].
// All kernels are fp32 SIMT with fixed summation orders (deterministic).
#include <math.h>

#include "common.cuh"

namespace sla {

namespace {

// ---------------------------------------------------------------------------
// Delta_t and g_t = dO_t W^T.  One CTA per (32 tokens, bh).
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(
    const T* __restrict__ dout, const float* __restrict__ o_s,
    const float* __restrict__ proj, float* __restrict__ delta,
    float* __restrict__ gbuf, int N) {
  extern __shared__ __align__(16) float sm[];
  float* Wt = sm;            // [D][D], Wt[c][a] = W[a][c]
  float* dO = Wt + D * D;    // [32][D]
  const int bh = blockIdx.y, t0 = blockIdx.x * 32, tid = threadIdx.x;
  const int t1 = min(t0 + 32, N);
  const i64 head = i64(bh) * N * D;
  for (int x = tid; x < D * D; x += 256) {
    const int a = x / D, c = x % D;
    Wt[c * D + a] = proj[x];
  }
  for (int x = tid; x < 32 * D; x += 256) {
    const int r = x / D, c = x % D;
    dO[x] = (t0 + r < t1) ? to_f32(dout[head + i64(t0 + r) * D + c]) : 0.f;
  }
  __syncthreads();
  const int w = tid / 32, lane = tid % 32;
  for (int r = w; r < t1 - t0; r += 8) {
    float s = 0.f;
    for (int c = lane; c < D; c += 32) s += dO[r * D + c] * o_s[head + i64(t0 + r) * D + c];
    s = warp_sum(s);
    if (lane == 0) delta[i64(bh) * N + t0 + r] = s;
  }
  constexpr int TL = 256 / D;
  const int a = tid % D;
  for (int r = tid / D; r < t1 - t0; r += TL) {
    float s = 0.f;
    for (int c = 0; c < D; ++c) s = fmaf(dO[r * D + c], Wt[c * D + a], s);
    gbuf[head + i64(t0 + r) * D + a] = s;
  }
}

// ---------------------------------------------------------------------------
// dW partials: one CTA per (split, bh) accumulates O_lin^T dO over its token
// range; a second kernel sums the partials in a fixed order.
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_dw_kernel(
    const T* __restrict__ dout, const float* __restrict__ o_lin,
    float* __restrict__ dw_part, int N, int per_split) {
  constexpr int MT = D / 16;
  __shared__ __align__(16) float ol[32][D];
  __shared__ __align__(16) float go[32][D];
  const int sp = blockIdx.x, bh = blockIdx.y;
  const int tb = sp * per_split, te = min(tb + per_split, N);
  const i64 head = i64(bh) * N * D;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[MT][MT] = {};
  for (int c0 = tb; c0 < te; c0 += 32) {
    __syncthreads();
    for (int x = threadIdx.x; x < 32 * D; x += 256) {
      const int r = x / D, c = x % D, t = c0 + r;
      ol[r][c] = t < te ? o_lin[head + i64(t) * D + c] : 0.f;
      go[r][c] = t < te ? to_f32(dout[head + i64(t) * D + c]) : 0.f;
    }
    __syncthreads();
    const int n = min(32, te - c0);
    for (int u = 0; u < n; ++u) {
      float a[MT], b[MT];
#pragma unroll
      for (int e = 0; e < MT; ++e) { a[e] = ol[u][ty * MT + e]; b[e] = go[u][tx * MT + e]; }
#pragma unroll
      for (int x = 0; x < MT; ++x)
#pragma unroll
        for (int y = 0; y < MT; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
    }
  }
  float* dst = dw_part + (i64(bh) * gridDim.x + sp) * D * D;
#pragma unroll
  for (int x = 0; x < MT; ++x)
#pragma unroll
    for (int y = 0; y < MT; ++y) dst[(ty * MT + x) * D + tx * MT + y] = acc[x][y];
}

__global__ void dw_reduce_kernel(const float* __restrict__ part,
                                 float* __restrict__ dproj, int nparts, int dd) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= dd) return;
  float s = 0.f;
  for (int p = 0; p < nparts; ++p) s += part[i64(p) * dd + x];
  dproj[x] = s;
}

// ---------------------------------------------------------------------------
// dQ for the critical part.  Same geometry as the SIMT forward: 64 query
// rows per CTA, 8 rows per warp, keys in chunks of 32 (lane = key).
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ dout, const float* __restrict__ lse,
    const float* __restrict__ delta, sla_block_lists rows,
    float* __restrict__ dq, int N, int bq, int bk, int nqb, int nkb, float scale) {
  constexpr int KP = D + 4, CPL = D / 32, R = 8;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;               // [64][D]
  float* Gs = Qs + 64 * D;      // [64][D]   dO rows
  float* Ks = Gs + 64 * D;      // [32][KP]
  float* Vs = Ks + 32 * KP;     // [32][KP]
  const int halves = bq / 64;
  const int qb = blockIdx.x / halves, half = blockIdx.x % halves, bh = blockIdx.y;
  const int row0 = qb * bq + half * 64;
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const i64 head = i64(bh) * N * D;
  const int list_row = bh * nqb + qb;
  const int ncrit = min(max(rows.crit_cnt[list_row], 0), nkb);
  const int32_t* crit = rows.crit_idx + i64(list_row) * nkb;
  for (int e = threadIdx.x * 4; e < 64 * D; e += 1024) {
    const int r = e / D, c = e % D, t = row0 + r;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (t < N) { a = load4(q + head + i64(t) * D + c); b = load4(dout + head + i64(t) * D + c); }
    *reinterpret_cast<float4*>(Qs + r * D + c) = a;
    *reinterpret_cast<float4*>(Gs + r * D + c) = b;
  }
  float lrow[R], drow[R], acc[R][CPL];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = row0 + w * R + r;
    lrow[r] = t < N ? lse[i64(bh) * N + t] : 0.f;
    drow[r] = t < N ? delta[i64(bh) * N + t] : 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[r][c] = 0.f;
  }
  const float* qw = Qs + w * R * D;
  const float* gw = Gs + w * R * D;
  for (int e = 0; e < ncrit; ++e) {
    if (crit[e] < 0 || crit[e] >= nkb) continue;  // malformed list entry
    const int k0 = crit[e] * bk, k1 = min(k0 + bk, N);
    for (int c0 = k0; c0 < k1; c0 += 32) {
      __syncthreads();
      for (int x = threadIdx.x * 4; x < 32 * D; x += 1024) {
        const int r = x / D, c = x % D, t = c0 + r;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (t < k1) { a = load4(k + head + i64(t) * D + c); b = load4(v + head + i64(t) * D + c); }
        *reinterpret_cast<float4*>(Ks + r * KP + c) = a;
        *reinterpret_cast<float4*>(Vs + r * KP + c) = b;
      }
      __syncthreads();
      const bool valid = c0 + lane < k1;
      float s[R], dp[R];
#pragma unroll
      for (int r = 0; r < R; ++r) { s[r] = 0.f; dp[r] = 0.f; }
      for (int c = 0; c < D; c += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(Ks + lane * KP + c);
        const float4 vv = *reinterpret_cast<const float4*>(Vs + lane * KP + c);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float4 a = *reinterpret_cast<const float4*>(qw + r * D + c);
          const float4 b = *reinterpret_cast<const float4*>(gw + r * D + c);
          s[r] = fmaf(a.x, kv.x, fmaf(a.y, kv.y, fmaf(a.z, kv.z, fmaf(a.w, kv.w, s[r]))));
          dp[r] = fmaf(b.x, vv.x, fmaf(b.y, vv.y, fmaf(b.z, vv.z, fmaf(b.w, vv.w, dp[r]))));
        }
      }
      float ds[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float p = valid ? expf(s[r] * scale - lrow[r]) : 0.f;
        ds[r] = p * (dp[r] - drow[r]);
      }
      for (int kk = 0; kk < 32; ++kk) {
        float kv[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) kv[c] = Ks[kk * KP + lane + 32 * c];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float d = __shfl_sync(0xffffffffu, ds[r], kk);
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[r][c] = fmaf(d, kv[c], acc[r][c]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = row0 + w * R + r;
    if (t >= N) continue;
#pragma unroll
    for (int c = 0; c < CPL; ++c) dq[head + i64(t) * D + lane + 32 * c] = scale * acc[r][c];
  }
}

// ---------------------------------------------------------------------------
// dK, dV for the critical part: one CTA per (64 keys of a key block, bh),
// 8 keys per warp; the query blocks holding this key block critically (CSC
// list) stream through shared memory in chunks of 32 rows (lane = row).
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_bwd_dkdv_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ dout, const float* __restrict__ lse,
    const float* __restrict__ delta, sla_block_lists cols,
    float* __restrict__ dk, float* __restrict__ dv, int N, int bq, int bk,
    int nqb, int nkb, float scale) {
  constexpr int QP = D + 4, CPL = D / 32, R = 8;
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;               // [64][D]
  float* Vs = Ks + 64 * D;      // [64][D]
  float* Qc = Vs + 64 * D;      // [32][QP]
  float* Gc = Qc + 32 * QP;     // [32][QP]
  __shared__ float Lc[32], Dc[32];
  const int halves = bk / 64;
  const int kb = blockIdx.x / halves, half = blockIdx.x % halves, bh = blockIdx.y;
  const int key0 = kb * bk + half * 64;
  const int kend = min((kb + 1) * bk, N);
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const i64 head = i64(bh) * N * D;
  const int col = bh * nkb + kb;
  const int nq = min(max(cols.crit_cnt[col], 0), nqb);
  const int32_t* qlist = cols.crit_idx + i64(col) * nqb;
  for (int e = threadIdx.x * 4; e < 64 * D; e += 1024) {
    const int r = e / D, c = e % D, t = key0 + r;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (t < kend) { a = load4(k + head + i64(t) * D + c); b = load4(v + head + i64(t) * D + c); }
    *reinterpret_cast<float4*>(Ks + r * D + c) = a;
    *reinterpret_cast<float4*>(Vs + r * D + c) = b;
  }
  float ak[R][CPL], av[R][CPL];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int c = 0; c < CPL; ++c) { ak[r][c] = 0.f; av[r][c] = 0.f; }
  const float* kw = Ks + w * R * D;
  const float* vw = Vs + w * R * D;
  for (int e = 0; e < nq; ++e) {
    if (qlist[e] < 0 || qlist[e] >= nqb) continue;  // malformed list entry
    const int q0 = qlist[e] * bq, q1 = min(q0 + bq, N);
    for (int c0 = q0; c0 < q1; c0 += 32) {
      __syncthreads();
      for (int x = threadIdx.x * 4; x < 32 * D; x += 1024) {
        const int r = x / D, c = x % D, t = c0 + r;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (t < q1) { a = load4(q + head + i64(t) * D + c); b = load4(dout + head + i64(t) * D + c); }
        *reinterpret_cast<float4*>(Qc + r * QP + c) = a;
        *reinterpret_cast<float4*>(Gc + r * QP + c) = b;
      }
      if (threadIdx.x < 32) {
        const int t = c0 + threadIdx.x;
        Lc[threadIdx.x] = t < q1 ? lse[i64(bh) * N + t] : 0.f;
        Dc[threadIdx.x] = t < q1 ? delta[i64(bh) * N + t] : 0.f;
      }
      __syncthreads();
      const bool valid = c0 + lane < q1;
      float s[R], dp[R];
#pragma unroll
      for (int r = 0; r < R; ++r) { s[r] = 0.f; dp[r] = 0.f; }
      for (int c = 0; c < D; c += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(Qc + lane * QP + c);
        const float4 gv = *reinterpret_cast<const float4*>(Gc + lane * QP + c);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float4 a = *reinterpret_cast<const float4*>(kw + r * D + c);
          const float4 b = *reinterpret_cast<const float4*>(vw + r * D + c);
          s[r] = fmaf(a.x, qv.x, fmaf(a.y, qv.y, fmaf(a.z, qv.z, fmaf(a.w, qv.w, s[r]))));
          dp[r] = fmaf(b.x, gv.x, fmaf(b.y, gv.y, fmaf(b.z, gv.z, fmaf(b.w, gv.w, dp[r]))));
        }
      }
      float p[R], ds[R];
      const float lt = Lc[lane], dt = Dc[lane];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const bool kvalid = key0 + w * R + r < kend;
        p[r] = (valid && kvalid) ? expf(s[r] * scale - lt) : 0.f;
        ds[r] = p[r] * (dp[r] - dt);
      }
      for (int tt = 0; tt < 32; ++tt) {
        float qv[CPL], gv[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) { qv[c] = Qc[tt * QP + lane + 32 * c]; gv[c] = Gc[tt * QP + lane + 32 * c]; }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float pp = __shfl_sync(0xffffffffu, p[r], tt);
          const float dd = __shfl_sync(0xffffffffu, ds[r], tt);
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            av[r][c] = fmaf(pp, gv[c], av[r][c]);
            ak[r][c] = fmaf(dd, qv[c], ak[r][c]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = key0 + w * R + r;
    if (t >= kend) continue;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      dk[head + i64(t) * D + lane + 32 * c] = scale * ak[r][c];
      dv[head + i64(t) * D + lane + 32 * c] = av[r][c];
    }
  }
}

// ---------------------------------------------------------------------------
// Linear part, query side: one CTA per (query block, bh) with a non-empty
// marginal list.  Adds df o phi'(q) into dq and writes dH^M_i, dz^M_i.
template <typename T, int D>
__global__ void __launch_bounds__(256) lin_bwd_q_kernel(
    const T* __restrict__ q, const float* __restrict__ hsum,
    const float* __restrict__ zsum, sla_block_lists rows,
    const float* __restrict__ gbuf, float* __restrict__ dq,
    float* __restrict__ dhm, float* __restrict__ dzm, int N, int bq, int nqb,
    int nkb) {
  constexpr int MT = D / 16;
  extern __shared__ __align__(16) float sm[];
  float* HM = sm;              // [D][D]
  float* zm = HM + D * D;      // [D]
  float* F = zm + D;           // [8][D]  phi(q)
  float* DN = F + 8 * D;       // [8][D]  g / den
  float* Gt = DN + 8 * D;      // [8][D]  g
  float* Q = Gt + 8 * D;       // [8][D]  q
  float* sc = Q + 8 * D;       // [8] den, [8] dden
  const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int list_row = bh * nqb + i;
  const int nmarg = min(max(rows.marg_cnt[list_row], 0), nkb);
  if (nmarg == 0) return;
  const int32_t* marg = rows.marg_idx + i64(list_row) * nkb;
  const i64 head = i64(bh) * N * D;
  const int t0 = i * bq, t1 = min(t0 + bq, N);
  for (int x = tid * 4; x < D * D; x += 1024) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = 0; e < nmarg; ++e) {
      if (marg[e] < 0 || marg[e] >= nkb) continue;
      const float4 h = *reinterpret_cast<const float4*>(hsum + (i64(bh) * nkb + marg[e]) * D * D + x);
      acc.x += h.x; acc.y += h.y; acc.z += h.z; acc.w += h.w;
    }
    *reinterpret_cast<float4*>(HM + x) = acc;
  }
  if (tid < D) {
    float acc = 0.f;
    for (int e = 0; e < nmarg; ++e)
      if (marg[e] >= 0 && marg[e] < nkb) acc += zsum[(i64(bh) * nkb + marg[e]) * D + tid];
    zm[tid] = acc;
  }
  __syncthreads();
  const int tx = tid % 16, ty = tid / 16;
  float ah[MT][MT] = {};
  float az = 0.f;
  const int w = tid / 32, lane = tid % 32;
  for (int g0 = t0; g0 < t1; g0 += 8) {
    const int ng = min(8, t1 - g0);
    for (int x = tid; x < 8 * D; x += 256) {
      const int r = x / D, c = x % D;
      const float qq = r < ng ? to_f32(q[head + i64(g0 + r) * D + c]) : 0.f;
      Q[x] = qq;
      F[x] = r < ng ? phi(qq) : 0.f;
      Gt[x] = r < ng ? gbuf[head + i64(g0 + r) * D + c] : 0.f;
    }
    __syncthreads();
    {  // warp r: den_r = f . z^M and (g . num)_r
      float sd = 0.f;
      for (int a = lane; a < D; a += 32) sd += F[w * D + a] * zm[a];
      sd = warp_sum(sd);
      float sg = 0.f;
      for (int c = lane; c < D; c += 32) {
        float num = 0.f;
        for (int a = 0; a < D; ++a) num = fmaf(F[w * D + a], HM[a * D + c], num);
        sg += Gt[w * D + c] * num;
      }
      sg = warp_sum(sg);
      if (lane == 0) { sc[w] = sd; sc[8 + w] = w < ng ? -sg / (sd * sd) : 0.f; }
    }
    __syncthreads();
    for (int x = tid; x < 8 * D; x += 256) {
      const int r = x / D;
      DN[x] = r < ng ? Gt[x] / sc[r] : 0.f;
    }
    __syncthreads();
    // df[a] = sum_c HM[a][c] DN[c] + zm[a] dden ; dq += df * phi'(q)
    for (int x = tid; x < ng * D; x += 256) {
      const int r = x / D, a = x % D;
      float s = 0.f;
      for (int c = 0; c < D; ++c) s = fmaf(HM[a * D + c], DN[r * D + c], s);
      s += zm[a] * sc[8 + r];
      dq[head + i64(g0 + r) * D + a] += s * dphi(Q[x]);
    }
    // dH^M += F^T DN, dz^M += F^T dden
    for (int u = 0; u < ng; ++u) {
      float a[MT], b[MT];
#pragma unroll
      for (int e = 0; e < MT; ++e) { a[e] = F[u * D + ty * MT + e]; b[e] = DN[u * D + tx * MT + e]; }
#pragma unroll
      for (int x = 0; x < MT; ++x)
#pragma unroll
        for (int y = 0; y < MT; ++y) ah[x][y] = fmaf(a[x], b[y], ah[x][y]);
    }
    if (tid < D)
      for (int u = 0; u < ng; ++u) az = fmaf(F[u * D + tid], sc[8 + u], az);
    __syncthreads();
  }
  float* dst = dhm + (i64(bh) * nqb + i) * D * D;
#pragma unroll
  for (int x = 0; x < MT; ++x)
#pragma unroll
    for (int y = 0; y < MT; ++y) dst[(ty * MT + x) * D + tx * MT + y] = ah[x][y];
  if (tid < D) dzm[(i64(bh) * nqb + i) * D + tid] = az;
}

// ---------------------------------------------------------------------------
// Linear part, key side: one CTA per (key block, bh) with a non-empty CSC
// marginal list.  dH_j = sum of dH^M_i over the query blocks i holding j.
template <typename T, int D>
__global__ void __launch_bounds__(256) lin_bwd_kv_kernel(
    const T* __restrict__ k, const T* __restrict__ v,
    const float* __restrict__ dhm, const float* __restrict__ dzm,
    sla_block_lists cols, float* __restrict__ dk, float* __restrict__ dv, int N,
    int bk, int nqb, int nkb) {
  extern __shared__ __align__(16) float sm[];
  float* DH = sm;              // [D][D]
  float* dz = DH + D * D;      // [D]
  float* Kt = dz + D;          // [8][D]
  float* Vt = Kt + 8 * D;      // [8][D]
  const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int col = bh * nkb + j;
  const int nq = min(max(cols.marg_cnt[col], 0), nqb);
  if (nq == 0) return;
  const int32_t* qlist = cols.marg_idx + i64(col) * nqb;
  const i64 head = i64(bh) * N * D;
  for (int x = tid * 4; x < D * D; x += 1024) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = 0; e < nq; ++e) {
      if (qlist[e] < 0 || qlist[e] >= nqb) continue;
      const float4 h = *reinterpret_cast<const float4*>(dhm + (i64(bh) * nqb + qlist[e]) * D * D + x);
      acc.x += h.x; acc.y += h.y; acc.z += h.z; acc.w += h.w;
    }
    *reinterpret_cast<float4*>(DH + x) = acc;
  }
  if (tid < D) {
    float acc = 0.f;
    for (int e = 0; e < nq; ++e)
      if (qlist[e] >= 0 && qlist[e] < nqb) acc += dzm[(i64(bh) * nqb + qlist[e]) * D + tid];
    dz[tid] = acc;
  }
  const int t0 = j * bk, t1 = min(t0 + bk, N);
  for (int g0 = t0; g0 < t1; g0 += 8) {
    const int ng = min(8, t1 - g0);
    __syncthreads();
    for (int x = tid; x < 8 * D; x += 256) {
      const int r = x / D, c = x % D;
      Kt[x] = r < ng ? to_f32(k[head + i64(g0 + r) * D + c]) : 0.f;
      Vt[x] = r < ng ? to_f32(v[head + i64(g0 + r) * D + c]) : 0.f;
    }
    __syncthreads();
    for (int x = tid; x < ng * D; x += 256) {
      const int r = x / D, a = x % D;
      // dphi(k)[a] = sum_c DH[a][c] v[c] + dz[a]
      float s = dz[a];
      for (int c = 0; c < D; ++c) s = fmaf(DH[a * D + c], Vt[r * D + c], s);
      const float kk = Kt[r * D + a];
      dk[head + i64(g0 + r) * D + a] += s * dphi(kk);
      // dv[c=a] = sum_a' phi(k)[a'] DH[a'][a]
      float sv = 0.f;
      for (int b = 0; b < D; ++b) sv = fmaf(phi(Kt[r * D + b]), DH[b * D + a], sv);
      dv[head + i64(g0 + r) * D + a] += sv;
    }
  }
}

template <typename T, int D>
struct Bwd {
  static cudaError_t prep(const void* dout, const float* o_s, const float* o_lin,
                          const float* proj, float* delta, float* gbuf,
                          float* dw_part, const Geom& g, cudaStream_t s) {
    const size_t smem = sizeof(float) * (D * D + 32 * D);
    cudaError_t e = cudaFuncSetAttribute(bwd_prep_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    bwd_prep_kernel<T, D><<<dim3((g.N + 31) / 32, g.BH), 256, smem, s>>>(
        static_cast<const T*>(dout), o_s, proj, delta, gbuf, g.N);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int nsplit = dw_splits(g);
    const int per = (g.N + nsplit - 1) / nsplit;
    bwd_dw_kernel<T, D><<<dim3(nsplit, g.BH), 256, 0, s>>>(
        static_cast<const T*>(dout), o_lin, dw_part, g.N, per);
    return cudaGetLastError();
  }
  static int dw_splits(const Geom& g) { return g.N >= 4096 ? 16 : 1; }
};

}  // namespace

int bwd_dw_parts(const Geom& g) { return g.BH * (g.N >= 4096 ? 16 : 1); }

cudaError_t launch_bwd_prep(const void* dout, const float* o_s,
                            const float* o_lin, const float* proj,
                            float* delta, float* gbuf, float* dw_part,
                            const Geom& g, cudaStream_t s) {
  if (g.dtype == SLA_BF16)
    return g.d == 128 ? Bwd<__nv_bfloat16, 128>::prep(dout, o_s, o_lin, proj, delta, gbuf, dw_part, g, s)
                      : Bwd<__nv_bfloat16, 64>::prep(dout, o_s, o_lin, proj, delta, gbuf, dw_part, g, s);
  return g.d == 128 ? Bwd<float, 128>::prep(dout, o_s, o_lin, proj, delta, gbuf, dw_part, g, s)
                    : Bwd<float, 64>::prep(dout, o_s, o_lin, proj, delta, gbuf, dw_part, g, s);
}

cudaError_t launch_bwd_dw_reduce(const float* dw_part, float* dproj,
                                 const Geom& g, cudaStream_t s) {
  const int dd = g.d * g.d;
  dw_reduce_kernel<<<(dd + 255) / 256, 256, 0, s>>>(dw_part, dproj, bwd_dw_parts(g), dd);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t dq_t(const void* q, const void* k, const void* v, const void* dout,
                        const float* lse, const float* delta,
                        const sla_block_lists& rows, float* dq, const Geom& g,
                        cudaStream_t s) {
  const size_t smem = sizeof(float) * (2 * 64 * D + 2 * 32 * (D + 4));
  auto kern = attn_bwd_dq_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(g.nqb * (g.bq / 64), g.BH), 256, smem, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(dout), lse, delta, rows, dq, g.N, g.bq, g.bk, g.nqb,
      g.nkb, g.scale);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_dq(const void* q, const void* k, const void* v,
                               const void* dout, const float* lse,
                               const float* delta, const sla_block_lists& rows,
                               float* dq, const Geom& g, cudaStream_t s) {
  if (g.dtype == SLA_BF16)
    return g.d == 128 ? dq_t<__nv_bfloat16, 128>(q, k, v, dout, lse, delta, rows, dq, g, s)
                      : dq_t<__nv_bfloat16, 64>(q, k, v, dout, lse, delta, rows, dq, g, s);
  return g.d == 128 ? dq_t<float, 128>(q, k, v, dout, lse, delta, rows, dq, g, s)
                    : dq_t<float, 64>(q, k, v, dout, lse, delta, rows, dq, g, s);
}

template <typename T, int D>
static cudaError_t dkdv_t(const void* q, const void* k, const void* v, const void* dout,
                          const float* lse, const float* delta,
                          const sla_block_lists& cols, float* dk, float* dv,
                          const Geom& g, cudaStream_t s) {
  const size_t smem = sizeof(float) * (2 * 64 * D + 2 * 32 * (D + 4));
  auto kern = attn_bwd_dkdv_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(g.nkb * (g.bk / 64), g.BH), 256, smem, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(dout), lse, delta, cols, dk, dv, g.N, g.bq, g.bk,
      g.nqb, g.nkb, g.scale);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_dkdv(const void* q, const void* k, const void* v,
                                 const void* dout, const float* lse,
                                 const float* delta,
                                 const sla_block_lists& cols, float* dk,
                                 float* dv, const Geom& g, cudaStream_t s) {
  if (g.dtype == SLA_BF16)
    return g.d == 128 ? dkdv_t<__nv_bfloat16, 128>(q, k, v, dout, lse, delta, cols, dk, dv, g, s)
                      : dkdv_t<__nv_bfloat16, 64>(q, k, v, dout, lse, delta, cols, dk, dv, g, s);
  return g.d == 128 ? dkdv_t<float, 128>(q, k, v, dout, lse, delta, cols, dk, dv, g, s)
                    : dkdv_t<float, 64>(q, k, v, dout, lse, delta, cols, dk, dv, g, s);
}

template <typename T, int D>
static cudaError_t lbq_t(const void* q, const float* hsum, const float* zsum,
                         const sla_block_lists& rows, const float* gbuf,
                         float* dq, float* dhm, float* dzm, const Geom& g,
                         cudaStream_t s) {
  const size_t smem = sizeof(float) * (D * D + D + 32 * D + 16);
  auto kern = lin_bwd_q_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(g.nqb, g.BH), 256, smem, s>>>(static_cast<const T*>(q), hsum, zsum,
                                             rows, gbuf, dq, dhm, dzm, g.N, g.bq,
                                             g.nqb, g.nkb);
  return cudaGetLastError();
}

cudaError_t launch_lin_bwd_q(const void* q, const float* hsum,
                             const float* zsum, const sla_block_lists& rows,
                             const float* gbuf, const float* o_lin, float* dq,
                             float* dhm, float* dzm, const Geom& g,
                             cudaStream_t s) {
  (void)o_lin;
  if (g.dtype == SLA_BF16)
    return g.d == 128 ? lbq_t<__nv_bfloat16, 128>(q, hsum, zsum, rows, gbuf, dq, dhm, dzm, g, s)
                      : lbq_t<__nv_bfloat16, 64>(q, hsum, zsum, rows, gbuf, dq, dhm, dzm, g, s);
  return g.d == 128 ? lbq_t<float, 128>(q, hsum, zsum, rows, gbuf, dq, dhm, dzm, g, s)
                    : lbq_t<float, 64>(q, hsum, zsum, rows, gbuf, dq, dhm, dzm, g, s);
}

template <typename T, int D>
static cudaError_t lbkv_t(const void* k, const void* v, const float* dhm,
                          const float* dzm, const sla_block_lists& cols,
                          float* dk, float* dv, const Geom& g, cudaStream_t s) {
  const size_t smem = sizeof(float) * (D * D + D + 16 * D);
  auto kern = lin_bwd_kv_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(g.nkb, g.BH), 256, smem, s>>>(static_cast<const T*>(k),
                                             static_cast<const T*>(v), dhm, dzm,
                                             cols, dk, dv, g.N, g.bk, g.nqb, g.nkb);
  return cudaGetLastError();
}

cudaError_t launch_lin_bwd_kv(const void* k, const void* v, const float* dhm,
                              const float* dzm, const sla_block_lists& cols,
                              float* dk, float* dv, const Geom& g,
                              cudaStream_t s) {
  if (g.dtype == SLA_BF16)
    return g.d == 128 ? lbkv_t<__nv_bfloat16, 128>(k, v, dhm, dzm, cols, dk, dv, g, s)
                      : lbkv_t<__nv_bfloat16, 64>(k, v, dhm, dzm, cols, dk, dv, g, s);
  return g.d == 128 ? lbkv_t<float, 128>(k, v, dhm, dzm, cols, dk, dv, g, s)
                    : lbkv_t<float, 64>(k, v, dhm, dzm, cols, dk, dv, g, s);
}

}  // namespace sla
