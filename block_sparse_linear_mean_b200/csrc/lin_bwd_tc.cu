// Backward of the linear (marginal) branch and of the output projection on
// the tensor cores (bf16 operands, fp32 accumulation, d = 128), plus the
// per-row Delta of the softmax backward.
//
// The SLA post ("fine-tuning") adapts a model with the hybrid attention in
// place; the marginal branch is linear attention with phi = elu + 1 and the
// output projection W (out = O_s + O_lin W).  For a token t of query block i
// with marginal set M_i, f = phi(q_t), den = f . z^M_i, o = f H^M_i / den and
// g = dO_t W^T (the gradient reaching o):
//   dnum = g / den,  dden = -(g . o) / den
//   dq_t  += (dnum H^M_i^T + dden z^M_i) o phi'(q_t)
//   dH^M_i = sum_t f^T dnum,  dz^M_i = sum_t f dden
// every key block j in M_i receives dH^M_i and dz^M_i (dH_j, dz_j), and for
// a token u of block j:
//   dk_u += (v_u dH_j^T + dz_j) o phi'(k_u),  dv_u += phi(k_u) dH_j
//   dW = sum over all tokens of O_lin^T dO.
// The gather dH_j = sum_{i : j in M_i} dH^M_i is the forward's indicator
// GEMM with the column lists.  phi(Q), phi(K) are rounded to bf16 exactly as
// in the forward, so the backward differentiates the forward's own
// arithmetic; g, dnum, dH^M and dH go through bf16 once as MMA operands.
//
// Kernels here (all waits bounded; timeouts set the status word):
//   delta_kernel   Delta_t = dO_t . O_s[t]                (HBM-bound)
//   dw_tc_kernel   dW partials, persistent over 128-token tiles
// The query side (g, dnum, dq, dH^M, dz^M) runs in the epilogue of the
// critical branch's dq kernel and the key side (dk, dv) in the epilogue of
// its dkdv kernel (attn_bwd_tc.cu), where the operands already sit on chip;
// between the two, the indicator GEMM over the column lists sums dH^M, dz^M
// into dH_j, dz_j.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace sla {

namespace {

constexpr long long kLbTimeout = 1ll << 31;
constexpr int kLD = 128;             // channels
constexpr int kLHElems = kLD * kLD;  // one d x d matrix

__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// ---------------------------------------------------------------------------
// Delta_t = dO_t . O_s[t] for every row (B*H*N rows of d channels): one warp
// per row, fixed summation order.
template <typename T>
__global__ void __launch_bounds__(256) delta_kernel(const T* __restrict__ dout,
                                                    const float* __restrict__ o_s,
                                                    float* __restrict__ delta, i64 rows, int d) {
  const i64 row = static_cast<i64>(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  float s = 0.f;
  for (int c = lane * 4; c < d; c += 128) {
    const float4 a = load4(dout + row * d + c);
    const float4 b = load4(o_s + row * d + c);
    s += a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
  }
  s = warp_sum(s);
  if (lane == 0) delta[row] = s;
}

// ---------------------------------------------------------------------------
// dW partials: dW = sum_t O_lin[t]^T dO[t] over all B*H*N rows, as one MMA
// chain per CTA (M = 128 channels a of O_lin, N = 128 channels c of dO,
// K = tokens; both operands MN-major).  CTA p takes 128-row tiles p, p + P,
// ...; O_lin is converted to bf16 into shared memory by all threads while
// the previous tile's MMAs run (two stages).  Partial p -> part[p] (fp32).
constexpr uint32_t kDwStage = 65536;  // dO tile + O_lin tile (bf16)

__global__ void __launch_bounds__(128, 1) dw_tc_kernel(const __grid_constant__ CUtensorMap tmdO,
                                                       const float* __restrict__ o_lin,
                                                       float* __restrict__ part, i64 rows,
                                                       int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1k(smem_raw);
  const uint32_t sb = smem_u32(base);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + 2 * kDwStage);
  auto b_full = [&](int s) { return smem_u32(&bars[s]); };
  auto b_done = [&](int s) { return smem_u32(&bars[2 + s]); };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(&bars[4]);
  const int tid = threadIdx.x, warp = tid / 32;
  const i64 ntiles = (rows + 127) / 128;
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) { mbar_init(b_full(s), 1); mbar_init(b_done(s), 1); }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(smem_u32(tslot), 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = true;
  int n = 0;
  for (i64 tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++n) {
    const int s = n & 1;
    if (n >= 2) ok = __syncthreads_and(wait_bounded(b_done(s), ((n >> 1) & 1) ^ 1, status, kLbTimeout));
    if (!ok) break;
    const uint32_t st = sb + s * kDwStage;
    const i64 r0 = tile * 128;
    if (tid == 0) {
      mbar_expect_tx(b_full(s), 32768);
      tma_load_2d(st, &tmdO, 0, static_cast<int>(r0), b_full(s));
      tma_load_2d(st + 16384, &tmdO, 64, static_cast<int>(r0), b_full(s));
    }
    // O_lin rows [r0, r0 + 128) -> bf16 [t][a] tile (16-byte units)
    uint8_t* ot = base + s * kDwStage + 32768;
    for (int x = tid; x < 128 * 16; x += 128) {
      const int row = x >> 4, u = x & 15;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (r0 + row < rows) {
        const float* src = o_lin + (r0 + row) * kLD + u * 8;
        const float4 a = *reinterpret_cast<const float4*>(src);
        const float4 b = *reinterpret_cast<const float4*>(src + 4);
        w = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                       pack_bf16x2(b.z, b.w));
      }
      *reinterpret_cast<uint4*>(ot + (u >> 3) * 16384 + sw128(row, u & 7)) = w;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      ok = wait_bounded(b_full(s), (n >> 1) & 1, status, kLbTimeout);
      if (ok) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16(128, 128, 1, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma(tmem, sdesc(st + 32768 + kk * 2048, 16384, 1024), sdesc(st + kk * 2048, 16384, 1024),
                 idesc, (n > 0 || kk > 0) ? 1u : 0u);
        tc_commit(b_done(s));
      }
    }
    ok = __syncthreads_and(ok);
  }
  // wait for the last tile's MMAs (tiles before it completed in order)
  if (ok && n > 0) ok = __syncthreads_and(wait_bounded(b_done((n - 1) & 1), ((n - 1) >> 1) & 1, status,
                                                       kLbTimeout));
  if (ok) {
    tc_fence_after();
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    float* dst = part + static_cast<i64>(blockIdx.x) * kLHElems + tid * kLD;
#pragma unroll
    for (int c0 = 0; c0 < kLD; c0 += 32) {
      float v[32];
      if (n > 0) {
        tmem_ld32(tmem + lane_off + c0, v);
        tmem_wait_ld();
        reg_fence<32>(v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(dst + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
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
    tmem_dealloc(tmem, 128);
  }
}

// dproj = sum of the partials in index order (deterministic)
__global__ void dw_sum_kernel(const float* __restrict__ part, float* __restrict__ dproj, int nparts) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= kLHElems) return;
  float s = 0.f;
  for (int p = 0; p < nparts; ++p) s += part[static_cast<i64>(p) * kLHElems + i];
  dproj[i] = s;
}

template <typename F>
cudaError_t lb_set_smem(F kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

constexpr int kDwParts = 148;

struct LinBwdWs {
  size_t lin, dhm, dzm, dh, dz, indt, part, total;
  int ldt;
};

LinBwdWs lin_bwd_ws(const Geom& g) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  LinBwdWs w;
  w.ldt = (g.nqb + 63) / 64 * 64;
  size_t off = 0;
  w.lin = off; off = al(off + lin_tc_scratch_bytes(g));
  w.dhm = off; off = al(off + size_t(g.BH) * g.nqb * kLHElems * 2);
  w.dzm = off; off = al(off + size_t(g.BH) * g.nqb * kLD * 4);
  w.dh = off; off = al(off + size_t(g.BH) * g.nkb * kLHElems * 2);
  w.dz = off; off = al(off + size_t(g.BH) * g.nkb * kLD * 4);
  w.indt = off; off = al(off + size_t(g.BH) * g.nkb * w.ldt * 2);
  w.part = off; off = al(off + size_t(kDwParts) * kLHElems * 4);
  w.total = off;
  return w;
}

}  // namespace

size_t lin_bwd_tc_scratch_bytes(const Geom& g) { return lin_bwd_ws(g).total; }

cudaError_t launch_delta(const void* dout, const float* o_s, float* delta, const Geom& g,
                         cudaStream_t s) {
  const i64 rows = static_cast<i64>(g.BH) * g.N;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  if (grid == 0) return cudaSuccess;
  if (g.dtype == SLA_BF16)
    delta_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(dout), o_s,
                                                     delta, rows, g.d);
  else
    delta_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(dout), o_s, delta, rows, g.d);
  return cudaGetLastError();
}

cudaError_t launch_lin_bwd_prepare(const void* k, const void* v, const float* proj,
                                   const sla_block_lists& rows, const float* o_lin,
                                   const Geom& g, void* scratch, int32_t* status,
                                   cudaStream_t s, LinBwdIn* lin) {
  if (!lin_tc_supported(g)) return cudaErrorNotSupported;
  const LinBwdWs w = lin_bwd_ws(g);
  char* sc = static_cast<char*>(scratch);
  cudaError_t e = launch_lin_tc_prepare(k, v, proj, rows, g, sc + w.lin, status, s);
  if (e != cudaSuccess) return e;
  const LinInputs li = lin_tc_inputs(g, sc + w.lin, rows);
  lin->hm = li.hm;
  lin->wb = li.wb;
  lin->zm = li.zm;
  lin->marg_cnt = rows.marg_cnt;
  lin->o_lin = o_lin;
  lin->dhm = sc + w.dhm;
  lin->dzm = reinterpret_cast<float*>(sc + w.dzm);
  return cudaSuccess;
}

cudaError_t launch_lin_bwd_gather(const sla_block_lists& cols, const Geom& g, void* scratch,
                                  int32_t* status, cudaStream_t s, LinBwdKIn* lin) {
  if (!lin_tc_supported(g)) return cudaErrorNotSupported;
  const LinBwdWs w = lin_bwd_ws(g);
  char* sc = static_cast<char*>(scratch);
  // dH^M, dz^M were written by the dq kernel (zeros for query blocks
  // without marginal sets)
  cudaError_t e = launch_list_gather(cols, g.BH, g.nkb, g.nqb, sc + w.dhm,
                                     reinterpret_cast<const float*>(sc + w.dzm), sc + w.dh,
                                     reinterpret_cast<float*>(sc + w.dz), sc + w.indt, w.ldt, status, g, s);
  if (e != cudaSuccess) return e;
  lin->dh = sc + w.dh;
  lin->dz = reinterpret_cast<const float*>(sc + w.dz);
  lin->marg_cnt = cols.marg_cnt;
  return cudaSuccess;
}

cudaError_t launch_lin_bwd_dw(const void* dout, const float* o_lin, float* dproj, const Geom& g,
                              void* scratch, int32_t* status, cudaStream_t s) {
  if (!g.linear) return cudaMemsetAsync(dproj, 0, sizeof(float) * kLHElems, s);
  const LinBwdWs w = lin_bwd_ws(g);
  char* sc = static_cast<char*>(scratch);
  const i64 R = static_cast<i64>(g.BH) * g.N;
  CUtensorMap mdO2;
  const uint64_t d2[2] = {kLD, static_cast<uint64_t>(R)}, s2[1] = {kLD * 2};
  const uint32_t box2[2] = {64, 128};
  if (!encode_bf16_map(&mdO2, dout, 2, d2, s2, box2)) return cudaErrorInvalidValue;
  const int parts = static_cast<int>(std::min<i64>(kDwParts, (R + 127) / 128));
  float* part = reinterpret_cast<float*>(sc + w.part);
  const size_t smem = 2 * kDwStage + 64 + 1024;
  cudaError_t e;
  if ((e = lb_set_smem(dw_tc_kernel, smem)) != cudaSuccess) return e;
  dw_tc_kernel<<<parts, 128, smem, s>>>(mdO2, o_lin, part, R, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dw_sum_kernel<<<kLHElems / 256, 256, 0, s>>>(part, dproj, parts);
  return cudaGetLastError();
}

}  // namespace sla
