// Token order of 3D tiles, and the row permutation that moves token tensors
// into and out of it.
//
// Veda article (mlllm.io, sections "Что произошло" / what happened and
// "Контекст" / context): attention is selected over tiles of tokens, with tile
// shapes fitted per head and layer.  With tokens in tile order, a block of
// consecutive tokens covers a compact (frames x rows x columns) box of the
// latent grid instead of a strip of raster rows, which is what the mean
// pooling of the block mask then summarises.
//
// Raster token t = (f R + r) C + c of a (F, R, C) grid.  Tiles of
// (tf, tr, tc) tokens are taken in raster order over the tile grid (the
// tiles at the far edges are partial), tokens in raster order inside each
// tile.  A tile starting at (f0, r0, c0) with extents (ef, er, ec) starts at
// position f0 R C + ef r0 C + ef er c0 of the new order: every earlier tile
// layer is made of whole frames, every earlier tile row of the layer of
// whole rows, and every earlier tile of the row has the same ef x er face.
#include "common.cuh"

namespace sla {

namespace {

__global__ void __launch_bounds__(256) tile_order_kernel(int F, int R, int C, int tf, int tr, int tc,
                                                         int32_t* __restrict__ perm) {
  const i64 n_tok = i64(F) * R * C;
  const i64 t = i64(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n_tok) return;
  const int c = static_cast<int>(t % C);
  const int r = static_cast<int>((t / C) % R);
  const int f = static_cast<int>(t / (i64(C) * R));
  const int f0 = f - f % tf, r0 = r - r % tr, c0 = c - c % tc;
  const int ef = min(tf, F - f0), er = min(tr, R - r0), ec = min(tc, C - c0);
  const i64 start = i64(f0) * R * C + i64(ef) * r0 * C + i64(ef) * er * c0;
  const i64 local = (i64(f - f0) * er + (r - r0)) * ec + (c - c0);
  perm[start + local] = static_cast<int32_t>(t);
}

// One thread per 16-byte unit of a row; dst row (bh, n) <- src row
// (bh, perm[n]) (gather), or dst row (bh, perm[n]) <- src row (bh, n)
// (scatter, its inverse).
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src,
                                                           uint4* __restrict__ dst,
                                                           const int32_t* __restrict__ perm, int N,
                                                           int units, i64 total, int scatter) {
  const i64 i = i64(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const i64 row = i / units;
  const int u = static_cast<int>(i - row * units);
  const i64 bh = row / N;
  const int n = static_cast<int>(row - bh * N);
  const i64 other = bh * N + perm[n];
  if (scatter) dst[other * units + u] = src[row * units + u];
  else dst[row * units + u] = src[other * units + u];
}

}  // namespace

cudaError_t launch_tile_order(int F, int R, int C, int tf, int tr, int tc, int32_t* perm,
                              cudaStream_t s) {
  const i64 n = i64(F) * R * C;
  tile_order_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(F, R, C, tf, tr, tc, perm);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(const void* src, void* dst, const int32_t* perm, i64 rows, int N,
                                int row_bytes, bool scatter, cudaStream_t s) {
  const int units = row_bytes / 16;
  const i64 total = rows * units;
  permute_rows_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), perm, N, units, total,
      scatter ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace sla
