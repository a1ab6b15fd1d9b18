"""GPU side of the 3D-tile token order (Veda article, sections "Что
произошло" / what happened and "Контекст" / context: attention is selected
over tiles of tokens).  The permutation is bit-exact against the oracle's;
moving tokens into and out of it is exact; the hybrid attention of tiled
blocks, run on permuted inputs and moved back, matches the oracle run on the
same permuted inputs; and on a smooth field tiled blocks raise the recall of
the pooled-score mask, measured with the library's own kernels."""

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import assert_close, compare_masks, feed_mask, gpu_inputs, to_np
from oracle import sla_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("grid,tile", [
    ((2, 2, 2), (2, 1, 2)),        # the hand-worked order of the oracle pins
    ((3, 5, 7), (2, 2, 4)),        # partial tiles on every axis
    ((3, 5, 7), (1, 1, 1)),        # degenerate: raster order
    ((3, 5, 7), (3, 5, 7)),        # one tile: raster order
    ((4, 16, 16), (4, 4, 4)),
    ((21, 30, 52), (1, 8, 8)),     # the 1.3B-DiT grid, 64-token tiles
    ((60, 64, 64), (2, 8, 8)),     # the long-clip grid, 128-token tiles
])
def test_tile_order_matches_oracle(grid, tile):
    perm = sla.tile_order(grid, tile, "cuda")
    torch.cuda.synchronize()
    np.testing.assert_array_equal(perm.cpu().numpy(), orc.tile_order(grid, tile))


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 128), (torch.float32, 64)])
def test_permute_tokens_is_exact(dtype, d):
    grid, tile = (3, 10, 22), (2, 4, 8)
    N = grid[0] * grid[1] * grid[2]
    x = torch.randn(2, 3, N, d, generator=torch.Generator().manual_seed(3)).to(dtype).cuda()
    wl = synth.small_case(d=d, grid=grid, H=3, B=2, dtype="bf16" if dtype == torch.bfloat16 else "f32")
    p = sla.params_from(x, wl)
    perm = sla.tile_order(grid, tile, "cuda")
    y = sla.permute_tokens(p, x, perm)
    z = sla.permute_tokens(p, y, perm, inverse=True)
    torch.cuda.synchronize()
    assert torch.equal(y, x[:, :, perm.long()])
    assert torch.equal(z, x)


def _tiled(x, perm):
    return x[:, :, perm]


def _untiled(x, perm):
    out = np.empty_like(x)
    out[..., perm, :] = x
    return out


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tiled_attention_matches_oracle_on_tiled_tokens(dtype):
    grid, tile = (4, 8, 32), (2, 4, 8)      # N = 1024, 64-token tiles
    wl = synth.small_case(d=128 if dtype == "bf16" else 64, grid=grid, H=2, dtype=dtype,
                          frac_crit=0.2, frac_marg=0.2)
    x, t = gpu_inputs(wl, seed=12, with_dout=True)
    p = sla.params_from(t["q"], wl)
    perm_d = sla.tile_order(grid, tile, "cuda")
    perm = orc.tile_order(grid, tile)
    qt, kt, vt, dot = (sla.permute_tokens(p, t[n], perm_d) for n in ("q", "k", "v", "dout"))
    # the mask of the tiled blocks against the oracle's on the tiled tokens
    xq, xk, xv, xd = (_tiled(a.double().numpy(), perm) for a in (x.q, x.k, x.v, x.dout))
    ref = orc.build_mask(xq, xk, wl.block_q, wl.block_k, wl.mode, wl.frac_crit, wl.frac_marg,
                         wl.thr)
    m = sla.build_mask(p, qt, kt)
    torch.cuda.synchronize()
    compare_masks(m["mask"].cpu().numpy(), ref["mask"], ref["margins"])
    # forward and backward with the oracle's mask, moved back to raster order
    _, rows, cols = feed_mask(p, ref["mask"])
    f = sla.forward(p, qt, kt, vt, t["proj"], rows, save_for_backward=True)
    g = sla.backward(p, qt, kt, vt, t["proj"], dot, rows, cols, f)
    out = sla.permute_tokens(p, f["out"], perm_d, inverse=True)
    grads = {k: sla.permute_tokens(p, g[k], perm_d, inverse=True) for k in ("dq", "dk", "dv")}
    torch.cuda.synchronize()
    assert sla.check_device_status(g["ws"]) == sla.SLA_OK
    o = orc.forward(xq, xk, xv, x.proj, ref["mask"], wl.block_q, wl.block_k)
    assert_close(to_np(out), _untiled(o["out"], perm), dtype, "tiled out", stored_bf16=True)
    gr = orc.backward(xq, xk, xv, x.proj, ref["mask"], xd, wl.block_q, wl.block_k)
    for k in ("dq", "dk", "dv"):
        assert_close(to_np(grads[k]), _untiled(gr[k], perm), dtype, f"tiled {k}", rel=True)
    assert_close(to_np(g["dproj"]), gr["dproj"], dtype, "tiled dproj", rel=True)


def test_tiled_blocks_raise_gpu_mask_recall():
    # a 4 x 32 x 32 field in bf16: 64-token blocks as 4 x 4 x 4 boxes against
    # raster strips of two rows, recall of the critical set against the dense
    # attention max-pooled over tiles (the library's quality kernels)
    grid, tile = (4, 32, 32), (4, 4, 4)
    wl = synth.small_case(d=64, grid=grid, H=2, dtype="bf16", frac_crit=0.1, frac_marg=0.1)
    x, t = gpu_inputs(wl, seed=0)
    p = sla.params_from(t["q"], wl)
    perm = sla.tile_order(grid, tile, "cuda")

    def recall(q, k):
        m = sla.build_mask(p, q, k)
        imp = sla.block_importance(p, q, k)
        return sla.mask_recall(p, m["mask"], imp)["recall_critical"]

    raster = recall(t["q"], t["k"])
    tiled = recall(sla.permute_tokens(p, t["q"], perm), sla.permute_tokens(p, t["k"], perm))
    print(f"critical recall: raster {raster:.3f}, 4x4x4 tiles {tiled:.3f}")
    assert tiled > raster + 0.1
