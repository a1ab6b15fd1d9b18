"""Pins of the 3D-tile token order, and the CPU measurement that motivates
it: on a smooth synthetic field, blocks of tiled tokens give pooled-score
masks with a higher recall against max-pooled dense attention than blocks
of raster tokens."""

import numpy as np

from block_sparse_linear_mean_b200 import synth
from oracle import sla_oracle as orc


def test_hand_worked_order():
    # grid (2, 2, 2), tile (2, 1, 2): tile r = 0 holds raster 0, 1, 4, 5
    # (f = 0, 1; c = 0, 1), tile r = 1 holds 2, 3, 6, 7
    np.testing.assert_array_equal(orc.tile_order((2, 2, 2), (2, 1, 2)), [0, 1, 4, 5, 2, 3, 6, 7])


def test_order_is_a_permutation_with_partial_edge_tiles():
    perm = orc.tile_order((3, 5, 7), (2, 2, 4))
    np.testing.assert_array_equal(np.sort(perm), np.arange(3 * 5 * 7))


def test_degenerate_tiles_keep_raster_order():
    for tile in [(1, 1, 1), (1, 1, 7), (3, 5, 7)]:
        np.testing.assert_array_equal(orc.tile_order((3, 5, 7), tile), np.arange(105))


def test_each_tile_is_a_box():
    F, R, C, t = 4, 8, 8, (2, 4, 4)
    perm = orc.tile_order((F, R, C), t)
    for n in range(len(perm) // 32):
        f, r, c = np.unravel_index(perm[32 * n:32 * (n + 1)], (F, R, C))
        assert (f.max() - f.min(), r.max() - r.min(), c.max() - c.min()) == (1, 3, 3)


def recall(q, k, frac_crit):
    m = orc.build_mask(q, k, 64, 64, "topk", frac_crit, 0.1)["mask"]
    imp = orc.max_pooled_attention(q, k, 64, 64)
    ch, ct, _, _ = orc.mask_recall_counts(m, imp)
    return ch / ct


def test_tiled_blocks_raise_mask_recall_on_a_smooth_field():
    # a 4 x 16 x 16 field: 64-token blocks as 4 x 4 x 4 boxes against raster
    # strips of four rows (measured: 0.812 against 0.453 critical recall)
    grid = (4, 16, 16)
    wl = synth.small_case(d=64, grid=grid, H=2, dtype="f32", frac_crit=0.1, frac_marg=0.1)
    x = synth.make_inputs(wl, seed=0, device="cpu")
    q, k = x.q.double().numpy(), x.k.double().numpy()
    perm = orc.tile_order(grid, (4, 4, 4))
    raster = recall(q, k, 0.1)
    tiled = recall(q[:, :, perm], k[:, :, perm], 0.1)
    print(f"critical recall: raster {raster:.3f}, 4x4x4 tiles {tiled:.3f}")
    assert tiled > raster + 0.2
