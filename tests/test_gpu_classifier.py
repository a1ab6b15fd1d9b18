"""The GPU classifier on crafted score rows (sla_classify_scores), bit for bit
against the oracle on the very same fp32 values: exact duplicates (index
tie-break), zeros, tiny and wide rows, and CDF rows whose dyadic masses put
tail sums exactly on thr (the strict 'exceeds 1 - thr' boundary)."""

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import expected_rows, lists_from_gpu
from oracle import sla_oracle as orc

pytestmark = pytest.mark.gpu


def _rows(kind, nkb, nrows, rng):
    if kind == "dups":
        p = rng.choice([1.0, 2.0, 3.0, 5.0, 8.0], size=(nrows, nkb))
    elif kind == "zeros":
        p = rng.random((nrows, nkb)) ** 6
        p[rng.random((nrows, nkb)) < 0.5] = 0.0
        p[:, 0] += 1e-3
    elif kind == "dyadic":
        p = 2.0 ** -rng.integers(1, 12, size=(nrows, nkb)).astype(np.float64)
    else:
        p = rng.random((nrows, nkb)) ** 4
    p = p / p.sum(axis=1, keepdims=True)
    return p.astype(np.float32)


def _params(nkb, nrows, mode, fc=0.0, fm=0.0, thr=0.0):
    wl = synth.Workload(name="cls", B=1, H=1, grid=(1, 1, nkb * 64), d=64, dtype="f32",
                        block_q=64, block_k=64, mode=mode, frac_crit=fc, frac_marg=fm, thr=thr)
    p = sla.params_for(wl)
    # one head of nrows query blocks: N spans max(nrows, nkb) blocks of 64
    return wl, p


@pytest.mark.parametrize("kind", ["dups", "zeros", "dyadic", "smooth"])
# rows of every length class of the one-warp-per-row kernel (shared memory
# per warp grows with the row; "dups" rows of 1920 and 2500 blocks overflow
# the 256 candidate slots and take the exact whole-row search)
@pytest.mark.parametrize("nkb", [1, 7, 64, 300, 512, 700, 1920, 2500])
@pytest.mark.parametrize("mode,fc,fm,thr", [("topk", 0.05, 0.10, 0.0), ("topk", 0.5, 0.25, 0.0),
                                            ("cdf", 0.0, 0.0, 0.2), ("cdf", 0.0, 0.1, 0.5),
                                            ("cdf", 0.0, 0.0, 0.0),
                                            # rows whose fp32 scores sum to just under 1
                                            # stay under thr: only the top rank is kept
                                            ("cdf", 0.0, 0.05, 0.99999999)])
def test_classifier_bit_exact_on_crafted_rows(kind, nkb, mode, fc, fm, thr):
    rng = np.random.default_rng(nkb * 7 + len(kind))
    nrows = nkb  # square: Nqb = Nkb
    s32 = _rows(kind, nkb, nrows, rng)
    wl, p = _params(nkb, nrows, mode, fc, fm, thr)
    got = sla.classify_scores(p, torch.from_numpy(s32.reshape(1, 1, nrows, nkb)).cuda())
    torch.cuda.synchronize()
    mask = got["mask"].cpu().numpy()[0, 0]
    ref, margins = orc.classify(s32.astype(np.float64), mode, fc, fm, thr)
    if mode == "topk":
        np.testing.assert_array_equal(mask, ref)
    else:
        # the decision may differ only where a tail sum lies within 1e-12 of
        # thr (fixed point vs binary64 summation order); dyadic rows are exact
        diff = (mask != ref).any(axis=-1)
        assert not (diff & (margins > 1e-12)).any()
        if kind == "dyadic":
            np.testing.assert_array_equal(mask, ref)
    assert lists_from_gpu(got["rows"], nrows, nkb) == expected_rows(mask[None, None])
    # the GPU's own tie count equals the oracle's on the same values
    if mode == "topk" or kind == "dyadic":
        assert int(got["ties"].item()) == int((margins <= 1e-5).sum())


@pytest.mark.parametrize("kind", ["smooth", "dups"])
@pytest.mark.parametrize("mode,fc,fm,thr", [("topk", 0.03, 0.02, 0.0), ("cdf", 0.0, 0.05, 0.2)])
def test_classifier_at_the_longest_rows(kind, mode, fc, fm, thr):
    # rows of 8192 key blocks, the most a mask supports (one warp per CTA,
    # 68 KB of shared memory); the GPU classifies all 4096 rows, the oracle
    # a spread of 48 of them
    nkb, bq = 8192, 128
    N = nkb * 64
    nqb = N // bq
    rng = np.random.default_rng(8192 + len(kind))
    s32 = _rows(kind, nkb, nqb, rng)
    wl = synth.Workload(name="cls", B=1, H=1, grid=(1, 1, N), d=64, dtype="f32", block_q=bq,
                        block_k=64, mode=mode, frac_crit=fc, frac_marg=fm, thr=thr)
    p = sla.params_for(wl)
    got = sla.classify_scores(p, torch.from_numpy(s32.reshape(1, 1, nqb, nkb)).cuda())
    torch.cuda.synchronize()
    sample = np.linspace(0, nqb - 1, 48).astype(int)
    mask = got["mask"].cpu().numpy()[0, 0][sample]
    ref, margins = orc.classify(s32[sample].astype(np.float64), mode, fc, fm, thr)
    if mode == "topk":
        np.testing.assert_array_equal(mask, ref)
    else:
        diff = (mask != ref).any(axis=-1)
        assert not (diff & (margins > 1e-12)).any()
    lists = lists_from_gpu(got["rows"], nqb, nkb)
    exp = expected_rows(mask[None, None])
    assert [lists[0][r] for r in sample] == exp[0]
    assert [lists[1][r] for r in sample] == exp[1]


@pytest.mark.parametrize("n_small", [40, 300])
@pytest.mark.parametrize("fm", [0.0, 0.05])
def test_cdf_cut_moved_to_a_lower_bin_by_the_exact_sums(n_small, fm):
    # n_small equal small scores whose 2^-24-unit truncation (the histogram's
    # approximate masses) loses almost a unit each, and 60 scores of 2^-7:
    # thr is exactly the small scores' total, so the approximate masses put
    # the cut in the large scores' bin and the exact fixed-point sums move it
    # down to the small scores' bin, whose scores are then collected anew
    # (40: a cut among 33-64 candidates; 300: more than the 256 slots, the
    # search over the whole row).  The one small score whose tail sum equals
    # thr exactly is kept, and every row is a near-tie row.
    a = np.float32((2046 + 1014 / 1024) * 2.0 ** -24)
    assert float(a) == (2046 + 1014 / 1024) * 2.0 ** -24
    thr = n_small * float(a)  # dyadic: exact in binary64 and in 2^-62 fixed point
    nkb = n_small + 60
    rng = np.random.default_rng(n_small)
    row = np.concatenate([np.full(n_small, a, np.float32), np.full(60, np.float32(2.0 ** -7))])
    s32 = np.stack([rng.permutation(row) for _ in range(nkb)]).astype(np.float32)
    wl, p = _params(nkb, nkb, "cdf", 0.0, fm, thr)
    got = sla.classify_scores(p, torch.from_numpy(s32.reshape(1, 1, nkb, nkb)).cuda())
    torch.cuda.synchronize()
    mask = got["mask"].cpu().numpy()[0, 0]
    ref, margins = orc.classify(s32.astype(np.float64), "cdf", 0.0, fm, thr)
    assert ((ref == 2).sum(axis=1) == 61).all()
    np.testing.assert_array_equal(mask, ref)
    assert lists_from_gpu(got["rows"], nkb, nkb) == expected_rows(mask[None, None])
    assert int(got["ties"].item()) == int((margins <= 1e-5).sum()) == nkb
