"""Pins for the oracle's pooling, block scores and classification (CPU only).

Each test checks the oracle against something other than itself: a closed
form, an invariant the definitions imply, or exhaustive enumeration on tiny
rows."""

import itertools
import math

import numpy as np
import pytest

from oracle import sla_oracle as orc


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- pooling


def test_pool_constant_block_and_tail():
    # a constant block pools to the constant; the ragged tail block is the
    # mean over its real tokens only (reading 1), not over zero padding
    x = np.zeros((1, 1, 10, 3))
    x[0, 0, :4] = 2.0
    x[0, 0, 4:8] = -1.5
    x[0, 0, 8:] = [[1.0, 2.0, 3.0], [3.0, 4.0, 5.0]]
    p = orc.pool_blocks(x, 4)
    assert p.shape == (1, 1, 3, 3)
    np.testing.assert_array_equal(p[0, 0, 0], [2.0, 2.0, 2.0])
    np.testing.assert_array_equal(p[0, 0, 1], [-1.5, -1.5, -1.5])
    np.testing.assert_array_equal(p[0, 0, 2], [2.0, 3.0, 4.0])


def test_pool_matches_numpy_mean():
    x = rng(1).standard_normal((2, 3, 37, 5))
    p = orc.pool_blocks(x, 8)
    for i in range(5):
        np.testing.assert_allclose(p[:, :, i], x[:, :, 8 * i:8 * i + 8].mean(axis=2),
                                   rtol=1e-14, atol=1e-14)


def test_scores_permutation_invariance_within_blocks():
    r = rng(2)
    q = r.standard_normal((1, 1, 48, 8))
    k = r.standard_normal((1, 1, 48, 8))
    m0 = orc.build_mask(q, k, 16, 16, "topk", 0.34, 0.34)
    perm_q, perm_k = q.copy(), k.copy()
    for i in range(3):
        perm_q[0, 0, 16 * i:16 * i + 16] = q[0, 0, 16 * i + r.permutation(16)]
        perm_k[0, 0, 16 * i:16 * i + 16] = k[0, 0, 16 * i + r.permutation(16)]
    m1 = orc.build_mask(perm_q, perm_k, 16, 16, "topk", 0.34, 0.34)
    np.testing.assert_allclose(m0["scores"], m1["scores"], rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(m0["mask"], m1["mask"])


def test_scores_rows_are_textbook_softmax():
    r = rng(3)
    qb = r.standard_normal((4, 6))
    kb = r.standard_normal((7, 6))
    s = 0.3
    p = orc.block_scores(qb, kb, s)
    for i in range(4):
        logits = [s * float(np.dot(qb[i], kb[j])) for j in range(7)]
        den = sum(math.exp(x) for x in logits)
        np.testing.assert_allclose(p[i], [math.exp(x) / den for x in logits],
                                   rtol=1e-13)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)


def test_key_shift_leaves_scores_and_mask_unchanged():
    # adding one vector c to every key adds s*qbar.c to a whole score row,
    # which the row softmax removes
    r = rng(4)
    q = r.standard_normal((1, 2, 64, 8))
    k = r.standard_normal((1, 2, 64, 8))
    c = r.standard_normal(8)
    m0 = orc.build_mask(q, k, 8, 8, "topk", 0.25, 0.25)
    m1 = orc.build_mask(q, k + c, 8, 8, "topk", 0.25, 0.25)
    np.testing.assert_allclose(m0["scores"], m1["scores"], rtol=1e-10)
    np.testing.assert_array_equal(m0["mask"], m1["mask"])


# ---------------------------------------------------------------- top-k


@pytest.mark.parametrize("fc,fm,nkb,expect", [
    (0.25, 0.25, 16, (4, 4)),
    (0.05, 0.10, 512, (26, 52)),     # 25.6 -> 26, 51.2 -> 52
    (0.03, 0.02, 1920, (58, 39)),    # 57.6 -> 58, 38.4 -> 39
    (0.07, 0.0, 100, (7, 0)),        # 0.07*100 = 7.000000000000001 in binary64
    (0.9, 0.5, 10, (9, 1)),          # marginal capped at Nkb - n_c
    (0.0, 0.0, 10, (0, 0)),
    (1.0, 0.0, 10, (10, 0)),
])
def test_topk_counts(fc, fm, nkb, expect):
    assert orc.topk_counts(fc, fm, nkb) == expect


def test_topk_invariants_random_rows():
    r = rng(5)
    for trial in range(200):
        nkb = int(r.integers(2, 40))
        p = r.random(nkb)
        p /= p.sum()
        n_c = int(r.integers(0, nkb + 1))
        n_m = int(r.integers(0, nkb - n_c + 1))
        lab, _ = orc.classify_topk_row(p, n_c, n_m)
        crit = p[lab == 2]
        marg = p[lab == 1]
        negl = p[lab == 0]
        assert crit.size == n_c and marg.size == n_m
        assert negl.size == nkb - n_c - n_m
        if crit.size and marg.size:
            assert crit.min() >= marg.max()
        if marg.size and negl.size:
            assert marg.min() >= negl.max()
        if crit.size and negl.size:
            assert crit.min() >= negl.max()


def test_topk_tie_break_prefers_lower_index():
    # exact ties (e.g. two identical key blocks) go to the lower block index
    p = np.array([0.1, 0.2, 0.2, 0.2, 0.3])
    lab, margin = orc.classify_topk_row(p, 2, 2)
    assert list(lab) == [0, 2, 1, 1, 2]
    assert margin == 0.0


def test_topk_on_identical_key_blocks_full_path():
    r = rng(6)
    q = r.standard_normal((1, 1, 32, 4))
    k = r.standard_normal((1, 1, 32, 4))
    k[0, 0, 8:16] = k[0, 0, 0:8]      # key blocks 0 and 1 are identical
    m = orc.build_mask(q, k, 8, 8, "topk", 0.25, 0.0)
    p = m["scores"][0, 0]
    for i in range(4):
        assert p[i, 0] == p[i, 1]
        # with one critical slot, a tie between blocks 0 and 1 at the top
        # resolves to block 0
        if p[i, 0] == p[i].max():
            assert m["mask"][0, 0, i, 0] == 2 and m["mask"][0, 0, i, 1] == 0


# ---------------------------------------------------------------- CDF


def test_cdf_threshold_zero_keeps_every_block():
    r = rng(7)
    p = r.random((5, 9, 23)) ** 8
    p /= p.sum(axis=-1, keepdims=True)
    mask, _ = orc.classify(p, "cdf", thr=0.0)
    assert (mask == 2).all()


def _brute_minimal_set(p, thr):
    """Smallest cardinality of a subset with mass > 1 - thr, by enumeration."""
    n = len(p)
    for size in range(1, n + 1):
        for sub in itertools.combinations(range(n), size):
            if sum(p[j] for j in sub) > 1.0 - thr:
                return size
    return n


def test_cdf_minimal_set_brute_force():
    r = rng(8)
    checked = 0
    for trial in range(300):
        nkb = int(r.integers(2, 11))
        p = r.random(nkb) ** 3
        p /= p.sum()
        thr = float(r.uniform(0.0, 0.95))
        lab, margin = orc.classify_cdf_row(p, thr)
        if margin < 1e-9:
            continue                       # boundary case: skip, not a pin
        kept = int((lab == 2).sum())
        assert kept == _brute_minimal_set(p, thr)
        # the kept set is the top-ranked one
        order = orc.rank_order(p)
        assert set(np.nonzero(lab == 2)[0]) == set(order[:kept])
        checked += 1
    assert checked > 250


def test_cdf_mass_and_minimality_and_monotone():
    r = rng(9)
    for trial in range(100):
        nkb = int(r.integers(3, 60))
        p = r.random(nkb) ** 4
        p /= p.sum()
        prev_kept = None
        for thr in (0.9, 0.7, 0.5, 0.3, 0.2, 0.1, 0.05, 0.0):
            lab, _ = orc.classify_cdf_row(p, thr)
            keep = lab == 2
            assert p[keep].sum() > 1.0 - thr - 1e-12
            smallest = p[keep].min()
            if keep.sum() > 1:
                assert p[keep].sum() - smallest <= 1.0 - thr + 1e-12
            if prev_kept is not None:
                assert (keep | ~prev_kept).all()   # kept set grows as thr falls
            prev_kept = keep


def test_cdf_with_marginal_fraction():
    p = np.array([0.5, 0.05, 0.3, 0.1, 0.05])
    # thr = 0.25: drop ranks while the tail stays < 0.25: 0.05 (idx4), 0.05
    # (idx1) -> 0.10, then 0.1 -> 0.20, then 0.3 -> 0.5 fails: keep {0, 2}
    lab, _ = orc.classify_cdf_row(p, 0.25, n_m=2)
    assert list(lab) == [2, 1, 2, 1, 0]


def test_cdf_worked_example_from_definition():
    # NABLA points 2-3 on a 4-block row: masses 0.6, 0.25, 0.1, 0.05 with
    # 1 - thr = 0.8 -> keep the two largest (0.85 > 0.8, 0.6 is not)
    p = np.array([0.05, 0.6, 0.1, 0.25])
    lab, margin = orc.classify_cdf_row(p, 0.2)
    assert list(lab) == [0, 2, 0, 2]
    assert margin == pytest.approx(0.05)


def test_mask_lists_ascending():
    mask = np.array([[[[2, 0, 1, 2], [0, 0, 0, 0]]]], dtype=np.int8)
    crit, marg = orc.mask_lists(mask)
    assert [list(c) for c in crit] == [[0, 3], []]
    assert [list(m) for m in marg] == [[2], []]


def test_cdf_exact_boundary_is_strict():
    # NABLA point 3: the kept blocks' sum must EXCEED 1 - thr.  With masses
    # exact in binary, {0.5, 0.25} sums to exactly 0.75 = 1 - thr, which does
    # not exceed it, so all three blocks are kept.
    p = np.array([0.5, 0.25, 0.25])
    lab, margin = orc.classify_cdf_row(p, 0.25)
    assert list(lab) == [2, 2, 2]
    assert margin == 0.0
    lab, _ = orc.classify_cdf_row(np.array([0.5, 0.25, 0.125, 0.125]), 0.25)
    # dropping 0.125 leaves a tail of 0.125 < 0.25; dropping the next 0.125
    # would make it 0.25, not below 0.25, so three blocks stay
    assert list(lab) == [2, 2, 2, 0]
