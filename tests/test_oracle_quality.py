"""Pins of the oracle's mask-quality measurement (max-pooled dense attention
and recall) against brute force, closed forms and hand-worked rows."""

import math

import numpy as np

from oracle import sla_oracle as orc


def brute_importance(q, k, bq, bk, scale):
    """Plain loops: each query token's softmax over every key, then the
    largest probability per (query block, key block)."""
    B, H, N, d = q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    out = np.zeros((B, H, nqb, nkb))
    for b in range(B):
        for h in range(H):
            for t in range(N):
                z = [scale * sum(float(q[b, h, t, c]) * float(k[b, h, s, c]) for c in range(d))
                     for s in range(N)]
                m = max(z)
                e = [math.exp(x - m) for x in z]
                tot = sum(e)
                for s in range(N):
                    i, j = t // bq, s // bk
                    out[b, h, i, j] = max(out[b, h, i, j], e[s] / tot)
    return out


def test_importance_matches_brute_force_with_ragged_blocks():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 2, 11, 5))
    k = rng.standard_normal((1, 2, 11, 5))
    for bq, bk in [(4, 3), (3, 4), (11, 2), (1, 1)]:
        got = orc.max_pooled_attention(q, k, bq, bk)
        ref = brute_importance(q, k, bq, bk, 1.0 / math.sqrt(5))
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=0)


def test_unit_blocks_give_the_dense_softmax():
    # blocks of one token: the importance is P itself, whose rows sum to one
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, 9, 4))
    k = rng.standard_normal((1, 1, 9, 4))
    imp = orc.max_pooled_attention(q, k, 1, 1, scale=0.7)
    np.testing.assert_allclose(imp.sum(axis=-1), 1.0, rtol=1e-13)
    logits = 0.7 * q[0, 0] @ k[0, 0].T
    p = np.exp(logits) / np.exp(logits).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(imp[0, 0], p, rtol=1e-12)


def test_identical_keys_give_uniform_importance():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, 10, 3))
    k = np.tile(rng.standard_normal((1, 1, 1, 3)), (1, 1, 10, 1))
    imp = orc.max_pooled_attention(q, k, 4, 3)
    np.testing.assert_allclose(imp, 0.1, rtol=1e-13)


def test_recall_of_the_importance_own_selection_is_full():
    rng = np.random.default_rng(6)
    imp = rng.random((2, 3, 5, 17))
    mask, _ = orc.classify(imp, "topk", 0.2, 0.3)
    ch, ct, kh, kt = orc.mask_recall_counts(mask, imp)
    assert ch == ct > 0 and kh == kt > ct


def test_recall_of_the_lowest_blocks_is_zero():
    rng = np.random.default_rng(7)
    imp = rng.random((1, 1, 4, 20))          # distinct values: no ties
    mask = np.zeros(imp.shape, dtype=np.int8)
    for i in range(4):
        low = np.argsort(imp[0, 0, i])[:5]   # five lowest: critical
        mask[0, 0, i, low] = orc.CRITICAL
    ch, ct, kh, kt = orc.mask_recall_counts(mask, imp)
    assert (ch, ct, kh, kt) == (0, 20, 0, 20)


def test_recall_on_hand_worked_rows():
    imp = np.array([[0.5, 0.5, 0.1, 0.2],
                    [0.1, 0.4, 0.3, 0.2]])
    # row 0: c = 1 and 1 kept, reference {0} (tie: lower index) -> misses
    # row 1: c = 1, reference {1} -> hit; 3 kept, reference {1, 2, 3}, of
    # which blocks 1 and 2 are kept -> 2 hits
    mask = np.array([[0, 2, 0, 0],
                     [1, 2, 1, 0]])
    assert orc.mask_recall_counts(mask, imp) == (0 + 1, 1 + 1, 0 + 2, 1 + 3)
