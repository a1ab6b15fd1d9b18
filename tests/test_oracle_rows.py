"""Pins for the oracle's per-row forward (``forward_rows``) and its per-block
summaries (``linear_summaries_of``), the functions that check sampled query
blocks of workloads too large for the whole oracle.

Both are compared with the token-level brute force (``tests/brute.py``, which
expands the block mask to token pairs and sums over keys directly, with no
block summaries), on every query block of every head, and with the whole-tensor
oracle.  Cases cover ragged tails, query blocks larger and smaller than key
blocks, rows with no critical block, rows that are linear only and rows with
nothing at all (SLA post, list "the idea", items 2-3: critical -> softmax
attention, marginal -> linear attention, negligible -> skipped)."""

import math

import numpy as np
import pytest

from brute import brute_forward, elu1
from oracle import sla_oracle as orc


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


CASES = [
    # n, d, block_q, block_k, seed
    (29, 4, 8, 8, 0),     # equal blocks, ragged tail of 5
    (31, 3, 12, 5, 1),    # query blocks larger than key blocks, both ragged
    (27, 4, 4, 10, 2),    # query blocks smaller than key blocks, both ragged
    (7, 2, 16, 3, 3),     # one ragged query block over three key blocks
]


def _mask(nqb, nkb, seed):
    r = np.random.default_rng(seed)
    m = r.choice([2, 1, 0], size=(1, 2, nqb, nkb), p=[0.35, 0.35, 0.3]).astype(np.int8)
    m[0, 0, 0] = 0                 # nothing at all
    m[0, 1, -1] = 1                # linear only
    if nqb > 1:
        m[0, 0, 1] = np.where(m[0, 0, 1] == 1, 2, m[0, 0, 1])  # no marginal
    return m


@pytest.mark.parametrize("n,d,bq,bk,seed", CASES)
def test_forward_rows_matches_brute_force_on_every_block(n, d, bq, bk, seed):
    q, k, v = (rnd((1, 2, n, d), seed + i) for i in range(3))
    w = rnd((d, d), seed + 7) / 8
    nqb, nkb = orc.n_blocks(n, bq), orc.n_blocks(n, bk)
    mask = _mask(nqb, nkb, seed + 11)
    s = 1 / math.sqrt(d)
    ref = brute_forward(q, k, v, w, mask, bq, bk, s)
    whole = orc.forward(q, k, v, w, mask, bq, bk, s)
    for h in range(2):
        for i in range(nqb):
            a, e = i * bq, min((i + 1) * bq, n)
            got = orc.forward_rows(q[0, h], k[0, h], v[0, h], w, mask[0, h, i],
                                   i, bq, bk, s)
            for key in ("out", "o_s", "o_lin"):
                np.testing.assert_allclose(got[key], ref[key][0, h, a:e],
                                           rtol=1e-11, atol=1e-12)
                np.testing.assert_allclose(got[key], whole[key][0, h, a:e],
                                           rtol=1e-12, atol=1e-13)
            fin = np.isfinite(ref["lse"][0, h, a:e])
            np.testing.assert_array_equal(np.isfinite(got["lse"]), fin)
            np.testing.assert_allclose(got["lse"][fin], ref["lse"][0, h, a:e][fin],
                                       rtol=1e-12)


def test_forward_rows_default_scale_is_inverse_sqrt_d():
    n, d = 20, 9
    q, k, v = (rnd((1, 1, n, d), 30 + i) for i in range(3))
    w = np.eye(d)
    mask = np.full((1, 1, 3, 3), 2, dtype=np.int8)
    ref = brute_forward(q, k, v, w, mask, 8, 8, 1 / 3.0)
    got = orc.forward_rows(q[0, 0], k[0, 0], v[0, 0], w, mask[0, 0, 2], 2, 8, 8)
    np.testing.assert_allclose(got["out"], ref["out"][0, 0, 16:20], rtol=1e-12)


@pytest.mark.parametrize("n,d,bk", [(23, 3, 5), (16, 4, 8), (5, 2, 8)])
def test_linear_summaries_of_are_outer_product_sums(n, d, bk):
    k = rnd((n, d), 40 + n)
    v = rnd((n, d), 41 + n)
    nkb = orc.n_blocks(n, bk)
    blocks = list(range(nkb - 1, -1, -1))          # any order, tail included
    got = orc.linear_summaries_of(k, v, blocks, bk)
    assert sorted(got) == list(range(nkb))
    hall, zall = orc.linear_summaries(k[None, None], v[None, None], bk)
    for j in range(nkb):
        a, b = j * bk, min((j + 1) * bk, n)
        h_ref = np.zeros((d, d))
        z_ref = np.zeros(d)
        for t in range(a, b):                       # token by token, by hand
            fk = np.array([elu1(x) for x in k[t]])
            h_ref += np.outer(fk, v[t])
            z_ref += fk
        np.testing.assert_allclose(got[j][0], h_ref, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(got[j][1], z_ref, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(got[j][0], hall[0, 0, j], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(got[j][1], zall[0, 0, j], rtol=1e-13, atol=1e-14)


def test_linear_summaries_of_subset_only():
    k, v = rnd((30, 3), 50), rnd((30, 3), 51)
    got = orc.linear_summaries_of(k, v, np.array([3, 1]), 8)
    assert sorted(got) == [1, 3]
    # block 3 is the ragged tail, tokens 24..29
    fk = np.array([[elu1(x) for x in row] for row in k[24:30]])
    np.testing.assert_allclose(got[3][0], fk.T @ v[24:30], rtol=1e-13)
