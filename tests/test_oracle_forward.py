"""Pins for the oracle's forward pass (sparse softmax part, linear part,
combine) against brute force, textbook special cases and closed forms."""

import json
import math
import os

import numpy as np
import pytest
import torch

from brute import brute_forward
from oracle import sla_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def random_mask(shape, seed, p=(0.3, 0.3, 0.4)):
    r = np.random.default_rng(seed)
    return r.choice([2, 1, 0], size=shape, p=p).astype(np.int8)


@pytest.mark.parametrize("n,d,bq,bk,seed", [
    (20, 4, 8, 8, 0),       # ragged tail (20 = 8 + 8 + 4)
    (23, 3, 8, 5, 1),       # query and key blocks differ, both ragged
    (16, 8, 4, 8, 2),
    (9, 2, 16, 16, 3),      # a single (ragged) block
])
def test_forward_matches_token_level_brute_force(n, d, bq, bk, seed):
    B, H = 1, 2
    q, k, v = (rnd((B, H, n, d), seed + i) for i in range(3))
    w = rnd((d, d), seed + 9) / 8
    nqb, nkb = orc.n_blocks(n, bq), orc.n_blocks(n, bk)
    mask = random_mask((B, H, nqb, nkb), seed + 17)
    mask[0, 0, 0] = 0                     # a row with nothing at all
    mask[0, 1, -1] = 1                    # a row that is linear only
    s = 1 / math.sqrt(d)
    got = orc.forward(q, k, v, w, mask, bq, bk, s)
    ref = brute_forward(q, k, v, w, mask, bq, bk, s)
    for key in ("out", "o_s", "o_lin"):
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(got["lse"]), np.isneginf(ref["lse"]))
    fin = np.isfinite(ref["lse"])
    np.testing.assert_allclose(got["lse"][fin], ref["lse"][fin], rtol=1e-12)


def test_all_critical_is_dense_softmax_attention():
    # textbook special case: every pair critical = dense attention, checked
    # against torch's scaled_dot_product_attention in float64
    B, H, N, d = 1, 2, 40, 8
    q, k, v = (rnd((B, H, N, d), 10 + i) for i in range(3))
    w = rnd((d, d), 20)
    mask = np.full((B, H, 5, 5), 2, dtype=np.int8)
    got = orc.forward(q, k, v, w, mask, 8, 8)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v)).numpy()
    np.testing.assert_allclose(got["out"], ref, rtol=1e-12, atol=1e-13)
    lse = torch.logsumexp(torch.tensor(q) @ torch.tensor(k).transpose(-1, -2)
                          / math.sqrt(d), dim=-1).numpy()
    np.testing.assert_allclose(got["lse"], lse, rtol=1e-13)


def test_all_negligible_gives_zero():
    B, H, N, d = 1, 1, 30, 4
    q, k, v = (rnd((B, H, N, d), 30 + i) for i in range(3))
    mask = np.zeros((B, H, 4, 4), dtype=np.int8)
    got = orc.forward(q, k, v, rnd((d, d), 33), mask, 8, 8)
    assert (got["out"] == 0).all()
    assert np.isneginf(got["lse"]).all()


def test_all_marginal_closed_form():
    # linear attention over all blocks equals
    #   phi(Q) (phi(K)^T V) / (phi(Q) sum_t phi(k_t)),  then @ W
    B, H, N, d = 2, 2, 37, 6
    q, k, v = (rnd((B, H, N, d), 40 + i) for i in range(3))
    w = rnd((d, d), 44) / 8
    mask = np.ones((B, H, 5, 4), dtype=np.int8)
    got = orc.forward(q, k, v, w, mask, 8, 10)

    def elu1(x):
        return np.where(x > 0, x + 1, np.exp(np.minimum(x, 0)))
    fq, fk = elu1(q), elu1(k)
    num = fq @ (np.swapaxes(fk, -1, -2) @ v)
    den = fq @ fk.sum(axis=-2)[..., None]
    np.testing.assert_allclose(got["out"], (num / den) @ w, rtol=1e-12, atol=1e-13)
    assert (got["o_s"] == 0).all()


def test_key_shift_leaves_sparse_output_and_shifts_lse():
    B, H, N, d = 1, 2, 48, 8
    q, k, v = (rnd((B, H, N, d), 50 + i) for i in range(3))
    c = rnd((d,), 54)
    mask = random_mask((B, H, 6, 6), 55, p=(0.5, 0.0, 0.5))
    o0, l0 = orc.sparse_attention(q, k, v, mask, 8, 8)
    o1, l1 = orc.sparse_attention(q, k + c, v, mask, 8, 8)
    np.testing.assert_allclose(o0, o1, rtol=1e-10, atol=1e-12)
    shift = (q @ c) / math.sqrt(d)
    fin = np.isfinite(l0)
    np.testing.assert_allclose(l1[fin], (l0 + shift)[fin], rtol=1e-10, atol=1e-12)


def test_phi_is_elu_plus_one():
    x = np.array([-3.0, -0.5, 0.0, 0.5, 2.0])
    np.testing.assert_allclose(
        orc.phi(x), torch.nn.functional.elu(torch.tensor(x)).numpy() + 1, rtol=1e-15)


def test_linear_summaries_are_outer_product_sums():
    k = rnd((1, 1, 10, 3), 60)
    v = rnd((1, 1, 10, 3), 61)
    h, z = orc.linear_summaries(k, v, 4)
    fk = orc.phi(k)
    for j, (a, b) in enumerate([(0, 4), (4, 8), (8, 10)]):
        ref = sum(np.outer(fk[0, 0, t], v[0, 0, t]) for t in range(a, b))
        np.testing.assert_allclose(h[0, 0, j], ref, rtol=1e-14)
        np.testing.assert_allclose(z[0, 0, j], fk[0, 0, a:b].sum(axis=0), rtol=1e-14)


def _load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_hand_worked_example():
    g = _load_golden("hand_worked_2blocks.json")
    q = np.array(g["q"], dtype=np.float64)[None, None]
    k = np.array(g["k"], dtype=np.float64)[None, None]
    v = np.array(g["v"], dtype=np.float64)[None, None]
    w = np.array(g["w"], dtype=np.float64)
    m = orc.build_mask(q, k, g["block"], g["block"], "topk", g["frac_crit"],
                       g["frac_marg"], scale=g["scale"])
    np.testing.assert_allclose(m["scores"][0, 0], g["expect_scores"], rtol=1e-14)
    np.testing.assert_array_equal(m["mask"][0, 0], g["expect_mask"])
    f = orc.forward(q, k, v, w, m["mask"], g["block"], g["block"], g["scale"])
    np.testing.assert_allclose(f["out"][0, 0], g["expect_out"], rtol=1e-14, atol=1e-15)
