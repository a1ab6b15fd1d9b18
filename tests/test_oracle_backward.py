"""Pins for the oracle's backward pass: central finite differences in float64,
torch autograd through the token-level brute-force formulation, and the
dense-attention special case."""

import math

import numpy as np
import pytest
import torch

from brute import torch_token_forward
from oracle import sla_oracle as orc


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def random_mask(shape, seed, p=(0.35, 0.35, 0.3)):
    r = np.random.default_rng(seed)
    return r.choice([2, 1, 0], size=shape, p=p).astype(np.int8)


def loss(q, k, v, w, mask, dout, bq, bk, s):
    return float((orc.forward(q, k, v, w, mask, bq, bk, s)["out"] * dout).sum())


@pytest.mark.parametrize("n,d,bq,bk,seed", [(12, 3, 4, 4, 0), (11, 2, 4, 3, 1)])
def test_backward_matches_finite_differences(n, d, bq, bk, seed):
    B, H = 1, 2
    q, k, v = (rnd((B, H, n, d), seed + i) for i in range(3))
    w = rnd((d, d), seed + 5, 0.3)
    dout = rnd((B, H, n, d), seed + 6)
    mask = random_mask((B, H, orc.n_blocks(n, bq), orc.n_blocks(n, bk)), seed + 7)
    s = 1 / math.sqrt(d)
    g = orc.backward(q, k, v, w, mask, dout, bq, bk, s)
    eps = 1e-6
    for name, arr in (("dq", q), ("dk", k), ("dv", v), ("dproj", w)):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(q, k, v, w, mask, dout, bq, bk, s)
            arr[idx] = orig - eps
            lm = loss(q, k, v, w, mask, dout, bq, bk, s)
            arr[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g[name], num, rtol=2e-6, atol=2e-7, err_msg=name)


@pytest.mark.parametrize("n,d,bq,bk,seed", [(40, 6, 8, 8, 10), (37, 5, 16, 8, 11)])
def test_backward_matches_autograd_of_token_formulation(n, d, bq, bk, seed):
    B, H = 1, 2
    q, k, v = (rnd((B, H, n, d), seed + i) for i in range(3))
    w = rnd((d, d), seed + 5, 1 / 8)
    dout = rnd((B, H, n, d), seed + 6)
    mask = random_mask((B, H, orc.n_blocks(n, bq), orc.n_blocks(n, bk)), seed + 7)
    s = 1 / math.sqrt(d)
    g = orc.backward(q, k, v, w, mask, dout, bq, bk, s)
    tq, tk, tv, tw = (torch.tensor(a, requires_grad=True) for a in (q, k, v, w))
    out = torch_token_forward(tq, tk, tv, tw, mask, bq, bk, s)
    (out * torch.tensor(dout)).sum().backward()
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv), ("dproj", tw)):
        np.testing.assert_allclose(g[name], t.grad.numpy(), rtol=1e-10, atol=1e-11,
                                   err_msg=name)


def test_all_critical_gradient_is_dense_attention_gradient():
    B, H, N, d = 1, 1, 24, 4
    q, k, v = (rnd((B, H, N, d), 20 + i) for i in range(3))
    dout = rnd((B, H, N, d), 23)
    w = rnd((d, d), 24)
    mask = np.full((B, H, 3, 3), 2, dtype=np.int8)
    g = orc.backward(q, k, v, w, mask, dout, 8, 8)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    (o * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(g["dq"], tq.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(g["dk"], tk.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(g["dv"], tv.grad.numpy(), rtol=1e-11, atol=1e-12)
    assert (g["dproj"] == 0).all()


def test_all_negligible_gradients_are_zero():
    B, H, N, d = 1, 1, 16, 3
    q, k, v = (rnd((B, H, N, d), 30 + i) for i in range(3))
    mask = np.zeros((B, H, 2, 2), dtype=np.int8)
    g = orc.backward(q, k, v, rnd((d, d), 33), mask, rnd((B, H, N, d), 34), 8, 8)
    for name in ("dq", "dk", "dv", "dproj"):
        assert (g[name] == 0).all()
