"""The seeded input generator: reproducible, correctly shaped, locally
correlated (spatio-temporally smooth), and bf16-exact where asked."""

import numpy as np
import torch

from block_sparse_linear_mean_b200 import synth


def test_reflect_index_half_sample_symmetric():
    n = 4
    assert [synth.reflect_index(i, n) for i in range(-3, 8)] == [2, 1, 0, 0, 1, 2, 3, 3, 2, 1, 0]


def test_gaussian_operator_rows_sum_to_one():
    for n in (4, 21, 64):
        m = synth.gaussian_operator(n, 3.0)
        np.testing.assert_allclose(m.sum(dim=1).numpy(), 1.0, rtol=1e-12)


def test_inputs_reproducible_and_shaped():
    wl = synth.small_case(d=16, grid=(2, 4, 10), H=2, dtype="bf16")
    a = synth.make_inputs(wl, seed=3, with_dout=True)
    b = synth.make_inputs(wl, seed=3, with_dout=True)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v), (a.proj, b.proj), (a.dout, b.dout)):
        assert torch.equal(x, y)
    assert a.q.shape == (1, 2, 80, 16) and a.q.dtype == torch.bfloat16
    assert a.proj.shape == (16, 16) and a.proj.dtype == torch.float32
    c = synth.make_inputs(wl, seed=4)
    assert not torch.equal(a.q, c.q)


def test_head_subset_equals_prefix_of_full_draw():
    wl = synth.small_case(d=8, grid=(2, 3, 8), H=3)
    full = synth.make_inputs(wl, seed=1)
    sub = synth.make_inputs(wl, seed=1, heads=2)
    assert torch.equal(full.q[:, :2], sub.q)
    assert torch.equal(full.v[:, :2], sub.v)


def test_queries_and_keys_are_locally_correlated():
    wl = synth.small_case(d=32, grid=(4, 16, 16), H=1, noise=0.5)
    x = synth.make_inputs(wl, seed=0)
    q = x.q[0, 0].double()
    k = x.k[0, 0].double()
    g = q.reshape(4, 16, 16, 32)
    cos = torch.nn.functional.cosine_similarity
    # neighbouring columns are strongly correlated, columns 8 apart much less
    # (Gaussian smoothing with sigma = 3 grid steps)
    near = cos(g[:, :, :-1], g[:, :, 1:], dim=-1).mean()
    far = cos(g[:, :, :-8], g[:, :, 8:], dim=-1).mean()
    assert near > 0.6 and far < near - 0.3
    # q and k share the smooth field
    same = torch.nn.functional.cosine_similarity(q, k, dim=1).mean()
    assert same > 0.6
