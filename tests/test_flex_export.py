"""The Flex Attention export of a block mask (NABLA post: the method is
compatible with PyTorch's Flex Attention): the BlockMask built from the CSR
lists marks exactly the critical blocks, and PyTorch's eager Flex attention
with it reproduces the oracle's sparse attention."""

import warnings

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from oracle import sla_oracle as orc


def lists_of(mask):
    """CPU BlockLists from an oracle mask ``[B,H,Nqb,Nkb]``."""
    nkb = mask.shape[-1]
    crit, marg = orc.mask_lists(mask)
    bl = sla.BlockLists.empty(len(crit), nkb, "cpu")
    for r, (c, m) in enumerate(zip(crit, marg)):
        bl.crit_cnt[r] = len(c)
        bl.crit_idx[r, :len(c)] = torch.as_tensor(c, dtype=torch.int32)
        bl.marg_cnt[r] = len(m)
        bl.marg_idx[r, :len(m)] = torch.as_tensor(m, dtype=torch.int32)
    return bl


CASES = {
    # 64/64 blocks with a 40-token tail, top-k
    "topk_64": synth.small_case(d=64, grid=(1, 5, 100), frac_crit=0.3, frac_marg=0.2),
    # 64-row query blocks, 128-key blocks with a tail, CDF
    "cdf_64_128": synth.small_case(d=64, grid=(1, 3, 111), block_q=64, block_k=128,
                                   mode="cdf", thr=0.3, frac_marg=0.0),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_flex_block_mask_marks_the_critical_blocks(name):
    wl = CASES[name]
    x = synth.make_inputs(wl, seed=3, device="cpu")
    ref = orc.build_mask(x.q, x.k, wl.block_q, wl.block_k, wl.mode, wl.frac_crit,
                         wl.frac_marg, wl.thr)
    mask = torch.from_numpy(ref["mask"])
    p = sla.params_from(x.q, wl)
    bm = sla.flex_block_mask(p, mask, lists_of(ref["mask"]))
    dense = bm.to_dense().numpy()
    np.testing.assert_array_equal(dense, (ref["mask"] == orc.CRITICAL).astype(dense.dtype))


@pytest.mark.parametrize("name", sorted(CASES))
def test_flex_attention_with_the_export_matches_the_oracle(name):
    from torch.nn.attention.flex_attention import flex_attention
    wl = CASES[name]
    x = synth.make_inputs(wl, seed=4, device="cpu")
    ref = orc.build_mask(x.q, x.k, wl.block_q, wl.block_k, wl.mode, wl.frac_crit,
                         wl.frac_marg, wl.thr)
    mask = torch.from_numpy(ref["mask"])
    p = sla.params_from(x.q, wl)
    bm = sla.flex_block_mask(p, mask, lists_of(ref["mask"]))
    q, k, v = (t.double() for t in (x.q, x.k, x.v))
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        o = flex_attention(q, k, v, block_mask=bm)
    o_ref, _ = orc.sparse_attention(x.q, x.k, x.v, ref["mask"], wl.block_q, wl.block_k)
    np.testing.assert_allclose(o.numpy(), o_ref, rtol=1e-10, atol=1e-12)
