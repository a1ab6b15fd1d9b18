"""Mask quality on the GPU (sla_block_importance, sla_mask_recall) against the
oracle's max-pooled dense attention and recall counts, plus the measured
recall of the pooled-score masks on the synthetic fields."""

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import gpu_inputs, to_np
from oracle import sla_oracle as orc

pytestmark = pytest.mark.gpu

CASES = {
    # bf16, d = 128, blocks 64 with a 16-token tail (two rows per lane)
    "bf16_d128_topk": synth.small_case(d=128, grid=(1, 4, 100), dtype="bf16",
                                       frac_crit=0.25, frac_marg=0.25),
    # fp32, d = 64, 128-row query blocks (four rows per lane), 64-key blocks
    "f32_d64_q128": synth.small_case(d=64, grid=(1, 5, 100), dtype="f32", block_q=128,
                                     block_k=64, frac_crit=0.2, frac_marg=0.1),
    # bf16, d = 128, CDF selection, 128-key blocks with a tail
    "bf16_cdf_k128": synth.small_case(d=128, grid=(1, 3, 111), dtype="bf16", block_q=64,
                                      block_k=128, mode="cdf", thr=0.3, frac_marg=0.0),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    wl = CASES[request.param]
    x, t = gpu_inputs(wl, seed=21)
    p = sla.params_from(t["q"], wl)
    imp = sla.block_importance(p, t["q"], t["k"])
    m = sla.build_mask(p, t["q"], t["k"])
    torch.cuda.synchronize()
    return request.param, wl, x, t, p, imp, m


def test_importance_matches_oracle(case):
    name, wl, x, t, p, imp, m = case
    ref = orc.max_pooled_attention(x.q, x.k, wl.block_q, wl.block_k)
    got = to_np(imp)
    # fp32 scores and exponentials against float64
    np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-7)


def test_recall_counts_are_exact(case):
    # the GPU counts equal the oracle's on the very same fp32 importance
    name, wl, x, t, p, imp, m = case
    got = sla.mask_recall(p, m["mask"], imp)
    ref = orc.mask_recall_counts(m["mask"].cpu().numpy(), to_np(imp))
    assert (got["critical_hits"], got["critical_total"], got["kept_hits"],
            got["kept_total"]) == ref
    print(f"{name}: recall critical {got['recall_critical']:.3f}, kept {got['recall_kept']:.3f}")


def test_recall_of_the_reference_selection_is_full():
    # a mask chosen by the importance itself keeps its whole reference set
    wl = CASES["bf16_d128_topk"]
    x, t = gpu_inputs(wl, seed=22)
    p = sla.params_from(t["q"], wl)
    imp = sla.block_importance(p, t["q"], t["k"])
    own = sla.classify_scores(p, imp)
    got = sla.mask_recall(p, own["mask"], imp)
    assert got["critical_hits"] == got["critical_total"] > 0
    assert got["kept_hits"] == got["kept_total"] > got["critical_total"]


def test_recall_at_a_longer_sequence():
    # the measurement on a 4096-token field: the GPU's counts equal the
    # oracle's on the GPU importance, and the importance matches the oracle
    wl = synth.small_case(d=128, grid=(2, 16, 128), H=2, dtype="bf16",
                          frac_crit=0.05, frac_marg=0.10)
    x, t = gpu_inputs(wl, seed=23)
    p = sla.params_from(t["q"], wl)
    imp = sla.block_importance(p, t["q"], t["k"])
    m = sla.build_mask(p, t["q"], t["k"])
    got = sla.mask_recall(p, m["mask"], imp)
    imp_np = to_np(imp)
    ref = orc.mask_recall_counts(m["mask"].cpu().numpy(), imp_np)
    assert (got["critical_hits"], got["critical_total"], got["kept_hits"],
            got["kept_total"]) == ref
    np.testing.assert_allclose(imp_np, orc.max_pooled_attention(x.q, x.k, 64, 64),
                               rtol=1e-4, atol=1e-7)
    print(f"N=4096: recall critical {got['recall_critical']:.3f}, "
          f"kept {got['recall_kept']:.3f}")
