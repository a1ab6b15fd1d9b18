"""The Flex Attention export on the GPU: the BlockMask built from the lists
the CUDA classifier wrote marks exactly the critical blocks, and PyTorch's
eager Flex attention with it agrees with the library's sparse attention."""

import warnings

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import assert_close, gpu_inputs, to_np

pytestmark = pytest.mark.gpu


def test_flex_export_of_gpu_lists():
    from torch.nn.attention.flex_attention import flex_attention
    wl = synth.small_case(d=128, grid=(1, 4, 100), dtype="bf16", frac_crit=0.3, frac_marg=0.2)
    x, t = gpu_inputs(wl, seed=31)
    p = sla.params_from(t["q"], wl)
    m = sla.build_mask(p, t["q"], t["k"])
    f = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], m["rows"], save_for_backward=True)
    bm = sla.flex_block_mask(p, m["mask"], m["rows"])
    torch.cuda.synchronize()
    dense = bm.to_dense().cpu().numpy()
    np.testing.assert_array_equal(dense, (m["mask"].cpu().numpy() == sla.CRITICAL).astype(dense.dtype))
    q, k, v = (t[n].float() for n in ("q", "k", "v"))
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        o = flex_attention(q, k, v, block_mask=bm)
    torch.cuda.synchronize()
    # the library's O_s (bf16 P) against Flex's fp32 attention on the same
    # bf16-valued inputs: the bf16 parity bound
    assert_close(to_np(f["o_s"]), to_np(o).astype(np.float64), wl.dtype, "flex o_s")
