"""Failure detection without a GPU fault: every device-side wait of the
tensor-core kernels is bounded.  Under SLA_FLAG_DEBUG_TIMEOUT the chosen
kernel's first CTA withholds one tile load (a barrier nothing will complete)
and every wait limit drops to ~1.7e7 cycles; the call must then report
SLA_ERR_TIMEOUT through the status word, and the context must stay usable:
a normal call afterwards gives the same result, bit for bit, as one made
before the failure."""

import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import gpu_inputs

pytestmark = pytest.mark.gpu


def _debug(p, kernel):
    p.flags = sla.SLA_FLAG_DEBUG_TIMEOUT | sla.SLA_DEBUG_WITHHOLD(kernel)
    return p


def _setup(block_k=64, seed=2):
    wl = synth.small_case(d=128, grid=(1, 4, 100), dtype="bf16", H=1, block_k=block_k)
    x, t = gpu_inputs(wl, seed=seed, with_dout=True)
    p = sla.params_from(t["q"], wl)
    return wl, t, p


def test_attention_forward_wait_times_out_and_context_survives():
    wl, t, p = _setup()
    m = sla.build_mask(p, t["q"], t["k"])
    before = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], m["rows"])
    pd = _debug(sla.params_from(t["q"], wl), sla.SLA_WITHHOLD_ATTENTION)
    assert sla.sla_forward_uses_tensor_cores(pd) == 1
    f = sla.forward(pd, t["q"], t["k"], t["v"], t["proj"], m["rows"])
    assert sla.check_device_status(f["ws"]) == sla.SLA_ERR_TIMEOUT
    g = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], m["rows"])
    assert sla.check_device_status(g["ws"]) == sla.SLA_OK
    assert torch.equal(g["out"], before["out"])


def test_logits_wait_times_out_and_context_survives():
    wl, t, p = _setup()
    ws = sla.workspace(p, sla.SLA_OP_MASK, "cuda")
    before = sla.build_mask(p, t["q"], t["k"], want_scores=True, ws=ws)
    torch.cuda.synchronize()
    ref = before["scores"].clone()
    pd = _debug(sla.params_from(t["q"], wl), sla.SLA_WITHHOLD_LOGITS)
    sla.build_mask(pd, t["q"], t["k"], ws=ws)
    assert sla.check_device_status(ws) == sla.SLA_ERR_TIMEOUT
    after = sla.build_mask(p, t["q"], t["k"], want_scores=True, ws=ws)
    assert sla.check_device_status(ws) == sla.SLA_OK
    assert torch.equal(after["scores"], ref)
    assert torch.equal(after["mask"], before["mask"])


@pytest.mark.parametrize("kernel,block_k", [
    (sla.SLA_WITHHOLD_SUMMARIES, 64),    # persistent summaries (64-token key blocks)
    (sla.SLA_WITHHOLD_SUMMARIES, 128),   # one CTA per 128-token key block
    (sla.SLA_WITHHOLD_GATHER, 64),       # marginal sums H^M
], ids=["summaries64", "summaries128", "gather"])
def test_linear_branch_wait_times_out_and_context_survives(kernel, block_k):
    wl, t, p = _setup(block_k=block_k)
    m = sla.build_mask(p, t["q"], t["k"])
    before = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], m["rows"], save_for_backward=True)
    torch.cuda.synchronize()
    assert (m["rows"].marg_cnt > 0).any()
    pd = _debug(sla.params_from(t["q"], wl), kernel)
    f = sla.forward(pd, t["q"], t["k"], t["v"], t["proj"], m["rows"])
    assert sla.check_device_status(f["ws"]) == sla.SLA_ERR_TIMEOUT
    g = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], m["rows"], save_for_backward=True)
    assert sla.check_device_status(g["ws"]) == sla.SLA_OK
    assert torch.equal(g["out"], before["out"])
    assert torch.equal(g["o_lin"], before["o_lin"])


@pytest.mark.parametrize("kernel", [sla.SLA_WITHHOLD_BWD_DQ, sla.SLA_WITHHOLD_BWD_DKDV],
                         ids=["dq", "dkdv"])
def test_backward_wait_times_out_and_context_survives(kernel):
    wl, t, p = _setup()
    m = sla.build_mask(p, t["q"], t["k"], want_cols=True)
    f = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], m["rows"], save_for_backward=True)
    before = sla.backward(p, t["q"], t["k"], t["v"], t["proj"], t["dout"], m["rows"], m["cols"], f)
    torch.cuda.synchronize()
    pd = _debug(sla.params_from(t["q"], wl), kernel)
    b = sla.backward(pd, t["q"], t["k"], t["v"], t["proj"], t["dout"], m["rows"], m["cols"], f)
    assert sla.check_device_status(b["ws"]) == sla.SLA_ERR_TIMEOUT
    g = sla.backward(p, t["q"], t["k"], t["v"], t["proj"], t["dout"], m["rows"], m["cols"], f)
    assert sla.check_device_status(g["ws"]) == sla.SLA_OK
    for key in ("dq", "dk", "dv", "dproj"):
        assert torch.equal(g[key], before[key]), key

