"""Failure detection without a GPU fault: every device-side wait of the
tensor-core kernel is bounded.  A test flag makes one CTA withhold a K/V tile
load (a barrier nothing will complete) and shortens the wait limit to ~1e7
cycles; the call must then report SLA_ERR_TIMEOUT through the status word,
and the context must stay usable for the next, normal call."""

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import gpu_inputs, oracle_mask, feed_mask

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    wl = synth.small_case(d=128, grid=(1, 4, 100), dtype="bf16", H=1)
    x, t = gpu_inputs(wl, seed=2)
    p = sla.params_from(t["q"], wl)
    m = sla.build_mask(p, t["q"], t["k"])
    pd = sla.params_from(t["q"], wl)
    pd.flags = sla.SLA_FLAG_DEBUG_TIMEOUT
    assert sla.sla_forward_uses_tensor_cores(pd) == 1
    f = sla.forward(pd, t["q"], t["k"], t["v"], t["proj"], m["rows"])
    assert sla.check_device_status(f["ws"]) == sla.SLA_ERR_TIMEOUT
    # the next normal call on the same context works and resets the status
    g = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], m["rows"])
    assert sla.check_device_status(g["ws"]) == sla.SLA_OK
    assert torch.isfinite(g["out"].float()).all()
