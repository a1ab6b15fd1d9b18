"""The workspace-free sparse attention entry point.

Callers that are handed only a stream and their buffers (runtime plugins
without an allocator, loops that must not allocate) use
sla_sparse_attention_noalloc, whose scratch is a static device array inside
the library.  Called through the C ABI twice in a row, it must give exactly
what the workspace-based sla_sparse_attention gives on the same inputs (the
same kernel runs on the same plan, so the results agree bit for bit, which is
inside the parity tolerances of the other tests), with and without a status
word of the caller's, and refuse problems whose scratch would exceed the
array.  This file is collected last on purpose."""

import math

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import assert_close, gpu_inputs, to_np

pytestmark = pytest.mark.gpu


def _workspace_reference(p, t, rows):
    ws = sla.workspace(p, sla.SLA_OP_FORWARD, "cuda")
    o_s = torch.empty(t["q"].shape, dtype=torch.float32, device="cuda")
    lse = torch.empty(t["q"].shape[:-1], dtype=torch.float32, device="cuda")
    st = sla.sla_sparse_attention(p, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
                                  rows.c(), o_s.data_ptr(), lse.data_ptr(), ws.data_ptr(),
                                  ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == sla.SLA_OK
    return o_s, lse


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    wl = synth.small_case(d=128 if dtype == "bf16" else 64, grid=(2, 5, 100), dtype=dtype)
    x, t = gpu_inputs(wl, seed=21)
    p = sla.params_from(t["q"], wl)
    m = sla.build_mask(p, t["q"], t["k"])
    ref_o, ref_l = _workspace_reference(p, t, m["rows"])
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    # two calls with a status word of the caller's, then two that leave the
    # status word in the library's array
    for call in range(4):
        o_s = torch.full(t["q"].shape, float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full(t["q"].shape[:-1], float("nan"), dtype=torch.float32, device="cuda")
        status = torch.full((4,), -1, dtype=torch.int32, device="cuda") if call < 2 else None
        st = sla.sla_sparse_attention_noalloc(p, t["q"].data_ptr(), t["k"].data_ptr(),
                                              t["v"].data_ptr(), m["rows"].c(),
                                              o_s.data_ptr(), lse.data_ptr(),
                                              status.data_ptr() if status is not None else None,
                                              stream)
        assert st == sla.SLA_OK, sla.status_string(st)
        torch.cuda.synchronize()
        if status is not None:
            assert int(status[0].item()) == sla.SLA_OK
        assert torch.equal(o_s, ref_o), f"noalloc o_s call {call}"
        assert torch.equal(lse, ref_l), f"noalloc lse call {call}"
        assert_close(to_np(o_s), to_np(ref_o), dtype, f"noalloc o_s call {call}")


def test_noalloc_refuses_problems_beyond_its_scratch():
    # the long-clip shape needs ~590 MB of plan; the call is refused on the
    # host before anything is launched (the small buffers are never touched)
    wl = synth.small_case(d=128, grid=(1, 2, 100), dtype="bf16", H=1)
    x, t = gpu_inputs(wl, seed=1)
    p = sla.params_for(synth.WORKLOADS["long_clip"])
    dummy = sla.BlockLists.empty(4, 4, "cuda")
    out = torch.empty(64, dtype=torch.float32, device="cuda")
    st = sla.sla_sparse_attention_noalloc(p, t["q"].data_ptr(), t["k"].data_ptr(),
                                          t["v"].data_ptr(), dummy.c(), out.data_ptr(),
                                          out.data_ptr(), None,
                                          torch.cuda.current_stream().cuda_stream)
    assert st == sla.SLA_ERR_WORKSPACE
