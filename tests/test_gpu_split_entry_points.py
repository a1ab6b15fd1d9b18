"""GPU parity of the two split entry points against the float64 oracle.

``sla_sparse_attention`` (the critical branch alone: NABLA post, point 4 --
attention only over the kept blocks) and ``sla_linear_combine`` (the
marginal branch and the combine: SLA post, list "the idea", item 3 --
intermediate blocks through linear attention, out = O_s + O_lin W) are
called through the C ABI with the oracle's mask fed in, on ragged shapes
that span several tiles, and compared element by element with the oracle at
the tolerances of the other parity tests."""

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import assert_close, feed_mask, gpu_inputs, oracle_mask, to_np
from oracle import sla_oracle as orc

pytestmark = pytest.mark.gpu

CASES = {
    # tcgen05 attention, 64/64 blocks, 1000 tokens (tail of 40)
    "bf16_d128_64_64": (synth.small_case(d=128, grid=(2, 5, 100), dtype="bf16"), False),
    # tcgen05 attention, 64-row query blocks over 128-token key blocks
    "bf16_d128_64_128": (synth.small_case(d=128, grid=(3, 3, 100), dtype="bf16", block_q=64,
                                          block_k=128, frac_crit=0.2, frac_marg=0.3), False),
    # 128-row query blocks (the linear apply kernel's BQ = 128 variant)
    "bf16_d128_128_64": (synth.small_case(d=128, grid=(2, 5, 110), dtype="bf16", block_q=128,
                                          block_k=64, frac_crit=0.2, frac_marg=0.2), False),
    # tcgen05 attention at d = 64 (linear branch on the SIMT kernels)
    "bf16_d64": (synth.small_case(d=64, grid=(4, 10, 50), dtype="bf16", frac_crit=0.1,
                                  frac_marg=0.2), False),
    # fp32 mode: SIMT everywhere, 1e-4
    "f32_d64": (synth.small_case(d=64, grid=(2, 5, 100), dtype="f32"), False),
    "f32_d128_cdf": (synth.small_case(d=128, grid=(1, 7, 111), dtype="f32", block_q=128,
                                      block_k=128, mode="cdf", thr=0.3, frac_marg=0.1), False),
    # bf16 inputs forced onto the SIMT kernels
    "bf16_d128_simt": (synth.small_case(d=128, grid=(2, 5, 100), dtype="bf16"), True),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    wl, simt = CASES[request.param]
    x, t = gpu_inputs(wl, seed=31)
    ref = oracle_mask(wl, x)
    o = orc.forward(x.q, x.k, x.v, x.proj, ref["mask"], wl.block_q, wl.block_k)
    return request.param, wl, simt, x, t, ref, o


def test_sparse_attention_matches_oracle(case):
    name, wl, simt, x, t, ref, o = case
    p = sla.params_from(t["q"], wl, simt=simt)
    _, rows, _ = feed_mask(p, ref["mask"])
    r = sla.sparse_attention(p, t["q"], t["k"], t["v"], rows)
    torch.cuda.synchronize()
    assert sla.check_device_status(r["ws"]) == sla.SLA_OK
    assert_close(to_np(r["o_s"]), o["o_s"], wl.dtype, f"{name}.o_s")
    lse = to_np(r["lse"])
    fin = np.isfinite(o["lse"])
    np.testing.assert_array_equal(np.isfinite(lse), fin)
    assert_close(lse[fin], o["lse"][fin], wl.dtype, f"{name}.lse")


def test_linear_combine_matches_oracle(case):
    # O_s is the oracle's (rounded to fp32), so out checks the linear branch
    # and the combine alone
    name, wl, simt, x, t, ref, o = case
    p = sla.params_from(t["q"], wl, simt=simt)
    _, rows, _ = feed_mask(p, ref["mask"])
    o_s = torch.from_numpy(o["o_s"].astype(np.float32)).cuda()
    r = sla.linear_combine(p, t["q"], t["k"], t["v"], t["proj"], rows, o_s, save_o_lin=True)
    torch.cuda.synchronize()
    assert sla.check_device_status(r["ws"]) == sla.SLA_OK
    assert_close(to_np(r["o_lin"]), o["o_lin"], wl.dtype, f"{name}.o_lin")
    assert_close(to_np(r["out"]), o["out"], wl.dtype, f"{name}.out", stored_bf16=True)


def test_split_entry_points_compose_to_the_forward(case):
    # sparse attention, then linear combine on its O_s, equals the oracle's
    # whole forward
    name, wl, simt, x, t, ref, o = case
    p = sla.params_from(t["q"], wl, simt=simt)
    _, rows, _ = feed_mask(p, ref["mask"])
    a = sla.sparse_attention(p, t["q"], t["k"], t["v"], rows)
    r = sla.linear_combine(p, t["q"], t["k"], t["v"], t["proj"], rows, a["o_s"])
    torch.cuda.synchronize()
    assert sla.check_device_status(r["ws"]) == sla.SLA_OK
    assert_close(to_np(r["out"]), o["out"], wl.dtype, f"{name}.out", stored_bf16=True)


def test_linear_combine_without_linear_branch_copies_o_s():
    wl = synth.small_case(d=128, grid=(1, 4, 100), dtype="bf16", frac_marg=0.0, H=1)
    x, t = gpu_inputs(wl, seed=4)
    p = sla.params_from(t["q"], wl)
    ref = oracle_mask(wl, x)
    _, rows, _ = feed_mask(p, ref["mask"])
    o_s = torch.randn(t["q"].shape, generator=torch.Generator().manual_seed(5)).cuda()
    r = sla.linear_combine(p, t["q"], t["k"], t["v"], t["proj"], rows, o_s, save_o_lin=True)
    torch.cuda.synchronize()
    assert torch.equal(r["out"], o_s.to(torch.bfloat16))
    assert (r["o_lin"] == 0).all()
