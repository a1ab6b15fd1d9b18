"""GPU parity at oracle-sized shapes: every step of the CUDA path, called
through the C ABI, against the float64 oracle on the same seeded inputs.
Shapes span several tiles and a ragged tail block."""

import math

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import (assert_close, compare_masks, expected_cols, expected_rows,
                      feed_mask, gpu_inputs, lists_from_gpu, oracle_mask, to_np)
from oracle import sla_oracle as orc

pytestmark = pytest.mark.gpu

CASES = {
    # fp32 mode (1e-4), d = 64, 16 blocks of 64 with a 40-token tail
    "f32_d64_topk": synth.small_case(d=64, grid=(2, 5, 100), dtype="f32"),
    # bf16, d = 128, 64/64, ragged
    "bf16_d128_topk": synth.small_case(d=128, grid=(2, 5, 100), dtype="bf16"),
    # odd number of query blocks (15), key blocks of 128
    "bf16_bq64_bk128": synth.small_case(d=128, grid=(3, 3, 100), dtype="bf16",
                                        block_q=64, block_k=128, frac_crit=0.2,
                                        frac_marg=0.3),
    # query blocks of 128, key blocks of 64, CDF with a marginal fraction
    "bf16_bq128_cdf": synth.small_case(d=128, grid=(2, 5, 110), dtype="bf16",
                                       block_q=128, block_k=64, mode="cdf",
                                       thr=0.2, frac_marg=0.1),
    # fp32, CDF only (NABLA-style), 128/128
    "f32_d128_cdf": synth.small_case(d=128, grid=(1, 7, 111), dtype="f32",
                                     block_q=128, block_k=128, mode="cdf",
                                     thr=0.3, frac_marg=0.0),
    # bf16, d = 64, longer
    "bf16_d64_long": synth.small_case(d=64, grid=(4, 10, 50), dtype="bf16",
                                      frac_crit=0.1, frac_marg=0.2),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    wl = CASES[request.param]
    x, t = gpu_inputs(wl, seed=11, with_dout=True)
    ref = oracle_mask(wl, x)
    return request.param, wl, x, t, ref


def test_mask_matches_oracle(case):
    name, wl, x, t, ref = case
    p = sla.params_from(t["q"], wl)
    ws = sla.workspace(p, sla.SLA_OP_MASK, "cuda")
    got = sla.build_mask(p, t["q"], t["k"], want_scores=True, want_cols=True, ws=ws)
    torch.cuda.synchronize()
    assert sla.check_device_status(ws) == sla.SLA_OK
    scores = to_np(got["scores"])
    np.testing.assert_allclose(scores, ref["scores"], rtol=2e-5, atol=1e-7)
    mask = got["mask"].cpu().numpy()
    ndiff, nties = compare_masks(mask, ref["mask"], ref["margins"])
    print(f"{name}: rows differing {ndiff}, oracle tie rows {nties}, "
          f"GPU tie count {int(got['ties'].item())}")
    # lists are the mask's, ascending
    nrows = mask.shape[0] * mask.shape[1] * mask.shape[2]
    assert lists_from_gpu(got["rows"], nrows, mask.shape[3]) == expected_rows(mask)
    ncols = mask.shape[0] * mask.shape[1] * mask.shape[3]
    assert lists_from_gpu(got["cols"], ncols, mask.shape[2]) == expected_cols(mask)


def test_classifier_alone_is_exact_on_given_scores(case):
    # The oracle's scores, rounded once to fp32, are classified by the GPU
    # (sla_classify_scores) and by the oracle on the very same fp32 values:
    # top-k must agree bit for bit; the CDF decision may differ only where a
    # tail sum lies within 1e-12 of thr.
    name, wl, x, t, ref = case
    p = sla.params_from(t["q"], wl)
    s32 = ref["scores"].astype(np.float32)
    got = sla.classify_scores(p, torch.from_numpy(s32).cuda(), want_cols=True)
    torch.cuda.synchronize()
    mask_ref, margins = orc.classify(s32.astype(np.float64), wl.mode, wl.frac_crit,
                                     wl.frac_marg, wl.thr)
    mask = got["mask"].cpu().numpy()
    if wl.mode == "topk":
        np.testing.assert_array_equal(mask, mask_ref)
    else:
        diff = (mask != mask_ref).any(axis=-1)
        assert not (diff & (margins > 1e-12)).any()
    ncols = mask.shape[0] * mask.shape[1] * mask.shape[3]
    assert lists_from_gpu(got["cols"], ncols, mask.shape[2]) == expected_cols(mask)


def test_mask_lists_from_oracle_mask(case):
    name, wl, x, t, ref = case
    p = sla.params_from(t["q"], wl)
    _, rows, cols = feed_mask(p, ref["mask"])
    torch.cuda.synchronize()
    m = ref["mask"]
    nrows = m.shape[0] * m.shape[1] * m.shape[2]
    ncols = m.shape[0] * m.shape[1] * m.shape[3]
    assert lists_from_gpu(rows, nrows, m.shape[3]) == expected_rows(m)
    assert lists_from_gpu(cols, ncols, m.shape[2]) == expected_cols(m)


@pytest.mark.parametrize("simt", [False, True])
def test_forward_matches_oracle_with_oracle_mask(case, simt):
    name, wl, x, t, ref = case
    if simt and wl.dtype == "f32":
        pytest.skip("fp32 always runs the SIMT kernels")
    p = sla.params_from(t["q"], wl, simt=simt)
    _, rows, _ = feed_mask(p, ref["mask"])
    f = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], rows, save_for_backward=True)
    torch.cuda.synchronize()
    st = sla.check_device_status(f["ws"])
    assert st == sla.SLA_OK, sla.status_string(st)
    o = orc.forward(x.q, x.k, x.v, x.proj, ref["mask"], wl.block_q, wl.block_k)
    res = {}
    for key in ("o_s", "o_lin", "out"):
        res[key] = assert_close(to_np(f[key]), o[key], wl.dtype, f"{name}.{key}",
                                stored_bf16=(key == "out"))
    lse = to_np(f["lse"])
    fin = np.isfinite(o["lse"])
    np.testing.assert_array_equal(np.isfinite(lse), fin)
    res["lse"] = assert_close(lse[fin], o["lse"][fin], wl.dtype, f"{name}.lse")
    print(name, "simt" if simt else "default", {k: f"{v[0]:.2e}/{v[1]:.2e}" for k, v in res.items()})


@pytest.mark.parametrize("simt", [False, True], ids=["default", "simt"])
def test_backward_matches_oracle(case, simt):
    name, wl, x, t, ref = case
    if simt and wl.dtype == "f32":
        pytest.skip("fp32 always runs the SIMT kernels")
    p = sla.params_from(t["q"], wl, simt=simt)
    _, rows, cols = feed_mask(p, ref["mask"])
    f = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], rows, save_for_backward=True)
    g = sla.backward(p, t["q"], t["k"], t["v"], t["proj"], t["dout"], rows, cols, f)
    torch.cuda.synchronize()
    st = sla.check_device_status(g["ws"])
    assert st == sla.SLA_OK, sla.status_string(st)
    o = orc.backward(x.q, x.k, x.v, x.proj, ref["mask"], x.dout, wl.block_q, wl.block_k)
    res = {}
    for key in ("dq", "dk", "dv", "dproj"):
        res[key] = assert_close(to_np(g[key]), o[key], wl.dtype, f"{name}.{key}", rel=True)
    print(name, "simt" if simt else "default", {k: f"{v[0]:.2e}/{v[1]:.2e}" for k, v in res.items()})


# ---------------------------------------------------------------- edge cases


def _run_with_mask(wl, mask_np, seed=3):
    x, t = gpu_inputs(wl, seed=seed, with_dout=True)
    p = sla.params_from(t["q"], wl)
    _, rows, cols = feed_mask(p, mask_np)
    f = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], rows, save_for_backward=True)
    g = sla.backward(p, t["q"], t["k"], t["v"], t["proj"], t["dout"], rows, cols, f)
    torch.cuda.synchronize()
    return x, f, g


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_all_critical_equals_dense_attention(dtype):
    wl = synth.small_case(d=64, grid=(1, 3, 100), dtype=dtype, H=2)
    nqb = nkb = math.ceil(wl.N / 64)
    mask = np.full((1, 2, nqb, nkb), 2, dtype=np.int8)
    x, f, g = _run_with_mask(wl, mask)
    ref = torch.nn.functional.scaled_dot_product_attention(
        x.q.double(), x.k.double(), x.v.double()).numpy()
    assert_close(to_np(f["out"]), ref, dtype, "dense", stored_bf16=True)


def test_all_negligible_gives_zero_and_neg_inf():
    wl = synth.small_case(d=128, grid=(1, 2, 100), dtype="bf16", H=1)
    mask = np.zeros((1, 1, 4, 4), dtype=np.int8)
    x, f, g = _run_with_mask(wl, mask)
    assert (f["out"] == 0).all() and (f["o_s"] == 0).all()
    assert torch.isneginf(f["lse"]).all()
    for key in ("dq", "dk", "dv", "dproj"):
        assert (g[key] == 0).all(), key


@pytest.mark.parametrize("n", [1, 50, 64, 65, 127])
def test_single_and_ragged_blocks(n):
    wl = synth.small_case(d=64, grid=(1, 1, n), dtype="f32", H=2,
                          frac_crit=0.5, frac_marg=0.5)
    x, t = gpu_inputs(wl, seed=5)
    ref = oracle_mask(wl, x)
    p = sla.params_from(t["q"], wl)
    got = sla.build_mask(p, t["q"], t["k"])
    f = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], got["rows"], save_for_backward=True)
    torch.cuda.synchronize()
    compare_masks(got["mask"].cpu().numpy(), ref["mask"], ref["margins"])
    o = orc.forward(x.q, x.k, x.v, x.proj, got["mask"].cpu().numpy(), 64, 64)
    assert_close(to_np(f["out"]), o["out"], "f32", f"n={n}")


def test_key_shift_invariance_on_gpu():
    # adding one vector to every key leaves scores, mask and O_s unchanged
    wl = synth.small_case(d=64, grid=(1, 4, 100), dtype="f32", H=2)
    x, t = gpu_inputs(wl, seed=8)
    p = sla.params_from(t["q"], wl)
    c = torch.randn(64, generator=torch.Generator().manual_seed(1)).cuda()
    a = sla.build_mask(p, t["q"], t["k"], want_scores=True)
    b = sla.build_mask(p, t["q"], t["k"] + c, want_scores=True)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_np(a["scores"]), to_np(b["scores"]), rtol=1e-4, atol=1e-7)


def test_device_status_ok_after_calls():
    wl = synth.small_case(d=128, grid=(1, 2, 100), dtype="bf16", H=1)
    x, t = gpu_inputs(wl, seed=1)
    p = sla.params_from(t["q"], wl)
    m = sla.build_mask(p, t["q"], t["k"])
    f = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], m["rows"])
    assert sla.check_device_status(f["ws"]) == sla.SLA_OK


def test_bf16_forward_runs_tensor_core_kernel():
    for name in ("sla_1p3b", "nabla_14b", "long_clip"):
        p = sla.params_for(synth.WORKLOADS[name])
        assert sla.sla_forward_uses_tensor_cores(p) == 1, name
    p = sla.params_for(synth.WORKLOADS["tiny"])
    assert sla.sla_forward_uses_tensor_cores(p) == 0        # fp32 mode: SIMT
    p = sla.params_for(synth.WORKLOADS["sla_1p3b"], simt=True)
    assert sla.sla_forward_uses_tensor_cores(p) == 0


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_batch_of_two_matches_oracle(dtype, d):
    # B = 2: every kernel indexes (batch, head) pairs as one flat index
    wl = synth.small_case(d=d, grid=(2, 4, 100), H=2, B=2, dtype=dtype, frac_crit=0.2,
                          frac_marg=0.2)
    x, t = gpu_inputs(wl, seed=17, with_dout=True)
    ref = oracle_mask(wl, x)
    p = sla.params_from(t["q"], wl)
    m = sla.build_mask(p, t["q"], t["k"], want_scores=True)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_np(m["scores"]), ref["scores"], rtol=2e-5, atol=1e-7)
    compare_masks(m["mask"].cpu().numpy(), ref["mask"], ref["margins"])
    _, rows, cols = feed_mask(p, ref["mask"])
    f = sla.forward(p, t["q"], t["k"], t["v"], t["proj"], rows, save_for_backward=True)
    g = sla.backward(p, t["q"], t["k"], t["v"], t["proj"], t["dout"], rows, cols, f)
    torch.cuda.synchronize()
    assert sla.check_device_status(g["ws"]) == sla.SLA_OK
    o = orc.forward(x.q, x.k, x.v, x.proj, ref["mask"], wl.block_q, wl.block_k)
    assert_close(to_np(f["out"]), o["out"], dtype, "B2 out", stored_bf16=True)
    gr = orc.backward(x.q, x.k, x.v, x.proj, ref["mask"], x.dout, wl.block_q, wl.block_k)
    for key in ("dq", "dk", "dv", "dproj"):
        assert_close(to_np(g[key]), gr[key], dtype, f"B2 {key}", rel=True)
