"""GPU parity when the scores of later key blocks grow far past those of the
earlier ones.  The tensor-core forward computes each tile's exponentials
with the running maximum of the earlier tiles and raises it lazily (a rise
beyond 2^8 takes effect on the warpgroup's next tile, a jump beyond 2^64 in
the exp2 domain redoes the tile with its own maximum first).  Growing key
scales exercise the lazy raises; one late key block scaled far up
exercises the redo.  Same bounds as the other parity tests, against the
float64 oracle on the oracle's own mask."""

import numpy as np
import pytest
import torch

from block_sparse_linear_mean_b200 import sla, synth
from gpu_util import assert_close, feed_mask, oracle_mask, to_np
from oracle import sla_oracle as orc

pytestmark = pytest.mark.gpu


def scaled_inputs(wl, ramp, spike, seed=5):
    """Keys of block j scaled by 1 + ramp * j; the second-to-last key block
    additionally by `spike`.  The inputs stay in the workload dtype."""
    x = synth.make_inputs(wl, seed=seed, device="cpu")
    k = x.k.float()
    nkb = -(-wl.N // wl.block_k)
    for j in range(nkb):
        f = 1.0 + ramp * j
        if j == nkb - 2:
            f *= spike
        k[..., j * wl.block_k:(j + 1) * wl.block_k, :] *= f
    x.k = k.to(x.k.dtype)
    return x


CASES = {
    # rising maxima across the tiles: lazy raises only
    "ramp": (synth.small_case(d=128, grid=(2, 5, 100), dtype="bf16", frac_crit=0.6,
                              frac_marg=0.2), 0.6, 1.0),
    # rising maxima and one late block 40x up: scores ~10^3 past the running
    # maximum, beyond the one-pass guard
    "ramp_spike": (synth.small_case(d=128, grid=(2, 5, 100), dtype="bf16", frac_crit=0.6,
                                    frac_marg=0.2), 0.6, 40.0),
    # 128-key blocks, 128-row query blocks
    "spike_128": (synth.small_case(d=128, grid=(2, 5, 110), dtype="bf16", block_q=128,
                                   block_k=128, frac_crit=0.7, frac_marg=0.0), 0.3, 40.0),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_with_growing_scores(name):
    wl, ramp, spike = CASES[name]
    x = scaled_inputs(wl, ramp, spike)
    dev = torch.device("cuda")
    q, k, v, proj = (t.to(dev) for t in (x.q, x.k, x.v, x.proj))
    ref = oracle_mask(wl, x)
    p = sla.params_from(q, wl)
    assert sla.sla_forward_uses_tensor_cores(p) == 1
    _, rows, _ = feed_mask(p, ref["mask"])
    f = sla.forward(p, q, k, v, proj, rows, save_for_backward=True)
    torch.cuda.synchronize()
    st = sla.check_device_status(f["ws"])
    assert st == sla.SLA_OK, sla.status_string(st)
    o = orc.forward(x.q, x.k, x.v, x.proj, ref["mask"], wl.block_q, wl.block_k)
    # the spread the test is about: row maxima of the raw scores (log2
    # domain) across a row's critical blocks
    res = {}
    for key in ("o_s", "out"):
        res[key] = assert_close(to_np(f[key]), o[key], wl.dtype, f"{name}.{key}",
                                stored_bf16=(key == "out"))
    lse = to_np(f["lse"])
    fin = np.isfinite(o["lse"])
    np.testing.assert_array_equal(np.isfinite(lse), fin)
    # LSE grows with the scores; its error bound is relative to its size
    res["lse"] = assert_close(lse[fin], o["lse"][fin], wl.dtype, f"{name}.lse", rel=True)
    print(name, {k2: f"{v2[0]:.2e}/{v2[1]:.2e}" for k2, v2 in res.items()})


def test_spike_reaches_the_redo_range():
    """The spiked case's scores do jump past the one-pass guard: some row's
    critical-score maximum in the exp2 domain exceeds that of its first key
    block by more than 64."""
    wl, ramp, spike = CASES["ramp_spike"]
    x = scaled_inputs(wl, ramp, spike)
    ref = oracle_mask(wl, x)
    q = x.q.double()[0, 0]
    k = x.k.double()[0, 0]
    s = (q @ k.T) / np.sqrt(wl.d) * np.log2(np.e)
    bq, bk = wl.block_q, wl.block_k
    mask = ref["mask"][0, 0]
    best = 0.0
    for i in range(mask.shape[0]):
        crit = np.nonzero(mask[i] == 2)[0]
        if len(crit) < 2:
            continue
        rows = s[i * bq:(i + 1) * bq]
        first = rows[:, crit[0] * bk:(crit[0] + 1) * bk].max(dim=1).values
        top = torch.stack([rows[:, j * bk:(j + 1) * bk].max(dim=1).values for j in crit]).max(dim=0).values
        best = max(best, float((top - first).max()))
    assert best > 64.0, best
