"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
binding and the oracle on the same seeded inputs, and compare."""

import math

import numpy as np
import torch

from block_sparse_linear_mean_b200 import sla, synth
from oracle import sla_oracle as orc

# Tolerances of the workload statement: bf16 inputs with fp32 accumulation
# (max abs 2e-2, mean abs 2e-3) and fp32 mode (1e-4).  Gradients use the same
# bounds on the error relative to the largest reference magnitude.
BF16_MAX, BF16_MEAN, F32_MAX = 2e-2, 2e-3, 1e-4
TIE_EPS = 1e-5


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got, ref):
    e = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    return float(e.max()) if e.size else 0.0, float(e.mean()) if e.size else 0.0


# Round-to-nearest-even to bf16 moves a value by at most half a unit in the
# last of its 8 significant bits: 2^-8 of the value at the bottom of a binade.
BF16_HALF_ULP_REL = 2.0 ** -8


def assert_close(got, ref, dtype, what, rel=False, stored_bf16=False):
    """Tolerances of the workload statement.  ``stored_bf16``: the value is
    an output stored in bf16, so each element may additionally carry its own
    output rounding (<= 2^-8 |ref|) on top of the computation's error."""
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    scale = max(1e-30, float(np.abs(ref).max())) if rel else 1.0
    err = np.abs(got - ref) / scale
    mx, mean = (float(err.max()), float(err.mean())) if err.size else (0.0, 0.0)
    if dtype == "f32":
        assert mx <= F32_MAX, f"{what}: max {mx:.3g} > {F32_MAX}"
    else:
        q = BF16_HALF_ULP_REL * np.abs(ref) / scale if stored_bf16 else np.zeros_like(ref)
        over = err - (BF16_MAX + q)
        assert (over <= 0).all(), f"{what}: max {mx:.3g} > {BF16_MAX} (+ bf16 output rounding)"
        lim = BF16_MEAN + (float(q.mean()) if q.size else 0.0)
        assert mean <= lim, f"{what}: mean {mean:.3g} > {lim:.3g}"
    return mx, mean


def gpu_inputs(wl, seed=0, with_dout=False):
    x = synth.make_inputs(wl, seed=seed, device="cpu", with_dout=with_dout)
    dev = torch.device("cuda")
    out = dict(q=x.q.to(dev), k=x.k.to(dev), v=x.v.to(dev), proj=x.proj.to(dev))
    if with_dout:
        out["dout"] = x.dout.to(dev)
    return x, out


def oracle_mask(wl, x):
    return orc.build_mask(x.q, x.k, wl.block_q, wl.block_k, wl.mode, wl.frac_crit,
                          wl.frac_marg, wl.thr)


def compare_masks(gpu_mask, ref_mask, margins):
    """Rows of the mask must match bit for bit, except rows whose decisive
    margin is within TIE_EPS (counted and returned)."""
    g = np.asarray(gpu_mask)
    r = np.asarray(ref_mask)
    diff_rows = (g != r).any(axis=-1)
    tie_rows = np.asarray(margins) <= TIE_EPS
    bad = diff_rows & ~tie_rows
    assert not bad.any(), f"{int(bad.sum())} non-tie rows differ, e.g. {np.argwhere(bad)[:3]}"
    return int(diff_rows.sum()), int(tie_rows.sum())


def lists_from_gpu(bl, nrows, width):
    cc = bl.crit_cnt.cpu().numpy()
    ci = bl.crit_idx.cpu().numpy().reshape(nrows, width)
    mc = bl.marg_cnt.cpu().numpy()
    mi = bl.marg_idx.cpu().numpy().reshape(nrows, width)
    return ([ci[r, :cc[r]].tolist() for r in range(nrows)],
            [mi[r, :mc[r]].tolist() for r in range(nrows)])


def expected_rows(mask):
    m = np.asarray(mask)
    rows = m.reshape(-1, m.shape[-1])
    return ([np.nonzero(r == 2)[0].tolist() for r in rows],
            [np.nonzero(r == 1)[0].tolist() for r in rows])


def expected_cols(mask):
    m = np.asarray(mask)
    B, H, nqb, nkb = m.shape
    crit, marg = [], []
    for b in range(B):
        for h in range(H):
            for j in range(nkb):
                crit.append(np.nonzero(m[b, h, :, j] == 2)[0].tolist())
                marg.append(np.nonzero(m[b, h, :, j] == 1)[0].tolist())
    return crit, marg


def feed_mask(p, mask_np):
    """Upload a mask (e.g. the oracle's) and build its CSR/CSC lists on GPU."""
    m = torch.as_tensor(np.asarray(mask_np, dtype=np.int8)).cuda()
    rows, cols = sla.mask_lists(p, m)
    return m, rows, cols
