"""The benchmark's host-side bookkeeping on CPU: the head groups of the mask
step (the library's 64 MB score slab), the algorithmic bytes of the two
memory-bound stages, the choice of the tensor-core peak by the timed
region's length, the launch counts and the head-restricted workloads."""

import math
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_sparse_linear_mean_b200 import synth  # noqa: E402

W = synth.WORKLOADS


@pytest.mark.parametrize("name,groups", [("sla_1p3b", 1), ("finetune", 1), ("tiny", 1),
                                         ("nabla_14b", 4), ("long_clip", 10)])
def test_mask_groups_follow_the_slab(name, groups):
    # 1.3B: 12 heads of 512 x 512 scores (1 MiB each) in one group; 14B: 11
    # heads of 1182 x 1182 (5.3 MiB) per group; long clip: 4 heads of
    # 1920 x 1920 (14 MiB) per group
    assert bench.mask_groups(W[name]) == groups


def test_stage_bytes_count_reads_writes_and_lists():
    wl = W["sla_1p3b"]
    nqb = nkb = 512
    mask = np.zeros((1, 12, nqb, nkb), dtype=np.int8)
    mask[..., :26] = 2
    mask[..., 26:78] = 1
    mask_b, prep_b = bench.stage_bytes(wl, mask)
    qk = 2 * 12 * 32760 * 128 * 2
    listed = 12 * nqb * 78
    assert mask_b == qk + 12 * nqb * nkb + 4 * listed + 8 * 12 * nqb
    summ = 2 * 128 * 128 + 4 * 128
    assert prep_b == qk + 2 * 12 * nkb * summ + 12 * nqb * summ
    # fp32 or no linear branch: no prepare figure
    assert bench.stage_bytes(W["tiny"], np.zeros((1, 2, 16, 16), np.int8))[1] is None
    assert bench.stage_bytes(W["nabla_14b"], np.zeros((1, 40, 4, 4), np.int8))[1] is None


def test_stage_bytes_of_the_finetune_step_add_the_column_lists():
    mask = np.zeros((1, 12, 512, 512), dtype=np.int8)
    mask[..., :10] = 2
    a, _ = bench.stage_bytes(W["sla_1p3b"], mask)
    b, _ = bench.stage_bytes(W["finetune"], mask)
    assert b - a == 4 * int(np.count_nonzero(mask)) + 8 * 12 * 512


def test_tensor_peak_burst_under_a_second_sustained_above():
    peaks = {"bf16_tflops": 1679.3, "bf16_tflops_sustained": 1437.5}
    assert bench.tensor_peak(peaks, "measured", 0.04)[0] == 1679.3
    assert "burst" in bench.tensor_peak(peaks, "measured", 0.04)[1]
    assert bench.tensor_peak(peaks, "measured", 2.5)[0] == 1437.5
    assert "sustained" in bench.tensor_peak(peaks, "measured", 2.5)[1]


def test_launch_counts_grow_with_the_head_groups():
    one = bench.launches_per_step(W["sla_1p3b"], True, False)
    assert one == 1 + 2 + 1 + 3 + 1           # pool, logits + select, plan, linear, attention
    assert bench.launches_per_step(W["long_clip"], True, False) == one + 2 * 9
    assert bench.launches_per_step(W["nabla_14b"], True, False) == 1 + 2 * 4 + 1 + 1


def test_with_heads_restricts_the_workload():
    wl = bench.with_heads(W["long_clip"], 3)
    assert wl.H == 3 and wl.N == W["long_clip"].N and "first 3 heads" in wl.description
    assert bench.with_heads(W["long_clip"], None) is W["long_clip"]
    assert bench.with_heads(W["long_clip"], 40) is W["long_clip"]
    assert bench.mask_groups(wl) == 1


def test_effective_flops_count_kept_pairs_with_ragged_tails():
    # one head, N = 100 with blocks of 64: a full and a 36-token block
    wl = synth.small_case(d=64, grid=(1, 1, 100), H=1, dtype="f32", frac_crit=0.5,
                          frac_marg=0.0)
    mask = np.array([[[[2, 0], [2, 2]]]], dtype=np.int8)
    total, pairs, crit, lin, apply = bench.effective_flops(wl, mask)
    assert pairs == 64 * 64 + 36 * 64 + 36 * 36
    assert crit == 4 * 64 * pairs and lin == 0 and apply == 0 and total == crit
    assert math.isclose(bench.backward_flops(wl, mask)[0], 10 * 64 * pairs)
