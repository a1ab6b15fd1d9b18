"""Benchmark: hybrid block-sparse + linear attention on B200.

One step = one pass of the forward hot path over one synthetic batch:
sla_build_mask (pool, score, classify) + sla_forward_prepare (attention
plan; linear-branch summaries and their per-query-block sums) +
sla_attention_combine (critical-block attention, linear apply, projection
and sum, fused into one kernel on the tensor-core path).  The
default workload is the 1.3B-DiT-shaped SLA forward (B=1, H=12, N=32760,
d=128, bf16, blocks of 64, 5% critical / 10% marginal); ``--workload``
selects another.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

Multi-GPU (launched by torchrun): every rank runs its own independent problem
(its own batch element, seed = rank) -- weak scaling, no collective on the
data path; the only collectives are the timing barrier and the max over
ranks of the elapsed device time.

``--impl reference`` times the float64 CPU oracle (test infrastructure, the
reference arm of this benchmark) on the host cores, on a bounded sample of the
same workload (one head per step), and reports the same metric.
"""

import argparse
import json
import math
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_linear_mean_b200 import synth  # noqa: E402

METRIC = ("hybrid sparse attention ms/call & effective TFLOP/s vs B200 roofline, "
          "32k–245k")
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
# fp32 FMA peak of a B200 from unit counts and clocks: 148 SMs x 128 FP32
# lanes x 2 flops x 1.965 GHz (max SM clock).
FP32_SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture of the current kernel version (dram__bytes_read.sum +
# dram__bytes_write.sum, the pipeline's own L2 contents, the timed step of
# `bench.py --steps 1 --warmup 1`); absent = null.
TRAFFIC_PER_LAUNCH = {
    ("sla_1p3b", "attn_tc"): 507_496_960 + 135_902_208,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="sla_1p3b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-range", action="store_true",
                    help="time only --workload (by default a single-GPU run of the 32k "
                         "workload also times the 75.6k and 245k workloads)")
    ap.add_argument("--clock-csv", default=None,
                    help="also write the raw clock samples of the timed region to this CSV "
                         "(rank r writes <path>.r when several ranks run)")
    ap.add_argument("--mask-quality", action="store_true",
                    help="instead of the timed step: recall of the workload's mask against "
                         "the dense attention max-pooled over tiles (one GPU; dense work)")
    ap.add_argument("--heads", type=int, default=None,
                    help="time only the first HEADS heads of the workload (a smaller case "
                         "for profiler captures; the reported workload says so)")
    ap.add_argument("--tile", default=None,
                    help="with --mask-quality: also measure blocks of tokens taken in 3D tiles "
                         "of this shape, e.g. 1,8,8 (frames, rows, columns)")
    return ap.parse_args()


def run_mask_quality(args):
    """Mask quality on the workload (one GPU): the pooled-score mask against
    the dense attention max-pooled over (query block, key block) tiles, both
    from the library's kernels.  Prints one JSON line."""
    from block_sparse_linear_mean_b200 import sla
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = with_heads(synth.WORKLOADS[args.workload], args.heads)
    x = synth.make_inputs(wl, seed=0, device=dev)
    p = sla.params_for(wl)

    def measure_recall(q, k):
        m = sla.build_mask(p, q, k)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        imp = sla.block_importance(p, q, k)
        e1.record()
        rec = sla.mask_recall(p, m["mask"], imp)
        return {**{k: (round(v, 4) if isinstance(v, float) else v) for k, v in rec.items()},
                "importance_ms": round(e0.elapsed_time(e1), 2)}

    res = {"workload": wl.name, "config": wl.description,
           "mask_quality": {"reference": "dense attention max-pooled over (query block, key block) "
                                         "tiles; per row as many reference blocks as the mask keeps",
                            **measure_recall(x.q, x.k)}}
    if args.tile:
        tile = tuple(int(v) for v in args.tile.split(","))
        perm = sla.tile_order(wl.grid, tile, dev)
        res["mask_quality_tiled"] = {"tile": list(tile),
                                     **measure_recall(sla.permute_tokens(p, x.q, perm),
                                                      sla.permute_tokens(p, x.k, perm))}
    return res


def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's milliseconds, on every rank (one all-reduce); the
    value itself on a single process."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, flops_per_step: float, steps: int, ms: float) -> float:
    """Whole-job TFLOP/s: each of the `world` ranks ran `steps` steps of its
    own problem within `ms` milliseconds (the slowest rank's time)."""
    return world * flops_per_step * steps / (ms * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


# --------------------------------------------------------------- work counts


def block_sizes(n, b):
    return np.array([min((i + 1) * b, n) - i * b for i in range(math.ceil(n / b))],
                    dtype=np.float64)


def effective_flops(wl, mask_np, N=None):
    """Algorithmic flops of one forward over ``mask_np [B,H,Nqb,Nkb]``:
    4*d per kept critical (query, key) token pair, plus the linear branch
    (2*Bk*d^2 + Bk*d per key block for the summaries, |M_i|*(d^2+d) per
    query block for the gather, 2*d^2 + 2*d per token for phi(q) H / phi(q).z,
    2*d^2 per token for the projection, tokens of rows with marginal blocks).
    Real tokens only (ragged tails at their true size)."""
    N = wl.N if N is None else N
    d = wl.d
    sq, sk = block_sizes(N, wl.block_q), block_sizes(N, wl.block_k)
    crit = (mask_np == 2).astype(np.float64)
    pairs = float(np.einsum("bhij,i,j->", crit, sq, sk))
    fl = 4.0 * d * pairs
    lin = 0.0
    tok = 0.0
    if wl.frac_marg > 0:
        marg = (mask_np == 1)
        nm = marg.sum(axis=-1).astype(np.float64)          # [B,H,Nqb]
        BH = mask_np.shape[0] * mask_np.shape[1]
        lin += BH * float(np.sum(2.0 * sk * d * d + sk * d))
        lin += float(nm.sum()) * (d * d + d)
        tok = float(np.einsum("bhi,i->", (nm > 0).astype(np.float64), sq))
        lin += tok * (2.0 * d * d + 2.0 * d + 2.0 * d * d)
    apply = 0.0
    if wl.frac_marg > 0:
        apply = tok * (2.0 * d * d + 2.0 * d + 2.0 * d * d)
    return fl + lin, pairs, fl, lin, apply


def backward_flops(wl, mask_np):
    """Algorithmic flops of one backward over ``mask_np``: 10*d per kept
    critical token pair (S and dP recomputed, dV, dK, dQ), plus the linear
    branch: per token of a query block with marginal blocks g = dO W^T,
    dW += O_lin^T dO, d phi(q) and the dH^M, dz^M outer products
    (8*d^2 + 4*d); per marginal (query block, key block) pair the scatter
    of dH^M, dz^M (d^2 + d); per token of a key block that is marginal for
    some query block dk, dv (4*d^2 + 2*d).  Returns (total, critical, linear)."""
    d = wl.d
    sq, sk = block_sizes(wl.N, wl.block_q), block_sizes(wl.N, wl.block_k)
    crit = (mask_np == 2).astype(np.float64)
    cfl = 10.0 * d * float(np.einsum("bhij,i,j->", crit, sq, sk))
    lfl = 0.0
    if wl.frac_marg > 0:
        marg = (mask_np == 1)
        nm = marg.sum(axis=-1).astype(np.float64)
        tok = float(np.einsum("bhi,i->", (nm > 0).astype(np.float64), sq))
        ktok = float(np.einsum("bhj,j->", (marg.sum(axis=-2) > 0).astype(np.float64), sk))
        lfl = tok * (8.0 * d * d + 4.0 * d) + float(nm.sum()) * (d * d + d) + \
            ktok * (4.0 * d * d + 2.0 * d)
    return cfl + lfl, cfl, lfl


# --------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and clock-event (throttle) reasons of one GPU every
    20 ms through NVML in a background thread while the timed region runs;
    with ``csv_path`` given, the raw samples are also written there as CSV."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
               "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, device_index, period_s=0.02, csv_path=None):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self.err = None
        self.path = csv_path

    def _sample_once(self):
        import pynvml as nv
        try:
            h = nv.nvmlDeviceGetHandleByIndex(self.idx)
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
            self.samples.append((time.time(), sm, rs, pw))
        except Exception as e:  # keep sampling; record the last error
            self.err = repr(e)

    def _run(self):
        import pynvml as nv
        try:
            h = nv.nvmlDeviceGetHandleByIndex(self.idx)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:
            self.err = repr(e)
            return
        while not self._stop.is_set():
            self._sample_once()
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self.thread = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            # the timed region starts only once sampling runs
            t0 = time.time()
            while not self.samples and self.err is None and time.time() - t0 < 5.0:
                time.sleep(0.001)
        except Exception as e:
            self.err = repr(e)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._sample_once()  # one sample at the end of the timed region
            self._stop.set()
            self.thread.join(timeout=5)
        if not self.path:
            return
        try:
            os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
            with open(self.path, "w") as f:
                f.write("t,sm_mhz,reasons_mask,power_w\n")
                for t, sm, rs, pw in self.samples:
                    f.write(f"{t:.3f},{sm},{rs:#x},{pw:.1f}\n")
        except OSError:
            pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": [f"no samples ({self.err})"]}
        reasons = sorted({name for _, _, rs, _ in self.samples
                          for name, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(sm for _, sm, _, _ in self.samples),
                "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": reasons,
                "samples": len(self.samples),
                "power_w_max": max(pw for _, _, _, pw in self.samples)}


# --------------------------------------------------------------- our arm

# The metric is quoted over 32k-245k tokens: a default single-GPU run also
# times these workloads, reported as sub-records of the one JSON line.
RANGE_WORKLOADS = ("nabla_14b", "long_clip")


def mask_groups(wl):
    """Head groups of the mask step: the logits of a group go through a slab
    of at most 64 MB (the library's constant), one logits and one selection
    launch per group."""
    nqb, nkb = math.ceil(wl.N / wl.block_q), math.ceil(wl.N / wl.block_k)
    bh = wl.B * wl.H
    per_group = max(1, min(bh, (64 << 20) // (4 * nqb * nkb)))
    return math.ceil(bh / per_group)


def launches_per_step(wl, fused, bwd):
    """Kernels the library launches per step, from the entry points' code
    (checked against the ncu launch lists)."""
    # pool (Q and K in one launch), logits + selection per head group | plan
    # (+ summaries, indicator, gather GEMM; W to bf16 rides in the indicator
    # kernel unless B*H*Nqb < 16, when it takes a launch of its own) | fused
    # attention (or attention + combine)
    nqb = -(-wl.N // wl.block_q)
    prep = 3 if wl.B * wl.H * nqb >= 16 else 4
    n = 1 + 2 * mask_groups(wl) + (1 if fused else 0) + (prep if (fused and wl.frac_marg > 0) else 0) \
        + (1 if (not fused and wl.frac_marg > 0) else 0) + (1 if fused else 2)
    if bwd:
        lin = wl.frac_marg > 0
        n += 1  # column lists
        if fused and wl.d == 128:
            # Delta | 2 tile plans, dq (+ linear query side), dkdv (+ linear
            # key side) | (summaries, indicator, gather of H^M -- W to bf16
            # as in the forward --, indicator + gather of dH, dW partials, dW
            # sum)
            n += 1 + 4 + ((prep + 4) if lin else 0)
        else:
            # Delta and g, dW partials | dq, dkdv (tcgen05: + 2 tile plans) |
            # (summaries, linear dq, linear dk dv) | dW reduction
            n += 2 + (4 if fused else 2) + (3 if lin else 0) + 1
    return n


def stage_bytes(wl, mask_np):
    """Algorithmic HBM bytes per step of the two memory-bound stages.

    mask: read Q and K once; write the int8 mask, the list entries (4 bytes
    per critical or marginal block) and the per-row counts (and, for the
    fine-tune step, the column lists).  The pooled means and scores are the
    implementation's intermediates, not counted.
    prepare (linear branch on the tensor cores): read K and V once; write the
    key-block summaries H_j (bf16 d x d) and z_j (fp32 d) once and read them
    once; write the per-query-block sums H^M_i, z^M_i once."""
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    esz = 2 if wl.dtype == "bf16" else 4
    nqb, nkb = math.ceil(N / wl.block_q), math.ceil(N / wl.block_k)
    listed = int(np.count_nonzero(mask_np))
    mask_b = 2 * B * H * N * d * esz + B * H * nqb * nkb + 4 * listed + 8 * B * H * nqb
    if wl.backward:
        mask_b += 4 * listed + 8 * B * H * nkb
    prep_b = None
    if wl.frac_marg > 0 and d == 128 and wl.dtype == "bf16":
        summ = 2 * d * d + 4 * d
        prep_b = 2 * B * H * N * d * esz + 2 * B * H * nkb * summ + B * H * nqb * summ
    return mask_b, prep_b


def tensor_peak(peaks, peak_src, timed_s):
    """The bf16 tensor-core denominator: the burst figure for a timed region
    under a second, the sustained one (measured under the power cap over
    seconds) for longer regions."""
    if timed_s < 1.0:
        return peaks["bf16_tflops"], f"bf16 dense, burst ({peak_src}; timed region {timed_s:.3f} s)"
    return (peaks["bf16_tflops_sustained"],
            f"bf16 dense, sustained ({peak_src}; timed region {timed_s:.3f} s)")


def measure(wl, args, rank, world, local_rank, steps, warmup, do_e2e, keep_sample=False):
    """Time `steps` steps of workload `wl` on this rank's GPU (after
    `warmup` untimed ones) and return the measurement record."""
    from block_sparse_linear_mean_b200 import sla
    import torch.distributed as dist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bwd = wl.backward
    x = synth.make_inputs(wl, seed=rank, device=dev, with_dout=bwd)
    p = sla.params_for(wl)
    ws_m = sla.workspace(p, sla.SLA_OP_MASK, dev)
    ws_f = sla.workspace(p, sla.SLA_OP_FORWARD, dev)
    ws_b = sla.workspace(p, sla.SLA_OP_BACKWARD, dev) if bwd else None
    N, nqb, nkb = wl.N, math.ceil(wl.N / wl.block_q), math.ceil(wl.N / wl.block_k)
    B, H, d = wl.B, wl.H, wl.d
    mask = torch.empty(B, H, nqb, nkb, dtype=torch.int8, device=dev)
    rows = sla.BlockLists.empty(B * H * nqb, nkb, dev)
    rc = rows.c()
    # the fine-tune step also needs the column lists and the saved O_s, O_lin
    cols = sla.BlockLists.empty(B * H * nkb, nqb, dev) if bwd else None
    cc = cols.c() if bwd else None
    out = torch.empty_like(x.q)
    f32 = dict(dtype=torch.float32, device=dev)
    o_s = torch.empty(x.q.shape, **f32) if bwd else None
    o_lin = torch.empty(x.q.shape, **f32) if bwd else None
    lse = torch.empty(x.q.shape[:-1], **f32)
    if bwd:
        dq, dk, dv = (torch.empty(x.q.shape, **f32) for _ in range(3))
        dproj = torch.empty(x.proj.shape, **f32)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    ties = torch.zeros(4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def chk(name, st):
        if st != sla.SLA_OK:
            raise sla.SlaError(name, st)

    def stage_mask(q, k, tie_ptr=None):
        chk("sla_build_mask", sla.sla_build_mask(p, q.data_ptr(), k.data_ptr(), mask.data_ptr(),
                                                 rc, cc, None, tie_ptr, ws_m.data_ptr(),
                                                 ws_m.numel(), sp))

    def stage_prepare(k, v):
        chk("sla_forward_prepare", sla.sla_forward_prepare(
            p, k.data_ptr(), v.data_ptr(), x.proj.data_ptr(), rc, ws_f.data_ptr(),
            ws_f.numel(), sp))

    def stage_combine(q, k, v, dst):
        chk("sla_attention_combine", sla.sla_attention_combine(
            p, q.data_ptr(), k.data_ptr(), v.data_ptr(), x.proj.data_ptr(), rc,
            dst.data_ptr(), lse.data_ptr(), o_s.data_ptr() if bwd else None,
            o_lin.data_ptr() if bwd else None, ws_f.data_ptr(), ws_f.numel(), sp))

    def stage_backward(q, k, v, dout, grads=None):
        gq, gk, gv, gw = grads if grads is not None else (dq, dk, dv, dproj)
        chk("sla_backward", sla.sla_backward(
            p, q.data_ptr(), k.data_ptr(), v.data_ptr(), x.proj.data_ptr(), dout.data_ptr(),
            rc, cc, o_s.data_ptr(), lse.data_ptr(), o_lin.data_ptr(), gq.data_ptr(),
            gk.data_ptr(), gv.data_ptr(), gw.data_ptr(), ws_b.data_ptr(), ws_b.numel(), sp))

    fused = sla.sla_forward_uses_tensor_cores(p) == 1 and (wl.frac_marg == 0 or wl.d == 128)
    n_launch = launches_per_step(wl, fused, bwd)

    # warm-up (also fixes the mask used to count the algorithmic work)
    for _ in range(max(warmup, 0)):
        stage_mask(x.q, x.k)
        stage_prepare(x.k, x.v)
        stage_combine(x.q, x.k, x.v, out)
        if bwd:
            stage_backward(x.q, x.k, x.v, x.dout)
    torch.cuda.synchronize(dev)
    assert sla.check_device_status(ws_m) == sla.SLA_OK
    assert sla.check_device_status(ws_f) == sla.SLA_OK
    if bwd:
        assert sla.check_device_status(ws_b) == sla.SLA_OK
    mask_np = mask.cpu().numpy()
    flops, pairs, crit_fl, lin_fl, apply_fl = effective_flops(wl, mask_np)
    bwd_fl = backward_flops(wl, mask_np) if bwd else (0.0, 0.0, 0.0)
    flops += bwd_fl[0]

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    csv_path = None
    if args.clock_csv:
        csv_path = args.clock_csv if world == 1 else f"{args.clock_csv}.{rank}"
        if wl.name != args.workload:
            csv_path = f"{csv_path}.{wl.name}"
    with ClockSampler(local_rank, csv_path=csv_path) as clocks:
        for s in range(steps):
            flush.zero_()                      # L2 flush, outside the timed events
            e = ev[s]
            e[0].record(stream)
            stage_mask(x.q, x.k)
            e[1].record(stream)
            stage_prepare(x.k, x.v)
            e[2].record(stream)
            stage_combine(x.q, x.k, x.v, out)
            e[3].record(stream)
            if bwd:
                stage_backward(x.q, x.k, x.v, x.dout)
            e[4].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t_mask = [e[0].elapsed_time(e[1]) for e in ev]
    t_prep = [e[1].elapsed_time(e[2]) for e in ev]
    t_comb = [e[2].elapsed_time(e[3]) for e in ev]
    t_bwd = [e[3].elapsed_time(e[4]) for e in ev]
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[4]) for e in ev), dev)
    ms_step = total_ms / steps
    value = job_rate(world, flops, steps, total_ms)

    # the GPU's near-tie count over the whole problem (one untimed call)
    stage_mask(x.q, x.k, ties.data_ptr())
    torch.cuda.synchronize(dev)
    gpu_ties = int(ties[0].item())

    # end to end through the C ABI with host buffers: every step copies its
    # inputs (q, k, v, and dO for the fine-tune step) from pinned host memory,
    # runs mask + forward (+ backward), and reads its output (and gradients)
    # back.  Steps are pipelined as a serving loop would run them: inputs and
    # outputs are double-buffered on the device, host-to-device copies run on
    # one stream, device-to-host copies on another, so the copies of steps
    # s + 1 and s - 1 overlap the compute of step s.  The timed region spans
    # the first input copy to the last output copy.  Each step's input copy
    # (> L2) replaces the L2 flush.
    e2e = None
    if do_e2e:
        ins = (x.q, x.k, x.v, x.dout) if bwd else (x.q, x.k, x.v)
        hosts = [t.cpu().pin_memory() for t in ins]
        nb = 2
        devs = [[torch.empty_like(t) for t in ins] for _ in range(nb)]
        outs = [torch.empty_like(out) for _ in range(nb)]
        gsrc = (dq, dk, dv, dproj) if bwd else ()
        grads = [[torch.empty_like(t) for t in gsrc] for _ in range(nb)]
        outs_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(nb)]
        grads_h = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in gsrc]
                   for _ in range(nb)]
        cs, ds = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        mk = lambda: torch.cuda.Event()  # noqa: E731
        ev_in = [mk() for _ in range(steps)]
        ev_comp = [mk() for _ in range(steps)]
        ev_out = [mk() for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        t0.record(cs)
        for s in range(steps):
            b = s % nb
            with torch.cuda.stream(cs):
                if s >= nb:
                    cs.wait_event(ev_comp[s - nb])   # buffer b read by step s - nb
                for d_, h_ in zip(devs[b], hosts):
                    d_.copy_(h_, non_blocking=True)
                ev_in[s].record(cs)
            stream.wait_event(ev_in[s])
            if s >= nb:
                stream.wait_event(ev_out[s - nb])    # outputs b read back
            qd, kd, vd = devs[b][:3]
            stage_mask(qd, kd)
            stage_prepare(kd, vd)
            stage_combine(qd, kd, vd, outs[b])
            if bwd:
                stage_backward(qd, kd, vd, devs[b][3], grads[b])
            ev_comp[s].record(stream)
            with torch.cuda.stream(ds):
                ds.wait_event(ev_comp[s])
                outs_h[b].copy_(outs[b], non_blocking=True)
                for h_, d_ in zip(grads_h[b], grads[b]):
                    h_.copy_(d_, non_blocking=True)
                ev_out[s].record(ds)
        ds.wait_event(ev_comp[steps - 1])
        t1.record(ds)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), dev)
        e2e = {"value": job_rate(world, flops, steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in ins)),
               "d2h_bytes_per_step": int(out.numel() * out.element_size() +
                                         sum(t.numel() * t.element_size() for t in gsrc)),
               "ms_per_step": e2e_ms / steps,
               "pipelining": "double-buffered, H2D / compute / D2H on three streams"}

    peaks, peak_src = load_peaks()
    comb_ms = statistics.mean(t_comb)
    tc = _tc_enabled(p)
    if tc:
        peak, peak_note = tensor_peak(peaks, peak_src, total_ms * 1e-3)
        bound, unit = "tensor", "TFLOP/s"
    else:
        peak, bound, unit = FP32_SIMT_PEAK_TFLOPS, "alu", "TFLOP/s"
        peak_note = "fp32 FMA: 148 SMs x 128 lanes x 2 x 1.965 GHz"
    # the combine stage is one fused kernel on the tensor-core path: critical
    # attention + phi(Q) H^M / normaliser + projection for tokens with
    # marginal blocks
    kern_fl = crit_fl + apply_fl
    achieved = kern_fl / (comb_ms * 1e-3) / 1e12
    roofline = {"bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 1),
                "unit": unit, "frac": round(achieved / peak, 4),
                "traffic": TRAFFIC_PER_LAUNCH.get((wl.name, "attn_tc" if tc else "attn_simt")),
                "kernel": ("fused tcgen05 attention + linear apply + projection + combine"
                           if fused else "sparse attention forward (SIMT fp32) + combine"),
                "peak_source": peak_note,
                "algorithmic": f"{kern_fl:.4g} flops per launch = 4*d*{pairs:.4g} kept critical "
                               f"token pairs + {apply_fl:.4g} linear apply/projection flops"}
    if tc:
        roofline["frac_of_sustained"] = round(achieved / peaks["bf16_tflops_sustained"], 4)
    mask_b, prep_b = stage_bytes(wl, mask_np)
    hbm = peaks["hbm_gbs"]
    mask_ms = statistics.mean(t_mask)
    prep_ms = statistics.mean(t_prep)
    stages = [{"stage": "mask (pool, score, classify, lists)", "bound": "hbm",
               "algorithmic_bytes": mask_b, "ms": round(mask_ms, 4),
               "achieved": round(mask_b / (mask_ms * 1e-3) / 1e9, 1), "peak": hbm,
               "unit": "GB/s", "frac": round(mask_b / (mask_ms * 1e-3) / 1e9 / hbm, 4)}]
    if prep_b is not None:
        stages.append({"stage": "prepare (plan, summaries, marginal sums)", "bound": "hbm",
                       "algorithmic_bytes": prep_b, "ms": round(prep_ms, 4),
                       "achieved": round(prep_b / (prep_ms * 1e-3) / 1e9, 1), "peak": hbm,
                       "unit": "GB/s",
                       "frac": round(prep_b / (prep_ms * 1e-3) / 1e9 / hbm, 4)})
    res = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic (smooth 3D-grid field + noise, seeded)",
        "config": {"workload": wl.description, "name": wl.name, "B": B, "H": H, "N": N, "d": d,
                   "block_q": wl.block_q, "block_k": wl.block_k, "mode": wl.mode,
                   "frac_crit": wl.frac_crit, "frac_marg": wl.frac_marg, "thr": wl.thr,
                   "parallelism": f"independent problem per GPU x{world}",
                   "l2": "256 MB write flushes L2 between steps, outside the timed events"},
        "breakdown_ms": {"mask": round(mask_ms, 4),
                         "prepare (plan + linear summaries + gather)": round(prep_ms, 4),
                         "attention_combine": round(comb_ms, 4),
                         **({"backward": round(statistics.mean(t_bwd), 4)} if bwd else {})},
        "work": {"effective_flops_per_step": flops, "critical_flops": crit_fl,
                 "linear_flops": lin_fl, "critical_token_pairs": pairs,
                 **({"backward_critical_flops": bwd_fl[1], "backward_linear_flops": bwd_fl[2]}
                    if bwd else {}),
                 "kept_fraction_of_dense_pairs": pairs / (B * H * float(N) * N)},
        "roofline": roofline,
        "stage_rooflines": stages,
        "mask_near_tie_rows": gpu_ties,
        "e2e": e2e,
        "gpu_launches": n_launch * steps,
        "clocks": clocks.summary(),
    }
    sample = None
    if keep_sample:
        # head 0 of batch 0, for the oracle comparison of the CPU-baseline
        # leg: inputs as drawn, the GPU's mask and the output rows of a few
        # query blocks spread over the sequence (the last one ragged)
        blocks = sorted({int(round(i * (nqb - 1) / 7)) for i in range(8)})
        rows_of = [np.arange(i * wl.block_q, min((i + 1) * wl.block_q, N)) for i in blocks]
        sample = {"q": x.q[:1, :1].cpu(), "k": x.k[:1, :1].cpu(), "v": x.v[:1, :1].cpu(),
                  "proj": x.proj.cpu(), "mask": mask_np[:1, :1].copy(), "blocks": blocks,
                  "out": [out[0, 0, r[0]:r[-1] + 1].float().cpu().numpy() for r in rows_of]}
    del x, ws_m, ws_f, ws_b, mask, rows, cols, out, o_s, o_lin, lse, flush
    if bwd:
        del dq, dk, dv, dproj
    torch.cuda.empty_cache()
    return res, sample


def with_heads(wl, heads):
    """The workload restricted to its first `heads` heads (profiling cases)."""
    if heads is None or heads == wl.H:
        return wl
    import dataclasses
    return dataclasses.replace(wl, H=heads, description=f"{wl.description} [first {heads} heads]")


def run_ours(args, rank, world, local_rank):
    wl = with_heads(synth.WORKLOADS[args.workload], args.heads)
    res, sample = measure(wl, args, rank, world, local_rank, args.steps, args.warmup,
                          not args.no_e2e, keep_sample=(rank == 0 and world == 1))
    if world == 1 and not args.no_range and wl.name == "sla_1p3b" and args.heads is None:
        subs = []
        for name in RANGE_WORKLOADS:
            r, _ = measure(synth.WORKLOADS[name], args, rank, world, local_rank,
                           min(args.steps, 10), max(3, min(args.warmup, 3)), False)
            subs.append({k: r[k] for k in ("value", "unit", "ms_per_step", "steps", "warmup",
                                           "breakdown_ms", "roofline", "stage_rooflines",
                                           "mask_near_tie_rows", "gpu_launches", "clocks",
                                           "work")}
                        | {"workload": r["config"]["workload"], "name": name,
                           "N": r["config"]["N"]})
        res["range"] = subs
    return res, sample


def _tc_enabled(p):
    """Whether the forward of ``p`` runs the tcgen05 kernel (library query)."""
    from block_sparse_linear_mean_b200 import sla
    return sla.sla_forward_uses_tensor_cores(p) == 1


# --------------------------------------------------------------- oracle arms


def oracle_sample(wl, heads, min_seconds=0.0):
    """Time the float64 oracle (mask + forward) head by head on the host."""
    from oracle import sla_oracle as orc
    x = synth.make_inputs(wl, seed=0, device="cpu", heads=heads)
    done, flops, t0 = 0, 0.0, time.perf_counter()
    while done < heads:
        h = done
        qh, kh, vh = (t[:, h:h + 1] for t in (x.q, x.k, x.v))
        m = orc.build_mask(qh, kh, wl.block_q, wl.block_k, wl.mode, wl.frac_crit,
                           wl.frac_marg, wl.thr)
        orc.forward(qh, kh, vh, x.proj, m["mask"], wl.block_q, wl.block_k)
        flops += effective_flops(wl, m["mask"])[0]
        done += 1
        if time.perf_counter() - t0 >= min_seconds and min_seconds > 0:
            break
    return done, flops, time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def cpu_baseline(wl):
    heads, flops, secs = oracle_sample(wl, heads=wl.H, min_seconds=12.0)
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"float64 oracle mask + forward on {heads} of {wl.H} heads "
                      f"({secs:.1f} s); value = effective flops of those heads / time",
            "ms_per_call_extrapolated": round(secs / heads * wl.H * 1e3, 1)}


def oracle_parity(wl, sample):
    """The CPU-baseline leg's check of the timed run: the oracle's mask of
    head 0 (all its rows) against the GPU's, and the oracle's output rows of
    a few sampled query blocks (with the oracle's own mask row) against the
    GPU's bf16 output, where the two masks agree on that row."""
    from oracle import sla_oracle as orc
    tie_eps = 1e-5
    ref = orc.build_mask(sample["q"], sample["k"], wl.block_q, wl.block_k, wl.mode,
                         wl.frac_crit, wl.frac_marg, wl.thr)
    gm, om = sample["mask"][0, 0], ref["mask"][0, 0]
    differ = (gm != om).any(axis=-1)
    ties = ref["margins"][0, 0] <= tie_eps
    q, k, v = (orc.f64(t[0, 0]) for t in (sample["q"], sample["k"], sample["v"]))
    w = orc.f64(sample["proj"])
    errs, over, skipped = [], 0, 0
    for i, got in zip(sample["blocks"], sample["out"]):
        if differ[i]:
            skipped += 1
            continue
        o = orc.forward_rows(q, k, v, w, om[i], i, wl.block_q, wl.block_k)["out"]
        e = np.abs(got.astype(np.float64) - o)
        errs.append(e)
        # tolerance: 2e-2 plus the bf16 rounding of the stored output
        over += int((e > 2e-2 + 2.0 ** -8 * np.abs(o)).sum())
    e = np.concatenate([x.ravel() for x in errs]) if errs else np.zeros(1)
    return {"head": 0, "mask_rows": int(gm.shape[0]),
            "mask_rows_differing": int(differ.sum()),
            "mask_rows_differing_outside_ties": int((differ & ~ties).sum()),
            "oracle_tie_rows": int(ties.sum()),
            "sampled_query_blocks": sample["blocks"], "blocks_skipped_mask_differs": skipped,
            "out_max_abs_err": float(e.max()), "out_mean_abs_err": float(e.mean()),
            "out_elements_over_tolerance": over,
            "tolerance": "max abs 2e-2 (+ bf16 output rounding 2^-8 |ref|), mean abs 2e-3"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wl = synth.WORKLOADS[args.workload]
    for _ in range(args.warmup):
        oracle_sample(wl, heads=1)
    tot_f, tot_s = 0.0, 0.0
    for _ in range(args.steps):
        _, f, s = oracle_sample(wl, heads=1)
        tot_f += f
        tot_s += s
    value = tot_f / tot_s / 1e12
    cores = blas_threads()
    return {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot_s / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": wl.description, "name": wl.name,
                   "sample": "one head per step (mask + forward) of the workload"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "kind": "oracle",
                         "cores": cores,
                         "sample": "float64 oracle, one head per step, host cores"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.mask_quality:
        if rank == 0:
            print(json.dumps(run_mask_quality(args)))
        return
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res))
        return
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res, sample = run_ours(args, rank, world, local_rank)
        if rank == 0:
            wl = synth.WORKLOADS[args.workload]
            if not args.no_cpu_baseline and world == 1:
                res["cpu_baseline"] = cpu_baseline(wl)
                res["parity"] = oracle_parity(wl, sample)
            print(json.dumps(res))
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
