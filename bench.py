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
# dram__bytes_write.sum; command and figures in profiles/); absent = null.
TRAFFIC_PER_LAUNCH = {
    ("sla_1p3b", "attn_tc"): 507_041_280 + 92_068_608,
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
    ap.add_argument("--mask-quality", action="store_true",
                    help="instead of the timed step: recall of the workload's mask against "
                         "the dense attention max-pooled over tiles (one GPU; dense work)")
    return ap.parse_args()


def run_mask_quality(args):
    """Mask quality on the workload (one GPU): the pooled-score mask against
    the dense attention max-pooled over (query block, key block) tiles, both
    from the library's kernels.  Prints one JSON line."""
    from block_sparse_linear_mean_b200 import sla
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]
    x = synth.make_inputs(wl, seed=0, device=dev)
    p = sla.params_for(wl)
    m = sla.build_mask(p, x.q, x.k)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    imp = sla.block_importance(p, x.q, x.k)
    e1.record()
    rec = sla.mask_recall(p, m["mask"], imp)
    return {"workload": wl.name, "config": wl.description,
            "mask_quality": {"reference": "dense attention max-pooled over (query block, key block) "
                                          "tiles; per row as many reference blocks as the mask keeps",
                             **{k: (round(v, 4) if isinstance(v, float) else v) for k, v in rec.items()},
                             "importance_ms": round(e0.elapsed_time(e1), 2)}}


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
    the raw samples are written as CSV, one file per rank, beside the other
    run outputs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
               "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, device_index, period_s=0.02):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self.err = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_rank{device_index}.csv")

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
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
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


def run_ours(args, rank, world, local_rank):
    from block_sparse_linear_mean_b200 import sla
    import torch.distributed as dist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]
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
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def chk(name, st):
        if st != sla.SLA_OK:
            raise sla.SlaError(name, st)

    def stage_mask(q, k):
        chk("sla_build_mask", sla.sla_build_mask(p, q.data_ptr(), k.data_ptr(), mask.data_ptr(),
                                                 rc, cc, None, None, ws_m.data_ptr(),
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
    # kernels per step: pool (Q and K in one launch), logits, classify | plan
    # (+ W to bf16, summaries, indicator, gather GEMM) | fused attention (or
    # attention + combine)
    launches_per_step = 3 + (1 if fused else 0) + (4 if (fused and wl.frac_marg > 0) else 0) \
        + (1 if (not fused and wl.frac_marg > 0) else 0) + (1 if fused else 2)
    if bwd:
        lin = wl.frac_marg > 0
        launches_per_step += 1  # column lists
        if fused and wl.d == 128:
            # Delta | 2 tile plans, dq (+ linear query side), dkdv (+ linear
            # key side) | (W to bf16, summaries, indicator, gather of H^M,
            # indicator + gather of dH, dW partials, dW sum)
            launches_per_step += 1 + 4 + (8 if lin else 0)
        else:
            # Delta and g, dW partials | dq, dkdv (tcgen05: + 2 tile plans) |
            # (summaries, linear dq, linear dk dv) | dW reduction
            launches_per_step += 2 + (4 if fused else 2) + (3 if lin else 0) + 1


    # warm-up (also fixes the mask used to count the algorithmic work)
    for _ in range(max(args.warmup, 0)):
        stage_mask(x.q, x.k)
        stage_prepare(x.k, x.v)
        stage_combine(x.q, x.k, x.v, out)
        if bwd:
            stage_backward(x.q, x.k, x.v, x.dout)
    torch.cuda.synchronize(dev)
    assert sla.check_device_status(ws_f) == sla.SLA_OK
    if bwd:
        assert sla.check_device_status(ws_b) == sla.SLA_OK
    mask_np = mask.cpu().numpy()
    flops, pairs, crit_fl, lin_fl, apply_fl = effective_flops(wl, mask_np)
    bwd_fl = backward_flops(wl, mask_np) if bwd else (0.0, 0.0, 0.0)
    flops += bwd_fl[0]

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clocks:
        for s in range(args.steps):
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
    ms_step = total_ms / args.steps
    value = job_rate(world, flops, args.steps, total_ms)

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
    if not args.no_e2e:
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
        ev_in = [mk() for _ in range(args.steps)]
        ev_comp = [mk() for _ in range(args.steps)]
        ev_out = [mk() for _ in range(args.steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        t0.record(cs)
        for s in range(args.steps):
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
        ds.wait_event(ev_comp[args.steps - 1])
        t1.record(ds)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), dev)
        e2e = {"value": job_rate(world, flops, args.steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in ins)),
               "d2h_bytes_per_step": int(out.numel() * out.element_size() +
                                         sum(t.numel() * t.element_size() for t in gsrc)),
               "ms_per_step": e2e_ms / args.steps,
               "pipelining": "double-buffered, H2D / compute / D2H on three streams"}

    peaks, peak_src = load_peaks()
    comb_ms = statistics.mean(t_comb)
    tc = _tc_enabled(p)
    if tc:
        peak, bound, unit = peaks["bf16_tflops_sustained"], "tensor", "TFLOP/s"
        peak_note = f"bf16 dense, sustained ({peak_src})"
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
                "traffic": TRAFFIC_PER_LAUNCH.get((args.workload, "attn_tc" if tc else "attn_simt")),
                "kernel": ("fused tcgen05 attention + linear apply + projection + combine"
                           if fused else "sparse attention forward (SIMT fp32) + combine"),
                "peak_source": peak_note,
                "algorithmic": f"{kern_fl:.4g} flops per launch = 4*d*{pairs:.4g} kept critical "
                               f"token pairs + {apply_fl:.4g} linear apply/projection flops"}
    res = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic (smooth 3D-grid field + noise, seeded)",
        "config": {"workload": wl.description, "name": wl.name, "B": B, "H": H, "N": N, "d": d,
                   "block_q": wl.block_q, "block_k": wl.block_k, "mode": wl.mode,
                   "frac_crit": wl.frac_crit, "frac_marg": wl.frac_marg, "thr": wl.thr,
                   "parallelism": f"independent problem per GPU x{world}",
                   "l2": "256 MB write flushes L2 between steps, outside the timed events"},
        "breakdown_ms": {"mask": round(statistics.mean(t_mask), 4),
                         "prepare (plan + linear summaries + gather)": round(statistics.mean(t_prep), 4),
                         "attention_combine": round(comb_ms, 4),
                         **({"backward": round(statistics.mean(t_bwd), 4)} if bwd else {})},
        "work": {"effective_flops_per_step": flops, "critical_flops": crit_fl,
                 "linear_flops": lin_fl, "critical_token_pairs": pairs,
                 **({"backward_critical_flops": bwd_fl[1], "backward_linear_flops": bwd_fl[2]}
                    if bwd else {}),
                 "kept_fraction_of_dense_pairs": pairs / (B * H * float(N) * N)},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    return res


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
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            wl = synth.WORKLOADS[args.workload]
            if not args.no_cpu_baseline and world == 1:
                res["cpu_baseline"] = cpu_baseline(wl)
            print(json.dumps(res))
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
