"""Benchmark of the Muon step on B200: prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gpt2_124m]
                    [--impl ours|reference]

A step is one Muon update (Nesterov momentum, NS5, W -= lr*O) over every
matrix of the workload, with inputs resident in HBM.  ``value`` is
algorithmic NS5 TFLOP/s of the whole job (symmetry of X X^T and A A
exploited, 5*(k(k+1)l + k^2(k+1) + 2k^2 l) per k x l matrix, k <= l);
``ms_per_step`` the device time per step; under torchrun the time is the
maximum over ranks.

``--impl reference`` times the CPU oracle (float64 numpy) on the host cores on
a bounded sample of the same workload, per the same metric.

Under torchrun (N > 1) the default is the data-parallel step: the ranks split
one model's matrices (greedy by flops) and exchange the updated weights with
an all_gather ("scaling": "strong"); ``--replicas`` runs an independent copy
per rank instead ("scaling": "weak").

The line also carries a ``sweep`` of the 64-matrix square batches
(n = 1024, 2048, 4096) with the GEMM kernel's throughput per size, so that the
fraction of the dense bf16 peak on those batches is measured in the same run
(``--sweep ""`` leaves it out).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Muon NS5 bf16 TFLOP/s (% of B200 tensor peak); ms per GPT-2-124M Muon step"
UNIT = "TFLOP/s"
# Used only when MEASURED_PEAKS.json is absent: an earlier measurement of a
# plain copy and of a cuBLAS bf16 GEMM (burst) on this machine's B200s.  There is
# no sustained GEMM figure without the measurement file.
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def ns_flops(shapes, ns_steps=5) -> float:
    tot = 0.0
    for r, c in shapes:
        k, l = min(r, c), max(r, c)
        tot += ns_steps * (k * (k + 1) * l + k * k * (k + 1) + 2 * k * k * l)
    return tot


def ns_flops_dense(shapes, ns_steps=5) -> float:
    """Dense-equivalent flops: the same products without the symmetry of X X^T
    and A A (every Gram and polynomial output element computed)."""
    tot = 0.0
    for r, c in shapes:
        k, l = min(r, c), max(r, c)
        tot += ns_steps * (4 * k * k * l + 2 * k * k * k)
    return tot


def flops_by_kind(shapes, ns_steps=5):
    g = p = u = 0.0
    for r, c in shapes:
        k, l = min(r, c), max(r, c)
        g += k * (k + 1) * l
        p += k * k * (k + 1)
        u += 2 * k * k * l
    return {"gram": g * ns_steps, "poly": p * ns_steps, "update": u * ns_steps}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The fused small-matrix kernels sit between these two markers of kernels.cuh;
# they are not part of the GEMM kernel whose DRAM traffic the summary records.
_FUSED_BEGIN = "// ================================================ small matrices, fused ==="
_FUSED_END = "// ======================================================= ns_steps == 0 ==="
_PRO_BEGIN = "// ============================================================ prologue ==="
_PRO_END = "// ====================================================== NS GEMM kernel ==="


def kernel_source_hash() -> str:
    """Hash of the device code the GEMM kernel's ncu figures were taken on:
    ptx.cuh and kernels.cuh without the prologue and the fused small-matrix
    kernels, comments and whitespace removed (a comment edit keeps it)."""
    h = hashlib.sha256()
    for f in ("kernels.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "muon_newton_schulz_02_b200", "csrc", f)) as fh:
            text = fh.read()
        for begin, end in ((_FUSED_BEGIN, _FUSED_END), (_PRO_BEGIN, _PRO_END)):
            a, b = text.find(begin), text.find(end)
            if a >= 0 and b > a:
                text = text[:a] + text[b:]
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic():
    """DRAM bytes per launch of the GEMM kernel from the committed ncu summary,
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "ns_gemm_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch_full_workload")


# ---------------------------------------------------------------- clocks ---
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = self._smi_id(device_index)

    @staticmethod
    def _smi_id(i):
        try:
            import torch
            p = torch.cuda.get_device_properties(i)
            return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            return vis.split(",")[i] if vis else str(i)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.dev, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------- CPU oracle ---
def cpu_oracle_rate(w, budget_s=12.0, threads=None):
    """Times the oracle as it stands on a bounded sample of the workload's
    matrices (cycling through its distinct shapes) on the host cores (all of
    them, or `threads`)."""
    import contextlib
    # all host cores for the BLAS pool, whatever OMP_NUM_THREADS a launcher set
    # (torchrun sets 1; under it only rank 0 runs this)
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        pool = threadpool_limits(limits=threads or os.cpu_count() or 1, user_api="blas")
    except Exception:
        threadpool_info, pool = None, contextlib.nullcontext()
    with pool:
        if threadpool_info is not None:
            cores = max([d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"] or [1])
        else:
            cores = os.cpu_count() or 1
        return _time_oracle(w, budget_s, cores)


def _time_oracle(w, budget_s, cores):
    import numpy as np
    from muon_newton_schulz_02_b200 import workloads
    from oracle import muon_oracle
    idx = workloads.sample_indices(w, per_shape=64)
    order = []
    by_shape = {}
    for i in idx:
        by_shape.setdefault(w.shapes[i], []).append(i)
    while any(by_shape.values()):
        for s in list(by_shape):
            if by_shape[s]:
                order.append(by_shape[s].pop(0))
    done, flops, t_used = [], 0.0, 0.0
    for i in order:
        g = workloads.grad(w, 0, i).numpy()
        W = workloads.weight(w, i).numpy()
        buf = np.zeros_like(g)
        t0 = time.perf_counter()
        muon_oracle.muon_update(W, g, buf, w.lr, w.mu)
        t_used += time.perf_counter() - t0
        flops += ns_flops([w.shapes[i]])
        done.append(w.shapes[i])
        if t_used >= budget_s:
            break
    shapes_desc = {}
    for s in done:
        shapes_desc[f"{s[0]}x{s[1]}"] = shapes_desc.get(f"{s[0]}x{s[1]}", 0) + 1
    return {"value": flops / t_used / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(done)} of {w.n_matrices} matrices ({shapes_desc}), one Muon step each, "
                      f"{t_used:.1f} s of float64 numpy",
            "seconds": t_used}


# ------------------------------------------------------------------ main ---
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from muon_newton_schulz_02_b200 import workloads
    w = workloads.get(args.workload)
    sharded = world > 1 and not args.replicas           # the GPU arm's configuration at this N
    # each step: a bounded sample (at least one matrix), sized so the whole
    # run stays within --ref-total seconds of CPU work
    per_step = args.ref_total / max(1, args.steps + args.warmup)
    flops = secs = 0.0
    base = None
    for s in range(args.warmup + args.steps):
        r = cpu_oracle_rate(w, budget_s=per_step)
        if s >= args.warmup:
            flops += r["value"] * 1e12 * r["seconds"]
            secs += r["seconds"]
        base = r
    val = flops / secs / 1e12
    flops_step = ns_flops(w.shapes)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": flops_step / (val * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,0.02) gradients of the GPT-2-124M hidden-matrix shapes)",
        "config": workload_config(w, args, sharded),
        "cpu_baseline": {k: base[k] for k in ("kind", "cores", "sample")} | {"value": val, "unit": UNIT},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, args, sharded=False):
    shapes = {}
    for s in w.shapes:
        shapes[f"{s[0]}x{s[1]}"] = shapes.get(f"{s[0]}x{s[1]}", 0) + 1
    return {"workload": w.name, "matrices": w.n_matrices, "shapes": shapes, "ns_steps": 5,
            "mu": w.mu, "lr": w.lr, "nesterov": True, "grad_sets": args.grad_sets,
            "l2": f"inputs larger than L2: W, g, buf are {w.n_elements * 12 / 1e9:.2f} GB per step",
            "parallelism": (f"matrices sharded over {args.gpus} ranks + all_gather of "
                            f"{'the bf16 update' if args.exchange == 'o16' else 'the fp32 weights'} in "
                            f"{args.buckets} run(s)" if sharded else f"independent replicas x{args.gpus}")}


def pick_peak(peaks, clk, timed_s):
    """The GEMM peak a kernel is judged against: the burst figure when the
    timed region is short (under a second) or ran at (nearly) full clock, the
    sustained figure when a long region settled under the power cap."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sust = peaks.get("bf16_tflops_sustained")
    full_clock = bool(clk) and clk["sm_mhz"] >= 0.95 * clk["sm_max_mhz"]
    if sust is None or timed_s < 1.0 or full_clock:
        why = ("no sustained figure" if sust is None else
               f"timed region {timed_s:.2f} s < 1 s" if timed_s < 1.0 else "median SM clock >= 0.95 of max")
        return burst, "bf16_tflops (burst: " + why + ")"
    return float(sust), "bf16_tflops_sustained (timed region >= 1 s below full clock)"


# Launch kinds of the tcgen05 GEMM kernel (ns_gemm_kernel): the chained launch
# of every phase but the last update, and the one-phase launches.
GEMM_KINDS = ("chain", "gram", "poly", "update", "update_apply")


def flush_l2(buf):
    buf.zero_()                      # writes more than the 126 MB L2: evicts every line


class StepTimer:
    """Runs `one_step` K times on `stream` with a CUDA event after every step
    (the loop total and per-step times from the same events)."""

    def __init__(self, torch, stream):
        self.torch, self.stream = torch, stream

    def run(self, one_step, steps, start=0):
        ev = [self.torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record(self.stream)
        for s in range(steps):
            one_step(start + s)
            ev[s + 1].record(self.stream)
        return ev

    @staticmethod
    def times(ev):
        return ev[0].elapsed_time(ev[-1]), [ev[i].elapsed_time(ev[i + 1]) for i in range(len(ev) - 1)]


def gemm_roofline(prof, flops, steps, peak):
    gemm_ms = sum(prof[k][0] for k in GEMM_KINDS)
    gemm_launches = sum(prof[k][1] for k in GEMM_KINDS)
    if not gemm_launches:
        return None
    per_launch = flops * steps / gemm_launches
    us = gemm_ms / gemm_launches * 1e3
    achieved = per_launch / (us / 1e6) / 1e12
    return {"achieved": achieved, "flops_per_launch": per_launch, "us_per_launch": us, "launches": gemm_launches,
            "frac": achieved / peak}


def alternate_fp8(args, muon, torch, dev, stream, w, W, bufs, gsets, stepper, blocks, per):
    """The reduced-precision variant (muon_step_fp8) against the bf16 step on
    the same workload, in alternating blocks so that both see the same clock
    and power state; the medians of the block means compare them."""
    stepper8 = muon.PreparedStep(W, bufs, lr=w.lr, mu=w.mu, fp8_iters=args.fp8_iters)
    for s in range(2):
        stepper8(gsets[s % len(gsets)], stream=stream)
    torch.cuda.synchronize(dev)
    timer = StepTimer(torch, stream)
    t16, t8 = [], []
    for _ in range(blocks):
        for st_, acc in ((stepper, t16), (stepper8, t8)):
            e = timer.run(lambda s: st_(gsets[s % len(gsets)], stream=stream), per)
            torch.cuda.synchronize(dev)
            acc.append(timer.times(e)[0] / per)
    m16, m8 = statistics.median(t16), statistics.median(t8)
    return {"fp8_iters": args.fp8_iters, "ms_per_step": m8, "ms_per_step_bf16": m16, "speedup": m16 / m8,
            "protocol": f"{blocks} alternating blocks of {per} bf16 and {per} e4m3 steps, medians of block means",
            "what": "muon_step_fp8: e4m3 operands for A*A (iterations 0..F-1) and X*X^T (1..F-1) in the "
                    "per-phase launches; a reduced-precision variant, not the headline"}


def run_sweep(args, muon, workloads, torch, dev, stream, peaks):
    """GEMM-kernel throughput on the 64-matrix square batches, each timed on
    its own (>= 3 warm-up and >= 5 timed steps, every launch bracketed by
    CUDA events), with its own clock record."""
    out = {}
    for n in [int(x) for x in args.sweep.split(",") if x.strip()]:
        w = workloads.get(f"square_n{n}")
        W = workloads.weights(w, device=dev)
        bufs = workloads.zero_bufs(w, device=dev)
        gsets = [workloads.grads(w, s, device=dev) for s in range(2)]
        stepper = muon.PreparedStep(W, bufs, lr=w.lr, mu=w.mu)
        steps, warm = max(5, args.sweep_steps), 3
        for s in range(warm):
            stepper(gsets[s % 2], stream=stream)
        torch.cuda.synchronize(dev)
        muon.profile_read()
        muon.profile_enable(True)
        clocks = ClockSampler(dev.index)
        clocks.start()
        time.sleep(0.2)
        timer = StepTimer(torch, stream)
        ev = timer.run(lambda s: stepper(gsets[s % 2], stream=stream), steps)
        torch.cuda.synchronize(dev)
        clk = clocks.stop()
        muon.profile_enable(False)
        prof = muon.profile_read()
        total, per = timer.times(ev)
        flops = ns_flops(w.shapes)
        peak, why = pick_peak(peaks, clk, total / 1e3)
        r = gemm_roofline(prof, flops, steps, peak)
        burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        entry = {"matrices": w.n_matrices, "steps": steps, "warmup": warm,
                 "ms_per_step_median": statistics.median(per), "step_tflops": flops * steps / (total / 1e3) / 1e12,
                 "gemm_tflops": r["achieved"] if r else None,
                 "gemm_frac_burst": r["achieved"] / burst if r else None, "clocks": clk, "peak_choice": why}
        if peaks.get("bf16_tflops_sustained") and r:
            entry["gemm_frac_sustained"] = r["achieved"] / float(peaks["bf16_tflops_sustained"])
        if r and clk:
            entry["gemm_kcycles_per_launch"] = r["us_per_launch"] * clk["sm_mhz"] / 1e3
        if args.fp8_iters and n > 1024:
            entry["fp8_variant"] = alternate_fp8(args, muon, torch, dev, stream, w, W, bufs, gsets, stepper,
                                                 blocks=2, per=2)
        out[f"n{n}"] = entry
        if muon.sync_status(stream) != 0:
            raise RuntimeError(f"device status after the n={n} sweep entry: " + muon.last_error())
        del W, bufs, gsets, stepper
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import __graft_entry__
    __graft_entry__.build()
    import muon_newton_schulz_02_b200 as muon
    from muon_newton_schulz_02_b200 import workloads

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.per_phase:
        muon.debug_set(4, 0)                    # one launch per Newton-Schulz phase, for comparisons
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    sharded = world > 1 and not args.replicas

    def barrier():
        if world > 1:
            dist.barrier()

    w = workloads.get(args.workload)
    W = workloads.weights(w, device=dev)
    bufs = workloads.zero_bufs(w, device=dev)
    gsets = [workloads.grads(w, s, device=dev) for s in range(args.grad_sets)]
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    from muon_newton_schulz_02_b200 import distributed as mdist

    stepper = muon.PreparedStep(W, bufs, lr=w.lr, mu=w.mu)    # the training-loop call: same W and buf

    def one_step(s):
        if sharded:
            mdist.sharded_step(W, gsets[s % args.grad_sets], bufs, lr=w.lr, mu=w.mu, nbuckets=args.buckets,
                               exchange=args.exchange)
        else:
            stepper(gsets[s % args.grad_sets], stream=stream)

    for s in range(args.warmup):
        one_step(s)
    torch.cuda.synchronize(dev)
    if muon.sync_status(stream) != 0:
        raise RuntimeError("device status after warm-up: " + muon.last_error())

    # ---- timed region: device time with CUDA events on the launching stream
    # (an event after every step gives the per-step times as well)
    muon.profile_read()                         # drop anything recorded so far
    clocks = ClockSampler(local_rank) if rank == 0 else None
    timer = StepTimer(torch, stream)
    barrier()
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.start()
        time.sleep(0.2)
    l0 = muon.launch_count()
    ev = timer.run(one_step, args.steps)
    torch.cuda.synchronize(dev)
    launches = muon.launch_count() - l0
    barrier()
    clk = clocks.stop() if clocks else None
    ms, per_step = timer.times(ev)

    # ---- second pass, same steps, every launch bracketed by CUDA events on its
    # stream: per-kernel device durations for the roofline (the events cost a
    # few percent, so the headline value comes from the pass above)
    prof = {k: (0.0, 0) for k in muon.KINDS}
    ms_prof = None
    if args.kernel_events:
        muon.profile_enable(True)
        barrier()
        torch.cuda.synchronize(dev)
        evp = timer.run(one_step, args.steps)
        torch.cuda.synchronize(dev)
        muon.profile_enable(False)
        prof = muon.profile_read()
        ms_prof, _ = timer.times(evp)

    # ---- cold-L2 pass: the L2 is flushed before every step, each step timed alone
    cold = []
    if args.cold_steps:
        flush = torch.empty(256 << 20, dtype=torch.float32, device=dev)     # 1 GiB
        barrier()
        for s in range(args.cold_steps):
            flush_l2(flush)
            e = timer.run(one_step, 1, start=s)
            torch.cuda.synchronize(dev)
            cold.append(timer.times(e)[0])
        del flush
    # ---- the reduced-precision variant (muon_step_fp8) on the same workload,
    # timed the same way; reported beside the bf16 line, never as its value
    if muon.sync_status(stream) != 0:
        raise RuntimeError("device status after timing: " + muon.last_error())
    ms_max = mdist.max_over_ranks(ms, device=dev)

    flops_step = ns_flops(w.shapes)
    jobs = 1 if sharded else world              # sharded: one model split over the ranks
    value = flops_step * args.steps * jobs / (ms_max / 1e3) / 1e12

    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    kinds = {}
    for k, (tms, cnt) in prof.items():
        if cnt:
            kinds[k] = {"launches": cnt, "ms_total": tms, "us_per_launch": tms / cnt * 1e3,
                        "share_of_step": tms / ms_prof}
    # algorithmic work of this rank's own GEMM launches
    own_flops = flops_step
    if sharded:
        own_flops = ns_flops([w.shapes[i] for i in mdist.partition(w.shapes, world)[rank]])
    peak, peak_why = pick_peak(peaks, clk, ms / 1e3)
    roofline = None
    r = gemm_roofline(prof, own_flops, args.steps, peak) if args.kernel_events else None
    if r is not None:
        roofline = {"bound": "tensor", "kernel": "ns_gemm_kernel", "achieved": r["achieved"], "peak": peak,
                    "unit": "TFLOP/s", "frac": r["frac"], "traffic": ncu_traffic(),
                    "peak_source": f"{peak_src} {peak_why}", "flops_per_launch": r["flops_per_launch"],
                    "us_per_launch": r["us_per_launch"], "frac_burst": r["achieved"] / burst}
        if peaks.get("bf16_tflops_sustained"):
            roofline["frac_sustained"] = r["achieved"] / float(peaks["bf16_tflops_sustained"])
        if clk:
            roofline["kcycles_per_launch"] = r["us_per_launch"] * clk["sm_mhz"] / 1e3
    fused = [k for k in ("small", "pair", "quad") if prof[k][1]]
    if r is None and fused and args.kernel_events:
        # every matrix ran in a fused on-chip kernel: its launches carry the whole step
        f_ms = sum(prof[k][0] for k in fused)
        f_launches = sum(prof[k][1] for k in fused)
        achieved = own_flops * args.steps / (f_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": " + ".join(f"ns_{k}_kernel" for k in fused), "achieved": achieved,
                    "peak": burst, "unit": "TFLOP/s", "frac": achieved / burst, "traffic": None,
                    "peak_source": f"{peak_src} bf16_tflops (burst: one short launch per step)",
                    "flops_per_launch": own_flops * args.steps / f_launches,
                    "us_per_launch": f_ms / f_launches * 1e3}
    if roofline is not None and "prologue" in kinds:
        pro_bytes = 14.0 * sum(w.shapes[i][0] * w.shapes[i][1] for i in
                               (mdist.partition(w.shapes, world)[rank] if sharded else range(w.n_matrices)))
        pro_s = prof["prologue"][0] / prof["prologue"][1] / 1e3
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        roofline["prologue"] = {"bound": "hbm", "achieved": pro_bytes / pro_s / 1e9, "peak": hbm, "unit": "GB/s",
                                "frac": pro_bytes / pro_s / 1e9 / hbm, "bytes_per_launch": pro_bytes}

    # ---- end to end through the host-buffer entry point
    e2e = None
    if not args.no_e2e:
        Wh = [x.cpu().pin_memory() for x in W]
        bh = [x.cpu().pin_memory() for x in bufs]
        gh = [[x.cpu().pin_memory() for x in gs] for gs in gsets[:2]]
        for s in range(2):
            muon.step_host(Wh, gh[s % 2], bh, lr=w.lr, mu=w.mu, stream=stream)
        barrier()
        k2 = max(2, min(args.steps, args.e2e_steps))
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for s in range(k2):
            muon.step_host(Wh, gh[s % 2], bh, lr=w.lr, mu=w.mu, stream=stream)
        el = mdist.max_over_ranks(time.perf_counter() - t0, device=dev)
        e2e = {"value": flops_step * k2 * world / el / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": 12 * w.n_elements, "d2h_bytes_per_step": 8 * w.n_elements,
               "ms_per_step": el / k2 * 1e3, "steps": k2,
               "path": "muon_step_host: pinned host W, g, buf -> device, step, W and buf -> host"}
        del Wh, bh, gh

    sweep = None
    if rank == 0 and world == 1 and args.sweep:
        del W, bufs, gsets, stepper
        torch.cuda.empty_cache()
        sweep = run_sweep(args, muon, workloads, torch, dev, stream, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r_all = cpu_oracle_rate(w, budget_s=args.ref_budget)
        cpu = {k: r_all[k] for k in ("value", "unit", "cores", "kind", "sample")}
        if args.ref_budget_1core > 0:
            r_one = cpu_oracle_rate(w, budget_s=args.ref_budget_1core, threads=1)
            cpu["one_core"] = {"value": r_one["value"], "unit": UNIT, "cores": r_one["cores"],
                               "sample": r_one["sample"]}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) gradients, N(0,0.02) weights, zero-initialised momentum; "
                "GPT-2-124M hidden-matrix shapes)",
        "config": workload_config(w, args, sharded),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "chain_clusters": muon.chain_clusters(),
        "clocks": clk,
        "step_times": {"ms_median": statistics.median(per_step), "ms_min": min(per_step), "ms_max": max(per_step),
                       "ms_cold_l2_median": statistics.median(cold) if cold else None,
                       "cold_l2_steps": len(cold),
                       "cold_l2": "a 1 GiB buffer is written before each cold step (evicts the 126 MB L2)"},
        "kernels": kinds,
        "sweep": sweep,
        "dense_equivalent": {"value": value * ns_flops_dense(w.shapes) / flops_step, "unit": UNIT,
                             "what": "the same step counted as dense products (X X^T and A A in full): "
                                     "a label for comparison, not work done"},
        "frac_of_dense_peak": value / world / burst,
        "frac_of_dense_spec": value / world / 2250.0,
        "peaks": {"source": peak_src, "bf16_tflops": peaks.get("bf16_tflops"),
                  "bf16_tflops_sustained": peaks.get("bf16_tflops_sustained"), "hbm_gbs": peaks.get("hbm_gbs")},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="gpt2_124m")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--grad-sets", type=int, default=10)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--ref-budget", type=float, default=12.0, help="seconds of CPU oracle work (cpu_baseline)")
    ap.add_argument("--ref-total", type=float, default=90.0, help="seconds of CPU oracle work (--impl reference)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-events", type=int, default=1, help="per-launch CUDA events in a second timed pass")
    ap.add_argument("--fp8-iters", type=int, default=2,
                    help="also time muon_step_fp8 (this many e4m3 iterations; 0: skip) beside the bf16 step on "
                         "the sweep's sizes above 1024, where it applies")
    ap.add_argument("--replicas", action="store_true",
                    help="under torchrun: an independent copy of the workload per rank instead of the sharded step")
    ap.add_argument("--per-phase", action="store_true",
                    help="run the Newton-Schulz phases as one launch per phase (the path of short sides "
                         "above 1024) instead of the chained launch")
    ap.add_argument("--sweep", default="1024,2048,4096",
                    help="square batch sizes n (64 matrices each) timed for the sweep object ('' to skip)")
    ap.add_argument("--sweep-steps", type=int, default=5)
    ap.add_argument("--cold-steps", type=int, default=5, help="steps timed one by one after an L2 flush")
    ap.add_argument("--ref-budget-1core", type=float, default=4.0,
                    help="seconds of single-threaded CPU oracle work (cpu_baseline.one_core)")
    ap.add_argument("--buckets", type=int, default=2,
                    help="with --sharded: runs per rank whose all_gather overlaps the next run's step")
    ap.add_argument("--exchange", choices=("w32", "o16"), default="w32",
                    help="sharded step: all_gather the updated fp32 weights, or the bf16 update (every rank applies)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
