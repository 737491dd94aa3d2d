"""Throughput of the Sign-Muon optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

A step is one full Sign-Muon step over every matrix and worker of the
workload: momentum + Frobenius norm, k Newton-Schulz iterations with the sign
fused into the last one, and the majority vote fused with the update (plus
the local polar step when the workload has it).  The metric is
params * workers / s (whole job); inputs are resident in HBM and larger than
L2.  The default workload is the batch of 32 square 4096 x 4096 matrices
(M = 16 workers, k = 5, 1-bit vote, local polar step); its line also carries
three more rows measured in the same run, each with its roofline: the vote +
update sweep point (2^30 parameters, M = 16, fp32 W), the majority-vote Signum
step (k = 0) and the step with spectral scaling, both on the nanoGPT-small
matrices (`--no-extras` skips them).  With N > 1 (torchrun) every rank runs an independent replica by default:
the M workers are buffers on one GPU, so the step has no exchange; with
--exchange every rank runs the workload's workers and the signs of all ranks
are exchanged (NCCL) before one vote over all of them.

Rank 0 prints one JSON line.  `--impl reference` times the CPU fp64 oracle on
a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
# stdout carries exactly one JSON line (see emit()): NCCL's own messages go to
# stderr unless the caller chose a file.
os.environ.setdefault("NCCL_DEBUG_FILE", "/dev/stderr")
_RESULT_FD = None


def _claim_stdout():
    """Keeps the real stdout for the result line and points file descriptor 1
    at stderr, so that whatever else writes to it (library banners printed
    from C, e.g. NCCL's version line at communicator setup) cannot add lines
    to stdout."""
    global _RESULT_FD
    if _RESULT_FD is None:
        sys.stdout.flush()
        _RESULT_FD = os.dup(1)
        os.dup2(2, 1)


def emit(obj):
    """Writes the one JSON result line to the real stdout."""
    data = (json.dumps(obj) + "\n").encode()
    if _RESULT_FD is None:
        sys.stdout.write(data.decode())
        sys.stdout.flush()
    else:
        os.write(_RESULT_FD, data)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "params·workers/s per Sign-Muon step"
UNIT = "params*workers/s"
DEFAULT_CONFIG = "square4096x32"
# Timed steps per workload when --steps is not given (about a second of GPU time).
DEFAULT_STEPS = {"single256": 200, "nanogpt_small": 60, "resnet50": 100, "square4096x32": 10,
                 "signum_nanogpt_small": 100}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# The sources of each kernel (for the Newton-Schulz kernel also the plan,
# which fixes its tile order); a captured traffic figure is used only while
# they are unchanged.
_CSRC = "sign_muon_optimizer_momentum_b200/csrc/"
KERNEL_SOURCES = {
    "ns_gemm_kernel": (_CSRC + "ns_gemm.cu", _CSRC + "common.cuh", _CSRC + "api.cu"),
    "momentum_kernel": (_CSRC + "elementwise.cu", _CSRC + "common.cuh"),
    "vote_kernel": (_CSRC + "elementwise.cu", _CSRC + "common.cuh"),
    "spectral_rowpass_kernel": (_CSRC + "elementwise.cu", _CSRC + "common.cuh"),
    "spectral_segment_kernel": (_CSRC + "elementwise.cu", _CSRC + "common.cuh"),
}


def kernel_source_hash(kernel):
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


def captured_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the ncu summary in
    profiles/dram_traffic.json, or None if absent or taken on other sources."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        entries = json.load(open(p))
    except ValueError:
        return None
    src = kernel_source_hash(kernel)
    for e in entries:
        if e.get("kernel") == kernel and e.get("workload") == workload and e.get("source_hash") == src:
            return e.get("bytes_per_launch")
    return None


def ns_flops(shapes, n_workers, k, dense=False):
    """Algorithmic Newton-Schulz FLOPs per step: per iteration and unit,
    Gram s^2 l (symmetric output), square s^3 (symmetric output) and apply
    2 s^2 l; dense counts 4 s^2 l + 2 s^3."""
    tot = 0
    for r, c in shapes:
        s, l = min(r, c), max(r, c)
        tot += (4 * s * s * l + 2 * s ** 3) if dense else (3 * s * s * l + s ** 3)
    return tot * n_workers * k


def max_over_ranks_value(x, world, device):
    """The slowest rank's value (every rank calls this at the same point)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_throughput(units_per_step, steps, world, max_ms):
    """Whole-job units/s: every rank processes units_per_step per step (weak
    scaling, independent replicas), timed by the slowest rank."""
    return units_per_step * steps * world / (max_ms / 1e3)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.skip = 0

    def mark(self):
        """Samples taken so far (before the timed region) are left out."""
        try:
            self.skip = len(open(self.path).read().splitlines())
        except Exception:
            self.skip = 0

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [ln.split(",") for ln in open(self.path).read().splitlines()[self.skip:] if ln.strip()]
        os.unlink(self.path)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower().startswith("active"):
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- oracle arm
def oracle_sample_step(wl, units, seed=0):
    """One oracle step over a sample of (matrix, worker) units: momentum,
    Newton-Schulz, sign (and pack) per unit, then the vote and update of each
    sampled matrix over its sampled workers.  Returns params*workers done."""
    import numpy as np
    from oracle import signmuon_oracle as O
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    by_mat = {}
    for i, m in units:
        by_mat.setdefault(i, []).append(m)
    done = 0
    for i, workers in by_mat.items():
        r, c = wl.shapes[i]
        g_star = syn.gaussian((r, c), wl.g_signal_std, "cpu", "Gstar", seed, i).double().numpy()
        w = O.round_to_dtype(syn.gaussian((r, c), wl.w_std, "cpu", "W", seed, i).double().numpy(), wl.w_dtype)
        grads = [O.round_to_dtype(g_star + syn.gaussian((r, c), wl.g_noise_std, "cpu", "eps", seed, i, m, 0)
                                  .double().numpy(), wl.w_dtype) for m in workers]
        O.signmuon_step(w, grads, [np.zeros((r, c)) for _ in workers], beta=float(np.float32(wl.beta)),
                        eta=wl.eta, k=wl.ns_iters, w_dtype=wl.w_dtype, polar=wl.polar,
                        int8_variant=(wl.variant == "int8"))
        done += r * c * len(workers)
    return done


def oracle_sample(wl, budget_s):
    """(matrix, worker) units whose oracle step fits in about budget_s: one
    unit of every distinct shape first (so that every shape, and both the
    wide and the tall Newton-Schulz branch, is in the sample), then further
    workers of those matrices, shape by shape in turn."""
    order, seen = [], set()
    for i, s in enumerate(wl.shapes):
        if s not in seen:
            seen.add(s)
            order.append(i)
    t0 = time.perf_counter()
    chosen = [(i, 0) for i in order]
    for u in chosen:
        oracle_sample_step(wl, [u])
    for m in range(1, wl.n_workers):
        for i in order:
            if time.perf_counter() - t0 > budget_s:
                return chosen
            chosen.append((i, m))
            oracle_sample_step(wl, [(i, m)])
    return chosen


def describe_sample(wl, units):
    mats = sorted({i for i, _ in units})
    shapes = ", ".join(f"{wl.shapes[i][0]}x{wl.shapes[i][1]}" for i in mats)
    return (f"{len(units)} of {wl.units} (matrix, worker) units over {len(mats)} matrices ({shapes}), "
            f"k={wl.ns_iters}, fp64 numpy")


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:
        return None


def cpu_baseline(wl, budget_s=15.0):
    units = oracle_sample(wl, budget_s * 0.4)
    t0 = time.perf_counter()
    done = oracle_sample_step(wl, units)
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": UNIT, "cores": blas_threads() or host_cores(), "kind": "oracle",
            "sample": f"one oracle step over {describe_sample(wl, units)}; {dt:.1f} s"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # Size each step's sample so that the whole --steps/--warmup run stays
    # within about three minutes of host time.
    per_step = max(0.2, 150.0 / (args.steps + args.warmup))
    mats = oracle_sample(wl, per_step * 0.6)
    for _ in range(args.warmup):
        oracle_sample_step(wl, mats[:1])
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += oracle_sample_step(wl, mats)
    dt = time.perf_counter() - t0
    value = done / dt
    sample = f"each step: one oracle step over {describe_sample(wl, mats)}"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": line_config(wl, args, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle",
                             "cores": blas_threads() or host_cores(), "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    emit(line)
    return 0


def workload_config(wl):
    return {"workload": wl.name, "matrices": len(wl.shapes), "params": wl.params, "workers": wl.n_workers,
            "ns_iters": wl.ns_iters, "variant": wl.variant, "w_dtype": wl.w_dtype, "polar": wl.polar,
            "beta": wl.beta, "eta": wl.eta}


def resident_bytes(wl):
    """Gradients (W's dtype) and fp32 momentum of every (matrix, worker) unit."""
    return wl.params * wl.n_workers * ((2 if wl.w_dtype == "bf16" else 4) + 4)


def line_config(wl, args, world):
    """The `config` of the result line; both arms print the same one."""
    cfg = dict(workload_config(wl), norm=args.norm)
    cfg["parallelism"] = (f"dp{world}-{'allgather' if wl.variant == 'pack1' else 'allreduce'}"
                          if args.exchange else f"replicas{world}")
    cfg["l2"] = f"inputs larger than L2 ({resident_bytes(wl) / 2**30:.1f} GiB gradients+momentum resident)"
    cfg["launch"] = "cuda_graph" if args.graph else "eager"
    return cfg


# --------------------------------------------------------------------------- GPU arm
class Ctx:
    """Process-group and device facts of this rank, shared by the timed runs."""

    def __init__(self, world, rank, local, dev):
        self.world, self.rank, self.local, self.dev = world, rank, local, dev

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
        import torch
        torch.cuda.synchronize()

    def max_over_ranks(self, x):
        return max_over_ranks_value(x, self.world, self.dev)


def ns_roofline(wl, ns_ms, ms_total, pk, steps):
    """Newton-Schulz roofline: algorithmic FLOPs of the step's NS call over
    its mean duration, against the sustained bf16 peak when the timed region
    lasts 0.5 s or more (the GPU then sits at its power cap, the condition of
    the sustained figure), else the burst peak."""
    flops = ns_flops(wl.shapes, wl.n_workers, wl.ns_iters)
    note = ("Newton-Schulz call of the step (the local polar step is timed with the vote)" if wl.polar
            else "Newton-Schulz call of the step")
    achieved = flops / (ns_ms / 1e3) / 1e12
    dense = ns_flops(wl.shapes, wl.n_workers, wl.ns_iters, True) / (ns_ms / 1e3) / 1e12
    sustained = ms_total >= 500.0
    peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    return {"bound": "tensor", "kernel": "ns_gemm_kernel", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": captured_traffic("ns_gemm_kernel", wl.name),
            "note": f"{note}: {flops / 1e12:.3f} TFLOP algorithmic (symmetric-aware: 3s^2l + s^3 per iteration "
                    f"and unit) per step over {ns_ms:.3f} ms (CUDA events, mean of {steps} timed steps, "
                    f"{ms_total / 1e3:.2f} s of timed work); dense-equivalent {dense:.1f} TFLOP/s; peak = "
                    f"{pk['source']} {'sustained' if sustained else 'burst'} bf16 cuBLAS (burst "
                    f"{pk['bf16_tflops']}, sustained {pk['bf16_tflops_sustained']}); frac of burst "
                    f"{achieved / pk['bf16_tflops']:.3f}, of sustained {achieved / pk['bf16_tflops_sustained']:.3f}"}


def momentum_roofline(wl, opt, mom_ms, pk):
    """k = 0 (majority-vote Signum): the momentum pass dominates.  Fused (the
    momentum kernel writes the signs) or momentum + bf16 copy."""
    fused = getattr(opt, "fused_sign", False)
    out_b = (1 / 8 if wl.variant == "pack1" else 1) if fused else 2
    gbytes = wl.params * wl.n_workers * ((2 if wl.w_dtype == "bf16" else 4) + 8 + out_b)
    achieved = gbytes / (mom_ms / 1e3) / 1e9
    out_what = ("packed sign" if wl.variant == "pack1" else "int8 sign") if fused else "bf16 copy"
    return {"bound": "hbm", "kernel": "momentum_kernel", "achieved": achieved, "peak": pk["hbm_gbs"],
            "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": captured_traffic("momentum_kernel", wl.name),
            "note": f"momentum call: {gbytes / 1e9:.3f} GB algorithmic (gradient read, fp32 momentum read+write, "
                    f"{out_what} write) per step over {mom_ms:.3f} ms"}


def time_workload(ctx, wl, args, *, norm, steps, warmup, graph=False, exchange=False, e2e=False, clocks=False):
    """Builds the workload's optimizer and inputs on this rank and times
    `steps` whole steps after `warmup` (CUDA events on the step's stream,
    max over ranks).  Returns the measured figures."""
    import torch
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    dev, rank, world = ctx.dev, ctx.rank, ctx.world
    dt = syn.torch_dtype(wl.w_dtype)
    if exchange:
        # One group of n_workers workers per GPU; the signs of all GPUs are
        # exchanged (1-bit all-gather for packed workloads, int8 SUM
        # all-reduce for int8 ones) and every GPU votes over all of them.
        from sign_muon_optimizer_momentum_b200.distributed import SignMuonDistStep
        if norm != "frobenius" or graph:
            raise SystemExit("--exchange runs eagerly with the Frobenius scaling only")
        opt = SignMuonDistStep(wl.shapes, wl.n_workers, wl.ns_iters, wl.variant, wl.beta, wl.eta, dt,
                               polar=wl.polar, device=dev)
    else:
        opt = SignMuonStep(wl.shapes, wl.n_workers, wl.ns_iters, wl.variant, wl.beta, wl.eta, dt,
                           polar=wl.polar, device=dev, norm=norm)
    # Replicas draw their own problem; with --exchange all ranks share W and
    # the gradient signal G* (one model, data-parallel), and their workers
    # differ through the per-rank noise drawn below.
    problem_seed = 0 if exchange else rank
    weights = [w.to(dev) for w in syn.initial_weights(wl, problem_seed)]
    signal = [g.to(dev) for g in syn.gradient_signal(wl, problem_seed)]
    n_sets = 2
    grad_sets = []
    for t in range(n_sets):
        gs = []
        for i in range(len(wl.shapes)):
            for m in range(wl.n_workers):
                gs.append(syn.worker_gradient(wl, signal[i], i, m, t, rank))
        grad_sets.append(gs)
    del signal
    stream = torch.cuda.current_stream(dev)
    s_ptr = stream.cuda_stream

    def one_step(t, ev=None):
        gs = grad_sets[t % n_sets]
        if ev is not None:
            ev[0].record(stream)
        opt.momentum_norm(gs, s_ptr)
        if ev is not None:
            ev[1].record(stream)
        opt.newton_schulz(s_ptr)
        if ev is not None:
            ev[2].record(stream)
        opt.vote_update(weights, s_ptr)
        if ev is not None:
            ev[3].record(stream)

    graphs = None
    if graph:
        # One CUDA graph per gradient set: each replay is a whole step.
        graphs = [opt.capture(weights, grad_sets[t]) for t in range(n_sets)]
    for t in range(warmup):
        if graphs:
            graphs[t % n_sets].replay()
        else:
            one_step(t)
    ctx.barrier()
    if graphs:
        # Phases from the captured kernels cannot be told apart on the host:
        # they are taken from eager steps (same kernels), the step time from
        # the replays.
        ph_ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(steps)]
        for t in range(steps):
            one_step(t, ph_ev[t])
        ctx.barrier()
    sampler = ClockSampler(ctx.local) if (clocks and rank == 0) else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
        sampler.mark()
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx.barrier()
    start.record(stream)
    for t in range(steps):
        if graphs:
            graphs[t % n_sets].replay()
        else:
            one_step(t, ev[t])
    stop.record(stream)
    ctx.barrier()
    ms = ctx.max_over_ranks(start.elapsed_time(stop))
    if graphs:
        ev = ph_ev
    phases = {"momentum": sum(e[0].elapsed_time(e[1]) for e in ev) / steps,
              "newton_schulz": sum(e[1].elapsed_time(e[2]) for e in ev) / steps,
              "vote_update": sum(e[2].elapsed_time(e[3]) for e in ev) / steps}
    clk = sampler.stop() if sampler else None
    units_per_step = wl.params * wl.n_workers
    out = {"ms_total": ms, "ms_per_step": ms / steps, "value": job_throughput(units_per_step, steps, world, ms),
           "phases_ms": phases, "gpu_launches": opt.kernel_launches_per_step() * steps, "clocks": clk, "opt": opt}
    if exchange:
        out["exchange_bytes_per_step"] = opt.exchange_bytes_per_step()
    if norm == "spectral":
        # The power iterations alone, timed on the step's own bf16 copies of
        # the momentum (they hold the last step's values).
        from sign_muon_optimizer_momentum_b200 import _lib as L
        xp = [x.data_ptr() for x in opt.x]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 200

        def spectral():
            L.signmuon_spectral_norm(opt.shapes, opt.n_workers, xp, opt.spectral_iters, opt.inv_norm.data_ptr(),
                                     opt.ws_spec.data_ptr(), opt.ws_spec.numel(), s_ptr)

        for _ in range(3):
            spectral()
        ctx.barrier()
        sp_sampler = ClockSampler(ctx.local) if (clocks and rank == 0) else None
        if sp_sampler:
            sp_sampler.start()
            time.sleep(0.3)
            sp_sampler.mark()
        a.record(stream)
        for _ in range(reps):
            spectral()
        b.record(stream)
        ctx.barrier()
        out["spectral_ms"] = ctx.max_over_ranks(a.elapsed_time(b)) / reps
        out["spectral_clocks"] = sp_sampler.stop() if sp_sampler else None
    if e2e:
        # End to end through the public step with HOST buffers: each step's
        # gradients come from pinned host memory and the updated weights go
        # back to host memory.  The next step's gradients are copied on a
        # second stream while the current step computes (copy engines overlap
        # the kernels).
        host_g = [g.cpu().pin_memory() for g in grad_sets[0]]
        host_w = [torch.empty(w.shape, dtype=w.dtype, pin_memory=True) for w in weights]
        h2d = sum(g.numel() * g.element_size() for g in host_g)
        d2h = sum(w.numel() * w.element_size() for w in weights)
        copy_stream = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        consumed = [torch.cuda.Event(), torch.cuda.Event()]

        def h2d_into(buf):
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(consumed[buf])
                for hg, dg in zip(host_g, grad_sets[buf]):
                    dg.copy_(hg, non_blocking=True)
                copied[buf].record(copy_stream)

        # The updated weights go back to the host on a third stream: the next
        # step reads them only in its final vote/update phase, which waits
        # for that copy, so the copy overlaps the next step's momentum and
        # Newton-Schulz work.
        d2h_stream = torch.cuda.Stream(dev)
        updated, read_back = torch.cuda.Event(), torch.cuda.Event()

        def e2e_steps(n):
            # Steady state: step t copies step t + 1's gradients while it
            # computes (the copy for the step after the last one included),
            # so n steps make n H2D copies and n D2H read-backs; the first
            # step's gradients were copied before.
            for t in range(n):
                buf = t % 2
                h2d_into(1 - buf)
                stream.wait_event(copied[buf])
                opt.momentum_norm(grad_sets[buf], s_ptr)
                consumed[buf].record(stream)
                opt.newton_schulz(s_ptr)
                if t > 0:
                    stream.wait_event(read_back)
                opt.vote_update(weights, s_ptr)
                updated.record(stream)
                with torch.cuda.stream(d2h_stream):
                    d2h_stream.wait_event(updated)
                    for hw, w in zip(host_w, weights):
                        hw.copy_(w, non_blocking=True)
                    read_back.record(d2h_stream)
            stream.wait_event(read_back)       # the last step's weights are on the host
            stream.wait_event(copied[n % 2])   # and the next step's gradients on the device

        h2d_into(0)
        stream.wait_event(copied[0])
        e2e_steps(2)
        ctx.barrier()
        e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(steps, 10))
        e_start.record(stream)
        e2e_steps(n_e2e)
        e_stop.record(stream)
        ctx.barrier()
        e_ms = ctx.max_over_ranks(e_start.elapsed_time(e_stop))
        out["e2e"] = {"value": units_per_step * n_e2e * world / (e_ms / 1e3), "unit": UNIT,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
                      "ms_per_step": e_ms / n_e2e,
                      "note": "gradients H2D from pinned host memory and weights D2H to pinned host memory, every "
                              "step, each on its own copy stream overlapped with the neighbouring step's compute "
                              "(steady state: each step copies the next step's gradients; the timed region holds "
                              "one H2D and one D2H per step)"}
        del host_g, host_w
    if graphs:
        del graphs
    return out


def extra_signum(ctx, args, pk):
    """Majority-vote Signum (k = 0) on the nanoGPT-small matrices: the fused
    momentum + sign pass, then the vote + update."""
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    wl = syn.WORKLOADS["signum_nanogpt_small"]
    r = time_workload(ctx, wl, args, norm="frobenius", steps=300, warmup=5, clocks=True)
    return {"workload": wl.name, "config": workload_config(wl), "metric": METRIC, "value": r["value"], "unit": UNIT,
            "ms_per_step": r["ms_per_step"], "steps": 300, "warmup": 5, "phases_ms": r["phases_ms"],
            "roofline": momentum_roofline(wl, r["opt"], r["phases_ms"]["momentum"], pk), "clocks": r["clocks"]}


def spectral_bytes_per_iteration(shapes, n_workers):
    """Algorithmic bytes of one power iteration: each unit's bf16 copy of M
    read once, and its partial sums of z written and read back (for widths
    that are multiples of 8 up to 4096 two per 128-row segment up to 1536
    columns and one beyond, else one per 32-row block), 4 B per column each."""
    total = 0
    for r, c in shapes:
        if c % 8 == 0 and c <= 4096:
            rs = 2 if c <= 1536 else 1
            parts = -(-r // 128) * rs
        else:
            parts = -(-r // 32)
        total += r * c * 2 + 2 * parts * c * 4
    return total * n_workers


def extra_spectral(ctx, args, pk):
    """The nanoGPT-small step with spectral scaling of the Newton-Schulz input
    (5 power iterations per unit); roofline of the power-iteration pass: per
    iteration each unit's bf16 copy of M is read once (2 B/param) and its
    partial sums of z written and read back."""
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    wl = syn.WORKLOADS["nanogpt_small"]
    r = time_workload(ctx, wl, args, norm="spectral", steps=30, warmup=3, clocks=True)
    iters = r["opt"].spectral_iters
    per_iter = spectral_bytes_per_iteration(wl.shapes, wl.n_workers)
    gbytes = iters * per_iter
    achieved = gbytes / (r["spectral_ms"] / 1e3) / 1e9
    kernel = "spectral_segment_kernel"
    return {"workload": wl.name, "config": dict(workload_config(wl), norm="spectral", spectral_iters=iters),
            "metric": METRIC, "value": r["value"], "unit": UNIT, "ms_per_step": r["ms_per_step"], "steps": 30,
            "warmup": 3, "phases_ms": dict(r["phases_ms"], spectral_alone=r["spectral_ms"]),
            "clocks": r["clocks"], "clocks_spectral_alone": r["spectral_clocks"],
            "roofline": {"bound": "hbm", "kernel": kernel, "achieved": achieved,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                         "traffic": captured_traffic(kernel, wl.name),
                         "note": f"{iters} power iterations: {gbytes / 1e9:.3f} GB algorithmic "
                                 f"({per_iter / (wl.params * wl.n_workers):.3f} B per param*worker and iteration: "
                                 f"the bf16 copy of M once, partial sums of z written and read back) over "
                                 f"{r['spectral_ms']:.3f} ms, timed alone"}}


def run_gpu(args, wl):
    import torch
    import torch.distributed as dist
    from sign_muon_optimizer_momentum_b200 import build as _build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = world > 1 or args.exchange
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
        if args.exchange:
            import datetime
            import socket
            sk = socket.socket()
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
            sk.close()
            dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                    timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", 0))
    _build.build()
    ctx = Ctx(world, rank, local, torch.device("cuda", torch.cuda.current_device()))
    pk = peaks()
    extras = {}
    if wl.name == DEFAULT_CONFIG and not args.no_extras and not args.exchange:
        # Rows measured beside the headline workload, each with its roofline
        # and the clocks sampled during its own timed region.  They run first:
        # after the seconds-long headline run the power-capped clock is lower
        # for a while, which would slow the short, clock-sensitive rows.
        extras["vote_sweep"] = time_vote_sweep(ctx, 1 << 30, 16, "f32", steps=200, warmup=5, clocks=True)
        torch.cuda.empty_cache()
        extras["signum"] = extra_signum(ctx, args, pk)
        torch.cuda.empty_cache()
        extras["spectral"] = extra_spectral(ctx, args, pk)
        torch.cuda.empty_cache()
    r = time_workload(ctx, wl, args, norm=args.norm, steps=args.steps, warmup=args.warmup, graph=args.graph,
                      exchange=args.exchange, e2e=not args.no_e2e, clocks=True)
    if wl.ns_iters > 0:
        roofline = ns_roofline(wl, r["phases_ms"]["newton_schulz"], r["ms_total"], pk, args.steps)
    else:
        roofline = momentum_roofline(wl, r["opt"], r["phases_ms"]["momentum"], pk)
    result = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
              "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
              "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
              "config": line_config(wl, args, world), "roofline": roofline, "e2e": r.get("e2e"),
              "phases_ms": r["phases_ms"], "gpu_launches": r["gpu_launches"], "clocks": r["clocks"]}
    if "spectral_ms" in r:
        result["phases_ms"]["spectral_alone"] = r["spectral_ms"]
    if args.exchange:
        result["config"]["vote_workers"] = world * wl.n_workers
        result["config"]["exchange_bytes_per_step"] = r["exchange_bytes_per_step"]
    del r
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl)
    result.update(extras)
    if pg:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        emit(result)
    return 0


def time_vote_sweep(ctx, P, M, w_dtype, steps, warmup, clocks=False):
    """Vote + update alone (the bandwidth-bound row): P params as (P/1024, 1024)
    W (fp32 or bf16), M packed sign buffers with P(+1) ~ U(0,1) per entry."""
    import torch
    from sign_muon_optimizer_momentum_b200 import _lib as L
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    dev, rank, world = ctx.dev, ctx.rank, ctx.world
    shape = (P // 1024, 1024)
    stream = torch.cuda.current_stream(dev)
    words = L.signmuon_packed_words(shape)
    signs = []
    for m, s8 in syn.vote_sweep_signs(P, M, seed=rank, device=dev):
        buf = torch.empty(words, dtype=torch.int32, device=dev)
        L.signmuon_sign_pack(shape, L.SIGNMUON_F32, s8.float().data_ptr(), 1024, 0, buf.data_ptr(),
                             stream.cuda_stream)
        torch.cuda.synchronize()
        signs.append(buf)
        del s8
    w_bf16 = w_dtype == "bf16"
    w = syn.gaussian(shape, 0.02, dev, "W", rank, 0, dtype=torch.bfloat16 if w_bf16 else torch.float32)
    w_code = L.SIGNMUON_BF16 if w_bf16 else L.SIGNMUON_F32
    w_bytes = 2 if w_bf16 else 4
    wsz = L.signmuon_vote_workspace_bytes([shape], M)
    wsb = torch.zeros(wsz, dtype=torch.uint8, device=dev)
    sp = [t.data_ptr() for t in signs]

    def step():
        L.signmuon_vote_update([shape], M, False, sp, w_code, [w.data_ptr()], 0.01, None, 0, 0,
                               wsb.data_ptr(), wsz, stream.cuda_stream)

    for _ in range(warmup):
        step()
    ctx.barrier()
    sampler = ClockSampler(ctx.local) if (clocks and rank == 0) else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
        sampler.mark()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    ctx.barrier()
    ms = ctx.max_over_ranks(a.elapsed_time(b))
    clk = sampler.stop() if sampler else None
    per = ms / steps
    bytes_per = P * (M / 8 + 2 * w_bytes)
    pk = peaks()
    gbs = bytes_per / (per / 1e3) / 1e9
    return {"metric": METRIC, "value": P * M * world / (per / 1e3), "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": per, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic",
            "config": {"workload": "vote_sweep", "params": P, "workers": M, "w_dtype": w_dtype, "eta": 0.01,
                       "l2": f"inputs larger than L2 ({bytes_per / 2**30:.2f} GiB per step)"},
            "roofline": {"bound": "hbm", "kernel": "vote_kernel", "achieved": gbs, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                         "traffic": captured_traffic("vote_kernel", f"vote_sweep_P{P}_M{M}_{w_dtype}"),
                         "note": f"algorithmic {M}/8 + {2 * w_bytes} B/param (packed signs read, "
                                 f"{w_dtype} W read+write); peak = {pk['source']} copy bandwidth"},
            "gpu_launches": 2 * steps, "clocks": clk}


def run_vote_sweep(args):
    import torch
    from sign_muon_optimizer_momentum_b200 import build as _build
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    _build.build()
    ctx = Ctx(world, rank, local, torch.device("cuda", torch.cuda.current_device()))
    res = time_vote_sweep(ctx, args.sweep_params, args.sweep_workers, args.sweep_w_dtype, args.steps, args.warmup,
                          clocks=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        emit(res)
    return 0


def main():
    _claim_stdout()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--mats", type=int, default=None,
                    help="keep only the first N matrices of the workload (small profiling cases)")
    ap.add_argument("--workers", type=int, default=None,
                    help="override the workload's number of workers (small profiling cases)")
    ap.add_argument("--sweep-params", type=int, default=1 << 30)
    ap.add_argument("--sweep-workers", type=int, default=16)
    ap.add_argument("--sweep-w-dtype", default="f32", choices=["f32", "bf16"],
                    help="weight dtype of the vote sweep")
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg with host buffers (profiling runs only: the line then has no e2e)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the vote-sweep, Signum and spectral rows measured beside the default workload")
    ap.add_argument("--norm", default="frobenius", choices=["frobenius", "spectral"],
                    help="scaling of the Newton-Schulz input (spectral: 5 power iterations)")
    ap.add_argument("--graph", action="store_true",
                    help="time the step as one CUDA graph replay (captured with SignMuonStep.capture)")
    ap.add_argument("--exchange", action="store_true",
                    help="each GPU runs the workload's workers and the signs of all GPUs are exchanged "
                         "(1-bit all-gather or int8 SUM all-reduce, NCCL) before one vote over all workers; "
                         "default: independent replicas")
    args = ap.parse_args()
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    if args.config == "vote_sweep":
        if args.steps is None:
            args.steps = 50
        return run_vote_sweep(args)
    wl = syn.WORKLOADS[args.config]
    if args.mats or args.workers:
        import dataclasses
        name = wl.name + (f"[:{args.mats}]" if args.mats else "") + (f"[M={args.workers}]" if args.workers else "")
        wl = dataclasses.replace(wl, name=name, shapes=wl.shapes[: args.mats] if args.mats else wl.shapes,
                                 n_workers=args.workers or wl.n_workers)
    if args.steps is None:
        args.steps = 10 if args.impl == "reference" else DEFAULT_STEPS.get(wl.name, 20)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
