"""Throughput of the Sign-Muon optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

A step is one full Sign-Muon step over every matrix and worker of the
workload: momentum + Frobenius norm, k Newton-Schulz iterations with the sign
fused into the last one, and the majority vote fused with the update (plus
the local polar step when the workload has it).  The metric is
params * workers / s (whole job); inputs are resident in HBM and larger than
L2.  With N > 1 (torchrun) every rank runs an independent replica: the path
has no exchange step because the M workers are buffers on one GPU.

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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "params·workers/s per Sign-Muon step"
UNIT = "params*workers/s"
DEFAULT_CONFIG = "nanogpt_small"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def ns_flops(shapes, n_workers, k, dense=False):
    """Algorithmic Newton-Schulz FLOPs per step: per iteration and unit,
    Gram s^2 l (symmetric output), square s^3 (symmetric output) and apply
    2 s^2 l; dense counts 4 s^2 l + 2 s^3."""
    tot = 0
    for r, c in shapes:
        s, l = min(r, c), max(r, c)
        tot += (4 * s * s * l + 2 * s ** 3) if dense else (3 * s * s * l + s ** 3)
    return tot * n_workers * k


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
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
        rows = [ln.split(",") for ln in open(self.path).read().splitlines() if ln.strip()]
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
def oracle_sample_step(wl, mats, seed=0):
    """One oracle step over the (matrix index) sample: returns params*workers processed."""
    import numpy as np
    from oracle import signmuon_oracle as O
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    done = 0
    for i in mats:
        r, c = wl.shapes[i]
        g_star = syn.gaussian((r, c), wl.g_signal_std, "cpu", "Gstar", seed, i).double().numpy()
        w = syn.gaussian((r, c), wl.w_std, "cpu", "W", seed, i).double().numpy()
        grads = [g_star + syn.gaussian((r, c), wl.g_noise_std, "cpu", "eps", seed, i, m, 0).double().numpy()
                 for m in range(wl.n_workers)]
        moms = [np.zeros((r, c)) for _ in range(wl.n_workers)]
        O.signmuon_step(O.round_to_dtype(w, wl.w_dtype), [O.round_to_dtype(g, wl.w_dtype) for g in grads], moms,
                        beta=float(np.float32(wl.beta)), eta=wl.eta, k=wl.ns_iters, w_dtype=wl.w_dtype,
                        polar=wl.polar, int8_variant=(wl.variant == "int8"))
        done += r * c * wl.n_workers
    return done


def oracle_sample(wl, budget_s):
    """Matrices (one of each shape first) whose oracle step fits in ~budget_s."""
    order, seen = [], set()
    for i, s in enumerate(wl.shapes):
        if s not in seen:
            seen.add(s)
            order.append(i)
    t0 = time.perf_counter()
    chosen = []
    for i in order:
        chosen.append(i)
        oracle_sample_step(wl, [i])
        if time.perf_counter() - t0 > budget_s:
            break
    return chosen


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
    mats = oracle_sample(wl, budget_s * 0.4)
    t0 = time.perf_counter()
    done = oracle_sample_step(wl, mats)
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": UNIT, "cores": blas_threads() or host_cores(), "kind": "oracle",
            "sample": f"one oracle step (fp64 numpy) over {len(mats)} of {len(wl.shapes)} matrices "
                      f"({', '.join(f'{wl.shapes[i][0]}x{wl.shapes[i][1]}' for i in mats)}) x "
                      f"{wl.n_workers} workers, k={wl.ns_iters}; {dt:.1f} s"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    mats = oracle_sample(wl, 10.0)
    for _ in range(args.warmup):
        oracle_sample_step(wl, mats[:1])
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += oracle_sample_step(wl, mats)
    dt = time.perf_counter() - t0
    value = done / dt
    sample = (f"each step: one oracle step (fp64 numpy) over {len(mats)} of {len(wl.shapes)} matrices x "
              f"{wl.n_workers} workers, k={wl.ns_iters}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle",
                             "cores": blas_threads() or host_cores(), "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl):
    return {"workload": wl.name, "matrices": len(wl.shapes), "params": wl.params, "workers": wl.n_workers,
            "ns_iters": wl.ns_iters, "variant": wl.variant, "w_dtype": wl.w_dtype, "polar": wl.polar,
            "beta": wl.beta, "eta": wl.eta}


# --------------------------------------------------------------------------- GPU arm
def run_gpu(args, wl):
    import torch
    import torch.distributed as dist
    from sign_muon_optimizer_momentum_b200 import build as _build
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    _build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    dt = syn.torch_dtype(wl.w_dtype)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return t.item()

    opt = SignMuonStep(wl.shapes, wl.n_workers, wl.ns_iters, wl.variant, wl.beta, wl.eta, dt,
                       polar=wl.polar, device=dev)
    weights = [w.to(dev) for w in syn.initial_weights(wl, rank)]
    signal = [g.to(dev) for g in syn.gradient_signal(wl, rank)]
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
    resident = sum(g.numel() * g.element_size() for g in grad_sets[0]) + sum(m.numel() * 4 for m in opt.mom)

    def one_step(t, ev=None):
        gs = grad_sets[t % n_sets]
        opt.momentum_norm(gs, s_ptr)
        if ev is not None:
            ev[0].record(stream)
        opt.newton_schulz(s_ptr)
        if ev is not None:
            ev[1].record(stream)
        opt.vote_update(weights, s_ptr)

    for t in range(args.warmup):
        one_step(t)
    barrier()

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    ns_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    start.record(stream)
    for t in range(args.steps):
        one_step(t, ns_ev[t])
    stop.record(stream)
    barrier()
    ms = max_over_ranks(start.elapsed_time(stop))
    ns_ms = sum(a.elapsed_time(b) for a, b in ns_ev) / args.steps
    clk = clocks.stop() if clocks else None

    units_per_step = wl.params * wl.n_workers
    value = units_per_step * args.steps * world / (ms / 1e3)

    # End to end through the public step: pinned host gradients -> device,
    # step, weights -> host, every step.
    host_g = [g.cpu().pin_memory() for g in grad_sets[0]]
    dev_g = grad_sets[1]
    host_w = [torch.empty(w.shape, dtype=w.dtype, pin_memory=True) for w in weights]
    h2d = sum(g.numel() * g.element_size() for g in host_g)
    d2h = sum(w.numel() * w.element_size() for w in weights)
    for _ in range(1):
        for hg, dg in zip(host_g, dev_g):
            dg.copy_(hg, non_blocking=True)
        opt.step(weights, dev_g)
    barrier()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(2, min(args.steps, 5))
    e_start.record(stream)
    for _ in range(e_steps):
        for hg, dg in zip(host_g, dev_g):
            dg.copy_(hg, non_blocking=True)
        opt.step(weights, dev_g)
        for hw, w in zip(host_w, weights):
            hw.copy_(w, non_blocking=True)
    e_stop.record(stream)
    barrier()
    e_ms = max_over_ranks(e_start.elapsed_time(e_stop))
    e2e = {"value": units_per_step * e_steps * world / (e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
           "ms_per_step": e_ms / e_steps}

    pk = peaks()
    flops = ns_flops(wl.shapes, wl.n_workers, wl.ns_iters)
    if wl.polar:
        flops_note = "Newton-Schulz call of the step (the local polar step is timed with the vote)"
    else:
        flops_note = "Newton-Schulz call of the step"
    achieved = flops / (ns_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": "ns_gemm_kernel", "achieved": achieved,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                "traffic": None,
                "note": f"{flops_note}: {flops / 1e12:.3f} TFLOP algorithmic (symmetric-aware) per step "
                        f"over {ns_ms:.3f} ms (CUDA events, mean of {args.steps} timed steps); "
                        f"dense-equivalent {ns_flops(wl.shapes, wl.n_workers, wl.ns_iters, True) / (ns_ms / 1e3) / 1e12:.1f} "
                        f"TFLOP/s; peak = {pk['source']} burst bf16 cuBLAS "
                        f"(sustained {pk['bf16_tflops_sustained']})"}
    result = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
              "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
              "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
              "config": dict(workload_config(wl), parallelism=f"replicas{world}",
                             l2=f"inputs larger than L2 ({resident / 2**30:.1f} GiB gradients+momentum resident)"),
              "roofline": roofline, "e2e": e2e,
              "gpu_launches": opt.kernel_launches_per_step() * args.steps,
              "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    from sign_muon_optimizer_momentum_b200 import synthetic as syn
    wl = syn.WORKLOADS[args.config]
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
