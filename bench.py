#!/usr/bin/env python
"""Throughput of the TensorGRaD optimizer step on B200: gradient elements/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle on the host cores

One step = one full optimizer step (sparse gather + masked projection + core
and sparse AdamW + reconstruction + in-place scatter-add + weight update, and
the refresh when the workload's period T says so) over one synthetic gradient
already resident in HBM. The default workload is the large complex fp16
spectral tensor (256, 256, 128, 65) with ranks (64, 64, 32, 16), 5% top-k
sparse, factors and index set fixed after one untimed refresh.

The default run also records the other workloads at their full step counts
under "workloads" (the 4-tensor mixed-precision set, the complex64 FNO
tensor, the 5-way refresh tensor and the small real tensor), each with its
time per step, roofline fraction, kernel times and clocks.

Multi-GPU (torchrun, one rank per GPU): every rank steps its own tensor
(independent problems, no data-path collective), value = elements of all
ranks / the slowest rank's time (weak scaling).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TensorGRaD step: gradient elems/s per B200 and % of HBM/tensor roofline"
UNIT = "gradient elements/s"
DEFAULT_WORKLOAD = "spectral_c32h_256x256x128x65"
L2_BYTES = 126 * 2 ** 20
ELEM = {"r32": 4, "c64": 8, "c32h": 4, "r16": 2}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def algorithmic_bytes(wl) -> dict:
    """Bytes one step must move at least (the per-element figure of the
    method: G read once, W read and written once, Omega's index and sparse
    moments read and written, core moments read and written, factors read)."""
    N, k = wl.N, wl.k
    cplx = wl.dtype in ("c64", "c32h")
    sm, sv = (8, 4) if cplx else (4, 4)
    ncore = math.prod(wl.ranks)
    su = 8 if cplx else 4
    parts = {
        "grad": N * ELEM[wl.dtype],
        "weight": 2 * N * ELEM[wl.weight_dtype],
        "sparse": k * (8 + 2 * (sm + sv)),
        "core": 2 * ncore * (sm + sv),
        "factors": sum(I * r * su for I, r in zip(wl.shape, wl.ranks) if r < I),
    }
    parts["total"] = sum(parts.values())
    return parts


def optimizer_state(wl, n_tensors: int, device_bytes: int) -> dict:
    """Optimizer-state memory of this rank's tensors: the method's count
    (core and sparse moments, factors, Omega's index; tgd_state_memory) next
    to AdamW's moments for the same tensors, and the device memory the
    handles hold (state plus work buffers)."""
    import rank_sparse_tensor_b200 as rst
    m = rst.state_memory(wl.shape, wl.ranks, wl.sparse_ratio, wl.dtype, 0)
    return {"bytes": m["total_bytes"] * n_tensors, "adamw_bytes": m["adamw_bytes"] * n_tensors,
            "ratio": m["ratio"], "device_bytes": int(device_bytes)}


def kernel_algorithmic_bytes(name: str, wl) -> float:
    """Algorithmic bytes of one launch of the named kernel: its share of the
    step's algorithmic bytes (the parts of the step it alone moves)."""
    a = algorithmic_bytes(wl)
    N = wl.N
    cplx = wl.dtype in ("c64", "c32h")
    moments = wl.k * 2 * ((8, 4) if cplx else (4, 4))[0] + wl.k * 2 * 4
    table = {
        # tensor-core path: G stream (mask, gather, Omega's index read once),
        # sparse AdamW stream (moments read and written), W stream
        "proj_stream": a["grad"] + 8 * wl.k,
        "sparse_adam": moments,
        "recon_stream": a["weight"],
        # fp32 tensor-core path: the last expansion updates W in place
        "expand_update32": a["weight"],
        # CUDA-core path
        "weight_update": a["weight"],
        "mode_product": a["grad"],
    }
    return float(table.get(name, 0.0))


POLLER = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[1]))
get = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
    pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    print(f"{time.time():.4f},{pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)},"
          f"{int(get(h)):#x},{pynvml.nvmlDeviceGetPowerUsage(h) / 1e3:.1f}", flush=True)
    time.sleep(0.002)
"""


class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region by a
    separate polling process (read-only NVML queries every 2 ms; a thread in
    this process would be starved while it launches). The samples inside the
    timed region are kept, and written as clocks_rank<i>.csv to out_dir."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown"}

    def __init__(self, index: int, out_dir: str):
        self.path = os.path.join(out_dir, f"clocks_rank{index}.csv")
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        self.raw = self.path + ".raw"
        self.t0, self.t1 = 0.0, float("inf")
        try:
            self.f = open(self.raw, "w")
            self.proc = subprocess.Popen([sys.executable, "-c", POLLER, str(index)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def mark(self, start: bool):
        """Bounds of the timed region (samples outside it are dropped)."""
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["sampler unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        smax, rows = None, []
        for line in open(self.raw):
            if line.startswith("max"):
                smax = float(line.split()[1])
                continue
            f = line.strip().split(",")
            if len(f) == 4:
                try:
                    rows.append((float(f[0]), float(f[1]), int(f[2], 16), float(f[3])))
                except ValueError:
                    pass
        os.remove(self.raw)
        inside = [r for r in rows if self.t0 <= r[0] <= self.t1]
        with open(self.path, "w") as out:
            out.write("time,sm_mhz,reasons_bits,power_w\n")
            for t, mhz, bits, pw in inside:
                out.write(f"{t:.4f},{mhz:.0f},{bits:#x},{pw:.1f}\n")
        sm = [r[1] for r in inside]
        reasons = sorted({nm for r in inside for b, nm in self.REASONS.items() if r[2] & b})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(sm), "source": "nvml (polling process)"}


def oracle_sample(wl, factor: int):
    """The workload with its leading mode divided by `factor` (rank scaled
    with it): the same trailing modes, ranks, dtype and generator."""
    import dataclasses
    sh, rk, gr = list(wl.shape), list(wl.ranks), list(wl.gen_ranks)
    f = max(1, min(factor, sh[0]))
    ratio = rk[0] / sh[0]
    sh[0] //= f
    rk[0] = max(1, min(sh[0], math.ceil(ratio * sh[0])))
    gr[0] = max(1, min(sh[0], math.ceil(gr[0] / f)))
    return dataclasses.replace(wl, name=f"{wl.name}/leading-mode/{f}", shape=tuple(sh),
                               ranks=tuple(rk), gen_ranks=tuple(gr))


class OracleRun:
    """The oracle, as it stands (test infrastructure, never tuned for this),
    on a sample of the workload: one untimed refresh, then timed steps."""

    def __init__(self, wl, seed=0):
        import oracle
        from rank_sparse_tensor_b200.synth import GradientStream, weights
        self.wl = wl
        gs = GradientStream(wl.shape, wl.gen_ranks, wl.dtype, seed, outlier_frac=wl.outlier_frac,
                            outlier_scale=wl.outlier_scale)
        self.g = [gs.next().numpy() for _ in range(2)]
        self.w = weights(wl.shape, wl.weight_dtype, seed).numpy()
        self.o = oracle.Oracle(wl.shape, wl.ranks, wl.sparse_ratio, 0, wl.lr, wl.betas, wl.eps,
                               wl.wd, wl.dtype, wl.weight_dtype, auto_refresh=0)
        self.o.refresh(self.g[0])
        self.i = 0

    def step(self) -> float:
        t0 = time.perf_counter()
        self.o.step(self.g[1 - self.i % 2], self.w)
        self.i += 1
        return time.perf_counter() - t0

    def describe(self, steps, seconds):
        wl = self.wl
        return (f"{steps} oracle steps (after one untimed refresh) on shape {tuple(wl.shape)} ranks "
                f"{tuple(wl.ranks)}, {wl.dtype} gradients, rho {wl.sparse_ratio}: the workload with "
                f"its leading mode cut down; {seconds:.1f} s of step time")


def oracle_threads() -> int:
    return int(os.environ.get("TGD_ORACLE_THREADS", "0")) or (os.cpu_count() or 1)


def cpu_baseline(wl, target_s=10.0):
    """Oracle throughput on a bounded sample (about `target_s` of step time)."""
    run = OracleRun(oracle_sample(wl, 16), seed=0)
    n, tot = 0, 0.0
    while tot < target_s and n < 64:
        tot += run.step()
        n += 1
    N = math.prod(run.wl.shape)
    return {"value": N * n / tot, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": run.describe(n, tot)}


def run_reference(args, wl):
    """The reference arm: the oracle on the host cores, on this arm's metric,
    each step a bounded sample of the workload (leading mode / 16). Under a
    multi-rank launch rank 0 alone runs and prints; the others exit."""
    _, rank, _ = rank_env()
    if rank != 0:
        return 0
    run = OracleRun(oracle_sample(wl, 16), seed=1)
    for _ in range(args.warmup):
        run.step()
    tot = sum(run.step() for _ in range(args.steps))
    N = math.prod(run.wl.shape)
    value = N * args.steps / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "shape": list(wl.shape), "ranks": list(wl.ranks),
                       "sparse_ratio": wl.sparse_ratio, "sample_shape": list(run.wl.shape),
                       "sample_ranks": list(run.wl.ranks)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(),
                             "kind": "oracle", "sample": run.describe(args.steps, tot)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- ranks
def rank_env():
    """(world, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def tensor_seeds(rank: int, n_tensors: int):
    """Seeds of the independent tensors a rank steps (gradient, weight):
    disjoint across ranks, so no two ranks hold the same problem."""
    return [(1000 * rank + 17 * j + 1, 1000 * rank + j) for j in range(n_tensors)]


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's value (all ranks take this collective)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, elems_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job gradient elements/s: every rank's elements over the slowest
    rank's time (weak scaling: each rank has its own tensors)."""
    return world * elems_per_rank * steps / (max_ms / 1e3)


def step_roofline(wl, n_tensors, step_ms, hbm_gbs):
    """Algorithmic bytes of one step over every tensor, and the fraction of
    the HBM roofline the step time reaches."""
    ab = algorithmic_bytes(wl)["total"] * n_tensors
    gbs = ab / (step_ms / 1e3) / 1e9
    return {"step_algorithmic_bytes": ab, "step_achieved_gbs": gbs, "step_frac": gbs / hbm_gbs}


class Bench:
    """One rank's tensors of one workload, resident in HBM, and their timing."""

    def __init__(self, wl, args, dev, rank, concurrent_default=True, opts=None):
        import torch
        import rank_sparse_tensor_b200 as rst
        from rank_sparse_tensor_b200.synth import GradientStream, weights
        self.wl, self.args, self.dev = wl, args, dev
        nt = wl.n_tensors
        self.concurrent = nt > 1 and not args.sequential and concurrent_default
        n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
        # tensors go round-robin onto ns streams, each with 1/ns of the SMs
        ns = min(nt, args.tensor_streams) if args.tensor_streams > 0 else nt
        self.n_streams = ns if self.concurrent else 1
        sm_budget = max(1, n_sms // ns) if self.concurrent and not args.full_sms else 0
        self.streams = [torch.cuda.Stream(device=dev) for _ in range(ns)] if self.concurrent else None
        self.tensors = []
        for gseed, wseed in tensor_seeds(rank, nt):
            gs = GradientStream(wl.shape, wl.gen_ranks, wl.dtype, seed=gseed,
                                outlier_frac=wl.outlier_frac, outlier_scale=wl.outlier_scale,
                                noise=wl.noise, drift=0.0, device=str(dev))
            grads = [gs.next() for _ in range(2)]
            w = weights(wl.shape, wl.weight_dtype, seed=wseed, device=str(dev))
            opt = rst.TensorGRaD(wl.shape, wl.ranks, wl.sparse_ratio, wl.T, wl.lr, wl.betas, wl.eps,
                                 wl.wd, wl.dtype, wl.weight_dtype, path=args.path, sm_budget=sm_budget,
                                 **(opts or {}))
            if wl.T == 0:
                opt.refresh(grads[0])
            self.tensors.append((opt, grads, w))
        torch.cuda.synchronize()
        in_bytes = sum(g[0].numel() * g[0].element_size() + w.numel() * w.element_size()
                       for _, g, w in self.tensors)
        self.flush = in_bytes < 2 * L2_BYTES
        self.scratch = torch.empty(256 * 2 ** 20 // 4, dtype=torch.float32, device=dev) if self.flush else None

    def one_step(self, i):
        import torch
        if self.streams is None:
            for opt, grads, w in self.tensors:
                opt.step(grads[i % 2], w)
            return
        # each tensor on its own stream, forked from and joined back into the
        # timed stream
        main = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(main)
        for st in self.streams:
            st.wait_event(fork)
        for j, (opt, grads, w) in enumerate(self.tensors):
            with torch.cuda.stream(self.streams[j % len(self.streams)]):
                opt.step(grads[i % 2], w)
        for st in self.streams:
            join = torch.cuda.Event()
            join.record(st)
            main.wait_event(join)

    def timed_steps(self, steps, profile, barrier):
        """`steps` steps between barriers, each bracketed by CUDA events on
        the launching stream (L2 flushed between steps when inputs fit in
        it). Returns (total ms, {kernel: [launches, ms]})."""
        import torch
        stream = torch.cuda.current_stream()
        for opt, _, _ in self.tensors:
            opt.profile(profile)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            evs[i][0].record(stream)
            self.one_step(i)
            evs[i][1].record(stream)
            if self.flush:
                self.scratch.add_(1.0)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        prof = {}
        for opt, _, _ in self.tensors:
            opt.profile(False)
            if profile:
                for kname, (n, ms) in opt.profile_read().items():
                    a = prof.setdefault(kname, [0, 0.0])
                    a[0] += n
                    a[1] += ms
        return sum(a.elapsed_time(b) for a, b in evs), prof

    def close(self):
        for opt, _, _ in self.tensors:
            opt.close()
        self.tensors = []


def measure(wl, args, dev, world, rank, local, barrier, steps, warmup, opts=None):
    """Warm-up, K timed steps with the clock sampler running, K more with
    per-kernel events; the per-rank numbers of one workload."""
    import torch
    b = Bench(wl, args, dev, rank, opts=opts)
    for i in range(warmup):
        b.one_step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(local, args.out_dir)
    time.sleep(1.0)  # the polling process is up before the timed region
    sampler.mark(True)
    total_ms, _ = b.timed_steps(steps, False, barrier)
    sampler.mark(False)
    clocks = sampler.stop()
    _, prof = b.timed_steps(steps, True, barrier)
    max_ms = max_over_ranks(total_ms, world, dev)
    return b, {"total_ms": total_ms, "max_ms": max_ms, "prof": prof, "clocks": clocks}


def kernel_roofline(wl, prof, hbm_gbs):
    """The slowest per-step kernel's algorithmic bytes per launch over its
    average launch time (a refresh kernel in the profiled pass is reported
    in "kernels" but is not a step kernel)."""
    refresh_kernels = {"select", "mode_gram", "eigh", "dct_select", "rebuild"}
    step_prof = {k: v for k, v in prof.items() if k not in refresh_kernels}
    dom = max(step_prof.items(), key=lambda kv: kv[1][1]) if step_prof else ("none", [1, 1.0])
    dom_name, (dom_n, dom_ms) = dom[0], dom[1]
    per_launch_ms = dom_ms / max(dom_n, 1)
    kbytes = kernel_algorithmic_bytes(dom_name, wl)
    achieved = kbytes / (per_launch_ms / 1e3) / 1e9 if kbytes else None
    return dom_name, achieved


def other_workload(name, args, dev, world, rank, local, barrier, hbm_gbs, opts=None, oracle_steps=0):
    """A compact record of one more workload at its full step count: time
    per step, throughput, the step's roofline fraction, kernel times and
    clocks (refreshes, where the workload's period T calls for them, run
    inside the timed steps). opts: options of the method's variants (the
    decomposition order, the factor basis). oracle_steps > 0: the oracle's
    throughput on the same workload (rank 0, after the GPU timing)."""
    import torch
    from rank_sparse_tensor_b200.synth import WORKLOADS
    wl = WORKLOADS[name]
    steps = wl.steps
    b, m = measure(wl, args, dev, world, rank, local, barrier, steps, 3, opts=opts)
    step_ms = m["max_ms"] / steps
    n_elems = wl.N * len(b.tensors)
    rec = {"steps": steps, "warmup": 3, "ms_per_step": step_ms,
           "value": job_throughput(world, n_elems, steps, m["max_ms"]), "unit": UNIT,
           "shape": list(wl.shape), "ranks": list(wl.ranks), "tensors_per_gpu": len(b.tensors),
           "T": wl.T, "grad_dtype": wl.dtype, "kernel_path": b.tensors[0][0].info["path"],
           "l2": "flushed between steps" if b.flush else "inputs larger than L2",
           "tensor_streams": ("%d streams, tensors round-robin, %s" % (b.n_streams, "all SMs each" if b.args.full_sms else "1/%d of the SMs each" % b.n_streams))
           if b.concurrent else "one stream",
           "roofline": dict(step_roofline(wl, len(b.tensors), step_ms, hbm_gbs), peak=hbm_gbs,
                            unit="GB/s", bound="hbm"),
           "kernels": {k: {"launches": v[0], "ms_total": round(v[1], 4)} for k, v in m["prof"].items()},
           "clocks": m["clocks"]}
    if opts:
        rec["options"] = dict(opts)
    b.close()
    if oracle_steps and rank == 0:
        rec["cpu_baseline"] = oracle_full(wl, oracle_steps, opts)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def oracle_full(wl, steps, opts=None):
    """The oracle on the whole workload (not a sample) for `steps` steps
    from create, its refreshes at the workload's period included."""
    import oracle
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    gs = GradientStream(wl.shape, wl.gen_ranks, wl.dtype, 1, outlier_frac=wl.outlier_frac,
                        outlier_scale=wl.outlier_scale)
    g = [gs.next().numpy() for _ in range(2)]
    w = weights(wl.shape, wl.weight_dtype, 1).numpy()
    o = oracle.Oracle(wl.shape, wl.ranks, wl.sparse_ratio, wl.T, wl.lr, wl.betas, wl.eps, wl.wd,
                      wl.dtype, wl.weight_dtype, **(opts or {}))
    t0 = time.perf_counter()
    for i in range(steps):
        o.step(g[i % 2], w)
    el = time.perf_counter() - t0
    return {"value": wl.N * steps / el, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{steps} oracle steps of the whole workload from create (refreshes every "
                      f"{wl.T} steps included): {el:.1f} s"}


def cpu_single_core(wl_name, target_s):
    """The oracle's throughput on one host thread, in a fresh process (the
    oracle fixes its thread count when it starts)."""
    env = dict(os.environ, TGD_ORACLE_THREADS="1")
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "--cpu-baseline-only",
                        "--workload", wl_name, "--cpu-seconds", str(target_s)],
                       env=env, capture_output=True, text=True, timeout=600)
    for line in r.stdout.splitlines()[::-1]:
        if line.startswith("{"):
            return json.loads(line)
    return {"error": (r.stderr or r.stdout)[-300:]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--path", default="auto", choices=["auto", "generic", "tcgen05"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--out-dir", default=os.path.join(ROOT, "bench_out"),
                    help="directory for the per-rank clock records")
    ap.add_argument("--tensor-streams", type=int, default=0,
                    help="streams the tensors of a multi-tensor workload are spread over "
                         "(each with that share of the SMs); 0 = one per tensor")
    ap.add_argument("--full-sms", action="store_true",
                    help="concurrent tensors' kernels each sized for all SMs (no SM budget)")
    ap.add_argument("--sequential", action="store_true",
                    help="step the tensors of a multi-tensor workload one after another on one "
                         "stream (default: each on its own stream with an equal share of the SMs)")
    ap.add_argument("--shrink", type=int, default=1,
                    help="divide the leading mode (and its rank) by this factor: small "
                         "cases of the same kernels, for profiler captures only")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the records of the other workloads in the default run")
    ap.add_argument("--cpu-baseline-only", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help=argparse.SUPPRESS)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    import dataclasses
    from rank_sparse_tensor_b200.synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.cpu_baseline_only:
        print(json.dumps(cpu_baseline(wl, args.cpu_seconds)), flush=True)
        return 0
    if args.shrink > 1:
        sh, rk, gr = list(wl.shape), list(wl.ranks), list(wl.gen_ranks)
        sh[0] //= args.shrink
        rk[0] = max(1, rk[0] // args.shrink)
        gr[0] = max(1, gr[0] // args.shrink)
        wl = dataclasses.replace(wl, name=f"{wl.name}/shrink{args.shrink}", shape=tuple(sh),
                                 ranks=tuple(rk), gen_ranks=tuple(gr))
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    if args.workload == DEFAULT_WORKLOAD:
        wl = dataclasses.replace(wl, n_tensors=1)
    b, m = measure(wl, args, dev, world, rank, local, barrier, args.steps, args.warmup)
    tensors, prof, clocks, max_ms = b.tensors, m["prof"], m["clocks"], m["max_ms"]
    n_elems = wl.N * len(tensors)
    value = job_throughput(world, n_elems, args.steps, max_ms)

    # End to end through the host-buffer entry point: H2D of the gradient and
    # the weights, the step, D2H of the updated weights, every step.
    e2e = None
    if args.e2e_steps > 0:
        opt, grads, w = tensors[0]
        gh = torch.empty(grads[0].shape, dtype=grads[0].dtype, pin_memory=True)
        wh = torch.empty(w.shape, dtype=w.dtype, pin_memory=True)
        gh.copy_(grads[0])
        wh.copy_(w)
        gh_np, wh_np = gh.numpy(), wh.numpy()
        opt.step_host(gh_np, wh_np)
        barrier()
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            opt.step_host(gh_np, wh_np)
        el = max_over_ranks(time.perf_counter() - t0, world, dev)
        e2e = {"value": job_throughput(world, wl.N, args.e2e_steps, 1e3 * el), "unit": UNIT,
               "h2d_bytes_per_step": gh.numel() * gh.element_size() + wh.numel() * wh.element_size(),
               "d2h_bytes_per_step": wh.numel() * wh.element_size()}
        del gh, wh

    hbm_gbs, bf16_tf, peak_src = load_peaks()
    dom_name, achieved = kernel_roofline(wl, prof, hbm_gbs)
    step_ms = max_ms / args.steps
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        tt = json.load(open(tpath)).get(wl.name, {}).get(dom_name)
        if tt and tt.get("valid", False):
            traffic = tt["bytes_per_launch"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"c32h": "f16", "c64": "f32", "r32": "f32", "r16": "f16"}[wl.dtype],
        "data": "synthetic",
        "config": {"workload": wl.name, "shape": list(wl.shape), "ranks": list(wl.ranks),
                   "sparse_ratio": wl.sparse_ratio, "k": wl.k, "T": wl.T, "tensors_per_gpu": len(tensors),
                   "grad_dtype": wl.dtype, "weight_dtype": wl.weight_dtype,
                   "kernel_path": tensors[0][0].info["path"],
                   "l2": "flushed between steps" if b.flush else "inputs larger than L2",
                   "parallelism": f"independent tensors per rank x{world}",
                   "tensor_streams": "%d streams, tensors round-robin, %s" % (b.n_streams, "all SMs each" if args.full_sms else "1/%d of the SMs each" % b.n_streams)
                   if b.concurrent else "one stream"},
        "roofline": dict({"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": hbm_gbs,
                          "unit": "GB/s", "frac": (achieved / hbm_gbs) if achieved else None,
                          "traffic": traffic, "peak_source": peak_src},
                         **step_roofline(wl, len(tensors), step_ms, hbm_gbs)),
        "kernels": {k: {"launches": v[0], "ms_total": round(v[1], 4)} for k, v in prof.items()},
        "gpu_launches": int(sum(v[0] for v in prof.values())),  # per K steps (profiled pass)
        "clocks": clocks,
        "e2e": e2e,
        "optimizer_state": optimizer_state(wl, len(tensors),
                                           sum(t[0].info["device_bytes"] for t in tensors)),
    }
    b.close()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    # the other workloads, each at its full step count (default run only)
    if args.workload == DEFAULT_WORKLOAD and not args.no_other_workloads and args.shrink == 1:
        line["workloads"] = {}
        ow = line["workloads"]
        cpu = world == 1 and not args.no_cpu_baseline
        ow["fno4_c32h_128x128x64x33"] = other_workload("fno4_c32h_128x128x64x33", args, dev, world, rank,
                                                       local, barrier, hbm_gbs)
        ow["fno_c64_64x64x32x17"] = other_workload("fno_c64_64x64x32x17", args, dev, world, rank, local,
                                                   barrier, hbm_gbs, oracle_steps=200 if cpu else 0)
        # the method's ablated variants on the same tensor: the low-rank part
        # first, and the DCT column-selection basis instead of HOSVD factors
        ow["fno_c64_64x64x32x17/lowrank_first"] = other_workload(
            "fno_c64_64x64x32x17", args, dev, world, rank, local, barrier, hbm_gbs, opts={"order": 1})
        ow["fno_c64_64x64x32x17/dct_basis"] = other_workload(
            "fno_c64_64x64x32x17", args, dev, world, rank, local, barrier, hbm_gbs, opts={"basis": 1})
        ow["refresh_c64_64x64x32x32x17"] = other_workload("refresh_c64_64x64x32x32x17", args, dev, world,
                                                          rank, local, barrier, hbm_gbs)
        ow["tiny_r32_16x16x8x8"] = other_workload("tiny_r32_16x16x8x8", args, dev, world, rank, local,
                                                  barrier, hbm_gbs, oracle_steps=10 if cpu else 0)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(wl)
        one = cpu_single_core(wl.name, 10.0)
        cb["single_core"] = {k: one.get(k) for k in ("value", "unit", "cores", "sample")} if "value" in one else one
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
