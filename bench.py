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
        # CUDA-core path
        "weight_update": a["weight"],
        "mode_product": a["grad"],
    }
    return float(table.get(name, 0.0))


class ClockSampler:
    def __init__(self, index: int):
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_rank{index}.csv")
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        self.proc = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_baseline_sample(wl, seed=0):
    """The oracle, as it stands, on a bounded sample of the workload: the same
    trailing modes and rank ratios with the leading modes cut down so that one
    step takes seconds; one timed step after one untimed refresh."""
    import numpy as np
    import oracle
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    shape, ranks = list(wl.shape), list(wl.ranks)
    budget = 2_500_000
    n = 0
    while math.prod(shape) > budget and n < len(shape) - 2:
        f = max(1, math.prod(shape) // budget)
        new = max(1, shape[n] // min(f, shape[n]))
        if new == shape[n]:
            n += 1
            continue
        ratio = ranks[n] / shape[n]
        shape[n] = new
        ranks[n] = max(1, min(new, math.ceil(ratio * new)))
        n += 1
    gen = [min(g, s) for g, s in zip(wl.gen_ranks, shape)]
    gs = GradientStream(shape, gen, wl.dtype, seed, outlier_frac=wl.outlier_frac,
                        outlier_scale=wl.outlier_scale)
    g0 = gs.next().numpy()
    g1 = gs.next().numpy()
    w = weights(shape, wl.weight_dtype, seed).numpy()
    o = oracle.Oracle(shape, ranks, wl.sparse_ratio, 0, wl.lr, wl.betas, wl.eps, wl.wd,
                      wl.dtype, wl.weight_dtype, auto_refresh=0)
    o.refresh(g0)
    t0 = time.perf_counter()
    o.step(g1, w)
    dt = time.perf_counter() - t0
    N = math.prod(shape)
    threads = int(os.environ.get("TGD_ORACLE_THREADS", "0")) or (os.cpu_count() or 1)
    return {"value": N / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "_seconds": dt, "_elements": N,
            "sample": f"one oracle step (after an untimed refresh) on shape {tuple(shape)} "
                      f"ranks {tuple(ranks)}, {wl.dtype}, rho {wl.sparse_ratio}: the workload "
                      f"with its leading modes cut down; {dt:.2f} s"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    samples = []
    for _ in range(args.warmup):
        cpu_baseline_sample(wl, seed=1)
    for s in range(args.steps):
        samples.append(cpu_baseline_sample(wl, seed=2 + s))
    tot_elems = sum(x["_elements"] for x in samples)
    tot_time = sum(x["_seconds"] for x in samples)
    value = tot_elems / tot_time
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_time / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "shape": list(wl.shape), "ranks": list(wl.ranks),
                       "sparse_ratio": wl.sparse_ratio},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": samples[0]["cores"],
                             "kind": "oracle", "sample": samples[0]["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--path", default="auto", choices=["auto", "generic", "tcgen05"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--shrink", type=int, default=1,
                    help="divide the leading mode (and its rank) by this factor: small "
                         "cases of the same kernels, for profiler captures only")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    import dataclasses
    from rank_sparse_tensor_b200.synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.shrink > 1:
        sh, rk, gr = list(wl.shape), list(wl.ranks), list(wl.gen_ranks)
        sh[0] //= args.shrink
        rk[0] = max(1, rk[0] // args.shrink)
        gr[0] = max(1, gr[0] // args.shrink)
        wl = dataclasses.replace(wl, name=f"{wl.name}/shrink{args.shrink}", shape=tuple(sh),
                                 ranks=tuple(rk), gen_ranks=tuple(gr))
    if args.impl == "reference":
        return run_reference(args, wl)

    import numpy as np
    import torch
    import torch.distributed as dist
    import rank_sparse_tensor_b200 as rst
    from rank_sparse_tensor_b200.synth import GradientStream, weights

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # Inputs resident in HBM before the timed region.
    nt = wl.n_tensors if args.workload != DEFAULT_WORKLOAD else 1
    tensors = []
    for j in range(nt):
        gs = GradientStream(wl.shape, wl.gen_ranks, wl.dtype, seed=1000 * rank + 17 * j + 1,
                            outlier_frac=wl.outlier_frac, outlier_scale=wl.outlier_scale,
                            noise=wl.noise, drift=0.0, device=str(dev))
        grads = [gs.next() for _ in range(2)]
        w = weights(wl.shape, wl.weight_dtype, seed=1000 * rank + j, device=str(dev))
        T = wl.T
        opt = rst.TensorGRaD(wl.shape, wl.ranks, wl.sparse_ratio, T, wl.lr, wl.betas, wl.eps, wl.wd,
                             wl.dtype, wl.weight_dtype, path=args.path)
        if T == 0:
            opt.refresh(grads[0])
        tensors.append((opt, grads, w))
    torch.cuda.synchronize()
    in_bytes = sum(g[0].numel() * g[0].element_size() + w.numel() * w.element_size()
                   for _, g, w in tensors)
    flush = in_bytes < 2 * L2_BYTES
    scratch = torch.empty(256 * 2 ** 20 // 4, dtype=torch.float32, device=dev) if flush else None

    def one_step(i):
        for opt, grads, w in tensors:
            opt.step(grads[i % 2], w)

    for i in range(args.warmup):
        one_step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    for opt, _, _ in tensors:
        opt.profile(True)
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        evs[i][0].record(stream)
        one_step(i)
        evs[i][1].record(stream)
        if flush:
            scratch.add_(1.0)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = sum(step_ms)
    prof = {}
    for opt, _, _ in tensors:
        opt.profile(False)
        for kname, (n, ms) in opt.profile_read().items():
            a = prof.setdefault(kname, [0, 0.0])
            a[0] += n
            a[1] += ms
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    n_elems = wl.N * len(tensors)
    value = world * n_elems * args.steps / (max_ms / 1e3)

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
        el = torch.tensor([time.perf_counter() - t0], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(el, op=dist.ReduceOp.MAX)
        e2e = {"value": world * wl.N * args.e2e_steps / float(el.item()), "unit": UNIT,
               "h2d_bytes_per_step": gh.numel() * gh.element_size() + wh.numel() * wh.element_size(),
               "d2h_bytes_per_step": wh.numel() * wh.element_size()}

    hbm_gbs, bf16_tf, peak_src = load_peaks()
    dom = max(prof.items(), key=lambda kv: kv[1][1]) if prof else ("none", [1, 1.0])
    dom_name, (dom_n, dom_ms) = dom[0], dom[1]
    per_launch_ms = dom_ms / max(dom_n, 1)
    kbytes = kernel_algorithmic_bytes(dom_name, wl)
    achieved = kbytes / (per_launch_ms / 1e3) / 1e9 if kbytes else None
    ab = algorithmic_bytes(wl)
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
                   "l2": "flushed between steps" if flush else "inputs larger than L2",
                   "parallelism": f"independent tensors per rank x{world}"},
        "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": hbm_gbs,
                     "unit": "GB/s", "frac": (achieved / hbm_gbs) if achieved else None,
                     "traffic": traffic, "peak_source": peak_src,
                     "step_algorithmic_bytes": ab["total"],
                     "step_achieved_gbs": ab["total"] / (step_ms / 1e3) / 1e9,
                     "step_frac": ab["total"] / (step_ms / 1e3) / 1e9 / hbm_gbs},
        "kernels": {k: {"launches": v[0], "ms_total": round(v[1], 4)} for k, v in prof.items()},
        "gpu_launches": int(sum(v[0] for v in prof.values())),
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline_sample(wl)
        line["cpu_baseline"] = {k: v for k, v in cb.items() if not k.startswith("_")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for opt, _, _ in tensors:
        opt.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
