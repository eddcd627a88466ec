#!/usr/bin/env python3
"""Benchmark of the fused verify + speculation-cache step (libssd) on B200.

One step = the whole hot path over one batch: the fan-out plan and the fused
verify kernel (softmax statistics, top-F, Saguaro reweighting, accept test,
residual bonus draw, cache build and lookup).  Inputs are seeded synthetic
Zipf logits, generated on the host, resident in HBM before timing starts; two
input copies rotate, each larger than the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle on host cores

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
rows (weak scaling, no collective on the data path); the step time is the
maximum over ranks.  Rank 0 prints one JSON line.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verify+cache rows/s and HBM GB/s (% of peak), B=64 K=6 V=128256 bf16"
L2_BYTES = 126 * 1024 * 1024
KERNEL_SOURCES = ["speculative_decoding_verify_ssd_b200/csrc/ssd_kernels.cuh",
                  "speculative_decoding_verify_ssd_b200/csrc/ssd_device.cuh",
                  "speculative_decoding_verify_ssd_b200/csrc/ssd_api.cu"]


# ssd_verify launches ssd_stats_kernel (softmax statistics, top-F, accept test,
# row decision) and then ssd_draw_kernel (residual / bonus draw, cache lookup).
KERNELS_PER_VERIFY = 2


def ssd_step_kernels():
    return "ssd_stats_kernel + ssd_draw_kernel (one ssd_verify call, timed as a whole)"


def kernel_sha():
    """Hash of the kernel sources with comments and whitespace removed, so
    that recorded counters stay valid across edits that change no code."""
    import re
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def recorded_traffic(workload):
    """DRAM bytes per launch of the verify kernel from a committed ncu
    summary, only if it was taken on the current kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "verify_traffic.json")) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel_sha") == kernel_sha():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thr = threading.Thread(target=self._read, daemon=True)
            self.thr.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def rank_workload(w, rank):
    """Rank `rank`'s share under weak scaling: the same workload shape with
    its own seeds, so every rank verifies different rows."""
    return w.replace(seed=w.seed + 7919 * rank, fallback_seed=w.fallback_seed + rank)


def max_over_ranks(value, dist, device):
    """The slowest rank's time: one all-reduce (MAX) of a scalar, taken by
    every rank at the same point."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rows_per_s(world, B, steps, max_ms):
    """Whole-job throughput: rows verified by all ranks over the slowest rank's time."""
    return world * B * steps / (max_ms / 1e3)


def workload_config(w, world):
    return {"workload": w.name, "B": w.B, "K": w.K, "V": w.V, "T": w.T, "budget": w.budget, "C": w.C,
            "fanout": "geometric" if w.fanout_mode == 0 else "uniform", "alpha": w.alpha,
            "parallelism": f"rows sharded, {world} independent GPU(s)"}


def algorithmic_bytes(w):
    s = 2 if w.dtype == "bf16" else 4
    logits = w.B * (2 * w.K + 1) * w.V * s
    inputs = w.B * (w.K * 4 + (w.K + 1) * 4 + (w.K + 1) * 4 + 4)           # tokens, uniforms, F, alpha
    outputs = w.B * (4 + 4 + (w.K + 1) * 4 + w.K * 4 + 4 + 4                  # verify outputs
                     + (w.K + 2) * 4 + w.budget * 4 + 1 + 4 + w.K * 4)        # cache
    return logits, logits + inputs + outputs


def run_ssd(args, rank, world, local_rank):
    import torch
    from speculative_decoding_verify_ssd_b200 import binding as ssd
    from speculative_decoding_verify_ssd_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ssd.load()
    w = synth.WORKLOADS[args.workload]
    w_rank = rank_workload(w, rank)
    logit_bytes, alg_bytes = algorithmic_bytes(w)
    n_copies = max(2, -(-2 * L2_BYTES // logit_bytes))
    n_copies = min(n_copies, 8)

    def dev_logits(x):
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(x).to(dev)

    sets = []
    host_first = None
    for c in range(n_copies):
        g = synth.generate(w_rank.replace(seed=w_rank.seed + 104729 * c))
        if c == 0:
            host_first = g
        t, d = dev_logits(g["target"]), dev_logits(g["draft"])
        alpha = torch.from_numpy(g["alpha"]).to(dev)
        u = torch.from_numpy(g["uniforms"]).to(dev)
        F = ssd.ssd_fanout_plan(alpha, w.K, w.budget, w.fanout_mode)
        # Draft tokens come from the draft side's own Saguaro sampler.
        rw = ssd.ssd_saguaro_reweight(d, w.T, F, w.C, w.budget,
                                      u_draft=torch.from_numpy(g["u_draft"]).to(dev))
        sets.append(dict(t=t, d=d, alpha=alpha, u=u, tok=rw.draft_tokens))
        del g
    torch.cuda.synchronize()
    ws = ssd.Workspace(w.B, w.K, dev, w.V, ssd.DTYPE_BF16 if w.dtype == "bf16" else ssd.DTYPE_FP32)
    outs = [ssd.alloc_verify_result(w.B, w.K, w.budget, dev, True) for _ in range(n_copies)]

    def step(i):
        # One launch: the fan-out plan is computed inside the fused kernel from alpha.
        s = sets[i % n_copies]
        ssd.ssd_verify(s["t"], s["d"], s["tok"], s["u"], w.T, alpha=s["alpha"], fanout_mode=w.fanout_mode,
                       C_coef=w.C, budget=w.budget, cache=True, fallback_seed=w_rank.fallback_seed,
                       workspace=ws, out=outs[i % n_copies])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    # The timed loop is one CUDA graph of `steps` back-to-back launches, so
    # host launch overhead never starves the GPU.
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap, capture_error_mode="thread_local"):
            for i in range(args.steps):
                step(i)
    torch.cuda.synchronize()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)

    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(1, args.repeat)
    per_rep = []
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    start.record(stream)
    for r in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        per_rep.append((e0, e1))
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = start.elapsed_time(end)
    steps_done = args.steps * reps
    # the graph holds `steps` verify calls back to back: per-step time = replay time / steps
    kernel_ms = [a.elapsed_time(b) / args.steps for a, b in per_rep]
    if world > 1:
        total_ms = max_over_ranks(total_ms, dist, dev)
    ms_per_step = total_ms / steps_done
    rows_per_s = job_rows_per_s(world, w.B, steps_done, total_ms)
    del graph

    # outcome statistics from the last step of each rotating copy
    r0 = outs[0]
    n_acc = r0.n_accepted.cpu().numpy()
    hit = r0.hit.cpu().numpy()
    st = r0.status.cpu().numpy()

    result = dict(rows_per_s=rows_per_s, ms_per_step=ms_per_step, kernel_ms=kernel_ms, clocks=clocks,
                  launches=steps_done * KERNELS_PER_VERIFY, mean_accepted=float(n_acc.mean()), hit_rate=float(hit.mean()),
                  near_tie_rows=int(((st & ssd.ROW_NEAR_TIE) != 0).sum()), n_copies=n_copies,
                  alg_bytes=alg_bytes, logit_bytes=logit_bytes)

    # End to end through the public API from pinned host buffers (rank 0, N=1 only).
    if rank == 0 and world == 1 and not args.no_e2e:
        ht = torch.from_numpy(host_first["target"].view(np.int16)).view(torch.bfloat16).pin_memory() \
            if host_first["target"].dtype == np.uint16 else torch.from_numpy(host_first["target"]).pin_memory()
        hd = torch.from_numpy(host_first["draft"].view(np.int16)).view(torch.bfloat16).pin_memory() \
            if host_first["draft"].dtype == np.uint16 else torch.from_numpy(host_first["draft"]).pin_memory()
        htok = sets[0]["tok"].cpu().pin_memory()
        hu = torch.from_numpy(host_first["uniforms"]).pin_memory()
        ha = torch.from_numpy(host_first["alpha"]).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (ht, hd, htok, hu, ha))
        probe = ssd.ssd_verify_host(ht, hd, htok, hu, w.T, ha, w.budget, w.C, dev,
                                    fallback_seed=w_rank.fallback_seed, workspace=ws)
        d2h = sum(v.numel() * v.element_size() for v in probe.__dict__.values() if isinstance(v, torch.Tensor))
        e_steps = max(3, min(args.steps, 10))
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(e_steps):
            ssd.ssd_verify_host(ht, hd, htok, hu, w.T, ha, w.budget, w.C, dev, fallback_seed=w_rank.fallback_seed,
                                workspace=ws)
        t1.record(stream)
        torch.cuda.synchronize()
        e_ms = t0.elapsed_time(t1) / e_steps
        result["e2e"] = {"value": w.B / (e_ms / 1e3), "unit": "rows/s", "h2d_bytes_per_step": int(h2d),
                         "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms}
    return result


def cpu_baseline(w, seconds_target=15.0, reference_rows=None):
    """The fp64 oracle as it stands, on the host cores, over a bounded sample
    of rows of the same workload."""
    import oracle
    from speculative_decoding_verify_ssd_b200 import synth

    cores = oracle.n_threads_default()
    n = reference_rows or max(1, cores)
    g = synth.generate(w, rows=min(w.B, n))
    F = oracle.fanout_plan_batch(g["alpha"], w.K, w.budget, w.fanout_mode)
    tok = oracle.reweight(g["draft"], w.T, F, w.C, w.budget, u_draft=g["u_draft"], n_threads=cores)["tokens"]
    rows_done, t_total = 0, 0.0
    while t_total < seconds_target:
        t0 = time.perf_counter()
        oracle.verify(g["target"], g["draft"], tok, g["uniforms"], w.T, F=F, C_coef=w.C, budget=w.budget,
                      fallback_seed=w.fallback_seed, n_threads=cores)
        t_total += time.perf_counter() - t0
        rows_done += g["target"].shape[0]
        if reference_rows:
            break
    return {"value": rows_done / t_total, "unit": "rows/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows_done} rows of {w.name} (fp64 C oracle, {cores} threads, {t_total:.1f} s)"}


def run_reference(args, rank, world):
    from speculative_decoding_verify_ssd_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if rank != 0:
        return
    import oracle
    cores = oracle.n_threads_default()
    for _ in range(args.warmup):
        cpu_baseline(w, reference_rows=cores)
    vals = []
    t_all = 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        cb = cpu_baseline(w, reference_rows=cores)
        t_all += time.perf_counter() - t0
        vals.append(cb["value"])
    value = float(statistics.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_all / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": cores, "kind": "oracle",
                             "sample": f"{min(w.B, cores)} row{'s' if min(w.B, cores) != 1 else ''} of {w.name} per step"},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--repeat", type=int, default=4, help="timed replays of the graph of --steps launches")
    ap.add_argument("--impl", default="ssd", choices=["ssd", "reference"])
    ap.add_argument("--workload", default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    from speculative_decoding_verify_ssd_b200 import synth
    if args.workload is None:
        args.workload = synth.HEADLINE
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus={args.gpus}", file=sys.stderr)

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res = run_ssd(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    peak, peak_kind = measured_peaks()
    kms = sorted(res["kernel_ms"])
    k_avg = sum(kms) / len(kms)   # average launch duration over the timed region
    achieved = res["alg_bytes"] / (k_avg / 1e3) / 1e9
    traffic = recorded_traffic(w.name)
    line = {
        "metric": METRIC,
        "value": res["rows_per_s"],
        "unit": "rows/s",
        "n_gpus": world,
        "steps": args.steps * max(1, args.repeat),
        "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": dict(workload_config(w, world),
                       l2=f"{res['n_copies']} rotating input copies of {res['logit_bytes'] / 1e6:.1f} MB "
                          f"(each > 126 MB L2)"),
        "hbm_gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": ssd_step_kernels(),
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_kind == "measured" else "fallback 6650 GB/s",
                     "kernel_us_avg": k_avg * 1e3, "kernel_us_min": kms[0] * 1e3,
                     "alg_bytes_per_launch": res["alg_bytes"]},
        "gpu_launches": res["launches"],
        "mean_accepted": res["mean_accepted"],
        "hit_rate": res["hit_rate"],
        "near_tie_rows": res["near_tie_rows"],
    }
    if res.get("clocks"):
        line["clocks"] = res["clocks"]
    if "e2e" in res:
        line["e2e"] = res["e2e"]
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
