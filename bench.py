#!/usr/bin/env python3
"""Benchmark of the fused verify + speculation-cache step (libssd) on B200.

One step = the whole hot path over one batch: the fan-out plan and the fused
verify (softmax statistics, top-F, Saguaro reweighting, accept test, residual
bonus draw, cache build and lookup).  Inputs are seeded synthetic Zipf
logits, generated on the host and resident in HBM before timing starts;
enough input copies rotate that their total exceeds twice the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --workload zipf_b256_k8_v151936_bf16_sweep --sweep
        # one line per (T, fan-out mode, C): rows/s, GB/s, hit rate
    python bench.py --workload zipf_b512_k4_v128256_bf16_miss --unfused
        # the five-call step (plan, reweight, verify, cache build, lookup)
    python bench.py --impl reference ...   # the fp64 CPU oracle on host cores

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
rows (weak scaling, no collective on the data path); the step time is the
maximum over ranks.  Rank 0 prints one JSON line (per sweep point).
"""
import argparse
import hashlib
import json
import os
import statistics
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
GRAPH_CALLS = 200  # verify calls captured per CUDA graph; the timed region replays graphs summing to --steps

# ssd_verify launches ssd_stats_kernel (softmax statistics, top-F, accept test,
# row decision) and then ssd_draw_kernel (residual / bonus draw, cache lookup).
KERNELS_PER_VERIFY = 2
# the unfused step: fan-out plan, reweight (its statistics kernel; no draft
# draw), verify without a cache (2), cache build, cache lookup
KERNELS_PER_UNFUSED = 6


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
    """DRAM bytes per launch of the verify kernels from a committed ncu
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
    """SM clock, max clock and throttle reasons sampled through NVML every
    few milliseconds while the timed region runs."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    r = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                    for name, bit in self.REASONS:
                        if r & bit:
                            self.reasons.add(name)
                except Exception:
                    pass
                time.sleep(0.002)

        self._thr = threading.Thread(target=loop, daemon=True)
        self._thr.start()

    def stop(self):
        if self._thr is None:
            return None
        self._stop.set()
        self._thr.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, every 2 ms"}


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


def n_rotating_copies(logit_bytes):
    """Input copies so that the rotation exceeds twice the L2 (small
    workloads would otherwise be served from L2), within 4 GB."""
    n = max(2, -(-2 * L2_BYTES // logit_bytes))
    return int(min(n, max(2, (4 << 30) // logit_bytes)))


def make_sets(w, n_copies, dev, ssd, synth):
    import torch

    def dev_logits(x):
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(x).to(dev)

    sets, host_first = [], None
    for c in range(n_copies):
        g = synth.generate(w.replace(seed=w.seed + 104729 * c))
        if c == 0:
            host_first = g
        sets.append(dict(t=dev_logits(g["target"]), d=dev_logits(g["draft"]),
                         u=torch.from_numpy(g["uniforms"]).to(dev), u_draft=torch.from_numpy(g["u_draft"]).to(dev)))
        del g
    return sets, host_first


def draw_tokens(w, sets, dev, ssd):
    """Draft tokens from the draft side's own Saguaro sampler (d_j ~ q'_j)."""
    import torch
    for s in sets:
        s["alpha"] = torch.full((w.B,), w.alpha, dtype=torch.float32, device=dev)
        s["F"] = ssd.ssd_fanout_plan(s["alpha"], w.K, w.budget, w.fanout_mode)
        rw = ssd.ssd_saguaro_reweight(s["d"], w.T, s["F"], w.C, w.budget, u_draft=s["u_draft"])
        s["tok"] = rw.draft_tokens
    torch.cuda.synchronize()


def time_steps(step, steps, warmup, dev, world, dist, sampler_index):
    """Warm up, capture CUDA graphs of up to GRAPH_CALLS steps, and time
    exactly `steps` steps (graph replays summing to `steps`) with CUDA events
    on the launching stream.  Returns (total_ms, per-step ms of each replay,
    clocks)."""
    import torch
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    per_graph = min(steps, GRAPH_CALLS)
    full, rest = divmod(steps, per_graph)
    graphs = []
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    for n in ([per_graph] if full else []) + ([rest] if rest else []):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                for i in range(n):
                    step(i)
        graphs.append((g, n))
    torch.cuda.synchronize()
    for g, _ in graphs:
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    plan = [graphs[0]] * full + ([graphs[-1]] if rest else [])
    sampler = ClockSampler(sampler_index) if sampler_index is not None else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    marks = []
    start.record(stream)
    for g, n in plan:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        marks.append((e0, e1, n))
    end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    per_step = [a.elapsed_time(b) / n for a, b, n in marks]
    del graphs, plan
    return total_ms, per_step, clocks


def run_ssd(args, rank, world, local_rank):
    import torch
    from speculative_decoding_verify_ssd_b200 import binding as ssd
    from speculative_decoding_verify_ssd_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ssd.load()
    dist = None
    if world > 1:
        import torch.distributed as dist
    w0 = synth.WORKLOADS[args.workload]
    w_rank = rank_workload(w0, rank)
    logit_bytes, alg_bytes = algorithmic_bytes(w0)
    n_copies = n_rotating_copies(logit_bytes)
    sets, host_first = make_sets(w_rank, n_copies, dev, ssd, synth)

    points = [dict()]
    if args.sweep:
        points = [dict(T=T, fanout_mode=m, C=C, alpha=synth.SWEEP_ALPHA[T])
                  for T in (0.0, 0.6, 1.0) for m in (0, 1) for C in (1.0, 0.5, 0.2)]
    results = []
    for pt in points:
        w = w_rank.replace(**pt)
        draw_tokens(w, sets, dev, ssd)
        ws = ssd.Workspace(w.B, w.K, dev, w.V, ssd.DTYPE_BF16 if w.dtype == "bf16" else ssd.DTYPE_FP32)
        outs = [ssd.alloc_verify_result(w.B, w.K, w.budget, dev, True) for _ in range(n_copies)]

        if args.unfused:
            def step(i, w=w, ws=ws, outs=outs):
                # the five calls of the unfused step on one stream
                s = sets[i % n_copies]
                o = outs[i % n_copies]
                F = ssd.ssd_fanout_plan(s["alpha"], w.K, w.budget, w.fanout_mode, F=s["F"])
                rw = ssd.ssd_saguaro_reweight(s["d"], w.T, F, w.C, w.budget, guess=s["t"][:, w.K, :],
                                              guess_row_stride=(w.K + 1) * w.V, workspace=ws)
                ver = ssd.ssd_verify(s["t"], s["d"], s["tok"], s["u"], w.T, F=F, C_coef=w.C, budget=w.budget,
                                     cache=False, workspace=ws, out=o)
                offs, toks = ssd.ssd_cache_build(F, rw.topf_tokens, w.budget)
                hit, slot, nxt = ssd.ssd_cache_lookup(offs, toks, ver.n_accepted, ver.bonus, w.V,
                                                      fallback_seed=w.fallback_seed)
                o.hit, o.slot, o.next_tokens = hit, slot, nxt
            kernels = KERNELS_PER_UNFUSED
        else:
            def step(i, w=w, ws=ws, outs=outs):
                # one launch pair: the fan-out plan is computed inside the fused kernel from alpha
                s = sets[i % n_copies]
                ssd.ssd_verify(s["t"], s["d"], s["tok"], s["u"], w.T, alpha=s["alpha"], fanout_mode=w.fanout_mode,
                               C_coef=w.C, budget=w.budget, cache=True, fallback_seed=w.fallback_seed,
                               workspace=ws, out=outs[i % n_copies], early_exit=args.early_exit)
            kernels = KERNELS_PER_VERIFY
        total_ms, per_step, clocks = time_steps(step, args.steps, args.warmup, dev, world, dist,
                                                local_rank if rank == 0 else None)
        if world > 1:
            total_ms = max_over_ranks(total_ms, dist, dev)
        skipped = None
        if args.early_exit:
            # target bytes left unread per call, counted on the device over one
            # pass of the rotating copies (outside the timed region)
            torch.cuda.synchronize()
            ws.skipped_bytes()
            for i in range(n_copies):
                step(i)
            skipped = ws.skipped_bytes() / n_copies
        # outcome statistics over every rotating copy's last step
        torch.cuda.synchronize()
        n_acc = np.concatenate([o.n_accepted.cpu().numpy() for o in outs])
        hit = np.concatenate([o.hit.cpu().numpy() for o in outs])
        st = np.concatenate([o.status.cpu().numpy() for o in outs])
        res = dict(point=pt, w=w, rows_per_s=job_rows_per_s(world, w.B, args.steps, total_ms),
                   ms_per_step=total_ms / args.steps, per_step_ms=per_step, clocks=clocks,
                   launches=args.steps * kernels, mean_accepted=float(n_acc.mean()), hit_rate=float(hit.mean()),
                   near_tie_rows=int(((st & ssd.ROW_NEAR_TIE) != 0).sum()), n_copies=n_copies, alg_bytes=alg_bytes,
                   logit_bytes=logit_bytes)
        if args.early_exit:
            # the early-exit count: every draft row, the target rows p_0..p_k*
            # and p_K, from this run's outcomes; the full read beside it
            s_b = 2 if w.dtype == "bf16" else 4
            kk = n_acc[n_acc >= 0]
            p_rows = np.where(kk >= w.K, w.K + 1, kk + 2).mean() if kk.size else w.K + 1
            ee_logits = w.B * (w.K + p_rows) * w.V * s_b
            res["alg_bytes"] = int(alg_bytes - logit_bytes + ee_logits)
            res["early_exit"] = {"alg_bytes_per_launch": res["alg_bytes"], "full_read_bytes_per_launch": alg_bytes,
                                 "target_bytes_not_read_per_launch": skipped,
                                 "logit_bytes_read_per_launch": logit_bytes - skipped}

        # End to end through the public API from pinned host buffers (rank 0,
        # N=1, default fused step only).
        if rank == 0 and world == 1 and not args.no_e2e and not args.unfused and not args.sweep and not args.early_exit:
            def pin(x):
                if x.dtype == np.uint16:
                    return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
                return torch.from_numpy(x).pin_memory()
            ht, hd = pin(host_first["target"]), pin(host_first["draft"])
            htok = sets[0]["tok"].cpu().pin_memory()
            hu = torch.from_numpy(host_first["uniforms"]).pin_memory()
            ha = torch.full((w.B,), w.alpha, dtype=torch.float32).pin_memory()
            h2d = sum(x.numel() * x.element_size() for x in (ht, hd, htok, hu, ha))
            probe = ssd.ssd_verify_host(ht, hd, htok, hu, w.T, ha, w.budget, w.C, dev,
                                        fallback_seed=w.fallback_seed, workspace=ws)
            d2h = sum(v.numel() * v.element_size() for v in probe.__dict__.values() if isinstance(v, torch.Tensor))
            e_steps = max(3, min(args.steps, 10))
            stream = torch.cuda.current_stream(dev)
            torch.cuda.synchronize()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(e_steps):
                ssd.ssd_verify_host(ht, hd, htok, hu, w.T, ha, w.budget, w.C, dev, fallback_seed=w.fallback_seed,
                                    workspace=ws)
            t1.record(stream)
            torch.cuda.synchronize()
            e_ms = t0.elapsed_time(t1) / e_steps
            res["e2e"] = {"value": w.B / (e_ms / 1e3), "unit": "rows/s", "h2d_bytes_per_step": int(h2d),
                          "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms}
        results.append(res)
        del ws, outs
    return results


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


def build_line(args, res, world):
    w = res["w"]
    peak, peak_kind = measured_peaks()
    per = res["per_step_ms"]
    k_avg = sum(per) / len(per)   # average launch duration over the timed region
    achieved = res["alg_bytes"] / (k_avg / 1e3) / 1e9
    traffic = recorded_traffic(w.name) if not args.unfused and not args.sweep else None
    cfg = dict(workload_config(w, world),
               l2=f"{res['n_copies']} rotating input copies of {res['logit_bytes'] / 1e6:.1f} MB "
                  f"(together > 2 x 126 MB L2)")
    if args.unfused:
        cfg["step"] = "unfused: fan-out plan, reweight, verify, cache build, cache lookup (one stream)"
    if args.early_exit:
        cfg["read_schedule"] = "early exit (ssd_verify_early_exit)"
    line = {
        "metric": METRIC,
        "value": res["rows_per_s"],
        "unit": "rows/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": cfg,
        "hbm_gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": ssd_step_kernels() if not args.unfused else "the five-call step, timed as a whole",
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_kind == "measured" else "fallback 6650 GB/s",
                     "kernel_us_avg": k_avg * 1e3, "kernel_us_min": min(per) * 1e3,
                     "alg_bytes_per_launch": res["alg_bytes"]},
        "gpu_launches": res["launches"],
        "mean_accepted": res["mean_accepted"],
        "hit_rate": res["hit_rate"],
        "miss_rate": 1.0 - res["hit_rate"],
        "near_tie_rows": res["near_tie_rows"],
    }
    if res.get("clocks"):
        line["clocks"] = res["clocks"]
    if "e2e" in res:
        line["e2e"] = res["e2e"]
    if "early_exit" in res:
        line["early_exit"] = res["early_exit"]
        line["roofline"]["traffic"] = None
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, seconds_target=5.0 if args.sweep else 15.0)
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ssd", choices=["ssd", "reference"])
    ap.add_argument("--workload", default=None)
    ap.add_argument("--sweep", action="store_true", help="temperature x fan-out mode x C grid, one line each")
    ap.add_argument("--unfused", action="store_true", help="time the five-call unfused step")
    ap.add_argument("--early-exit", action="store_true", help="the early-exit read schedule (ssd_verify_early_exit)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    from speculative_decoding_verify_ssd_b200 import synth
    if args.workload is None:
        args.workload = synth.HEADLINE
    args.warmup = max(args.warmup, 3)
    args.steps = max(args.steps, 1)

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
    results = run_ssd(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    for res in results:
        print(json.dumps(build_line(args, res, world)), flush=True)


if __name__ == "__main__":
    main()
