"""Measure each synthetic workload's mean acceptance overlap with the oracle.

alpha (the fan-out's per-token acceptance estimate) is stated per workload as
the mean over rows and draft positions of sum_v min(p_j(v), q_j(v)) on the
pre-reweight distributions, rounded to 0.01.  For the headline workload the
draft noise sigma is found by bisection so that this mean is 0.70.

Calls only oracle/ and the seeded generator.  Run:
    python tests/golden/calibrate_workloads.py
and copy the printed values into speculative_decoding_verify_ssd_b200/synth.py.
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from speculative_decoding_verify_ssd_b200 import synth  # noqa: E402


def mean_overlap(w, rows=8):
    g = synth.generate(w, rows=rows)
    vals = [oracle.overlap(g["target"][b, j], g["draft"][b, j], w.T if w.T > 0 else 1e-9)
            if w.T > 0 else float(np.argmax(synth.to_f32(g["target"][b, j])) ==
                                  np.argmax(synth.to_f32(g["draft"][b, j])))
            for b in range(rows) for j in range(w.K)]
    return float(np.mean(vals))


def main():
    head = synth.WORKLOADS[synth.HEADLINE]
    lo, hi = 0.05, 3.0
    for _ in range(18):
        mid = 0.5 * (lo + hi)
        a = mean_overlap(head.replace(draft_sigma=mid), rows=16)
        if a > 0.70:
            lo = mid
        else:
            hi = mid
    sigma = round(0.5 * (lo + hi), 2)
    print(f"{synth.HEADLINE}: draft_sigma={sigma} alpha={mean_overlap(head.replace(draft_sigma=sigma), 16):.4f}")
    for name, w in synth.WORKLOADS.items():
        if name == synth.HEADLINE:
            continue
        print(f"{name}: alpha={mean_overlap(w, rows=min(w.B, 8)):.4f}")
    sweep = synth.WORKLOADS["zipf_b256_k8_v151936_bf16_sweep"]
    for T in (0.0, 0.6, 1.0):
        print(f"sweep T={T}: alpha={mean_overlap(sweep.replace(T=T), rows=8):.4f}")


if __name__ == "__main__":
    main()
