"""The N > 1 host logic of bench.py on CPU: two `gloo` ranks.  Each rank
shards by rows (its own seeds), verifies its shard with the oracle, and the
job's time is the slowest rank's (one MAX all-reduce taken by every rank at
the same point).  No GPU and no data-path collective."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    import oracle
    from speculative_decoding_verify_ssd_b200 import synth

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.WORKLOADS["zipf_b16_k5_v32000_bf16"].replace(B=4, V=2048)
        wr = bench.rank_workload(w, rank)
        g = synth.generate(wr)
        F = oracle.fanout_plan_batch(g["alpha"], wr.K, wr.budget, wr.fanout_mode)
        tok = oracle.reweight(g["draft"], wr.T, F, wr.C, wr.budget, u_draft=g["u_draft"])["tokens"]
        r = oracle.verify(g["target"], g["draft"], tok, g["uniforms"], wr.T, F=F, C_coef=wr.C, budget=wr.budget,
                          fallback_seed=wr.fallback_seed)
        fake_ms = 10.0 + 5.0 * rank  # a slower rank 1
        slowest = bench.max_over_ranks(fake_ms, dist, "cpu")
        value = bench.job_rows_per_s(world, w.B, 20, slowest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"seed": wr.seed, "fallback_seed": wr.fallback_seed, "slowest": slowest, "value": value,
                       "first_logits": g["target"][0, 0, :8].astype(np.int64).tolist(),
                       "n_accepted": r["n_accepted"].tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_rows_and_take_the_slowest_time(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert res[0]["seed"] != res[1]["seed"] and res[0]["fallback_seed"] != res[1]["fallback_seed"]
    assert res[0]["first_logits"] != res[1]["first_logits"], "ranks must verify different rows"
    for r in res:
        assert r["slowest"] == pytest.approx(15.0)
        assert r["value"] == pytest.approx(world * 4 * 20 / 15e-3)
        assert all(0 <= k <= 5 for k in r["n_accepted"])
