"""The early-exit read schedule (ssd_verify_early_exit) through the C ABI:
against the oracle run with the same schedule, against the full read of the
same inputs, with the rows it need not read filled with garbage, and at the
headline size, where it must leave target rows unread."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_ssd_b200 import binding as ssd
from speculative_decoding_verify_ssd_b200 import synth

from ssd_testlib import Case, check_row_properties, compare, to_dev

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS

SMALL = [
    ("zipf_b16_k5_v32000_bf16", {}),
    ("zipf_b16_k5_v32000_bf16", {"V": 8003, "seed": 21}),   # ragged rows: the unaligned path
    ("tiny_b1_k4_v1024_fp32", {}),
    ("zipf_b16_k5_v32000_bf16", {"T": 0.0, "seed": 22}),    # greedy
    ("zipf_b64_k6_v128256_bf16", {"B": 24, "seed": 23}),
    ("zipf_b16_k5_v32000_bf16", {"B": 6, "K": 32, "V": 4096, "budget": 512, "seed": 32}),  # largest K and budget
]


@pytest.mark.parametrize("name,over", SMALL, ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in o.items())}" for n, o in SMALL])
def test_early_exit_matches_oracle(name, over):
    w = W[name].replace(**over)
    case = Case(w)
    gpu = case.run_gpu(early_exit=True)
    orc = case.run_oracle(early_exit=True)
    compare(case, gpu, orc, early_exit=True)
    check_row_properties(case, gpu, early_exit=True)


def _fields(r):
    return {k: v.cpu().numpy() for k, v in r.__dict__.items() if isinstance(v, torch.Tensor)}


def test_early_exit_equals_full_read():
    """Same inputs, both schedules: the same outcome and cache on every row;
    a_j equal up to k* and absent after it."""
    w = W["zipf_b64_k6_v128256_bf16"].replace(B=32, seed=24)
    case = Case(w)
    full = case.run_gpu()
    ee = case.run_gpu(early_exit=True)
    for k in ("n_accepted", "bonus", "out_tokens", "residual_mass", "cache_offsets", "cache_tokens", "hit", "slot",
              "next_tokens"):
        np.testing.assert_array_equal(ee[k], full[k], err_msg=k)
    K = w.K
    for b, ks in enumerate(full["n_accepted"]):
        np.testing.assert_array_equal(ee["accept_prob"][b, :min(ks + 1, K)], full["accept_prob"][b, :min(ks + 1, K)])
        assert np.all(np.isnan(ee["accept_prob"][b, ks + 1:]))
    assert np.all((ee["status"] ^ full["status"]) & ~ssd.ROW_ZERO_Q == 0)


def test_early_exit_ignores_target_rows_past_k_star():
    """Target rows p_j with k* < j < K hold NaN or huge values: the early-exit
    call must give the outcome of the clean inputs and flag nothing, while
    the full read flags those rows as non-finite."""
    w = W["zipf_b16_k5_v32000_bf16"].replace(seed=25)
    case = Case(w)
    clean = case.run_gpu()
    K = w.K
    t = case.g["target"].copy()
    dirty = 0
    for b, ks in enumerate(clean["n_accepted"]):
        for j in range(ks + 1, K):
            t[b, j, :] = 0x7FC0 if (b + j) % 2 else 0x7F7F  # bf16 NaN / largest finite
            dirty += 1
    assert dirty > 5
    d_t = to_dev(t)
    d = to_dev(case.g["draft"])
    tok, u, F = to_dev(case.tokens), to_dev(case.g["uniforms"]), to_dev(case.F)
    ee = _fields(ssd.ssd_verify(d_t, d, tok, u, w.T, F=F, C_coef=w.C, budget=w.budget, cache=True,
                                fallback_seed=w.fallback_seed, early_exit=True))
    full = _fields(ssd.ssd_verify(d_t, d, tok, u, w.T, F=F, C_coef=w.C, budget=w.budget, cache=True,
                                  fallback_seed=w.fallback_seed))
    torch.cuda.synchronize()
    for k in ("n_accepted", "bonus", "cache_tokens", "hit", "slot", "next_tokens"):
        np.testing.assert_array_equal(ee[k], clean[k], err_msg=k)
    assert np.all(ee["status"] & ssd.ROW_INVALID == 0)
    nan_rows = np.array([any((t[b, j] == 0x7FC0).any() for j in range(K)) for b in range(w.B)])
    assert np.all(full["status"][nan_rows] & ssd.ROW_NONFINITE)
    orc = oracle.verify(t, case.g["draft"], case.tokens, case.g["uniforms"], w.T, F=case.F, C_coef=w.C,
                        budget=w.budget, fallback_seed=w.fallback_seed, early_exit=True)
    np.testing.assert_array_equal(ee["n_accepted"], orc["n_accepted"])
    np.testing.assert_array_equal(ee["status"] & ssd.ROW_INVALID, orc["status"] & oracle.ROW_INVALID)


def test_early_exit_headline_reads_less_and_matches_sampled_rows():
    """The headline shape in the launch configuration the bench times:
    sampled rows against the oracle, every row's properties, and target rows
    left unread (the counted bytes never exceed what the outcome allows)."""
    w = W["zipf_b64_k6_v128256_bf16"]
    rows = np.arange(0, w.B, 3)
    case = Case(w, check_rows=rows)
    dev = torch.device("cuda")
    ws = ssd.Workspace(w.B, w.K, dev, w.V, ssd.DTYPE_BF16)
    ws.skipped_bytes()
    r = ssd.ssd_verify(to_dev(case.g["target"]), to_dev(case.g["draft"]), to_dev(case.tokens),
                       to_dev(case.g["uniforms"]), w.T, F=to_dev(case.F), C_coef=w.C, budget=w.budget, cache=True,
                       fallback_seed=w.fallback_seed, workspace=ws, early_exit=True)
    torch.cuda.synchronize()
    gpu = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in r.__dict__.items()}
    skipped = ws.skipped_bytes()
    compare(case, gpu, case.run_oracle(early_exit=True), early_exit=True)
    check_row_properties(case, gpu, early_exit=True)
    k = gpu["n_accepted"]
    allowed = int(np.sum(np.clip(w.K - 1 - k, 0, None))) * w.V * 2
    assert 0 < skipped <= allowed, (skipped, allowed)
