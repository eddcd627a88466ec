"""The one-pass cluster form of ssd_verify against the fp64 oracle.

A build of the library with SSD_CLUSTER_VERIFY=1 runs bf16 verify calls
(T > 0, rows of a multiple of 8 tokens, budget <= 256) as one kernel of
thread-block clusters: one cluster per (row, position) unit, the slice
statistics, top-F candidates and slice masses exchanged over distributed
shared memory between cluster barriers, and the bonus drawn inside the
cluster.  The default build keeps the two-kernel form, which measures faster
on B200; this build must still give the oracle's answers, element by element,
on the same cases the default build is held to.
"""
import numpy as np
import pytest

from speculative_decoding_verify_ssd_b200 import _build
from speculative_decoding_verify_ssd_b200 import binding as ssd
from speculative_decoding_verify_ssd_b200 import synth

from ssd_testlib import Case, check_row_properties, compare, draft_tokens_for

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def cluster_build():
    path = _build.build_variant("cluster", ["SSD_CLUSTER_VERIFY=1"])
    saved_path, saved_lib = _build.LIB, ssd._lib
    _build.LIB = path
    ssd._lib = None
    ssd._default_ws.clear()
    ssd.load(build_if_missing=False)
    yield
    _build.LIB, ssd._lib = saved_path, saved_lib
    ssd._default_ws.clear()


CASES = [
    ("headline_b8", W["zipf_b64_k6_v128256_bf16"].replace(B=8)),           # 4 CTAs per unit
    ("v32000_full", W["zipf_b16_k5_v32000_bf16"]),                         # 8 CTAs per unit
    ("miss_b12", W["zipf_b512_k4_v128256_bf16_miss"].replace(B=12)),
    ("sweep_t06_uniform", W["zipf_b256_k8_v151936_bf16_sweep"].replace(
        B=6, T=0.6, alpha=synth.SWEEP_ALPHA[0.6], fanout_mode=1)),           # 5 CTAs per unit
    ("sweep_t1_c02", W["zipf_b256_k8_v151936_bf16_sweep"].replace(B=6, C=0.2)),
    ("k1_v2048", W["zipf_b16_k5_v32000_bf16"].replace(B=16, K=1, V=2048, budget=4)),
    ("max_vocab_one_row", W["zipf_b64_k6_v128256_bf16"].replace(B=1, V=262144, K=3, budget=16)),
]


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_cluster_form_matches_oracle(name, w):
    case = Case(w)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)
    check_row_properties(case, gpu)


def test_cluster_form_headline_sampled_rows():
    w = W["zipf_b64_k6_v128256_bf16"]
    rows = np.sort(np.random.default_rng(99).choice(w.B, size=16, replace=False)).astype(np.int32)
    case = Case(w, check_rows=rows)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)
    check_row_properties(case, gpu)


def test_cluster_form_draft_next_payload_and_no_plan():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=12)
    case = Case(w, with_draft_next=True)
    payload = np.random.default_rng(5).integers(0, w.V, (w.B, w.budget, w.K)).astype(np.int32)
    gpu = case.run_gpu(payload=payload)
    compare(case, gpu, case.run_oracle(payload=payload))
    case2 = Case(w.replace(B=8))
    gpu2 = case2.run_gpu(cache=False, with_F=False)
    compare(case2, gpu2, case2.run_oracle(with_F=False), with_cache=False)


def test_cluster_form_exact_select_on_ties():
    """Logits on three values: every slice's candidate list overflows, and the
    cluster's exact bitwise select with ties in token order takes over."""
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=4, V=3000 - 3000 % 8, budget=200, alpha=0.05)
    case = Case(w)
    rng = np.random.default_rng(4)
    for key in ("target", "draft"):
        vals = rng.integers(0, 3, case.g[key].shape).astype(np.float32) * 0.25
        case.g[key] = synth.f32_to_bf16_bits(vals)
    case.tokens = draft_tokens_for(w, case.g, case.F)
    gpu = case.run_gpu()
    compare(case, gpu, case.run_oracle())


def test_cluster_form_invalid_rows_and_full_acceptance():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=6, C=1.0)
    case = Case(w)
    case.g["target"][0, 2, 17] = 0x7FC0          # NaN: row 0 is void
    case.g["draft"][1] = case.g["target"][1, :w.K]  # q = p: row 1 accepts every draft
    case.tokens = draft_tokens_for(w, case.g, case.F)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    assert orc["n_accepted"][1] == w.K
    assert gpu["n_accepted"][0] == -1 and (gpu["status"][0] & ssd.ROW_INVALID) != 0
    compare(case, gpu, orc)
