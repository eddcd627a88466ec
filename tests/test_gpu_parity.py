"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small cases span several CTA slices and a ragged tail; the full-size cases run
every row of the workload in the launch configuration the benchmark uses and
compare a sample of rows with the oracle, plus properties checked on all rows.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_ssd_b200 import binding as ssd
from speculative_decoding_verify_ssd_b200 import synth

from ssd_testlib import Case, check_row_properties, compare, draft_tokens_for, to_dev, PROB_ATOL, LSE_RTOL

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ssd.load()
    yield


# ---------------------------------------------------------------------------
# Small / mid-size cases: every row compared with the oracle.
# ---------------------------------------------------------------------------
SMALL = [
    ("tiny_fp32_full", W["tiny_b1_k4_v1024_fp32"]),
    ("tiny_fp32_b48", W["tiny_b1_k4_v1024_fp32"].replace(B=48)),
    ("zipf_v32000_full", W["zipf_b16_k5_v32000_bf16"]),
    ("zipf_v128256_b8", W["zipf_b64_k6_v128256_bf16"].replace(B=8)),
    ("miss_v128256_b12", W["zipf_b512_k4_v128256_bf16_miss"].replace(B=12)),
    ("ragged_v5003_bf16", W["zipf_b16_k5_v32000_bf16"].replace(B=10, V=5003, budget=24)),
    ("ragged_v777_fp32", W["tiny_b1_k4_v1024_fp32"].replace(B=20, V=777, budget=12, K=6)),
    ("k1_v2048", W["zipf_b16_k5_v32000_bf16"].replace(B=16, K=1, V=2048, budget=4)),
]


@pytest.mark.parametrize("name,w", SMALL, ids=[s[0] for s in SMALL])
def test_verify_matches_oracle_small(name, w):
    case = Case(w)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    near = compare(case, gpu, orc)
    check_row_properties(case, gpu)
    print(f"{name}: {near} near-tie rows of {w.B}")


@pytest.mark.parametrize("T", [0.0, 0.6, 1.0])
@pytest.mark.parametrize("mode", [0, 1])
def test_sweep_temperature_and_fanout(T, mode):
    w = W["zipf_b256_k8_v151936_bf16_sweep"].replace(B=8, T=T, alpha=synth.SWEEP_ALPHA[T], fanout_mode=mode)
    case = Case(w)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)
    check_row_properties(case, gpu)


@pytest.mark.parametrize("C", [1.0, 0.5, 0.2])
def test_sweep_saguaro_coefficient(C):
    w = W["zipf_b256_k8_v151936_bf16_sweep"].replace(B=6, C=C)
    case = Case(w)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)


def test_draft_next_and_payload():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=12)
    case = Case(w, with_draft_next=True)
    payload = np.random.default_rng(5).integers(0, w.V, (w.B, w.budget, w.K)).astype(np.int32)
    gpu = case.run_gpu(payload=payload)
    orc = case.run_oracle(payload=payload)
    compare(case, gpu, orc)
    check_row_properties(case, gpu)


def test_no_plan_means_no_reweight():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=8)
    case = Case(w)
    gpu = case.run_gpu(cache=False, with_F=False)
    orc = case.run_oracle(with_F=False)
    compare(case, gpu, orc, with_cache=False)


# ---------------------------------------------------------------------------
# Full-size workloads in the benchmark's launch configuration.
# ---------------------------------------------------------------------------
FULL = ["zipf_b16_k5_v32000_bf16", "zipf_b64_k6_v128256_bf16", "zipf_b256_k8_v151936_bf16_sweep",
        "zipf_b512_k4_v128256_bf16_miss"]


@pytest.mark.parametrize("name", FULL)
def test_verify_full_size_sampled(name):
    w = W[name]
    rng = np.random.default_rng(99)
    rows = np.sort(rng.choice(w.B, size=min(w.B, 24), replace=False)).astype(np.int32)
    case = Case(w, check_rows=rows)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)
    check_row_properties(case, gpu)


# ---------------------------------------------------------------------------
# Edge cases.
# ---------------------------------------------------------------------------
def _edge_case(w, mutate):
    case = Case(w)
    mutate(case)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)
    return case, gpu, orc


def test_invalid_rows_flagged_not_trapped():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=8)

    def mutate(c):
        bits = c.g["target"]
        bits[0, 2, 17] = 0x7FC0          # NaN
        bits[1, 0, 3] = 0x7F80           # +inf
        c.g["draft"][2, 1, :] = 0xFF80   # a whole draft row at -inf
        c.tokens[3, 0] = w.V             # token out of range
        c.g["uniforms"][4, w.K] = 1.0    # uniform outside [0, 1)
        c.F[5, 0] += 1                   # plan no longer sums to the budget

    case, gpu, orc = _edge_case(w, mutate)
    for b, bit in ((0, 1), (1, 1), (2, 1), (3, 2), (4, 4), (5, 64)):
        assert gpu["status"][b] & bit, (b, gpu["status"][b])
        assert gpu["n_accepted"][b] == -1 and gpu["bonus"][b] == -1
        assert np.all(gpu["cache_tokens"][b] == -1)
    assert np.all((gpu["status"][6:] & ssd.ROW_INVALID) == 0)


def test_neg_inf_logits_and_zero_draft_probability():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=8)

    def mutate(c):
        rng = np.random.default_rng(3)
        for b in range(w.B):
            for j in range(w.K):
                idx = rng.choice(w.V, 500, replace=False)
                c.g["draft"][b, j, idx] = 0xFF80
                c.g["target"][b, j, idx[:250]] = 0xFF80
            # the draft token sits where the draft has zero probability
            c.tokens[b, 0] = idx_first = int(np.nonzero(c.g["draft"][b, 0] == 0xFF80)[0][0])
            assert idx_first >= 0

    case, gpu, orc = _edge_case(w, mutate)
    assert np.all(orc["status"] & oracle.ROW_ZERO_Q)


def test_greedy_with_ties():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=16, T=0.0)

    def mutate(c):
        # heavy ties: quantise logits to a coarse grid so several ids share the max
        for key in ("target", "draft"):
            f = synth.bf16_bits_to_f32(c.g[key])
            c.g[key] = synth.f32_to_bf16_bits(np.round(f * 2) / 2)
        am = np.argmax(synth.bf16_bits_to_f32(c.g["target"][:, :w.K]), axis=2)
        keep = np.random.default_rng(1).random((w.B, w.K)) < 0.85
        c.tokens = np.where(keep, am, c.tokens).astype(np.int32)

    _edge_case(w, mutate)


def test_topf_slow_path_many_ties_and_big_F():
    # Every logit in a handful of values: the candidate filter overflows and
    # the exact global radix select takes over; F also exceeds the group count.
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=4, V=3000, budget=400, alpha=0.05)

    def mutate(c):
        rng = np.random.default_rng(4)
        for key in ("target", "draft"):
            vals = rng.integers(0, 3, c.g[key].shape).astype(np.float32) * 0.25
            c.g[key] = synth.f32_to_bf16_bits(vals)

    _edge_case(w, mutate)


def test_F_zero_budget_K_plus_1_and_C_one():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=8, budget=6, C=1.0)
    case = Case(w)
    case.F[:] = 1
    case.F[0] = [6, 0, 0, 0, 0, 0]
    case.F[1] = [0, 0, 0, 0, 0, 6]
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)


def test_max_draft_length_and_max_budget():
    """K = 32, the largest draft length (its unit 32 rides in the second word
    a lane of the draw's decision wait holds), with the largest budget, 512
    (top-F sets above a slice's candidate slots take the exact global
    path).  Rows 0 and 1 have draft rows equal to their target rows and
    C = 1, so every position is accepted and the bonus comes from p_K."""
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=4, K=32, V=4096, budget=512, C=1.0, seed=31)
    case = Case(w)
    for b in (0, 1):
        case.g["draft"][b] = case.g["target"][b, :w.K]
    case.tokens = draft_tokens_for(w, case.g, case.F)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    assert list(orc["n_accepted"][:2]) == [32, 32]
    compare(case, gpu, orc)
    check_row_properties(case, gpu)


def test_empty_batch():
    """B = 0: the call succeeds, launches nothing and returns empty outputs."""
    w = W["zipf_b16_k5_v32000_bf16"]
    dev = torch.device("cuda")
    t = torch.zeros(0, w.K + 1, w.V, dtype=torch.bfloat16, device=dev)
    d = torch.zeros(0, w.K, w.V, dtype=torch.bfloat16, device=dev)
    tok = torch.zeros(0, w.K, dtype=torch.int32, device=dev)
    u = torch.zeros(0, w.K + 1, dtype=torch.float32, device=dev)
    F = torch.zeros(0, w.K + 1, dtype=torch.int32, device=dev)
    r = ssd.ssd_verify(t, d, tok, u, w.T, F=F, C_coef=w.C, budget=w.budget, cache=True)
    torch.cuda.synchronize()
    assert r.n_accepted.numel() == 0 and r.bonus.numel() == 0 and r.status.numel() == 0


def test_single_row_and_max_vocab():
    w = W["zipf_b64_k6_v128256_bf16"].replace(B=1, V=262144, K=3, budget=16)
    case = Case(w)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)


# ---------------------------------------------------------------------------
# The other entry points.
# ---------------------------------------------------------------------------
def test_fanout_plan_bit_exact():
    rng = np.random.default_rng(0)
    for K in (1, 4, 6, 8, 32):
        for budget in (0, 1, 7, 64, 128, 512):
            alpha = rng.random(200).astype(np.float32)
            alpha[:3] = [0.0, 1.0, 0.5]
            for mode in (0, 1):
                Fg = ssd.ssd_fanout_plan(to_dev(alpha), K, budget, mode).cpu().numpy()
                Fo = oracle.fanout_plan_batch(alpha, K, budget, mode)
                np.testing.assert_array_equal(Fg, Fo, err_msg=f"K={K} budget={budget} mode={mode}")


@pytest.mark.parametrize("name", ["zipf_b16_k5_v32000_bf16", "tiny_b1_k4_v1024_fp32"])
@pytest.mark.parametrize("T", [0.0, 0.8])
def test_saguaro_reweight_and_draft_draw(name, T):
    w = W[name].replace(B=max(W[name].B, 8), T=T)
    g = synth.generate(w)
    F = oracle.fanout_plan_batch(g["alpha"], w.K, w.budget)
    r = ssd.ssd_saguaro_reweight(to_dev(g["draft"]), T, to_dev(F), w.C, w.budget, u_draft=to_dev(g["u_draft"]))
    torch.cuda.synchronize()
    o = oracle.reweight(g["draft"], T, F, w.C, w.budget, u_draft=g["u_draft"])
    np.testing.assert_array_equal(r.offsets.cpu().numpy(), o["offsets"])
    n_keys = o["offsets"][:, w.K]
    tg = r.topf_tokens.cpu().numpy()
    for b in range(w.B):
        np.testing.assert_array_equal(tg[b, :n_keys[b]], o["topf_tokens"][b, :n_keys[b]])
    assert np.max(np.abs(r.Z.cpu().numpy() - o["Z"])) < PROB_ATOL
    ql = r.q_lse.cpu().numpy().astype(np.float64)
    lse_err = np.max(np.abs(ql - o["q_lse"]) / np.maximum(1.0, np.abs(o["q_lse"])))
    print(f"q_lse error relative to max(1, |lse|): {lse_err:.3g}")
    assert lse_err < LSE_RTOL
    # every draft token is bit-exact, or inside the oracle's near-tie window
    # of its draw when that draw's margin is below 1e-5
    dg = r.draft_tokens.cpu().numpy()
    assert np.all((o["tok_lo"] <= dg) & (dg <= o["tok_hi"]))
    near = (o["status"] & oracle.ROW_NEAR_TIE) != 0
    np.testing.assert_array_equal(dg[~near], o["tokens"][~near])


def test_unfused_pipeline_equals_fused():
    """fan-out -> reweight (with the target's last position as the guess rows)
    -> verify without a cache -> cache build -> lookup gives what the fused
    verify + cache call gives."""
    w = W["zipf_b512_k4_v128256_bf16_miss"].replace(B=24)
    case = Case(w)
    fused = case.run_gpu()
    dev = "cuda"
    K, V, B = w.K, w.V, w.B
    F = ssd.ssd_fanout_plan(to_dev(case.g["alpha"]), K, w.budget)
    tgt = case.d_target
    guess = tgt[:, K, :]
    rw = ssd.ssd_saguaro_reweight(case.d_draft, w.T, F, w.C, w.budget, guess=guess,
                                  guess_row_stride=(K + 1) * V)
    ver = ssd.ssd_verify(tgt, case.d_draft, to_dev(case.tokens), to_dev(case.g["uniforms"]), w.T, F=F,
                         C_coef=w.C, budget=w.budget, cache=False)
    offs, toks = ssd.ssd_cache_build(F, rw.topf_tokens, w.budget)
    hit, slot, nxt = ssd.ssd_cache_lookup(offs, toks, ver.n_accepted, ver.bonus, V,
                                          fallback_seed=w.fallback_seed)
    torch.cuda.synchronize()
    orc = case.run_oracle()
    np.testing.assert_array_equal(offs.cpu().numpy(), orc["offsets"])
    np.testing.assert_array_equal(toks.cpu().numpy(), orc["cache_tokens"])
    np.testing.assert_array_equal(offs.cpu().numpy(), fused["cache_offsets"])
    np.testing.assert_array_equal(toks.cpu().numpy(), fused["cache_tokens"])
    for a, bname in ((ver.n_accepted, "n_accepted"), (ver.bonus, "bonus"), (hit, "hit"), (slot, "slot"),
                     (nxt, "next_tokens")):
        np.testing.assert_array_equal(a.cpu().numpy(), fused[bname], err_msg=bname)
    assert dev == "cuda"


def test_cache_lookup_against_oracle():
    rng = np.random.default_rng(13)
    B, K, budget, V = 300, 5, 40, 50000
    offsets = np.zeros((B, K + 2), np.int32)
    tokens = np.zeros((B, budget), np.int32)
    for b in range(B):
        cuts = np.sort(rng.integers(0, budget + 1, K))
        offsets[b] = np.concatenate([[0], cuts, [budget]])
        tokens[b] = rng.choice(V, budget, replace=False)
    k = rng.integers(0, K + 1, B).astype(np.int32)
    bonus = np.where(rng.random(B) < 0.5, tokens[np.arange(B), rng.integers(0, budget, B)],
                     rng.integers(0, V, B)).astype(np.int32)
    payload = rng.integers(0, V, (B, budget, K)).astype(np.int32)
    for pl in (None, payload):
        hit, slot, nxt = ssd.ssd_cache_lookup(to_dev(offsets), to_dev(tokens), to_dev(k), to_dev(bonus), V,
                                              payload=None if pl is None else to_dev(pl), fallback_seed=77)
        o = oracle.cache_lookup(offsets, tokens, k, bonus, V, payload=pl, fallback_seed=77)
        np.testing.assert_array_equal(hit.cpu().numpy(), o["hit"])
        np.testing.assert_array_equal(slot.cpu().numpy(), o["slot"])
        np.testing.assert_array_equal(nxt.cpu().numpy(), o["next_tokens"])


def test_repeat_calls_reuse_workspace():
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=8)
    case = Case(w)
    ws = ssd.Workspace(w.B, w.K, torch.device("cuda"), w.V, ssd.DTYPE_BF16)
    outs = []
    for _ in range(3):
        r = ssd.ssd_verify(to_dev(case.g["target"]), to_dev(case.g["draft"]), to_dev(case.tokens),
                           to_dev(case.g["uniforms"]), w.T, F=to_dev(case.F), C_coef=w.C, budget=w.budget,
                           cache=True, workspace=ws)
        outs.append((r.n_accepted.cpu().numpy(), r.bonus.cpu().numpy(), r.hit.cpu().numpy()))
    for o in outs[1:]:
        for x, y in zip(o, outs[0]):
            np.testing.assert_array_equal(x, y)
    assert ws.device_error() == 0


def test_host_argument_errors_do_not_launch():
    dev = torch.device("cuda")
    t = torch.zeros((2, 3, 64), dtype=torch.bfloat16, device=dev)
    d = torch.zeros((2, 2, 64), dtype=torch.bfloat16, device=dev)
    tok = torch.zeros((2, 2), dtype=torch.int32, device=dev)
    u = torch.zeros((2, 3), dtype=torch.float32, device=dev)
    F = torch.zeros((2, 3), dtype=torch.int32, device=dev)
    for kw in (dict(T=-1.0), dict(T=float("inf")), dict(T=1.0, F=F, C_coef=0.0, budget=0),
               dict(T=1.0, F=F, C_coef=0.5, budget=65)):
        with pytest.raises(ssd.SsdError):
            ssd.ssd_verify(t, d, tok, u, **kw)
    big = torch.zeros(2 * 3 * 64 + 8, dtype=torch.bfloat16, device=dev)
    t_mis = big[1:1 + 2 * 3 * 64].view(2, 3, 64)          # 2-byte offset: not 16-byte aligned
    with pytest.raises(ssd.SsdError, match="misaligned"):
        ssd.ssd_verify(t_mis, d, tok, u, 1.0)


def test_in_kernel_plan_equals_given_plan():
    """alpha given instead of F: the fused kernel plans the fan-out itself,
    bit-identically to ssd_fanout_plan and the oracle."""
    for mode in (0, 1):
        w = W["zipf_b64_k6_v128256_bf16"].replace(B=6, fanout_mode=mode)
        case = Case(w)
        given = case.run_gpu()
        r = ssd.ssd_verify(case.d_target, case.d_draft, to_dev(case.tokens), to_dev(case.g["uniforms"]), w.T,
                           alpha=to_dev(case.g["alpha"]), fanout_mode=mode, C_coef=w.C, budget=w.budget,
                           cache=True, fallback_seed=w.fallback_seed)
        torch.cuda.synchronize()
        for key in ("n_accepted", "bonus", "out_tokens", "cache_offsets", "cache_tokens", "hit", "slot",
                    "next_tokens", "status"):
            np.testing.assert_array_equal(getattr(r, key).cpu().numpy(), given[key], err_msg=key)
        np.testing.assert_array_equal(r.accept_prob.cpu().numpy(), given["accept_prob"])
