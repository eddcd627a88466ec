"""The fan-out variants, the per-row alpha update, the batch-size fallback
policy and the payload pre-speculation, through the C ABI against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_ssd_b200 import binding as ssd
from speculative_decoding_verify_ssd_b200 import synth

from ssd_testlib import Case, check_row_properties, compare, to_dev

W = synth.WORKLOADS


@pytest.mark.gpu
def test_power_plan_bit_exact():
    rng = np.random.default_rng(7)
    for K in (1, 4, 6, 8, 32):
        for budget in (0, 1, 7, 64, 128, 512):
            alpha = rng.random(300).astype(np.float32)
            alpha[:4] = [0.0, 1.0, 0.5, 0.25]
            for q in range(1, 9):
                Fg = ssd.ssd_fanout_plan_power(to_dev(alpha), K, budget, q).cpu().numpy()
                Fo = oracle.fanout_plan_power_batch(alpha, K, budget, q)
                np.testing.assert_array_equal(Fg, Fo, err_msg=f"K={K} budget={budget} q={q}")


@pytest.mark.gpu
@pytest.mark.parametrize("q", [2, 4, 6])
def test_verify_with_power_plan(q):
    w = W["zipf_b256_k8_v151936_bf16_sweep"].replace(B=8)
    case = Case(w)
    case.F = oracle.fanout_plan_power_batch(case.g["alpha"], w.K, w.budget, q)
    from ssd_testlib import draft_tokens_for
    case.tokens = draft_tokens_for(w, case.g, case.F)
    gpu = case.run_gpu()
    orc = case.run_oracle()
    compare(case, gpu, orc)
    check_row_properties(case, gpu)


@pytest.mark.gpu
def test_alpha_update_bit_exact():
    rng = np.random.default_rng(9)
    B, K = 1000, 6
    alpha = rng.random(B).astype(np.float32)
    ap = rng.random((B, K)).astype(np.float32)
    st = np.zeros(B, np.int32)
    st[rng.choice(B, 40, replace=False)] = ssd.ROW_NONFINITE
    ap[rng.choice(B, 30, replace=False), 3] = np.nan
    for lam in (0.0, 0.1, 0.37, 1.0):
        g = ssd.ssd_alpha_update(to_dev(alpha), to_dev(ap), to_dev(st), lam).cpu().numpy()
        np.testing.assert_array_equal(g, oracle.alpha_update(alpha, ap, st, lam))


@pytest.mark.gpu
def test_alpha_update_after_verify():
    """History loop: verify, then update alpha from the step's accept_prob."""
    w = W["zipf_b16_k5_v32000_bf16"]
    case = Case(w)
    gpu = case.run_gpu()
    a2 = ssd.ssd_alpha_update(to_dev(case.g["alpha"]), to_dev(gpu["accept_prob"]), to_dev(gpu["status"]), 0.25)
    orc = case.run_oracle()
    ref = oracle.alpha_update(case.g["alpha"], orc["accept_prob"].astype(np.float32), orc["status"], 0.25)
    np.testing.assert_allclose(a2.cpu().numpy(), ref, rtol=0, atol=1e-5)


def test_fallback_bstar_matches_oracle():
    """Host function of the library (no GPU) against the oracle's."""
    rng = np.random.default_rng(11)
    for _ in range(300):
        args = (float(rng.uniform(0.3, 0.999)), float(rng.uniform(0.2, 0.95)), int(rng.integers(1, 10)),
                float(rng.uniform(1, 30)), float(rng.uniform(0, 20)), float(rng.uniform(0, 0.5)),
                float(rng.uniform(0.5, 2.0)), int(rng.integers(1, 600)))
        bs, ch = ssd.ssd_fallback_bstar(*args)
        bo, cho = oracle.fallback_bstar(*args)
        assert bs == bo
        np.testing.assert_array_equal(ch, cho)
    with pytest.raises(ssd.SsdError):
        ssd.ssd_fallback_bstar(1.5, 0.5, 4, 1.0, 1.0, 0.0, 1.0, 8)


@pytest.mark.gpu
@pytest.mark.parametrize("T,C", [(0.8, 0.5), (1.0, 1.0), (0.0, 0.5)])
def test_prespeculate_matches_oracle(T, C):
    """Every key's K payload tokens equal the oracle's draft draws on the same
    rows (or lie in the oracle's near-tie window of that draw)."""
    B, n_keys, K, V, nb = 3, 5, 4, 3001, 6
    w = W["zipf_b16_k5_v32000_bf16"].replace(B=B * n_keys, K=K, V=V, T=T, budget=nb, C=C)
    g = synth.generate(w)
    logits = g["draft"].reshape(B, n_keys, K, V)
    F = oracle.fanout_plan_batch(np.full(B * n_keys, 0.6, np.float32), K, nb)
    F[0] = 0
    F[0, K] = nb
    u = synth.uniforms(w.seed + 9, B * n_keys, K, 3)
    pay, st = ssd.ssd_prespeculate(to_dev(logits), T, to_dev(F), C, nb, to_dev(u.reshape(B, n_keys, K)))
    torch.cuda.synchronize()
    o = oracle.reweight(g["draft"], T, F, C, nb, u_draft=u)
    got = pay.cpu().numpy().reshape(B * n_keys, K)
    assert np.all((o["tok_lo"] <= got) & (got <= o["tok_hi"]))
    near = (o["status"] & oracle.ROW_NEAR_TIE) != 0
    np.testing.assert_array_equal(got[~near], o["tokens"][~near])
    np.testing.assert_array_equal(st.cpu().numpy() & ssd.ROW_INVALID, o["status"] & oracle.ROW_INVALID)
