"""Pins for the fp64 CPU oracle: each test checks the oracle against something
other than itself -- a closed form, a property the pages state, a brute force
on tiny inputs, or an independent implementation of a published definition.

Sources: "Speculative Speculative Decoding" (gist.science, Chinese and Dutch
editions), technical summary sections 2 and 3; Salmon et al., "Parallel Random
Numbers: As Easy as 1, 2, 3" (SC'11) for Philox.
"""
import itertools
import os

import numpy as np
import pytest

import oracle
from speculative_decoding_verify_ssd_b200 import synth

GRID = 1 << 24  # uniforms are m * 2^-24, m in [0, 2^24)


def softmax64(l, T):
    x = np.asarray(l, dtype=np.float64) / T
    e = np.exp(x - x.max())
    return e / e.sum()


def grid_u(m):
    return (np.asarray(m, dtype=np.float64) / GRID).astype(np.float32)


def grid_bisect(pred, n):
    """Smallest m in [0, GRID] with pred(m) False, for n monotone predicates
    (True below the breakpoint).  pred takes an int64 array of length n."""
    lo = np.zeros(n, dtype=np.int64)        # pred(lo) assumed True (or lo == breakpoint)
    hi = np.full(n, GRID, dtype=np.int64)   # GRID stands for "never False"
    first = pred(lo)
    lo_done = ~first                        # already False at m = 0
    while np.any((hi - lo > 1) & ~lo_done):
        mid = (lo + hi) // 2
        ok = pred(mid)
        lo = np.where(ok & ~lo_done, mid, lo)
        hi = np.where(~ok & ~lo_done, mid, hi)
    return np.where(lo_done, 0, hi)


def tile_rows(x, n):
    return np.ascontiguousarray(np.broadcast_to(x, (n,) + x.shape))


class Case:
    """One fixed row of small logits, replicated over a batch of probes."""

    def __init__(self, lp, lq, T, F, C, budget):
        self.lp, self.lq, self.T, self.F, self.C, self.budget = lp, lq, T, F, C, budget
        self.K = lq.shape[0]
        self.V = lq.shape[1]

    def verify(self, D, U, **kw):
        n = D.shape[0]
        F = None if self.F is None else tile_rows(self.F, n)
        return oracle.verify(tile_rows(self.lp, n), tile_rows(self.lq, n), D, U, self.T, F=F,
                             C_coef=self.C, budget=self.budget, n_threads=1, **kw)

    def sample(self, Ud):
        n = Ud.shape[0]
        return oracle.reweight(tile_rows(self.lq, n), self.T, tile_rows(self.F, n), self.C,
                               self.budget, u_draft=Ud, n_threads=1)["tokens"]

    def draft_dist(self):
        """q'_j measured from the oracle's own draft sampler (inverse CDF)."""
        K, V = self.K, self.V
        jj, vv = np.meshgrid(np.arange(K), np.arange(V - 1), indexing="ij")
        jj, vv = jj.ravel(), vv.ravel()

        def pred(m):
            Ud = np.zeros((m.size, K), np.float32)
            Ud[np.arange(m.size), jj] = grid_u(m)
            tok = self.sample(Ud)
            return tok[np.arange(m.size), jj] <= vv

        beta = grid_bisect(pred, jj.size).reshape(K, V - 1)
        edges = np.concatenate([np.zeros((K, 1), np.int64), beta, np.full((K, 1), GRID)], axis=1)
        return np.diff(edges, axis=1) / GRID

    def accept_grid(self):
        """A_j(v): fraction of the uniform grid on which token v is accepted at j."""
        K, V = self.K, self.V
        jj, vv = np.meshgrid(np.arange(K), np.arange(V), indexing="ij")
        jj, vv = jj.ravel(), vv.ravel()

        def pred(m):
            D = np.zeros((m.size, K), np.int32)
            D[np.arange(m.size), jj] = vv
            U = np.zeros((m.size, K + 1), np.float32)
            U[np.arange(m.size), jj] = grid_u(m)
            out = self.verify(D, U)
            return out["n_accepted"] > jj

        return (grid_bisect(pred, jj.size) / GRID).reshape(K, V)

    def bonus_dist(self, k, d_reject):
        """Distribution of the bonus token when k* = k (k < K: rejection at k
        with draft token d_reject; k = K: full acceptance)."""
        K, V = self.K, self.V
        vv = np.arange(V - 1)

        def pred(m):
            D = np.zeros((m.size, K), np.int32)
            U = np.zeros((m.size, K + 1), np.float32)
            if k < K:
                D[:, k] = d_reject
                U[:, k] = np.float32((GRID - 1) / GRID)
            U[:, K] = grid_u(m)
            out = self.verify(D, U)
            assert np.all(out["n_accepted"] == k)
            return out["bonus"] <= vv

        beta = grid_bisect(pred, V - 1)
        edges = np.concatenate([[0], beta, [GRID]])
        return np.diff(edges) / GRID


def make_case(K, V, T, C, seed, budget=6, alpha=0.6, draft_scale=1.0):
    rng = np.random.default_rng(seed)
    lp = rng.normal(0.0, 1.5, (K + 1, V)).astype(np.float32)
    lq = (lp[:K] + rng.normal(0.0, draft_scale, (K, V))).astype(np.float32)
    F = oracle.fanout_plan(alpha, K, budget)
    return Case(lp, lq, T, F, C, budget)


# ---------------------------------------------------------------------------
# Losslessness: the whole draft-sample + verify step reproduces p exactly.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("K", [2, 3])
@pytest.mark.parametrize("C", [1.0, 0.5, 0.2])
@pytest.mark.parametrize("T", [1.0, 0.7])
def test_lossless_by_enumeration(K, C, T):
    """[ZH] section 2 / [NL] section 2: the method is lossless.  With d_j drawn
    by the oracle's Saguaro sampler and every uniform on the 2^-24 grid
    enumerated interval by interval, the token emitted at each position j,
    given that position j is reached, is distributed exactly as p_j."""
    case = make_case(K, 8, T, C, seed=10 * K + int(C * 10))
    qp = case.draft_dist()
    A = case.accept_grid()
    for j in range(K + 1):
        p = softmax64(case.lp[j], T)
        if j < K:
            rej_tok = int(np.argmin(A[j]))
            g = case.bonus_dist(j, rej_tok) if A[j, rej_tok] < 1.0 else np.zeros(case.V)
            emitted = qp[j] * A[j] + np.sum(qp[j] * (1.0 - A[j])) * g
        else:
            emitted = case.bonus_dist(K, None)
        np.testing.assert_allclose(emitted, p, atol=2e-6, rtol=0)
        assert abs(emitted.sum() - 1.0) < 2e-6


def test_lossless_detects_plain_q_in_accept_test():
    """The enumeration is sensitive: drafting from q' but scoring against q
    (a plausible slip) breaks losslessness for C < 1, so the check above would
    catch it.  Here the mistake is planted in the test's own composition."""
    case = make_case(2, 8, 1.0, 0.3, seed=7)
    qp = case.draft_dist()
    q = softmax64(case.lq[0], 1.0)
    p = softmax64(case.lp[0], 1.0)
    a_wrong = np.minimum(1.0, p / q)
    r = np.maximum(0.0, p - q)
    emitted = qp[0] * a_wrong + np.sum(qp[0] * (1 - a_wrong)) * r / r.sum()
    assert np.max(np.abs(emitted - p)) > 1e-3


# ---------------------------------------------------------------------------
# Saguaro sampling: the structure the pages describe, measured from the sampler.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("C", [1.0, 0.6, 0.25])
def test_saguaro_downweights_topF_by_C(C):
    """[ZH] section 2 challenge 2 / [NL] section 3B: the draft's top-F tokens
    are down-weighted by C and the distribution renormalised.  Measured q'
    must equal q scaled by C/Z on the top-F set and by 1/Z elsewhere, with S
    the top-F of the raw logits (brute-force sort)."""
    K, V = 2, 12
    case = make_case(K, V, 0.8, C, seed=3, budget=7, alpha=0.5)
    qp = case.draft_dist()
    for j in range(K):
        q = softmax64(case.lq[j], 0.8)
        S = sorted(range(V), key=lambda v: (-float(case.lq[j, v]), v))[: case.F[j]]
        w = np.ones(V)
        w[S] = C
        expect = w * q / np.sum(w * q)
        np.testing.assert_allclose(qp[j], expect, atol=2e-6, rtol=0)


def test_saguaro_C1_is_identity_and_outputs_match_unweighted():
    case = make_case(3, 16, 1.0, 1.0, seed=5, budget=9)
    rng = np.random.default_rng(1)
    n = 64
    D = rng.integers(0, 16, (n, 3)).astype(np.int32)
    U = synth.uniforms(11, n, 4, 0)
    with_plan = case.verify(D, U)
    plain = Case(case.lp, case.lq, 1.0, None, 1.0, 0).verify(D, U)
    assert np.all(with_plan["Z"] == 1.0)
    for key in ("n_accepted", "bonus", "out_tokens"):
        np.testing.assert_array_equal(with_plan[key], plain[key])
    np.testing.assert_array_equal(with_plan["accept_prob"], plain["accept_prob"])


def test_saguaro_raises_bonus_mass_on_cached_set():
    """[ZH] section 2 challenge 2: lowering C moves residual mass onto the
    cached top-F tokens, so the bonus lands in S more often (at rejection)."""
    K, V = 2, 10
    masses = []
    for C in (1.0, 0.7, 0.4, 0.1):
        case = make_case(K, V, 1.0, C, seed=21, budget=6, alpha=0.5)
        A = case.accept_grid()
        tok = int(np.argmin(A[0]))
        g = case.bonus_dist(0, tok)
        S = sorted(range(V), key=lambda v: (-float(case.lq[0, v]), v))[: case.F[0]]
        masses.append(g[S].sum())
    assert all(masses[i] <= masses[i + 1] + 1e-7 for i in range(len(masses) - 1)), masses
    assert masses[-1] > masses[0] + 0.05


# ---------------------------------------------------------------------------
# Identities.
# ---------------------------------------------------------------------------
def test_q_equals_p_accepts_everything():
    rng = np.random.default_rng(2)
    K, V, n = 4, 50, 200
    lp = rng.normal(0, 2, (K + 1, V)).astype(np.float32)
    case = Case(lp, lp[:K].copy(), 1.0, oracle.fanout_plan(0.7, K, 10), 1.0, 10)
    D = rng.integers(0, V, (n, K)).astype(np.int32)
    U = synth.uniforms(3, n, K + 1, 0)
    out = case.verify(D, U)
    assert np.all(out["n_accepted"] == K)
    assert np.all(out["accept_prob"] == 1.0)


def test_residual_mass_identity():
    """R = sum max(0, p - q') = 1 - sum min(p, q'), with q' measured from the
    sampler and p from the definition."""
    case = make_case(2, 8, 1.0, 0.4, seed=9)
    qp = case.draft_dist()
    A = case.accept_grid()
    tok = int(np.argmin(A[1]))
    D = np.zeros((1, 2), np.int32)
    D[0, 1] = tok
    U = np.zeros((1, 3), np.float32)
    U[0, 1] = np.float32((GRID - 1) / GRID)
    out = case.verify(D, U)
    assert out["n_accepted"][0] == 1
    p = softmax64(case.lp[1], 1.0)
    assert abs(out["residual_mass"][0] - (1.0 - np.minimum(p, qp[1]).sum())) < 2e-6


def test_accept_prob_matches_grid_and_ratio_bound():
    case = make_case(3, 8, 1.0, 0.5, seed=4)
    A = case.accept_grid()
    n = 8
    D = np.tile(np.arange(8, dtype=np.int32)[:, None], (1, 3))
    out = case.verify(D, np.zeros((n, 4), np.float32))
    a = out["accept_prob"]  # [8 tokens, 3 positions]
    np.testing.assert_allclose(a.T, A, atol=1.0 / GRID + 1e-12)
    assert np.all((a >= 0) & (a <= 1))


# ---------------------------------------------------------------------------
# Temperature 0: textbook greedy verification.
# ---------------------------------------------------------------------------
def test_greedy_is_textbook():
    rng = np.random.default_rng(8)
    K, V, n = 5, 40, 300
    lp = np.round(rng.normal(0, 1, (n, K + 1, V)) * 4) / 4  # ties on purpose
    lp = lp.astype(np.float32)
    lq = (lp[:, :K] + rng.normal(0, 0.5, (n, K, V))).astype(np.float32)
    am = np.argmax(lp, axis=2)  # numpy: first index of the maximum
    D = np.where(rng.random((n, K)) < 0.8, am[:, :K], rng.integers(0, V, (n, K))).astype(np.int32)
    U = synth.uniforms(5, n, K + 1, 0)
    F = np.tile(oracle.fanout_plan(0.7, K, 12), (n, 1))
    out = oracle.verify(lp, lq, D, U, 0.0, F=F, C_coef=0.5, budget=12, n_threads=2)
    for b in range(n):
        mism = [j for j in range(K) if D[b, j] != am[b, j]]
        k = mism[0] if mism else K
        assert out["n_accepted"][b] == k
        assert out["bonus"][b] == am[b, k]
        assert list(out["out_tokens"][b]) == list(D[b, :k]) + [am[b, k]] + [-1] * (K - k)
        assert np.all(out["Z"][b] == 1.0)


# ---------------------------------------------------------------------------
# Top-F and the cache.
# ---------------------------------------------------------------------------
def brute_topf(x, F):
    return [v for v in sorted(range(len(x)), key=lambda v: (-float(x[v]), v))][:F]


@pytest.mark.parametrize("seed", range(6))
def test_topf_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    V = int(rng.integers(1, 300))
    x = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.round(rng.normal(0, 1, V) * 3) / 3))
    x = x.astype(np.float64)
    x[rng.random(V) < 0.1] = -np.inf
    z = rng.random(V) < 0.1
    x[z] = np.where(rng.random(z.sum()) < 0.5, -0.0, 0.0)
    for F in sorted({0, 1, min(5, V), V // 2, V}):
        assert list(oracle.topf(x, F)) == brute_topf(x, F)


def test_cache_segments_are_topf_sets():
    rng = np.random.default_rng(12)
    B, K, V, budget = 6, 3, 64, 11
    lp = rng.normal(0, 1, (B, K + 1, V)).astype(np.float32)
    lq = (lp[:, :K] + rng.normal(0, 0.7, (B, K, V))).astype(np.float32)
    ln = rng.normal(0, 1, (B, V)).astype(np.float32)
    F = np.stack([oracle.fanout_plan(a, K, budget) for a in (0.2, 0.5, 0.9, 0.6, 0.7, 0.99)])
    D = rng.integers(0, V, (B, K)).astype(np.int32)
    U = synth.uniforms(1, B, K + 1, 0)
    for nxt in (None, ln):
        out = oracle.verify(lp, lq, D, U, 1.0, F=F, C_coef=0.5, budget=budget, draft_next=nxt)
        for b in range(B):
            off = out["offsets"][b]
            assert list(off) == [0] + list(np.cumsum(F[b]))
            for k in range(K + 1):
                src = lq[b, k] if k < K else (ln[b] if nxt is not None else lp[b, K])
                seg = out["cache_tokens"][b, off[k]:off[k + 1]]
                assert list(seg) == brute_topf(src, F[b, k])
            k = out["n_accepted"][b]
            seg = list(out["cache_tokens"][b, off[k]:off[k + 1]])
            bon = out["bonus"][b]
            assert out["hit"][b] == (bon in seg)
            assert out["slot"][b] == (off[k] + seg.index(bon) if bon in seg else -1)


def test_lookup_brute_force():
    rng = np.random.default_rng(13)
    B, K, budget, V = 50, 4, 20, 1000
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
    out = oracle.cache_lookup(offsets, tokens, k, bonus, V, payload=payload, fallback_seed=77)
    for b in range(B):
        seg = list(tokens[b, offsets[b, k[b]]:offsets[b, k[b] + 1]])
        if bonus[b] in seg:
            s = offsets[b, k[b]] + seg.index(bonus[b])
            assert out["hit"][b] == 1 and out["slot"][b] == s
            assert list(out["next_tokens"][b]) == list(payload[b, s])
        else:
            assert out["hit"][b] == 0 and out["slot"][b] == -1
            words = synth.philox4x32_10(np.array([[b, i, 2, 0] for i in range(K)], np.uint32),
                                        synth.seed_key(77))[:, 0]
            expect = (words.astype(np.uint64) * np.uint64(V)) >> np.uint64(32)
            assert list(out["next_tokens"][b]) == list(expect.astype(np.int32))


# ---------------------------------------------------------------------------
# Fan-out plan.
# ---------------------------------------------------------------------------
def test_fanout_worked_examples():
    """Hand-derived from the geometric reading (not printed on the pages):
    alpha = 0.7 quotas rounded by largest remainder."""
    assert list(oracle.fanout_plan(0.7, 6, 64)) == [19, 13, 9, 7, 5, 3, 8]
    assert list(oracle.fanout_plan(0.7, 4, 8)) == [2, 2, 1, 1, 2]
    assert list(oracle.fanout_plan(0.7, 8, 128)) == [38, 27, 19, 13, 9, 7, 5, 3, 7]


def test_fanout_extremes_and_uniform():
    assert list(oracle.fanout_plan(0.0, 5, 30)) == [30, 0, 0, 0, 0, 0]
    assert list(oracle.fanout_plan(1.0, 5, 30)) == [0, 0, 0, 0, 0, 30]
    assert list(oracle.fanout_plan(0.3, 6, 64, mode=1)) == [10, 9, 9, 9, 9, 9, 9]
    assert list(oracle.fanout_plan(0.3, 3, 0)) == [0, 0, 0, 0]


def quotas(alpha, K, budget):
    P = [alpha ** k * (1 - alpha) for k in range(K)] + [alpha ** K]
    return [budget * p for p in P]


def test_fanout_sum_rank_and_quota_bounds():
    rng = np.random.default_rng(0)
    for _ in range(400):
        K = int(rng.integers(1, 12))
        budget = int(rng.integers(0, 300))
        alpha = float(np.float32(rng.random()))
        F = oracle.fanout_plan(alpha, K, budget)
        Q = quotas(alpha, K, budget)
        assert F.sum() == budget and np.all(F >= 0)
        for a, b in itertools.combinations(range(K + 1), 2):
            if Q[a] > Q[b] + 1e-9:
                assert F[a] >= F[b]
        assert all(abs(F[k] - Q[k]) < 1.0 + 1e-9 for k in range(K + 1))
        if 0 < alpha < 1:   # geometric: successive quota ratio alpha for k+1 < K
            for k in range(K - 1):
                assert abs(Q[k + 1] / Q[k] - alpha) < 1e-12 if Q[k] > 0 else True


def test_fanout_largest_remainder_is_optimal_apportionment():
    """Brute force: among all integer splits of the budget, the plan minimises
    the total absolute deviation from the quotas."""
    for alpha in (0.15, 0.5, 0.73, 0.9):
        for K in (1, 2, 3):
            for budget in range(0, 11):
                Q = np.array(quotas(alpha, K, budget))
                F = oracle.fanout_plan(alpha, K, budget)
                best = min(np.abs(np.array(c) - Q).sum()
                           for c in itertools.product(range(budget + 1), repeat=K + 1)
                           if sum(c) == budget)
                assert np.abs(F - Q).sum() <= best + 1e-9


# ---------------------------------------------------------------------------
# Philox4x32-10 and the uniform / fallback encodings.
# ---------------------------------------------------------------------------
def load_philox_kat():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "philox4x32_10_kat.txt")
    rows = []
    for line in open(path):
        line = line.split("#", 1)[0].split()
        if line:
            rows.append([int(w, 16) for w in line])
    a = np.array(rows, dtype=np.uint64).astype(np.uint32)
    return a[:, 0:4], a[:, 4:6], a[:, 6:10]


def test_philox_known_answers():
    """Both Philox4x32-10 implementations (the oracle's C and the seeded
    generator's numpy) reproduce the published known-answer vectors."""
    ctr, key, expect = load_philox_kat()
    assert ctr.shape[0] == 3
    for i in range(ctr.shape[0]):
        np.testing.assert_array_equal(oracle.philox4x32_10(ctr[i:i + 1], key[i])[0], expect[i])
        np.testing.assert_array_equal(synth.philox4x32_10(ctr[i:i + 1], key[i])[0], expect[i])


def test_philox_two_implementations_agree():
    rng = np.random.default_rng(0)
    ctr = rng.integers(0, 2 ** 32, (20000, 4), dtype=np.uint64).astype(np.uint32)
    key = rng.integers(0, 2 ** 32, (20000, 2), dtype=np.uint64).astype(np.uint32)
    np.testing.assert_array_equal(oracle.philox4x32_10(ctr, key), synth.philox4x32_10(ctr, key))


def test_philox_statistics():
    n = 1 << 18
    ctr = np.stack([np.arange(n), np.zeros(n), np.zeros(n), np.zeros(n)], axis=1).astype(np.uint32)
    out = oracle.philox4x32_10(ctr, np.array([123, 456], np.uint32))
    assert len(np.unique(out[:, 0])) > n - 20        # a bijection of the counter
    for w in range(4):
        counts = np.bincount(out[:, w] >> 24, minlength=256)
        chi2 = ((counts - n / 256) ** 2 / (n / 256)).sum()
        assert chi2 < 400                             # 255 dof; p ~ 1e-8 tail
    bits = np.unpackbits(out.view(np.uint8)).reshape(n, 128).mean(axis=0)
    assert np.all(np.abs(bits - 0.5) < 0.01)


def test_uniform_encoding_and_range():
    u = synth.uniforms(5, 100, 7, 0)
    assert u.dtype == np.float32 and np.all(u >= 0) and np.all(u < 1)
    assert np.all(u * GRID == np.floor(u * GRID))
    ctr = np.array([[3, 4, 0, 0]], np.uint32)
    x = oracle.philox4x32_10(ctr, synth.seed_key(5))[0, 0]
    assert u[3, 4] == np.float32((x >> 8) / GRID)


# ---------------------------------------------------------------------------
# Invalid inputs and the diagnostic hit probability.
# ---------------------------------------------------------------------------
def test_invalid_rows_are_flagged():
    rng = np.random.default_rng(3)
    B, K, V, budget = 5, 2, 32, 6
    lp = rng.normal(0, 1, (B, K + 1, V)).astype(np.float32)
    lq = rng.normal(0, 1, (B, K, V)).astype(np.float32)
    D = rng.integers(0, V, (B, K)).astype(np.int32)
    U = synth.uniforms(1, B, K + 1, 0)
    F = np.tile(oracle.fanout_plan(0.5, K, budget), (B, 1))
    lp[0, 1, 3] = np.nan
    lq[1, 0, :] = -np.inf
    D[2, 1] = V
    U[3, 2] = 1.0
    F[4, 0] += 1
    out = oracle.verify(lp, lq, D, U, 1.0, F=F, C_coef=0.5, budget=budget, fallback_seed=9)
    assert list(out["status"] & oracle.ROW_INVALID) == [oracle.ROW_NONFINITE, oracle.ROW_NONFINITE,
                                                         oracle.ROW_BAD_TOKEN, oracle.ROW_BAD_UNIFORM,
                                                         oracle.ROW_BAD_PLAN]
    assert np.all(out["n_accepted"] == -1) and np.all(out["bonus"] == -1)
    assert np.all(out["out_tokens"] == -1) and np.all(np.isnan(out["accept_prob"]))
    assert np.all(out["hit"] == 0) and np.all(out["slot"] == -1)
    assert np.all(out["cache_tokens"] == -1)


def test_expected_hit_probability_matches_frequency():
    rng = np.random.default_rng(17)
    K, V, n, budget = 3, 24, 40000, 9
    lp = rng.normal(0, 1.2, (K + 1, V)).astype(np.float32)
    lq = (lp[:K] + rng.normal(0, 0.8, (K, V))).astype(np.float32)
    case = Case(lp, lq, 1.0, oracle.fanout_plan(0.6, K, budget), 0.4, budget)
    D = np.tile(np.array([[3, 7, 11]], np.int32), (n, 1))
    U = synth.uniforms(23, n, K + 1, 0)
    out = case.verify(D, U, want_phit=True)
    ph = out["p_hit"][0]
    assert np.allclose(out["p_hit"], ph)
    freq = out["hit"].mean()
    assert abs(freq - ph) < 4.5 * np.sqrt(ph * (1 - ph) / n) + 1e-9


# ---------------------------------------------------------------------------
# Exact boundaries of the accept test and the bonus draw.  Logits of 0 and
# -inf make every probability dyadic, so each comparison below is exact in
# fp32 and fp64; the expected outcomes are worked out by hand.
# ---------------------------------------------------------------------------
NEG = -np.inf


def _one_row(p_logits, q_logits, d, u):
    """K = len(q_logits), V = 4, T = 1, no reweighting."""
    target = np.array([p_logits], dtype=np.float32)
    draft = np.array([q_logits], dtype=np.float32)
    return oracle.verify(target, draft, np.array([d], np.int32), np.array([u], np.float32), 1.0)


def test_accept_test_is_strict_at_a():
    # p_0 uniform (1/4 each), q_0 = (1/2, 1/2, 0, 0), d_0 = 0: a_0 = (1/4)/(1/2) = 1/2
    p = [[0, 0, 0, 0], [0, 0, 0, 0]]
    q = [[0, 0, NEG, NEG]]
    below = _one_row(p, q, [0], [0.5 - 2.0 ** -24, 0.3])
    at = _one_row(p, q, [0], [0.5, 0.3])
    assert below["accept_prob"][0, 0] == 0.5 and at["accept_prob"][0, 0] == 0.5
    assert below["n_accepted"][0] == 1          # u < a accepts
    assert at["n_accepted"][0] == 0             # u = a rejects
    # after the rejection: r = max(0, p - q) = (0, 0, 1/4, 1/4), R = 1/2
    assert at["residual_mass"][0] == 0.5


def test_bonus_inverse_cdf_is_strict_in_token_order():
    # continuing the case above (k* = 0, r = (0, 0, 1/4, 1/4), R = 1/2):
    # u_K R = 1/4 equals the CDF step at token 2, strict > moves past it
    p = [[0, 0, 0, 0], [0, 0, 0, 0]]
    q = [[0, 0, NEG, NEG]]
    at_step = _one_row(p, q, [0], [0.5, 0.5])
    assert at_step["bonus"][0] == 3
    below_step = _one_row(p, q, [0], [0.5, 0.5 - 2.0 ** -24])
    assert below_step["bonus"][0] == 2
    assert list(at_step["out_tokens"][0]) == [3, -1]


def test_bonus_uses_the_last_uniform_whatever_k_star():
    # K = 2, rejection at position 0 (p_0(d_0) = 0): r = p_0 = (1/2, 1/2, 0, 0),
    # R = 1.  The bonus takes u_K = u_2 = 1/2 -> strict > gives token 1; u_1
    # (0.1, unused) would have given token 0.
    p = [[0, 0, NEG, NEG], [0, 0, 0, 0], [0, 0, 0, 0]]
    q = [[NEG, NEG, 0, 0], [0, 0, 0, 0]]
    out = _one_row(p, q, [2, 0], [0.25, 0.1, 0.5])
    assert out["n_accepted"][0] == 0 and out["accept_prob"][0, 0] == 0.0
    assert out["residual_mass"][0] == 1.0
    assert out["bonus"][0] == 1


# ---------------------------------------------------------------------------
# The decision margins and near-tie windows (the 1e-5 decision tolerance):
# exact on the dyadic cases above, where every CDF step and every a_j is a
# power of two, and by brute force over the CDF intervals on small rows.
# ---------------------------------------------------------------------------
def test_decision_margins_exact_at_dyadic_boundaries():
    p = [[0, 0, 0, 0], [0, 0, 0, 0]]
    q = [[0, 0, NEG, NEG]]
    u3 = float(np.float32(0.3))
    # u_0 = a_0 = 1/2: rejected with margin 0.  r = (0, 0, 1/4, 1/4), R = 1/2,
    # t = u_K R with u_K = 0.3 falls inside token 2's interval [0, 1/4): its
    # distance to the step at 1/4, over R, is 1/2 - u_K.
    at = _one_row(p, q, [0], [0.5, 0.3])
    assert at["accept_margin"][0] == 0.0
    assert at["bonus_margin"][0] == (0.25 - u3 * 0.5) / 0.5
    assert at["bonus_lo"][0] == 2 and at["bonus_hi"][0] == 2
    # u_0 one grid step below a_0: accepted with margin 2^-24, then the full
    # acceptance draw from p_1 = (1/4, 1/4, 1/4, 1/4): t = 0.3 lies between the
    # steps 1/4 and 1/2, margin min(0.3 - 1/4, 1/2 - 0.3) / 1.
    below = _one_row(p, q, [0], [0.5 - 2.0 ** -24, 0.3])
    assert below["n_accepted"][0] == 1 and below["bonus"][0] == 1
    assert below["accept_margin"][0] == 2.0 ** -24
    assert below["bonus_margin"][0] == min(u3 - 0.25, 0.5 - u3)
    assert below["bonus_lo"][0] == 1 and below["bonus_hi"][0] == 1
    # t exactly on the step at 1/4 between tokens 2 and 3: margin 0, and the
    # window holds both neighbours; one grid step below it, margin 2^-25 / R.
    on = _one_row(p, q, [0], [0.5, 0.5])
    assert on["bonus"][0] == 3 and on["bonus_margin"][0] == 0.0
    assert on["bonus_lo"][0] == 2 and on["bonus_hi"][0] == 3
    near = _one_row(p, q, [0], [0.5, 0.5 - 2.0 ** -24])
    assert near["bonus"][0] == 2 and near["bonus_margin"][0] == 2.0 ** -24
    assert near["bonus_lo"][0] == 2 and near["bonus_hi"][0] == 3
    # a row that never reaches a tie: its margin is the smallest |u_j - a_j|
    # over the tests it ran (positions 0..k*), here u_0 = 1/8 vs a_0 = 1/2
    far = _one_row(p, q, [0], [0.125, 0.3])
    assert far["accept_margin"][0] == 0.375


def _window_brute(r, t, delta):
    """Tokens with mass whose CDF interval [c(v-1), c(v)) meets [t - delta, t + delta]."""
    c = np.cumsum(r)
    prev = c - r
    hit = (r > 0) & (c > t - delta) & (prev <= t + delta)
    idx = np.nonzero(hit)[0]
    return int(idx.min()), int(idx.max())


@pytest.mark.parametrize("seed", range(4))
def test_bonus_window_matches_brute_force(seed):
    """Full acceptance (q = p, C = 1) makes k* = K, so the bonus is the inverse
    CDF of p_K at u_K: the oracle's window equals the set of tokens whose CDF
    interval meets [t - 1e-5, t + 1e-5], found by brute force here, and it
    always contains the drawn token.  Quantised logits put many tiny steps
    close together, so the windows are wide."""
    rng = np.random.default_rng(seed)
    K, V, n = 2, 64, 200
    lp = np.round(rng.normal(0, 3, (K + 1, V)) * 2) / 2
    lp[K, rng.choice(V, 5, replace=False)] = -np.inf
    lp = lp.astype(np.float32)
    target = tile_rows(lp, n)
    draft = tile_rows(lp[:K], n)
    D = np.zeros((n, K), np.int32)
    U = np.zeros((n, K + 1), np.float32)
    U[:, K] = synth.uniforms(seed, n, 1, 0)[:, 0]
    out = oracle.verify(target, draft, D, U, 1.0, n_threads=1)
    assert np.all(out["n_accepted"] == K)
    pK = softmax64(lp[K], 1.0)
    for i in range(n):
        t = float(U[i, K]) * pK.sum()
        lo, hi = _window_brute(pK, t, 1e-5 * pK.sum())
        assert (out["bonus_lo"][i], out["bonus_hi"][i]) == (lo, hi), i
        assert lo <= out["bonus"][i] <= hi


def test_draft_draw_window_on_a_dyadic_case():
    """The draft draw d ~ q' shares the inverse CDF: q_0 = (1/4, 1/4, 1/2, 0)
    with C = 1; u = 1/2 sits exactly on the step after token 1."""
    with np.errstate(divide="ignore"):
        lq = np.log(np.array([[[1.0, 1.0, 2.0, 0.0]]], np.float64)).astype(np.float32)
    F = np.array([[0, 0]], np.int32)
    r = oracle.reweight(lq, 1.0, F, 1.0, 0, u_draft=np.array([[0.5]], np.float32), n_threads=1)
    assert r["tokens"][0, 0] == 2
    assert r["tok_lo"][0, 0] == 1 and r["tok_hi"][0, 0] == 2
    r = oracle.reweight(lq, 1.0, F, 1.0, 0, u_draft=np.array([[0.75]], np.float32), n_threads=1)
    assert r["tokens"][0, 0] == 2 and r["tok_lo"][0, 0] == 2 and r["tok_hi"][0, 0] == 2


# ---------------------------------------------------------------------------
# Log-normalisers: closed forms, and the library log-sum-exp on random rows.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T", [1.0, 0.7, 2.5])
def test_log_normalisers_closed_forms(T):
    """A row of V equal logits L has lse = L / T + ln V; a row with n zeros
    and the rest -inf has lse = ln n (any T).  Checked for the target rows
    (p_lse) and the draft rows (q_lse)."""
    K, V = 2, 24
    L = np.float32(1.75)
    lp = np.full((K + 1, V), L, np.float32)
    lq = np.full((K, V), NEG, np.float32)
    lq[0, :5] = 0.0
    lq[1, :16] = 0.0
    out = oracle.verify(lp[None], lq[None], np.zeros((1, K), np.int32), np.zeros((1, K + 1), np.float32), T,
                        n_threads=1)
    np.testing.assert_allclose(out["p_lse"][0], float(L) / T + np.log(V), rtol=0, atol=1e-14)
    np.testing.assert_allclose(out["q_lse"][0], [np.log(5.0), np.log(16.0)], rtol=0, atol=1e-14)


def test_log_normalisers_match_library_logsumexp():
    from scipy.special import logsumexp
    rng = np.random.default_rng(8)
    K, V, T = 3, 1000, 0.8
    lp = rng.normal(0, 4, (2, K + 1, V)).astype(np.float32)
    lq = rng.normal(0, 4, (2, K, V)).astype(np.float32)
    lq[1, 0, :900] = -np.inf
    out = oracle.verify(lp, lq, np.zeros((2, K), np.int32), np.zeros((2, K + 1), np.float32), T, n_threads=1)
    np.testing.assert_allclose(out["p_lse"], logsumexp(lp.astype(np.float64) / T, axis=2), rtol=1e-14, atol=0)
    np.testing.assert_allclose(out["q_lse"], logsumexp(lq.astype(np.float64) / T, axis=2), rtol=1e-14, atol=0)


# ---------------------------------------------------------------------------
# Fan-out variants: the power-law plan (gamma = q/8) and the per-row alpha
# update from history.
# ---------------------------------------------------------------------------
def power_quotas(alpha, K, budget, gamma):
    P = np.array([alpha ** k * (1 - alpha) for k in range(K)] + [alpha ** K])
    w = P ** gamma
    return budget * w / w.sum()


def test_power_plan_gamma_one_is_the_geometric_plan():
    rng = np.random.default_rng(2)
    for _ in range(200):
        K, budget, alpha = int(rng.integers(1, 12)), int(rng.integers(0, 300)), float(np.float32(rng.random()))
        np.testing.assert_array_equal(oracle.fanout_plan_power(alpha, K, budget, 8), oracle.fanout_plan(alpha, K, budget))


def test_power_plan_sum_rank_quota_bounds_and_ratio():
    """Sum = budget; every F_k is the floor or the ceiling of its quota
    budget * P(k)^gamma / sum P^gamma (quotas computed here with pow); F is
    non-increasing in quota rank; successive real quotas have ratio alpha^gamma."""
    rng = np.random.default_rng(3)
    for _ in range(400):
        K = int(rng.integers(1, 12))
        budget = int(rng.integers(0, 300))
        alpha = float(np.float32(rng.uniform(0.01, 0.99)))
        q = int(rng.integers(1, 8))
        F = oracle.fanout_plan_power(alpha, K, budget, q)
        Q = power_quotas(alpha, K, budget, q / 8)
        assert F.sum() == budget and np.all(F >= 0)
        assert np.all(np.abs(F - Q) < 1.0 + 1e-9), (alpha, K, budget, q, F, Q)
        for a, b in itertools.combinations(range(K + 1), 2):
            if Q[a] > Q[b] + 1e-9:
                assert F[a] >= F[b]
        for k in range(K - 1):
            if budget > 0:
                assert abs(Q[k + 1] / Q[k] - alpha ** (q / 8)) < 1e-12


def test_power_plan_flattens_as_gamma_falls():
    """A smaller gamma moves branches from the most likely outcome to the
    least likely one: as gamma grows, the most likely outcome never loses a
    branch and the least likely never gains one."""
    for alpha in (0.3, 0.6, 0.85):
        P = [alpha ** k * (1 - alpha) for k in range(6)] + [alpha ** 6]
        hi, lo = int(np.argmax(P)), int(np.argmin(P))
        plans = [oracle.fanout_plan_power(alpha, 6, 96, q) for q in range(1, 9)]
        for a, b in zip(plans, plans[1:]):
            assert b[hi] >= a[hi] and b[lo] <= a[lo]


def test_power_plan_is_the_hit_optimal_split_under_a_power_law_hit_curve():
    """The reading behind gamma: with a hit curve h(F) = 1 - (1 + F)^-beta per
    outcome, maximising sum_k P(k) h(F_k) under sum F = budget (solved
    numerically here, over real F) gives F ~ P^(1/(1+beta)) up to the +1
    offset; for a large budget the integer plan at gamma = 1/(1+beta) must be
    within a few branches of that optimum."""
    from scipy.optimize import minimize
    for alpha, beta, q in ((0.7, 1.0, 4), (0.6, 1.0 / 3.0, 6), (0.8, 3.0, 2)):
        K, budget = 6, 4096
        P = np.array([alpha ** k * (1 - alpha) for k in range(K)] + [alpha ** K])

        def neg(x):
            F = budget * np.exp(x) / np.exp(x).sum()
            return -np.sum(P * (1 - (1 + F) ** -beta))

        res = minimize(neg, np.log(P ** (q / 8)), method="Nelder-Mead",
                       options=dict(xatol=1e-10, fatol=1e-14, maxiter=20000))
        Fopt = budget * np.exp(res.x) / np.exp(res.x).sum()
        F = oracle.fanout_plan_power(alpha, K, budget, q)
        assert abs(q / 8 - 1 / (1 + beta)) < 1e-12
        assert np.max(np.abs(F - Fopt)) < 0.01 * budget, (F, Fopt)


def test_alpha_update_closed_forms():
    rng = np.random.default_rng(4)
    B, K = 16, 5
    alpha = rng.random(B).astype(np.float32)
    ap = rng.random((B, K)).astype(np.float32)
    st = np.zeros(B, np.int32)
    st[3] = oracle.ROW_BAD_TOKEN
    ap[5, 2] = np.nan
    st[6] = oracle.ROW_NEAR_TIE          # informational: still updated
    full = oracle.alpha_update(alpha, ap, st, 1.0)
    none = oracle.alpha_update(alpha, ap, st, 0.0)
    half = oracle.alpha_update(alpha, ap, st, 0.5)
    keep = np.zeros(B, bool)
    keep[[3, 5]] = True
    np.testing.assert_array_equal(full[keep], alpha[keep])
    np.testing.assert_array_equal(none, alpha)
    mean = ap.astype(np.float64).mean(axis=1)
    np.testing.assert_allclose(full[~keep], mean[~keep].astype(np.float32), rtol=0, atol=6e-8)
    np.testing.assert_allclose(half[~keep], (0.5 * alpha + 0.5 * mean)[~keep], rtol=0, atol=6e-8)


# ---------------------------------------------------------------------------
# The batch-size fallback policy b*: the crossing in closed form.
# ---------------------------------------------------------------------------
def bstar_closed_form(h, alpha, K, Lt, Lp, Lf, Ef, b_max):
    """The fast fallback wins iff m = 1 - h^b exceeds
    m* = (1-h) Lt (Ep - Ef) / (Lp (h Ep + (1-h) Ef) - Ep Lf)  (denominator > 0)."""
    Ep = sum(alpha ** i for i in range(K + 1))
    den = Lp * (h * Ep + (1 - h) * Ef) - Ep * Lf
    if den <= 0:
        return b_max + 1
    mstar = (1 - h) * Lt * (Ep - Ef) / den
    for b in range(1, b_max + 1):
        if 1 - h ** b > mstar * (1 + 1e-12) + 1e-15:
            return b
    return b_max + 1


def test_fallback_bstar_matches_the_closed_form():
    rng = np.random.default_rng(5)
    for _ in range(300):
        h = float(rng.uniform(0.5, 0.999))
        alpha = float(rng.uniform(0.3, 0.9))
        K = int(rng.integers(2, 9))
        Lt, Lp = float(rng.uniform(5, 30)), float(rng.uniform(0.5, 20))
        Lf, Ef = float(rng.uniform(0.0, 0.2)), 1.0
        bs, choice = oracle.fallback_bstar(h, alpha, K, Lt, Lp, Lf, Ef, 512)
        assert bs == bstar_closed_form(h, alpha, K, Lt, Lp, Lf, Ef, 512)
        # below b* the primary speculator, from b* on the fast one
        assert np.all(choice[:bs - 1] == 0) and np.all(choice[bs - 1:] == 1)


def test_fallback_small_batches_primary_large_batches_fast():
    """The pages' qualitative rule: a batch of one keeps the primary
    speculator when its fallback is cheap relative to a round; very large
    batches switch to the fast one."""
    bs, choice = oracle.fallback_bstar(0.95, 0.7, 6, 20.0, 2.0, 0.05, 1.0, 4096)
    assert choice[0] == 0 and 1 < bs <= 4096 and choice[-1] == 1


# ---------------------------------------------------------------------------
# Early-exit read schedule: the outcome depends on p_0..p_{k*} and p_K only.
# ---------------------------------------------------------------------------
def _ee_batch(seed, B=24, K=5, V=64, T=1.0):
    rng = np.random.default_rng(seed)
    lp = rng.normal(0.0, 1.5, (B, K + 1, V)).astype(np.float32)
    lq = (lp[:, :K] + rng.normal(0.0, 1.2, (B, K, V))).astype(np.float32)
    D = rng.integers(0, V, (B, K)).astype(np.int32)
    if T == 0.0:  # greedy: row i drafts the target argmax at its first i mod (K+1) positions
        for i in range(B):
            for j in range(i % (K + 1)):
                D[i, j] = int(np.argmax(lp[i, j]))
    U = synth.uniforms(seed + 7, B, K + 1, 0)
    F = np.tile(oracle.fanout_plan(0.6, K, 8), (B, 1))
    return lp, lq, D, U, F


def _verify(lp, lq, D, U, F, T, early_exit):
    return oracle.verify(lp, lq, D, U, T, F=F, C_coef=0.5, budget=8, fallback_seed=5, early_exit=early_exit)


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_early_exit_outcome_equals_full_read(T):
    lp, lq, D, U, F = _ee_batch(11, T=T)
    full = _verify(lp, lq, D, U, F, T, False)
    ee = _verify(lp, lq, D, U, F, T, True)
    K = D.shape[1]
    assert len(set(full["n_accepted"].tolist())) > 2  # rows stop at several positions
    for k in ("n_accepted", "bonus", "out_tokens", "offsets", "cache_tokens", "hit", "slot", "next_tokens",
              "bonus_lo", "bonus_hi"):
        np.testing.assert_array_equal(ee[k], full[k], err_msg=k)
    np.testing.assert_array_equal(ee["residual_mass"], full["residual_mass"])
    np.testing.assert_array_equal(ee["accept_margin"], full["accept_margin"])
    # a_j up to k*, nothing past it
    for i, ks in enumerate(full["n_accepted"]):
        np.testing.assert_array_equal(ee["accept_prob"][i, :min(ks + 1, K)], full["accept_prob"][i, :min(ks + 1, K)])
        assert np.all(np.isnan(ee["accept_prob"][i, ks + 1:]))
    # the only status difference allowed is q'(d) = 0 past k*
    assert np.all((ee["status"] ^ full["status"]) & ~oracle.ROW_ZERO_Q == 0)


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_early_exit_ignores_rows_it_does_not_read(T):
    """Target rows past k* (other than p_K) can hold anything, NaN included:
    the early-exit outcome equals the full read of the same batch with those
    rows replaced by finite ones; a NaN at or before k*, or in p_K, still
    makes the row invalid."""
    lp, lq, D, U, F = _ee_batch(12, T=T)
    base = _verify(lp, lq, D, U, F, T, False)
    K = D.shape[1]
    junk = lp.copy()
    unread = np.zeros(lp.shape[:2], bool)
    for i, ks in enumerate(base["n_accepted"]):
        for j in range(ks + 1, K):
            junk[i, j, :] = np.nan if (i + j) % 2 else 1e30
            unread[i, j] = True
    assert unread.sum() > 10
    ee = _verify(junk, lq, D, U, F, T, True)
    for k in ("n_accepted", "bonus", "out_tokens", "cache_tokens", "hit", "slot", "next_tokens"):
        np.testing.assert_array_equal(ee[k], base[k], err_msg=k)
    assert np.all(ee["status"] & oracle.ROW_INVALID == 0)
    full_junk = _verify(junk, lq, D, U, F, T, False)
    nan_rows = np.array([np.isnan(junk[i]).any() for i in range(junk.shape[0])])
    assert np.all(full_junk["status"][nan_rows] & oracle.ROW_NONFINITE)  # the full read sees them
    # a NaN in a row that is read: p_{k*} or p_K
    bad = lp.copy()
    i0 = int(np.argmax(base["n_accepted"] < K))
    bad[i0, base["n_accepted"][i0], 3] = np.nan
    bad[i0 + 1, K, 0] = np.nan
    ee_bad = _verify(bad, lq, D, U, F, T, True)
    assert ee_bad["status"][i0] & oracle.ROW_NONFINITE and ee_bad["n_accepted"][i0] == -1
    assert ee_bad["status"][i0 + 1] & oracle.ROW_NONFINITE and ee_bad["n_accepted"][i0 + 1] == -1


def test_early_exit_zero_q_only_up_to_k_star():
    """q'(d_j) = 0 (a draft token outside the reweighted support) is reported
    by the full read at any position, by the early-exit read only up to k*."""
    rng = np.random.default_rng(13)
    B, K, V = 1, 3, 16
    lp = rng.normal(0.0, 1.0, (B, K + 1, V)).astype(np.float32)
    lq = lp[:, :K].copy()
    D = np.array([[2, 5, 7]], np.int32)
    lq[0, 2, 7] = -np.inf  # q_2(d_2) = 0
    U = np.array([[0.999, 0.5, 0.5, 0.5]], np.float32)  # position 0 rejects unless a_0 = 1
    lp[0, 0, 2] = -8.0  # small p_0(d_0): a_0 < 0.999
    F = np.array([[1, 1, 1, 1]], np.int32)
    full = oracle.verify(lp, lq, D, U, 1.0, F=F, C_coef=1.0, budget=4, early_exit=False)
    ee = oracle.verify(lp, lq, D, U, 1.0, F=F, C_coef=1.0, budget=4, early_exit=True)
    assert full["n_accepted"][0] == 0 and ee["n_accepted"][0] == 0
    assert full["status"][0] & oracle.ROW_ZERO_Q
    assert not ee["status"][0] & oracle.ROW_ZERO_Q
