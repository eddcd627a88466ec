"""Shared helpers for the parity tests: build one seeded case, run the oracle
and the CUDA library on identical inputs, compare element by element.

Bars (from the method's own decision structure):
* integer outputs (accepted length, bonus, out_tokens, cache keys, hit, slot,
  next tokens, fan-out plans, top-F sets, invalid-row bits) bit-exact, except
  at rows the oracle flags as near-ties (a decision margin below 1e-5, where
  the fp32 GPU and the fp64 oracle may legitimately decide differently);
* probabilities (accept_prob, residual_mass, Z) within 1e-5 absolute;
  log-normalisers within 1e-6 relative.
"""
import numpy as np
import torch

import oracle
from speculative_decoding_verify_ssd_b200 import binding as ssd
from speculative_decoding_verify_ssd_b200 import synth

PROB_ATOL = 1e-5
LSE_RTOL = 1e-6


def to_dev(x: np.ndarray, device="cuda"):
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)


def draft_tokens_for(w, g, F, rows=None):
    """Draft tokens d_j ~ q'_j drawn by the oracle's sampler with the
    workload's u_draft stream; rows outside `rows` get tokens drawn uniformly
    from the generator's own stream (still valid inputs)."""
    B, K = g["u_draft"].shape
    toks = np.floor(synth.uniforms(w.seed + 1000, B, K, 1) * w.V).astype(np.int32)
    r = oracle.reweight(g["draft"], w.T, F, w.C, w.budget, u_draft=g["u_draft"], rows=rows)
    if rows is None:
        toks[:] = r["tokens"]
    else:
        toks[np.asarray(rows)] = r["tokens"]
    return toks


def _f32_row(x):
    return synth.to_f32(x).astype(np.float64)


def segments_ok(case, offsets, tokens, rows=None):
    """Property check at any size: every segment k of every checked row is
    the top-F_k of its source row by (logit desc, id asc).  Source rows are
    converted one at a time, so full-size batches fit in host memory."""
    g, K, F = case.g, case.K, case.F
    dn = case.draft_next
    rows = range(F.shape[0]) if rows is None else rows
    for b in rows:
        for k in range(K + 1):
            src = _f32_row(g["draft"][b, k]) if k < K else _f32_row(dn[b] if dn is not None else g["target"][b, K])
            seg = tokens[b, offsets[b, k]:offsets[b, k + 1]]
            f = F[b, k]
            if len(seg) != f:
                return False
            if f == 0:
                continue
            vals = src[seg]
            keys = list(zip(-vals, seg))
            if keys != sorted(keys):
                return False
            last_v, last_i = vals[-1], seg[-1]
            mask = np.ones(src.size, bool)
            mask[seg] = False
            rest = np.nonzero(mask)[0]
            better = (src[rest] > last_v) | ((src[rest] == last_v) & (rest < last_i))
            if better.any():
                return False
    return True


class Case:
    def __init__(self, w, with_draft_next=False, check_rows=None, mode=None, tokens=None):
        self.w = w
        self.g = synth.generate(w, with_draft_next=with_draft_next)
        self.K = w.K
        self.mode = w.fanout_mode if mode is None else mode
        self.F = oracle.fanout_plan_batch(self.g["alpha"], w.K, w.budget, self.mode)
        self.rows = check_rows
        self.tokens = tokens if tokens is not None else draft_tokens_for(w, self.g, self.F, check_rows)
        self.draft_next = self.g.get("draft_next")
        self.payload = None
        self.with_F = True

    def run_gpu(self, cache=True, with_F=True, payload=None, early_exit=False):
        w, g = self.w, self.g
        self.payload = payload
        self.with_F = with_F
        self.d_target = to_dev(g["target"])
        self.d_draft = to_dev(g["draft"])
        dn = to_dev(self.draft_next) if self.draft_next is not None else None
        r = ssd.ssd_verify(self.d_target, self.d_draft, to_dev(self.tokens), to_dev(g["uniforms"]), w.T,
                           F=to_dev(self.F) if with_F else None, C_coef=w.C, budget=w.budget,
                           draft_next=dn, cache=cache and with_F,
                           payload=to_dev(payload) if payload is not None else None,
                           fallback_seed=w.fallback_seed, early_exit=early_exit)
        torch.cuda.synchronize()
        return {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in r.__dict__.items()}

    def run_oracle(self, with_F=True, payload=None, want_phit=False, early_exit=False):
        w, g = self.w, self.g
        self.with_F = with_F
        self.payload = payload
        return oracle.verify(g["target"], g["draft"], self.tokens, g["uniforms"], w.T,
                             F=self.F if with_F else None, C_coef=w.C, budget=w.budget,
                             draft_next=self.draft_next, payload=payload, fallback_seed=w.fallback_seed,
                             rows=self.rows, want_phit=want_phit, early_exit=early_exit)


NEAR_TIE = 1e-5


def _flip_uniform(a, accepted):
    """A uniform on the other side of a: the largest float32 below a when the
    oracle accepted (u < a), the smallest float32 >= a when it rejected.  None
    when no uniform in [0, 1) can take the other side."""
    u = np.float32(a)
    if accepted:   # want u' >= a (reject)
        if float(u) < a:
            u = np.nextafter(u, np.float32(1))
        return None if float(u) >= 1.0 else u
    if float(u) >= a:  # want u' < a (accept)
        u = np.nextafter(u, np.float32(0))
    return None if float(u) < 0.0 or float(u) >= a else u


def _alternative(case, orc, i, b):
    """The oracle's outcome for row b with its closest accept decision taken
    the other way (the only decision an fp32 evaluation may take otherwise
    when |u_j - a_j| < 1e-5)."""
    K = case.K
    k_o = int(orc["n_accepted"][i])
    u = case.g["uniforms"][b].astype(np.float64)
    a = orc["accept_prob"][i]
    jmax = min(k_o, K - 1)
    j = int(np.argmin(np.abs(u[:jmax + 1] - a[:jmax + 1])))
    nu = _flip_uniform(float(a[j]), accepted=j < k_o)
    if nu is None:
        return None
    uni = case.g["uniforms"].copy()
    uni[b, j] = nu
    w = case.w
    return oracle.verify(case.g["target"], case.g["draft"], case.tokens, uni, w.T,
                         F=case.F if case.with_F else None, C_coef=w.C, budget=w.budget,
                         draft_next=case.draft_next, payload=case.payload, fallback_seed=w.fallback_seed,
                         rows=np.array([b], np.int32))


def _outcome_ok(gk, gb, grm, o, i):
    """The GPU's (k*, bonus, R) against one exact outcome o (row i of it):
    k* equal; the bonus equal, or inside o's near-tie window when o's bonus
    margin is below 1e-5; R within the probability tolerance."""
    if gk != o["n_accepted"][i]:
        return False
    if o["bonus_margin"][i] >= NEAR_TIE:
        if gb != o["bonus"][i]:
            return False
    elif not (o["bonus_lo"][i] <= gb <= o["bonus_hi"][i]):
        return False
    return abs(float(grm) - o["residual_mass"][i]) < PROB_ATOL


def compare(case, gpu, orc, with_cache=True, early_exit=False):
    """Element-by-element comparison; returns the number of near-tie rows.

    Rows whose every decision margin is at least 1e-5 are bit-exact.  A row
    with a bonus margin below 1e-5 has several correct bonus tokens: the GPU's
    must lie in the oracle's near-tie window.  A row with an accept margin
    below 1e-5 has two correct accepted lengths: the GPU's outcome must equal
    the oracle's or the oracle's outcome with that one decision flipped.  The
    cache keys are checked bit for bit on every row, and hit / slot / next
    tokens must be what a brute-force lookup of the GPU's own (k*, bonus) in
    the oracle's cache gives.  early_exit: the oracle ran the early-exit
    schedule (no a_j past k*); a_j is compared where both report one, and a
    row with the oracle's own k* must report none past it."""
    rows = np.arange(case.w.B) if case.rows is None else np.asarray(case.rows)
    K = case.K
    st_o = orc["status"]
    st_g = gpu["status"][rows]
    np.testing.assert_array_equal(st_g & ssd.ROW_INVALID, st_o & oracle.ROW_INVALID,
                                  err_msg="invalid-row bits differ")
    invalid = (st_o & oracle.ROW_INVALID) != 0
    ap_g, ap_o = gpu["accept_prob"][rows], orc["accept_prob"]
    assert np.all(np.isnan(ap_g[invalid])), "invalid rows must carry NaN accept_prob"
    v = ~invalid
    if v.any() and not early_exit:
        err = np.max(np.abs(ap_g[v].astype(np.float64) - ap_o[v]))
        assert err < PROB_ATOL, f"accept_prob max err {err}"
    if v.any() and early_exit:
        both = v[:, None] & np.isfinite(ap_o) & np.isfinite(ap_g)
        if both.any():
            err = np.max(np.abs(ap_g[both].astype(np.float64) - ap_o[both]))
            assert err < PROB_ATOL, f"accept_prob max err {err}"
        same_k = v & (gpu["n_accepted"][rows] == orc["n_accepted"])
        np.testing.assert_array_equal(np.isnan(ap_g[same_k]), np.isnan(ap_o[same_k]),
                                      err_msg="early exit: a_j reported past k*, or missing before it")
    np.testing.assert_array_equal(gpu["n_accepted"][rows][invalid], -1)
    np.testing.assert_array_equal(gpu["bonus"][rows][invalid], -1)
    near = 0
    for i in np.nonzero(v)[0]:
        b = int(rows[i])
        gk, gb, grm = int(gpu["n_accepted"][b]), int(gpu["bonus"][b]), gpu["residual_mass"][b]
        amarg, bmarg = orc["accept_margin"][i], orc["bonus_margin"][i]
        near += int(amarg < NEAR_TIE or bmarg < NEAR_TIE)
        ok = _outcome_ok(gk, gb, grm, orc, i)
        if not ok and amarg < NEAR_TIE:
            alt = _alternative(case, orc, i, b)
            ok = alt is not None and _outcome_ok(gk, gb, grm, alt, 0)
        assert ok, (f"row {b}: gpu (k*={gk}, bonus={gb}, R={grm}) vs oracle (k*={orc['n_accepted'][i]}, "
                    f"bonus={orc['bonus'][i]} in [{orc['bonus_lo'][i]}, {orc['bonus_hi'][i]}], "
                    f"R={orc['residual_mass'][i]}, margins {amarg:.3g}/{bmarg:.3g})")
        ot = gpu["out_tokens"][b]
        assert list(ot[:gk]) == list(case.tokens[b, :gk]) and ot[gk] == gb and np.all(ot[gk + 1:] == -1), b
    if with_cache:
        np.testing.assert_array_equal(gpu["cache_offsets"][rows], orc["offsets"], err_msg="offsets")
        np.testing.assert_array_equal(gpu["cache_tokens"][rows], orc["cache_tokens"], err_msg="cache tokens")
        k_g = np.where(invalid, -1, gpu["n_accepted"][rows]).astype(np.int32)
        look = oracle.cache_lookup(orc["offsets"], orc["cache_tokens"], k_g, gpu["bonus"][rows].astype(np.int32),
                                   case.w.V, payload=None if case.payload is None else case.payload[rows],
                                   fallback_seed=case.w.fallback_seed)
        # the lookup numbers rows by position in the subset: fallback tokens
        # of a miss depend on the batch row, so compare misses separately
        hit_g = gpu["hit"][rows]
        np.testing.assert_array_equal(hit_g, look["hit"], err_msg="hit vs lookup of the gpu's own outcome")
        np.testing.assert_array_equal(gpu["slot"][rows], look["slot"], err_msg="slot")
        hits = hit_g == 1
        np.testing.assert_array_equal(gpu["next_tokens"][rows][hits], look["next_tokens"][hits], err_msg="payload")
        miss = np.nonzero(~hits)[0]
        if miss.size:
            ctr = np.array([[rows[i], t, 2, 0] for i in miss for t in range(K)], dtype=np.uint32)
            words = synth.philox4x32_10(ctr, synth.seed_key(case.w.fallback_seed))[:, 0]
            expect = ((words.astype(np.uint64) * np.uint64(case.w.V)) >> np.uint64(32)).astype(np.int32)
            np.testing.assert_array_equal(gpu["next_tokens"][rows][miss].ravel(), expect, err_msg="fallback")
    return near


def check_row_properties(case, gpu, with_cache=True, early_exit=False):
    """Properties that hold for every row at any size.  early_exit: a_j is
    reported up to k* only."""
    K, V = case.K, case.w.V
    st = gpu["status"]
    valid = (st & ssd.ROW_INVALID) == 0
    k = gpu["n_accepted"]
    assert np.all((k[valid] >= 0) & (k[valid] <= K))
    bon = gpu["bonus"]
    assert np.all((bon[valid] >= 0) & (bon[valid] < V))
    ap = gpu["accept_prob"][valid]
    if early_exit:
        past = np.arange(K)[None, :] > k[valid][:, None]
        assert np.all(np.isnan(ap[past])), "early exit: a_j reported past k*"
        ap = ap[~past]
    assert np.all((ap >= 0) & (ap <= 1))
    for b in np.nonzero(valid)[0]:
        kk = k[b]
        row = gpu["out_tokens"][b]
        assert list(row[:kk]) == list(case.tokens[b, :kk])
        assert row[kk] == bon[b] and np.all(row[kk + 1:] == -1)
    if with_cache:
        offs, toks = gpu["cache_offsets"], gpu["cache_tokens"]
        np.testing.assert_array_equal(offs[:, 1:], np.cumsum(case.F, axis=1))
        for b in np.nonzero(valid)[0]:
            kk = k[b]
            seg = list(toks[b, offs[b, kk]:offs[b, kk + 1]])
            inseg = bon[b] in seg
            assert gpu["hit"][b] == inseg
            assert gpu["slot"][b] == (offs[b, kk] + seg.index(bon[b]) if inseg else -1)
        miss = np.nonzero(valid & (gpu["hit"] == 0))[0]
        if miss.size:
            ctr = np.array([[b, i, 2, 0] for b in miss for i in range(K)], dtype=np.uint32)
            words = synth.philox4x32_10(ctr, synth.seed_key(case.w.fallback_seed))[:, 0]
            expect = ((words.astype(np.uint64) * np.uint64(V)) >> np.uint64(32)).astype(np.int32)
            np.testing.assert_array_equal(gpu["next_tokens"][miss].ravel(), expect)
        plan_ok = (st & ssd.ROW_BAD_PLAN) == 0
        assert segments_ok(case, offs, toks, rows=np.nonzero(plan_ok & ((st & ssd.ROW_NONFINITE) == 0))[0]), \
            "a cache segment is not the top-F of its source row"
