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


def segments_ok(draft_f32, lp_f32, dn_f32, F, offsets, tokens, K):
    """Property check at any size: every segment k is the top-F_k of its
    source row by (logit desc, id asc)."""
    B = F.shape[0]
    for b in range(B):
        for k in range(K + 1):
            src = draft_f32[b, k] if k < K else (dn_f32[b] if dn_f32 is not None else lp_f32[b, K])
            seg = tokens[b, offsets[b, k]:offsets[b, k + 1]]
            f = F[b, k]
            if len(seg) != f:
                return False
            if f == 0:
                continue
            vals = src[seg].astype(np.float64)
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

    def run_gpu(self, cache=True, with_F=True, payload=None):
        w, g = self.w, self.g
        self.payload = payload
        self.d_target = to_dev(g["target"])
        self.d_draft = to_dev(g["draft"])
        dn = to_dev(self.draft_next) if self.draft_next is not None else None
        r = ssd.ssd_verify(self.d_target, self.d_draft, to_dev(self.tokens), to_dev(g["uniforms"]), w.T,
                           F=to_dev(self.F) if with_F else None, C_coef=w.C, budget=w.budget,
                           draft_next=dn, cache=cache and with_F,
                           payload=to_dev(payload) if payload is not None else None,
                           fallback_seed=w.fallback_seed)
        torch.cuda.synchronize()
        return {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in r.__dict__.items()}

    def run_oracle(self, with_F=True, payload=None, want_phit=False):
        w, g = self.w, self.g
        return oracle.verify(g["target"], g["draft"], self.tokens, g["uniforms"], w.T,
                             F=self.F if with_F else None, C_coef=w.C, budget=w.budget,
                             draft_next=self.draft_next, payload=payload, fallback_seed=w.fallback_seed,
                             rows=self.rows, want_phit=want_phit)


def compare(case, gpu, orc, with_cache=True):
    """Element-by-element comparison; returns the number of near-tie rows."""
    rows = np.arange(case.w.B) if case.rows is None else np.asarray(case.rows)
    K = case.K
    st_o = orc["status"]
    st_g = gpu["status"][rows]
    np.testing.assert_array_equal(st_g & ssd.ROW_INVALID, st_o & oracle.ROW_INVALID,
                                  err_msg="invalid-row bits differ")
    invalid = (st_o & oracle.ROW_INVALID) != 0
    near = ((st_o & oracle.ROW_NEAR_TIE) != 0) & ~invalid
    ok = ~invalid & ~near
    ap_g, ap_o = gpu["accept_prob"][rows], orc["accept_prob"]
    assert np.all(np.isnan(ap_g[invalid])), "invalid rows must carry NaN accept_prob"
    v = ~invalid
    if v.any():
        err = np.max(np.abs(ap_g[v].astype(np.float64) - ap_o[v]))
        assert err < PROB_ATOL, f"accept_prob max err {err}"
    for key in ("n_accepted", "bonus", "out_tokens"):
        np.testing.assert_array_equal(gpu[key][rows][ok], orc[key][ok], err_msg=key)
    np.testing.assert_array_equal(gpu["n_accepted"][rows][invalid], -1)
    if ok.any():
        err = np.max(np.abs(gpu["residual_mass"][rows][ok].astype(np.float64) - orc["residual_mass"][ok]))
        assert err < PROB_ATOL, f"residual_mass max err {err}"
    if with_cache:
        np.testing.assert_array_equal(gpu["cache_offsets"][rows], orc["offsets"], err_msg="offsets")
        np.testing.assert_array_equal(gpu["cache_tokens"][rows], orc["cache_tokens"], err_msg="cache tokens")
        for key, okey in (("hit", "hit"), ("slot", "slot"), ("next_tokens", "next_tokens")):
            np.testing.assert_array_equal(gpu[key][rows][ok], orc[okey][ok], err_msg=key)
        np.testing.assert_array_equal(gpu["hit"][rows][invalid], 0)
        np.testing.assert_array_equal(gpu["next_tokens"][rows][invalid], orc["next_tokens"][invalid])
    return int(near.sum())


def check_row_properties(case, gpu, with_cache=True):
    """Properties that hold for every row at any size."""
    K, V = case.K, case.w.V
    st = gpu["status"]
    valid = (st & ssd.ROW_INVALID) == 0
    k = gpu["n_accepted"]
    assert np.all((k[valid] >= 0) & (k[valid] <= K))
    bon = gpu["bonus"]
    assert np.all((bon[valid] >= 0) & (bon[valid] < V))
    ap = gpu["accept_prob"][valid]
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
