"""Seeded synthetic inputs for the verify + speculation-cache step.

This module draws random numbers and shapes them into logits; it holds none of
the method's arithmetic (no softmax, no top-F, no acceptance test).  The draft
tokens are not made here: the draft side draws them from the reweighted draft
distribution, which is part of the method (see ``ssd_saguaro_reweight``).

Random streams
--------------
* Uniforms are Philox4x32-10 (Salmon et al., SC'11) words, key = seed,
  counter = (row b, position j, stream, 0), u = (x >> 8) * 2^-24 in [0, 1).
  Stream 0 = accept tests and the bonus draw, stream 1 = draft-token draws.
* Logit noise and vocabulary permutations come from numpy's Philox bit
  generator seeded with the workload seed.

Logit recipes (one vocabulary permutation per (row, position))
-------------------------------------------------------------
* ``iid``: target logits N(0, s_t^2); draft = target + N(0, s_d^2).
* ``zipf``: the token at rank r gets logit -s * ln(r) + N(0, s_t^2); the draft
  uses the same ranking with ``shuffle`` of its rank positions permuted among
  themselves and fresh N(0, s_d^2) noise, or (``draft_mode='additive'``) the
  target logits plus N(0, s_d^2).
Values are generated in float64, rounded to float32 and then, for bf16, to
bf16, each step round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

STREAM_ACCEPT = 0
STREAM_DRAFT = 1

# ---------------------------------------------------------------------------
# Philox4x32-10, vectorised over counters (Salmon, Moraes, Dror, Shaw, SC'11).
# ---------------------------------------------------------------------------
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """ctr [n,4] uint32, key [2] or [n,2] uint32 -> [n,4] uint32."""
    ctr = np.asarray(ctr, dtype=np.uint32).reshape(-1, 4)
    key = np.broadcast_to(np.asarray(key, dtype=np.uint32), (ctr.shape[0], 2))
    x0, x1, x2, x3 = (ctr[:, i].astype(np.uint64) for i in range(4))
    k0 = key[:, 0].astype(np.uint64)
    k1 = key[:, 1].astype(np.uint64)
    for _ in range(10):
        p0 = _M0 * x0
        p1 = _M1 * x2
        y0 = (p1 >> np.uint64(32)) ^ x1 ^ k0
        y1 = p1 & _MASK
        y2 = (p0 >> np.uint64(32)) ^ x3 ^ k1
        y3 = p0 & _MASK
        x0, x1, x2, x3 = y0 & _MASK, y1, y2 & _MASK, y3
        k0 = (k0 + _W0) & _MASK
        k1 = (k1 + _W1) & _MASK
    return np.stack([x0, x1, x2, x3], axis=1).astype(np.uint32)


def seed_key(seed: int):
    return np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint32)


def uniforms(seed: int, rows: int, cols: int, stream: int, row_offset: int = 0) -> np.ndarray:
    """[rows, cols] float32 uniforms in [0, 1): word 0 of Philox at (b, j, stream, 0)."""
    b, j = np.meshgrid(np.arange(rows, dtype=np.uint64) + np.uint64(row_offset),
                       np.arange(cols, dtype=np.uint64), indexing="ij")
    ctr = np.stack([b.ravel(), j.ravel(), np.full(b.size, stream, np.uint64),
                    np.zeros(b.size, np.uint64)], axis=1).astype(np.uint32)
    x = philox4x32_10(ctr, seed_key(seed))[:, 0]
    return ((x >> np.uint32(8)).astype(np.float64) * 2.0 ** -24).astype(np.float32).reshape(rows, cols)


# ---------------------------------------------------------------------------
# bf16 bit patterns.
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(x) -> np.ndarray:
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    bits = (r & np.uint64(0xFFFF)).astype(np.uint16)
    bits[np.isnan(f)] = 0x7FC0
    return bits


def bf16_bits_to_f32(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def as_dtype(x64: np.ndarray, dtype: str) -> np.ndarray:
    f = x64.astype(np.float32)
    return f32_to_bf16_bits(f) if dtype == "bf16" else f


def to_f32(x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(x) if x.dtype == np.uint16 else x.astype(np.float32)


# ---------------------------------------------------------------------------
# Workloads.
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    K: int
    V: int
    dtype: str              # "bf16" | "fp32"
    recipe: str             # "iid" | "zipf"
    zipf_s: float
    target_sigma: float
    draft_sigma: float
    draft_shuffle: float    # fraction of rank positions permuted in the draft
    draft_mode: str         # "shuffle" | "additive"
    T: float
    budget: int
    C: float
    seed: int
    alpha: float            # fan-out acceptance estimate: the mean overlap sum(min(p, q)), calibrated offline
    fallback_seed: int
    fanout_mode: int = 0    # 0 geometric, 1 uniform

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# alpha values: mean over rows and positions of sum_v min(p, q) on the
# pre-reweight distributions, rounded to 0.01, measured by
# tests/golden/calibrate_workloads.py (which calls only the oracle).
WORKLOADS = {
    "tiny_b1_k4_v1024_fp32": Workload(
        "tiny_b1_k4_v1024_fp32", B=1, K=4, V=1024, dtype="fp32", recipe="iid", zipf_s=0.0,
        target_sigma=2.0, draft_sigma=0.5, draft_shuffle=0.0, draft_mode="additive", T=1.0,
        budget=8, C=0.5, seed=0, alpha=0.80, fallback_seed=0),
    "zipf_b16_k5_v32000_bf16": Workload(
        "zipf_b16_k5_v32000_bf16", B=16, K=5, V=32000, dtype="bf16", recipe="zipf", zipf_s=1.1,
        target_sigma=0.3, draft_sigma=0.8, draft_shuffle=0.10, draft_mode="shuffle", T=0.7,
        budget=32, C=0.5, seed=1, alpha=0.56, fallback_seed=1),
    "zipf_b64_k6_v128256_bf16": Workload(
        "zipf_b64_k6_v128256_bf16", B=64, K=6, V=128256, dtype="bf16", recipe="zipf", zipf_s=1.0,
        target_sigma=0.3, draft_sigma=0.77, draft_shuffle=0.0, draft_mode="additive", T=1.0,
        budget=64, C=0.3, seed=2, alpha=0.70, fallback_seed=2),
    "zipf_b256_k8_v151936_bf16_sweep": Workload(
        "zipf_b256_k8_v151936_bf16_sweep", B=256, K=8, V=151936, dtype="bf16", recipe="zipf",
        zipf_s=1.2, target_sigma=0.3, draft_sigma=0.8, draft_shuffle=0.10, draft_mode="shuffle",
        T=1.0, budget=128, C=0.5, seed=3, alpha=0.62, fallback_seed=3),
    "zipf_b512_k4_v128256_bf16_miss": Workload(
        "zipf_b512_k4_v128256_bf16_miss", B=512, K=4, V=128256, dtype="bf16", recipe="zipf",
        zipf_s=1.0, target_sigma=0.3, draft_sigma=1.2, draft_shuffle=0.10, draft_mode="shuffle",
        T=1.0, budget=64, C=0.3, seed=4, alpha=0.49, fallback_seed=4),
}

HEADLINE = "zipf_b64_k6_v128256_bf16"

# The temperature sweep's alpha per temperature (same calibration script).
SWEEP_ALPHA = {0.0: 0.59, 0.6: 0.54, 1.0: 0.62}


ROW_CHUNK = 4  # batch rows generated per draw block (fixed: values do not depend on B)


def _zipf_block(rng, n_rows, V, base, sigma):
    """Rows of Zipf logits and the per-row ranking (token at rank r)."""
    order = rng.permuted(np.broadcast_to(np.arange(V, dtype=np.int32), (n_rows, V)), axis=1)
    vals = base[None, :] + sigma * rng.standard_normal((n_rows, V))
    out = np.empty((n_rows, V), dtype=np.float64)
    np.put_along_axis(out, order, vals, axis=1)
    return out, order


def _zipf_draft_block(rng, orders, V, base, sigma, shuffle):
    n_rows = orders.shape[0]
    m = int(round(shuffle * V))
    orders = orders.copy()
    if m > 1:
        for i in range(n_rows):
            pos = rng.choice(V, size=m, replace=False)
            orders[i, pos] = orders[i, pos[rng.permutation(m)]]
    vals = base[None, :] + sigma * rng.standard_normal((n_rows, V))
    out = np.empty((n_rows, V), dtype=np.float64)
    np.put_along_axis(out, orders, vals, axis=1)
    return out


def _block(w: Workload, rng, nb: int, with_draft_next: bool):
    K, V = w.K, w.V
    if w.recipe == "iid":
        tgt = w.target_sigma * rng.standard_normal((nb, K + 1, V))
        drf = tgt[:, :K, :] + w.draft_sigma * rng.standard_normal((nb, K, V))
        nxt = (tgt[:, K, :] + w.draft_sigma * rng.standard_normal((nb, V))) if with_draft_next else None
        return tgt, drf, nxt
    base = -w.zipf_s * np.log(np.arange(1, V + 1, dtype=np.float64))
    tgt, orders = _zipf_block(rng, nb * (K + 1), V, base, w.target_sigma)
    tgt = tgt.reshape(nb, K + 1, V)
    orders = orders.reshape(nb, K + 1, V)
    if w.draft_mode == "additive":
        drf = tgt[:, :K, :] + w.draft_sigma * rng.standard_normal((nb, K, V))
        nxt = (tgt[:, K, :] + w.draft_sigma * rng.standard_normal((nb, V))) if with_draft_next else None
    else:
        drf = _zipf_draft_block(rng, orders[:, :K, :].reshape(nb * K, V), V, base, w.draft_sigma,
                                w.draft_shuffle).reshape(nb, K, V)
        nxt = (_zipf_draft_block(rng, orders[:, K, :], V, base, w.draft_sigma, w.draft_shuffle)
               if with_draft_next else None)
    return tgt, drf, nxt


def generate(w: Workload, with_draft_next: bool = False, rows: Optional[int] = None):
    """Return dict(target [B,K+1,V], draft [B,K,V], uniforms [B,K+1],
    u_draft [B,K], alpha [B] (+ draft_next [B,V])).  Logits are float32 or
    uint16 bf16 bit patterns.  Rows are drawn in blocks of ROW_CHUNK batch
    rows, each block from its own Philox stream (seed, block), so the first
    ``rows`` rows equal those of the full batch."""
    if w.recipe not in ("iid", "zipf"):
        raise ValueError(w.recipe)
    B = w.B if rows is None else rows
    K, V = w.K, w.V
    odt = np.uint16 if w.dtype == "bf16" else np.float32
    target = np.empty((B, K + 1, V), dtype=odt)
    draft = np.empty((B, K, V), dtype=odt)
    dnext = np.empty((B, V), dtype=odt) if with_draft_next else None
    for b0 in range(0, B, ROW_CHUNK):
        nb = min(ROW_CHUNK, B - b0)
        rng = np.random.Generator(np.random.Philox(key=[w.seed, b0 // ROW_CHUNK]))
        tgt, drf, nxt = _block(w, rng, ROW_CHUNK, with_draft_next)
        target[b0:b0 + nb] = as_dtype(tgt[:nb], w.dtype)
        draft[b0:b0 + nb] = as_dtype(drf[:nb], w.dtype)
        if with_draft_next:
            dnext[b0:b0 + nb] = as_dtype(nxt[:nb], w.dtype)
    out = dict(
        target=target,
        draft=draft,
        uniforms=uniforms(w.seed, B, K + 1, STREAM_ACCEPT),
        u_draft=uniforms(w.seed, B, K, STREAM_DRAFT),
        alpha=np.full(B, w.alpha, dtype=np.float32),
    )
    if with_draft_next:
        out["draft_next"] = dnext
    return out
