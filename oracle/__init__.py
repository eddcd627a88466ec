"""ctypes wrapper of the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE.  Only tests/, the package smoke check and bench.py's
CPU-baseline leg import this module.  The product library never does.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

DTYPE_FP32 = 0
DTYPE_BF16 = 1

ROW_NONFINITE = 1
ROW_BAD_TOKEN = 2
ROW_BAD_UNIFORM = 4
ROW_ZERO_Q = 8
ROW_ZERO_RESIDUAL = 16
ROW_NEAR_TIE = 32
ROW_BAD_PLAN = 64
ROW_INVALID = ROW_NONFINITE | ROW_BAD_TOKEN | ROW_BAD_UNIFORM | ROW_BAD_PLAN

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        vp, i32p, f32p, f64p, u8p, u32p = (C.c_void_p, C.POINTER(C.c_int32), C.POINTER(C.c_float),
                                           C.POINTER(C.c_double), C.POINTER(C.c_uint8),
                                           C.POINTER(C.c_uint32))
        L.ssdo_philox_batch.argtypes = [C.c_long, u32p, u32p, u32p]
        L.ssdo_philox_batch.restype = None
        L.ssdo_fallback_token.argtypes = [C.c_uint64, C.c_int, C.c_int, C.c_int]
        L.ssdo_fallback_token.restype = C.c_int32
        L.ssdo_fanout_plan.argtypes = [C.c_double, C.c_int, C.c_int, C.c_int, i32p]
        L.ssdo_fanout_plan.restype = C.c_int
        L.ssdo_fanout_plan_power.argtypes = [C.c_double, C.c_int, C.c_int, C.c_int, i32p]
        L.ssdo_fanout_plan_power.restype = C.c_int
        L.ssdo_alpha_update.argtypes = [C.c_int, C.c_int, f32p, f32p, i32p, C.c_double, f32p]
        L.ssdo_alpha_update.restype = None
        L.ssdo_fallback_bstar.argtypes = [C.c_double, C.c_double, C.c_int, C.c_double, C.c_double, C.c_double,
                                          C.c_double, C.c_int, u8p]
        L.ssdo_fallback_bstar.restype = C.c_int
        L.ssdo_topf.argtypes = [f64p, C.c_int, C.c_int, i32p]
        L.ssdo_topf.restype = C.c_int
        L.ssdo_verify_batch.argtypes = (
            [C.c_int] * 5 + [vp, vp, vp, i32p, f32p, C.c_double, i32p, C.c_double, i32p, C.c_uint64,
                             i32p, C.c_int, C.c_int,
                             i32p, i32p, i32p, f64p, f64p, f64p, f64p, f64p, f64p, i32p, i32p,
                             u8p, i32p, i32p, i32p, f64p, f64p, f64p, i32p, i32p, C.c_int])
        L.ssdo_verify_batch.restype = C.c_int
        L.ssdo_reweight_batch.argtypes = (
            [C.c_int] * 5 + [vp, C.c_double, i32p, C.c_double, f32p, i32p, C.c_int, C.c_int,
                             i32p, i32p, f64p, f64p, f64p, i32p, f64p, i32p, i32p, i32p])
        L.ssdo_reweight_batch.restype = C.c_int
        L.ssdo_overlap.argtypes = [C.c_int, vp, vp, C.c_int, C.c_double]
        L.ssdo_overlap.restype = C.c_double
        L.ssdo_cache_lookup.argtypes = [C.c_int, C.c_int, C.c_int, i32p, i32p, i32p, i32p, i32p,
                                        C.c_uint64, C.c_int, u8p, i32p, i32p]
        L.ssdo_cache_lookup.restype = C.c_int
        _lib = L
    return _lib


def _p(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(C.POINTER(ctype))


def _vp(a):
    return None if a is None else C.c_void_p(a.ctypes.data)


def _dtype_code(arr):
    if arr.dtype == np.float32:
        return DTYPE_FP32
    if arr.dtype == np.uint16:  # bf16 bit patterns
        return DTYPE_BF16
    raise TypeError("logits must be float32 or uint16 (bf16 bits)")


def n_threads_default():
    return max(1, len(os.sched_getaffinity(0)))


def philox4x32_10(ctr, key):
    """ctr [n,4] uint32, key [n,2] uint32 -> [n,4] uint32."""
    ctr = np.ascontiguousarray(ctr, dtype=np.uint32).reshape(-1, 4)
    key = np.ascontiguousarray(np.broadcast_to(np.asarray(key, dtype=np.uint32), (ctr.shape[0], 2)))
    out = np.empty_like(ctr)
    lib().ssdo_philox_batch(ctr.shape[0], _p(ctr, C.c_uint32), _p(key, C.c_uint32), _p(out, C.c_uint32))
    return out


def fallback_token(seed, b, i, V):
    return int(lib().ssdo_fallback_token(seed, b, i, V))


def fanout_plan(alpha, K, budget, mode=0):
    F = np.zeros(K + 1, dtype=np.int32)
    rc = lib().ssdo_fanout_plan(float(alpha), K, budget, mode, _p(F, C.c_int32))
    if rc != 0:
        raise ValueError("bad fan-out arguments")
    return F


def fanout_plan_batch(alpha, K, budget, mode=0):
    alpha = np.asarray(alpha, dtype=np.float32)
    return np.stack([fanout_plan(float(a), K, budget, mode) for a in alpha])


def fanout_plan_power(alpha, K, budget, q):
    """Power-law plan, gamma = q / 8 (q = 8: the geometric plan)."""
    F = np.zeros(K + 1, dtype=np.int32)
    if lib().ssdo_fanout_plan_power(float(alpha), K, budget, int(q), _p(F, C.c_int32)) != 0:
        raise ValueError("bad fan-out arguments")
    return F


def fanout_plan_power_batch(alpha, K, budget, q):
    alpha = np.asarray(alpha, dtype=np.float32)
    return np.stack([fanout_plan_power(float(a), K, budget, q) for a in alpha])


def alpha_update(alpha, accept_prob, status, lam):
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    ap = np.ascontiguousarray(accept_prob, dtype=np.float32)
    st = np.ascontiguousarray(status, dtype=np.int32)
    B, K = ap.shape
    out = np.zeros(B, np.float32)
    lib().ssdo_alpha_update(B, K, _p(alpha, C.c_float), _p(ap, C.c_float), _p(st, C.c_int32), float(lam),
                            _p(out, C.c_float))
    return out


def fallback_bstar(h, alpha, K, L_target, L_primary, L_fast, E_fast, b_max):
    """(b*, choice[b_max]) of the batch-size fallback policy."""
    choice = np.zeros(b_max, np.uint8)
    bs = lib().ssdo_fallback_bstar(float(h), float(alpha), int(K), float(L_target), float(L_primary),
                                   float(L_fast), float(E_fast), int(b_max), _p(choice, C.c_uint8))
    return int(bs), choice


def topf(logits, F):
    l = np.ascontiguousarray(logits, dtype=np.float64)
    out = np.zeros(max(F, 0), dtype=np.int32)
    if lib().ssdo_topf(_p(l, C.c_double), l.size, F, _p(out, C.c_int32)) != 0:
        raise ValueError("bad top-F arguments")
    return out


def overlap(lp_row, lq_row, T):
    lp_row = np.ascontiguousarray(lp_row)
    lq_row = np.ascontiguousarray(lq_row)
    return lib().ssdo_overlap(_dtype_code(lp_row), _vp(lp_row), _vp(lq_row), lp_row.size, float(T))


def verify(target, draft, tokens, uniforms, T, F=None, C_coef=1.0, budget=0, draft_next=None,
           payload=None, fallback_seed=0, rows=None, n_threads=None, want_phit=False, early_exit=False):
    """Oracle verify + cache step.  target [B,K+1,V], draft [B,K,V] as float32 or
    uint16 bf16 bits; tokens [B,K] int32; uniforms [B,K+1] float32; F [B,K+1]
    int32 or None.  rows: optional subset of batch rows; outputs are indexed by
    position in that subset.  early_exit: the early-exit read schedule (target
    rows p_j past k* other than p_K are not read: no a_j, no flags from them)."""
    target = np.ascontiguousarray(target)
    draft = np.ascontiguousarray(draft)
    B, K1, V = target.shape
    K = K1 - 1
    assert draft.shape == (B, K, V) and draft.dtype == target.dtype
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    uniforms = np.ascontiguousarray(uniforms, dtype=np.float32)
    if draft_next is not None:
        draft_next = np.ascontiguousarray(draft_next)
        assert draft_next.shape == (B, V) and draft_next.dtype == target.dtype
    if F is not None:
        F = np.ascontiguousarray(F, dtype=np.int32)
    if payload is not None:
        payload = np.ascontiguousarray(payload, dtype=np.int32)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n = B if rows_arr is None else rows_arr.size
    out = dict(
        n_accepted=np.zeros(n, np.int32), bonus=np.zeros(n, np.int32),
        out_tokens=np.zeros((n, K + 1), np.int32), accept_prob=np.zeros((n, K)),
        residual_mass=np.zeros(n), Z=np.zeros((n, K)), QS=np.zeros((n, K)),
        q_lse=np.zeros((n, K)), p_lse=np.zeros((n, K + 1)),
        offsets=np.zeros((n, K + 2), np.int32), cache_tokens=np.zeros((n, max(budget, 1)), np.int32),
        hit=np.zeros(n, np.uint8), slot=np.zeros(n, np.int32), next_tokens=np.zeros((n, K), np.int32),
        status=np.zeros(n, np.int32), accept_margin=np.zeros(n), bonus_margin=np.zeros(n),
        p_hit=np.zeros(n), bonus_lo=np.zeros(n, np.int32), bonus_hi=np.zeros(n, np.int32))
    rc = lib().ssdo_verify_batch(
        _dtype_code(target), B, K, V, budget, _vp(target), _vp(draft), _vp(draft_next),
        _p(tokens, C.c_int32), _p(uniforms, C.c_float), float(T), _p(F, C.c_int32), float(C_coef),
        _p(payload, C.c_int32), fallback_seed, _p(rows_arr, C.c_int32), n,
        n_threads or n_threads_default(),
        _p(out["n_accepted"], C.c_int32), _p(out["bonus"], C.c_int32), _p(out["out_tokens"], C.c_int32),
        _p(out["accept_prob"], C.c_double), _p(out["residual_mass"], C.c_double),
        _p(out["Z"], C.c_double), _p(out["QS"], C.c_double), _p(out["q_lse"], C.c_double),
        _p(out["p_lse"], C.c_double), _p(out["offsets"], C.c_int32),
        _p(out["cache_tokens"], C.c_int32) if F is not None else None,
        _p(out["hit"], C.c_uint8), _p(out["slot"], C.c_int32), _p(out["next_tokens"], C.c_int32),
        _p(out["status"], C.c_int32), _p(out["accept_margin"], C.c_double),
        _p(out["bonus_margin"], C.c_double), _p(out["p_hit"], C.c_double) if want_phit else None,
        _p(out["bonus_lo"], C.c_int32), _p(out["bonus_hi"], C.c_int32), 1 if early_exit else 0)
    if rc != 0:
        raise ValueError("oracle verify rejected its arguments")
    if F is None:
        for k in ("offsets", "cache_tokens", "hit", "slot"):
            out.pop(k)
    if not want_phit:
        out.pop("p_hit")
    return out


def reweight(draft, T, F, C_coef, budget, u_draft=None, rows=None, n_threads=None):
    """Oracle Saguaro reweighting (+ optional draft-token draw d_j ~ q'_j)."""
    draft = np.ascontiguousarray(draft)
    B, K, V = draft.shape
    F = np.ascontiguousarray(F, dtype=np.int32)
    assert F.shape == (B, K + 1)
    if u_draft is not None:
        u_draft = np.ascontiguousarray(u_draft, dtype=np.float32)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n = B if rows_arr is None else rows_arr.size
    out = dict(topf_tokens=np.full((n, max(budget, 1)), -2, np.int32),
               offsets=np.zeros((n, K + 2), np.int32), Z=np.zeros((n, K)), QS=np.zeros((n, K)),
               q_lse=np.zeros((n, K)), tokens=np.zeros((n, K), np.int32) if u_draft is not None else None,
               margin=np.zeros(n), status=np.zeros(n, np.int32),
               tok_lo=np.zeros((n, K), np.int32), tok_hi=np.zeros((n, K), np.int32))
    rc = lib().ssdo_reweight_batch(
        _dtype_code(draft), B, K, V, budget, _vp(draft), float(T), _p(F, C.c_int32), float(C_coef),
        _p(u_draft, C.c_float), _p(rows_arr, C.c_int32), n, n_threads or n_threads_default(),
        _p(out["topf_tokens"], C.c_int32), _p(out["offsets"], C.c_int32), _p(out["Z"], C.c_double),
        _p(out["QS"], C.c_double), _p(out["q_lse"], C.c_double), _p(out["tokens"], C.c_int32),
        _p(out["margin"], C.c_double), _p(out["status"], C.c_int32),
        _p(out["tok_lo"], C.c_int32) if u_draft is not None else None,
        _p(out["tok_hi"], C.c_int32) if u_draft is not None else None)
    if rc != 0:
        raise ValueError("oracle reweight rejected its arguments")
    if u_draft is None:
        for k in ("tokens", "tok_lo", "tok_hi"):
            out.pop(k)
    return out


def cache_lookup(offsets, tokens, k, bonus, V, payload=None, fallback_seed=0):
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    B, K2 = offsets.shape
    K = K2 - 2
    budget = tokens.shape[1]
    k = np.ascontiguousarray(k, dtype=np.int32)
    bonus = np.ascontiguousarray(bonus, dtype=np.int32)
    if payload is not None:
        payload = np.ascontiguousarray(payload, dtype=np.int32)
    hit = np.zeros(B, np.uint8)
    slot = np.zeros(B, np.int32)
    nxt = np.zeros((B, K), np.int32)
    lib().ssdo_cache_lookup(B, K, budget, _p(offsets, C.c_int32), _p(tokens, C.c_int32),
                            _p(k, C.c_int32), _p(bonus, C.c_int32), _p(payload, C.c_int32),
                            fallback_seed, V, _p(hit, C.c_uint8), _p(slot, C.c_int32), _p(nxt, C.c_int32))
    return dict(hit=hit, slot=slot, next_tokens=nxt)
