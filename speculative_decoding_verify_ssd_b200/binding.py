"""Thin ctypes binding of libssd.so (include/ssd.h).

Argument marshalling only: shapes, dtypes and devices of torch tensors are
checked, pointers and the current CUDA stream are handed to the C ABI, and a
non-zero ssd_status becomes an exception.  Every step of the computation runs
in libssd's CUDA kernels; there is no CPU path.  Functions keep the C names.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional

import torch

from . import _build

SSD_OK = 0
DTYPE_FP32 = 0
DTYPE_BF16 = 1
FANOUT_GEOMETRIC = 0
FANOUT_UNIFORM = 1

ROW_NONFINITE = 1
ROW_BAD_TOKEN = 2
ROW_BAD_UNIFORM = 4
ROW_ZERO_Q = 8
ROW_ZERO_RESIDUAL = 16
ROW_NEAR_TIE = 32
ROW_BAD_PLAN = 64
ROW_DEVICE_TIMEOUT = 128
ROW_INVALID = ROW_NONFINITE | ROW_BAD_TOKEN | ROW_BAD_UNIFORM | ROW_BAD_PLAN | ROW_DEVICE_TIMEOUT

MAX_K = 32
MAX_BUDGET = 512


class SsdError(RuntimeError):
    pass


class _Cache(C.Structure):
    _fields_ = [("offsets", C.c_void_p), ("tokens", C.c_void_p), ("payload", C.c_void_p),
                ("hit", C.c_void_p), ("slot", C.c_void_p), ("next_tokens", C.c_void_p),
                ("fallback_seed", C.c_uint64)]


_lib = None


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True):
    """Load libssd.so from the package directory (building it with nvcc if it
    is missing or older than its sources)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build() if build_if_missing else _build.LIB
    if not os.path.exists(path):
        raise SsdError(f"libssd.so not found at {path}")
    L = C.CDLL(path)
    vp, i32, i64, f32, sz = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t
    L.ssd_version.restype = C.c_char_p
    L.ssd_status_string.restype = C.c_char_p
    L.ssd_status_string.argtypes = [i32]
    L.ssd_workspace_bytes.restype = sz
    L.ssd_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.ssd_read_device_error.restype = i32
    L.ssd_read_device_error.argtypes = [vp, i32, i32, i32, i32, vp, C.POINTER(C.c_int32)]
    L.ssd_fanout_plan.restype = i32
    L.ssd_fanout_plan.argtypes = [vp, i32, i32, i32, i32, vp, vp]
    L.ssd_saguaro_reweight.restype = i32
    L.ssd_saguaro_reweight.argtypes = [vp, i32, i32, i32, i32, f32, vp, f32, i32, vp, i64, vp, vp, vp,
                                       vp, vp, vp, vp, vp, sz, vp]
    L.ssd_verify.restype = i32
    L.ssd_verify.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, f32, vp, vp, i32, f32, i32, vp, vp,
                             vp, vp, vp, C.POINTER(_Cache), vp, vp, sz, vp]
    L.ssd_verify_early_exit.restype = i32
    L.ssd_verify_early_exit.argtypes = L.ssd_verify.argtypes
    L.ssd_read_skipped_bytes.restype = i32
    L.ssd_read_skipped_bytes.argtypes = [vp, i32, i32, i32, i32, vp, C.POINTER(C.c_uint64)]
    L.ssd_verify_noalloc.restype = i32
    L.ssd_verify_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, f32, vp, vp, i32, f32, i32, vp, vp,
                                     vp, vp, vp, C.POINTER(_Cache), vp, vp]
    L.ssd_fanout_plan_power.restype = i32
    L.ssd_fanout_plan_power.argtypes = [vp, i32, i32, i32, i32, vp, vp]
    L.ssd_alpha_update.restype = i32
    L.ssd_alpha_update.argtypes = [vp, vp, vp, i32, i32, C.c_double, vp, vp]
    L.ssd_fallback_bstar.restype = i32
    L.ssd_fallback_bstar.argtypes = [C.c_double, C.c_double, i32, C.c_double, C.c_double, C.c_double, C.c_double,
                                     i32, vp]
    L.ssd_prespeculate.restype = i32
    L.ssd_prespeculate.argtypes = [vp, i32, i32, i32, i32, i32, f32, vp, f32, i32, vp, vp, vp, vp, sz, vp]
    L.ssd_cache_build.restype = i32
    L.ssd_cache_build.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp]
    L.ssd_cache_lookup.restype = i32
    L.ssd_cache_lookup.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, C.c_uint64, i32, vp, vp, vp, vp]
    _lib = L
    return L


def version() -> str:
    return load().ssd_version().decode()


def status_string(code: int) -> str:
    return load().ssd_status_string(code).decode()


def _check(code: int, what: str):
    if code != SSD_OK:
        raise SsdError(f"{what}: {status_string(code)} ({code})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _logit_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_FP32
    raise ValueError("logits must be torch.bfloat16 or torch.float32")


def workspace_bytes(B: int, K: int, V: int = 0, dtype: int = DTYPE_BF16) -> int:
    return int(load().ssd_workspace_bytes(B, K, V, dtype))


class Workspace:
    """Caller-owned, zero-filled device workspace for (B, K, V, dtype),
    reusable across calls on one stream (each completed call leaves its
    counters zero)."""

    def __init__(self, B: int, K: int, device, V: int = 262144, dtype: int = DTYPE_BF16):
        self.B, self.K, self.V, self.dtype = B, K, V, dtype
        self.nbytes = workspace_bytes(B, K, V, dtype)
        self.buf = torch.zeros(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + self.nbytes]

    def ptr(self):
        return C.c_void_p(self.view.data_ptr())

    def reset(self):
        """Zero-fill the workspace again (needed after a device timeout, which
        may leave arrival counters non-zero).  Synchronises the device, so the
        next call on any stream sees the zeros."""
        self.view.zero_()
        torch.cuda.synchronize(self.view.device)

    def device_error(self, stream=None) -> int:
        """SSD_OK, or SSD_ERR_TIMEOUT if a bounded device wait of an earlier
        call gave up; in that case the workspace is zero-filled again."""
        out = C.c_int32(0)
        _check(load().ssd_read_device_error(self.ptr(), self.B, self.K, self.V, self.dtype, _stream(stream),
                                            C.byref(out)),
               "ssd_read_device_error")
        if out.value != 0:
            self.reset()
        return out.value

    def skipped_bytes(self, stream=None) -> int:
        """Target-logit bytes that early-exit calls on this workspace did not
        read since the last query (the counter is cleared)."""
        out = C.c_uint64(0)
        _check(load().ssd_read_skipped_bytes(self.ptr(), self.B, self.K, self.V, self.dtype, _stream(stream),
                                             C.byref(out)),
               "ssd_read_skipped_bytes")
        return int(out.value)


_default_ws = {}


def default_workspace(device, B: int, K: int, V: int, dtype: int) -> Workspace:
    """The workspace used when a call passes none: one per (device, B, K, V,
    dtype), made on first use and kept, so repeated calls of one shape do not
    allocate.  Calls that share it must not overlap on the GPU (one stream);
    calls on several streams pass a Workspace each."""
    key = (torch.device(device).index, B, K, V, dtype)
    ws = _default_ws.get(key)
    if ws is None:
        ws = Workspace(B, K, device, V, dtype)
        _default_ws[key] = ws
    return ws


def ssd_fanout_plan(alpha: torch.Tensor, K: int, budget: int, mode: int = FANOUT_GEOMETRIC,
                    F: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    B = alpha.shape[0]
    _need(alpha, "alpha", torch.float32, (B,), alpha.device)
    if F is None:
        F = torch.empty((B, K + 1), dtype=torch.int32, device=alpha.device)
    _need(F, "F", torch.int32, (B, K + 1), alpha.device)
    with torch.cuda.device(alpha.device):
        _check(load().ssd_fanout_plan(_ptr(alpha), B, K, budget, mode, _ptr(F), _stream(stream)),
               "ssd_fanout_plan")
    return F


def ssd_fanout_plan_power(alpha: torch.Tensor, K: int, budget: int, gamma_eighths: int,
                          F: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Power-law fan-out plan, gamma = gamma_eighths / 8 (see ssd.h)."""
    B = alpha.shape[0]
    _need(alpha, "alpha", torch.float32, (B,), alpha.device)
    if F is None:
        F = torch.empty((B, K + 1), dtype=torch.int32, device=alpha.device)
    _need(F, "F", torch.int32, (B, K + 1), alpha.device)
    with torch.cuda.device(alpha.device):
        _check(load().ssd_fanout_plan_power(_ptr(alpha), B, K, budget, int(gamma_eighths), _ptr(F),
                                            _stream(stream)), "ssd_fanout_plan_power")
    return F


def ssd_alpha_update(alpha: torch.Tensor, accept_prob: torch.Tensor, status: torch.Tensor, lam: float,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """alpha' = (1 - lam) alpha + lam * mean_j accept_prob[:, j] per valid row."""
    B, K = accept_prob.shape
    dev = alpha.device
    _need(alpha, "alpha", torch.float32, (B,), dev)
    _need(accept_prob, "accept_prob", torch.float32, (B, K), dev)
    _need(status, "status", torch.int32, (B,), dev)
    if out is None:
        out = torch.empty_like(alpha)
    with torch.cuda.device(dev):
        _check(load().ssd_alpha_update(_ptr(alpha), _ptr(accept_prob), _ptr(status), B, K, float(lam), _ptr(out),
                                       _stream(stream)), "ssd_alpha_update")
    return out


def ssd_fallback_bstar(h: float, alpha: float, K: int, L_target: float, L_primary: float, L_fast: float,
                       E_fast: float, b_max: int):
    """(b*, choice[b_max] as a numpy uint8 array) of the batch-size fallback policy (host)."""
    import numpy as np
    choice = np.zeros(b_max, np.uint8)
    r = load().ssd_fallback_bstar(float(h), float(alpha), int(K), float(L_target), float(L_primary),
                                  float(L_fast), float(E_fast), int(b_max), C.c_void_p(choice.ctypes.data))
    if r < 0:
        raise SsdError("ssd_fallback_bstar: arguments out of range")
    return int(r), choice


def ssd_prespeculate(key_logits: torch.Tensor, T: float, F_next: torch.Tensor, C_coef: float, next_budget: int,
                     uniforms: torch.Tensor, workspace: Optional["Workspace"] = None, payload=None, stream=None):
    """Draw the K-token payload of every cache key (see ssd.h); returns (payload, status)."""
    B, n_keys, K, V = key_logits.shape
    dev = key_logits.device
    dt = _logit_dtype(key_logits)
    _need(key_logits, "key_logits", key_logits.dtype, (B, n_keys, K, V), dev)
    _need(F_next, "F_next", torch.int32, (B * n_keys, K + 1), dev)
    _need(uniforms, "uniforms", torch.float32, (B, n_keys, K), dev)
    if payload is None:
        payload = torch.empty((B, n_keys, K), dtype=torch.int32, device=dev)
    _need(payload, "payload", torch.int32, (B, n_keys, K), dev)
    status = torch.empty(B * n_keys, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = default_workspace(dev, B * n_keys, K, V, dt)
    with torch.cuda.device(dev):
        _check(load().ssd_prespeculate(_ptr(key_logits), dt, B, n_keys, K, V, float(T), _ptr(F_next),
                                       float(C_coef), int(next_budget), _ptr(uniforms), _ptr(payload),
                                       _ptr(status), workspace.ptr(), workspace.nbytes, _stream(stream)),
               "ssd_prespeculate")
    return payload, status


@dataclass
class VerifyResult:
    n_accepted: torch.Tensor
    bonus: torch.Tensor
    out_tokens: torch.Tensor
    accept_prob: torch.Tensor
    residual_mass: torch.Tensor
    status: torch.Tensor
    cache_offsets: Optional[torch.Tensor] = None
    cache_tokens: Optional[torch.Tensor] = None
    hit: Optional[torch.Tensor] = None
    slot: Optional[torch.Tensor] = None
    next_tokens: Optional[torch.Tensor] = None


def alloc_verify_result(B: int, K: int, budget: int, device, with_cache: bool) -> VerifyResult:
    i32 = dict(dtype=torch.int32, device=device)
    r = VerifyResult(
        n_accepted=torch.empty(B, **i32), bonus=torch.empty(B, **i32),
        out_tokens=torch.empty((B, K + 1), **i32),
        accept_prob=torch.empty((B, K), dtype=torch.float32, device=device),
        residual_mass=torch.empty(B, dtype=torch.float32, device=device), status=torch.empty(B, **i32))
    if with_cache:
        r.cache_offsets = torch.empty((B, K + 2), **i32)
        r.cache_tokens = torch.empty((B, max(budget, 1)), **i32)
        r.hit = torch.empty(B, dtype=torch.uint8, device=device)
        r.slot = torch.empty(B, **i32)
        r.next_tokens = torch.empty((B, K), **i32)
    return r


def ssd_verify(target: torch.Tensor, draft: torch.Tensor, draft_tokens: torch.Tensor,
               uniforms: torch.Tensor, T: float, F: Optional[torch.Tensor] = None, C_coef: float = 1.0,
               budget: int = 0, draft_next: Optional[torch.Tensor] = None, cache: bool = False,
               alpha: Optional[torch.Tensor] = None, fanout_mode: int = FANOUT_GEOMETRIC,
               payload: Optional[torch.Tensor] = None, fallback_seed: int = 0,
               workspace: Optional[Workspace] = None, out: Optional[VerifyResult] = None,
               stream=None, early_exit: bool = False) -> VerifyResult:
    """Fused verify + speculation-cache step on the GPU (see ssd_verify in ssd.h);
    early_exit=True calls ssd_verify_early_exit (the early-exit read schedule)."""
    B, K1, V = target.shape
    K = K1 - 1
    dev = target.device
    if dev.type != "cuda":
        raise ValueError("ssd_verify runs on a CUDA device; use ssd_verify_host for host tensors")
    dt = _logit_dtype(target)
    _need(target, "target", target.dtype, (B, K + 1, V), dev)
    _need(draft, "draft", target.dtype, (B, K, V), dev)
    if draft_next is not None:
        _need(draft_next, "draft_next", target.dtype, (B, V), dev)
    _need(draft_tokens, "draft_tokens", torch.int32, (B, K), dev)
    _need(uniforms, "uniforms", torch.float32, (B, K + 1), dev)
    if F is not None:
        _need(F, "F", torch.int32, (B, K + 1), dev)
    if alpha is not None:
        _need(alpha, "alpha", torch.float32, (B,), dev)
    if payload is not None:
        _need(payload, "payload", torch.int32, (B, budget, K), dev)
    if cache and F is None and alpha is None:
        raise ValueError("a cache needs a fan-out plan (F or alpha)")
    if workspace is None:
        workspace = default_workspace(dev, B, K, V, dt)
    if out is None:
        out = alloc_verify_result(B, K, budget, dev, cache)
    cstruct = None
    if cache:
        cstruct = _Cache(out.cache_offsets.data_ptr(), out.cache_tokens.data_ptr(),
                         None if payload is None else payload.data_ptr(), out.hit.data_ptr(),
                         out.slot.data_ptr(), out.next_tokens.data_ptr(), fallback_seed)
    fn = load().ssd_verify_early_exit if early_exit else load().ssd_verify
    with torch.cuda.device(dev):
        code = fn(
            _ptr(target), _ptr(draft), _ptr(draft_next), dt, B, K, V, _ptr(draft_tokens), _ptr(uniforms),
            float(T), _ptr(F), _ptr(alpha), int(fanout_mode), float(C_coef), int(budget),
            _ptr(out.n_accepted), _ptr(out.bonus),
            _ptr(out.out_tokens), _ptr(out.accept_prob), _ptr(out.residual_mass),
            C.byref(cstruct) if cstruct is not None else None, _ptr(out.status), workspace.ptr(),
            workspace.nbytes, _stream(stream))
    _check(code, "ssd_verify_early_exit" if early_exit else "ssd_verify")
    return out


NOALLOC_MAX_WORKSPACE = 16 << 20


def ssd_verify_noalloc(target: torch.Tensor, draft: torch.Tensor, draft_tokens: torch.Tensor,
                       uniforms: torch.Tensor, T: float, out: VerifyResult, F: Optional[torch.Tensor] = None,
                       C_coef: float = 1.0, budget: int = 0, draft_next: Optional[torch.Tensor] = None,
                       cache: bool = False, alpha: Optional[torch.Tensor] = None,
                       fanout_mode: int = FANOUT_GEOMETRIC, payload: Optional[torch.Tensor] = None,
                       fallback_seed: int = 0, stream=None) -> VerifyResult:
    """ssd_verify with the library's static scratch instead of a workspace
    (see ssd_verify_noalloc in ssd.h).  The caller passes `out` (from
    alloc_verify_result, made once ahead of time), so the call itself makes no
    device allocation.  Calls on one device must not overlap."""
    B, K1, V = target.shape
    K = K1 - 1
    dev = target.device
    if dev.type != "cuda":
        raise ValueError("ssd_verify_noalloc runs on a CUDA device")
    dt = _logit_dtype(target)
    _need(target, "target", target.dtype, (B, K + 1, V), dev)
    _need(draft, "draft", target.dtype, (B, K, V), dev)
    if draft_next is not None:
        _need(draft_next, "draft_next", target.dtype, (B, V), dev)
    _need(draft_tokens, "draft_tokens", torch.int32, (B, K), dev)
    _need(uniforms, "uniforms", torch.float32, (B, K + 1), dev)
    if F is not None:
        _need(F, "F", torch.int32, (B, K + 1), dev)
    if alpha is not None:
        _need(alpha, "alpha", torch.float32, (B,), dev)
    if payload is not None:
        _need(payload, "payload", torch.int32, (B, budget, K), dev)
    if cache and F is None and alpha is None:
        raise ValueError("a cache needs a fan-out plan (F or alpha)")
    cstruct = None
    if cache:
        cstruct = _Cache(out.cache_offsets.data_ptr(), out.cache_tokens.data_ptr(),
                         None if payload is None else payload.data_ptr(), out.hit.data_ptr(),
                         out.slot.data_ptr(), out.next_tokens.data_ptr(), fallback_seed)
    with torch.cuda.device(dev):
        code = load().ssd_verify_noalloc(
            _ptr(target), _ptr(draft), _ptr(draft_next), dt, B, K, V, _ptr(draft_tokens), _ptr(uniforms),
            float(T), _ptr(F), _ptr(alpha), int(fanout_mode), float(C_coef), int(budget),
            _ptr(out.n_accepted), _ptr(out.bonus),
            _ptr(out.out_tokens), _ptr(out.accept_prob), _ptr(out.residual_mass),
            C.byref(cstruct) if cstruct is not None else None, _ptr(out.status), _stream(stream))
    _check(code, "ssd_verify_noalloc")
    return out


def ssd_verify_host(target: torch.Tensor, draft: torch.Tensor, draft_tokens: torch.Tensor,
                    uniforms: torch.Tensor, T: float, alpha: torch.Tensor, budget: int, C_coef: float,
                    device, fallback_seed: int = 0, mode: int = FANOUT_GEOMETRIC,
                    workspace: Optional[Workspace] = None, stream=None) -> VerifyResult:
    """The whole step from host (ideally pinned) tensors: copy the inputs to
    the device, plan the fan-out, verify + build + look up, and copy the
    results back to host memory.  Returns host tensors."""
    nb = dict(device=device, non_blocking=True)
    t, d = target.to(**nb), draft.to(**nb)
    tok, u, al = draft_tokens.to(**nb), uniforms.to(**nb), alpha.to(**nb)
    r = ssd_verify(t, d, tok, u, T, alpha=al, fanout_mode=mode, C_coef=C_coef, budget=budget, cache=True,
                   fallback_seed=fallback_seed, workspace=workspace, stream=stream)
    host = {k: (v.to("cpu", non_blocking=True) if isinstance(v, torch.Tensor) else v)
            for k, v in r.__dict__.items()}
    (stream or torch.cuda.current_stream()).synchronize()
    return VerifyResult(**host)


@dataclass
class ReweightResult:
    topf_tokens: torch.Tensor
    offsets: torch.Tensor
    Z: torch.Tensor
    q_lse: torch.Tensor
    status: torch.Tensor
    draft_tokens: Optional[torch.Tensor] = None


def ssd_saguaro_reweight(draft: torch.Tensor, T: float, F: torch.Tensor, C_coef: float, budget: int,
                         u_draft: Optional[torch.Tensor] = None, guess: Optional[torch.Tensor] = None,
                         guess_row_stride: Optional[int] = None, workspace: Optional[Workspace] = None,
                         stream=None) -> ReweightResult:
    """Draft-side Saguaro reweighting (+ optional draw d_j ~ q'_j)."""
    B, K, V = draft.shape
    dev = draft.device
    dt = _logit_dtype(draft)
    _need(draft, "draft", draft.dtype, (B, K, V), dev)
    _need(F, "F", torch.int32, (B, K + 1), dev)
    if u_draft is not None:
        _need(u_draft, "u_draft", torch.float32, (B, K), dev)
    stride = 0
    if guess is not None:
        if guess.dtype != draft.dtype or guess.device != dev:
            raise ValueError("guess rows must match the draft dtype and device")
        stride = int(guess_row_stride if guess_row_stride is not None else guess.stride(0))
    if workspace is None:
        workspace = default_workspace(dev, B, K, V, dt)
    i32 = dict(dtype=torch.int32, device=dev)
    r = ReweightResult(topf_tokens=torch.full((B, max(budget, 1)), -2, **i32),
                       offsets=torch.empty((B, K + 2), **i32),
                       Z=torch.empty((B, K), dtype=torch.float32, device=dev),
                       q_lse=torch.empty((B, K), dtype=torch.float32, device=dev),
                       status=torch.empty(B, **i32),
                       draft_tokens=torch.empty((B, K), **i32) if u_draft is not None else None)
    with torch.cuda.device(dev):
        code = load().ssd_saguaro_reweight(
            _ptr(draft), dt, B, K, V, float(T), _ptr(F), float(C_coef), int(budget), _ptr(guess), stride,
            _ptr(u_draft), _ptr(r.topf_tokens), _ptr(r.offsets), _ptr(r.Z), _ptr(r.q_lse),
            _ptr(r.draft_tokens), _ptr(r.status), workspace.ptr(), workspace.nbytes, _stream(stream))
    _check(code, "ssd_saguaro_reweight")
    return r


def ssd_cache_build(F: torch.Tensor, topf_tokens: torch.Tensor, budget: int,
                    guess_K: Optional[torch.Tensor] = None, stream=None):
    B, K1 = F.shape
    K = K1 - 1
    dev = F.device
    _need(F, "F", torch.int32, (B, K + 1), dev)
    _need(topf_tokens, "topf_tokens", torch.int32, (B, budget), dev)
    if guess_K is not None:
        _need(guess_K, "guess_K", torch.int32, (B, budget), dev)
    offsets = torch.empty((B, K + 2), dtype=torch.int32, device=dev)
    tokens = torch.empty((B, budget), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(load().ssd_cache_build(_ptr(F), _ptr(topf_tokens), _ptr(guess_K), B, K, budget, _ptr(offsets),
                                      _ptr(tokens), _stream(stream)), "ssd_cache_build")
    return offsets, tokens


def ssd_cache_lookup(offsets: torch.Tensor, tokens: torch.Tensor, k: torch.Tensor, bonus: torch.Tensor,
                     V: int, payload: Optional[torch.Tensor] = None, fallback_seed: int = 0, stream=None):
    B, K2 = offsets.shape
    K = K2 - 2
    budget = tokens.shape[1]
    dev = offsets.device
    _need(offsets, "offsets", torch.int32, (B, K + 2), dev)
    _need(tokens, "tokens", torch.int32, (B, budget), dev)
    _need(k, "k", torch.int32, (B,), dev)
    _need(bonus, "bonus", torch.int32, (B,), dev)
    if payload is not None:
        _need(payload, "payload", torch.int32, (B, budget, K), dev)
    hit = torch.empty(B, dtype=torch.uint8, device=dev)
    slot = torch.empty(B, dtype=torch.int32, device=dev)
    nxt = torch.empty((B, K), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(load().ssd_cache_lookup(_ptr(offsets), _ptr(tokens), B, K, budget, _ptr(k), _ptr(bonus),
                                       _ptr(payload), fallback_seed, V, _ptr(hit), _ptr(slot), _ptr(nxt),
                                       _stream(stream)), "ssd_cache_lookup")
    return hit, slot, nxt
