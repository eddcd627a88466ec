"""ssd_verify_noalloc (the static-scratch variant of ssd_verify) against
ssd_verify on the same inputs, through the C ABI.

Some callers cannot allocate device memory when they verify: a serving loop
that gave all of HBM to its KV cache at start-up, a host program with no
device allocator, code that must not let cudaMalloc/cudaFree synchronise the
device mid-step.  They use the entry point whose scratch is a static device
buffer of the library.  That buffer is shared by every call on a device and
keeps the last call's contents, so these tests run calls back to back -- the
same shape twice, and different shapes one after another with fresh inputs
-- and compare each with ssd_verify on a workspace of its own.

Kept in its own file, collected last, so it runs both alone and after the
other GPU tests (the static scratch must not depend on what ran before)."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_ssd_b200 import binding as ssd
from speculative_decoding_verify_ssd_b200 import synth

from ssd_testlib import draft_tokens_for, to_dev

pytestmark = pytest.mark.gpu


def _inputs(w):
    g = synth.generate(w)
    F = oracle.fanout_plan_batch(g["alpha"], w.K, w.budget, w.fanout_mode)
    tok = draft_tokens_for(w, g, F)
    return dict(t=to_dev(g["target"]), d=to_dev(g["draft"]), tok=to_dev(tok), u=to_dev(g["uniforms"]),
                alpha=to_dev(g["alpha"]))


def _fields(r):
    return {k: v.cpu().numpy() for k, v in r.__dict__.items() if isinstance(v, torch.Tensor)}


def _kw(w, x):
    return dict(alpha=x["alpha"], fanout_mode=w.fanout_mode, C_coef=w.C, budget=w.budget, cache=True,
                fallback_seed=w.fallback_seed)


def _with_workspace(w, x):
    """ssd_verify on a fresh workspace of its own: the reference outputs."""
    ws = ssd.Workspace(w.B, w.K, x["t"].device, w.V, ssd.DTYPE_BF16 if w.dtype == "bf16" else ssd.DTYPE_FP32)
    return _fields(ssd.ssd_verify(x["t"], x["d"], x["tok"], x["u"], w.T, workspace=ws, **_kw(w, x)))


def _assert_same(got, ref, what):
    assert np.all((got["status"] & ssd.ROW_DEVICE_TIMEOUT) == 0), f"{what}: a device wait timed out"
    for k, v in ref.items():
        np.testing.assert_array_equal(got[k], v, err_msg=f"{what}: {k}")


@pytest.mark.parametrize("name,B,V", [("zipf_b16_k5_v32000_bf16", 16, 32000),
                                      ("zipf_b64_k6_v128256_bf16", 8, 128256),
                                      ("tiny_b1_k4_v1024_fp32", 1, 1024)])
def test_noalloc_matches_workspace_entry_point(name, B, V):
    w = synth.WORKLOADS[name].replace(B=B, V=V)
    x = _inputs(w)
    dev = x["t"].device
    ref = _with_workspace(w, x)
    outs = [ssd.alloc_verify_result(w.B, w.K, w.budget, dev, True) for _ in range(2)]
    for out in outs:  # two calls in a row on the same static scratch
        ssd.ssd_verify_noalloc(x["t"], x["d"], x["tok"], x["u"], w.T, out, **_kw(w, x))
    torch.cuda.synchronize()
    for i, out in enumerate(outs):
        _assert_same(_fields(out), ref, f"call {i}")


def test_noalloc_shape_changes_between_calls():
    """The headline shape, then a smaller shape with other inputs, then the
    headline shape again with new uniforms: each call's counters and decision
    words sit at offsets of its own shape, over what the previous call left
    there, and every call must still equal ssd_verify on a fresh workspace."""
    head = synth.WORKLOADS["zipf_b64_k6_v128256_bf16"]
    small = synth.WORKLOADS["zipf_b16_k5_v32000_bf16"].replace(seed=11)
    x1 = _inputs(head)
    x2 = _inputs(small)
    x3 = dict(x1)
    x3["u"] = to_dev(synth.uniforms(head.seed + 500, head.B, head.K + 1, synth.STREAM_ACCEPT))
    dev = x1["t"].device
    seq = [(head, x1), (small, x2), (head, x3)]
    refs = [_with_workspace(w, x) for w, x in seq]
    torch.cuda.synchronize()
    outs = []
    for w, x in seq:
        out = ssd.alloc_verify_result(w.B, w.K, w.budget, dev, True)
        ssd.ssd_verify_noalloc(x["t"], x["d"], x["tok"], x["u"], w.T, out, **_kw(w, x))
        outs.append(out)
    torch.cuda.synchronize()
    for i, (out, ref) in enumerate(zip(outs, refs)):
        _assert_same(_fields(out), ref, f"call {i} ({seq[i][0].name})")
    # the third call really saw new uniforms
    assert not np.array_equal(refs[0]["n_accepted"], refs[2]["n_accepted"]) or \
        not np.array_equal(refs[0]["bonus"], refs[2]["bonus"])


def test_noalloc_rejects_problems_beyond_its_buffer():
    L = ssd.load()
    B, K, V = 256, 8, 151936
    assert L.ssd_workspace_bytes(B, K, V, ssd.DTYPE_BF16) > ssd.NOALLOC_MAX_WORKSPACE
    dev = torch.device("cuda")
    t = torch.zeros((B, K + 1, V), dtype=torch.bfloat16, device=dev)
    d = torch.zeros((B, K, V), dtype=torch.bfloat16, device=dev)
    tok = torch.zeros((B, K), dtype=torch.int32, device=dev)
    u = torch.zeros((B, K + 1), dtype=torch.float32, device=dev)
    out = ssd.alloc_verify_result(B, K, 0, dev, False)
    with pytest.raises(ssd.SsdError, match="ssd_verify_noalloc"):
        ssd.ssd_verify_noalloc(t, d, tok, u, 1.0, out)
    torch.cuda.synchronize()
