"""ssd_verify_noalloc (the static-scratch variant of ssd_verify) against
ssd_verify on the same inputs: two calls in a row, identical outputs.  Kept
in its own file, collected last, so it runs both alone and after the other
GPU tests (the static scratch must not depend on what ran before)."""
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


@pytest.mark.parametrize("name,B,V", [("zipf_b16_k5_v32000_bf16", 16, 32000),
                                      ("zipf_b64_k6_v128256_bf16", 8, 128256),
                                      ("tiny_b1_k4_v1024_fp32", 1, 1024)])
def test_noalloc_matches_workspace_entry_point(name, B, V):
    w = synth.WORKLOADS[name].replace(B=B, V=V)
    x = _inputs(w)
    dev = x["t"].device
    kw = dict(alpha=x["alpha"], fanout_mode=w.fanout_mode, C_coef=w.C, budget=w.budget, cache=True,
              fallback_seed=w.fallback_seed)
    ref = _fields(ssd.ssd_verify(x["t"], x["d"], x["tok"], x["u"], w.T, **kw))
    outs = [ssd.alloc_verify_result(w.B, w.K, w.budget, dev, True) for _ in range(2)]
    for out in outs:  # two calls in a row on the same static scratch
        ssd.ssd_verify_noalloc(x["t"], x["d"], x["tok"], x["u"], w.T, out, **kw)
    torch.cuda.synchronize()
    for out in outs:
        got = _fields(out)
        for k, v in ref.items():
            np.testing.assert_array_equal(got[k], v, err_msg=k)


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
