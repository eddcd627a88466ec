"""Failure detection on the GPU without a fault: a test build of the library
whose waits for another CTA's result (a slice partial, a unit record, a row's
decision word) give up after 200 ns instead of 1 s.  Only the two-kernel
form (the default) has such waits; the optional cluster form's CTAs meet at
hardware cluster barriers and never poll another CTA's flag, so the test
build names the two-kernel form explicitly.  The waits then run out
on an ordinary call; the call must still return, the rows whose waits gave up
must carry SSD_ROW_DEVICE_TIMEOUT with the void-row outputs, and the
workspace's error word must read SSD_ERR_TIMEOUT.  The waits on the CTA's own
bulk copies keep their limit, so no copy is left in flight.  Afterwards the
normal library on a reset workspace must match the oracle again."""
import ctypes as C

import numpy as np
import pytest
import torch

from speculative_decoding_verify_ssd_b200 import _build
from speculative_decoding_verify_ssd_b200 import binding as ssd
from speculative_decoding_verify_ssd_b200 import synth

from ssd_testlib import Case, compare, to_dev

pytestmark = pytest.mark.gpu

SSD_ERR_TIMEOUT = 6


@pytest.fixture(scope="module")
def short_wait_lib():
    path = _build.build_variant("shortwait", ["SSD_DEP_WAIT_NS=200ull", "SSD_CLUSTER_VERIFY=0"])
    L = C.CDLL(path)
    vp, i32, f32, sz = C.c_void_p, C.c_int, C.c_float, C.c_size_t
    L.ssd_verify.restype = i32
    L.ssd_verify.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, f32, vp, vp, i32, f32, i32, vp, vp,
                             vp, vp, vp, C.POINTER(ssd._Cache), vp, vp, sz, vp]
    L.ssd_read_device_error.restype = i32
    L.ssd_read_device_error.argtypes = [vp, i32, i32, i32, i32, vp, C.POINTER(C.c_int32)]
    return L


@pytest.mark.parametrize("V", [8003, 8000], ids=["unaligned rows", "aligned rows (bulk-copy ring)"])
def test_short_waits_give_up_and_report(short_wait_lib, V):
    L = short_wait_lib
    w = synth.WORKLOADS["zipf_b16_k5_v32000_bf16"].replace(B=4, V=V)
    case = Case(w)
    dev = torch.device("cuda")
    t, d = to_dev(case.g["target"]), to_dev(case.g["draft"])
    tok, u, F = to_dev(case.tokens), to_dev(case.g["uniforms"]), to_dev(case.F)
    ws = ssd.Workspace(w.B, w.K, dev, w.V, ssd.DTYPE_BF16)
    out = ssd.alloc_verify_result(w.B, w.K, w.budget, dev, True)
    cs = ssd._Cache(out.cache_offsets.data_ptr(), out.cache_tokens.data_ptr(), None, out.hit.data_ptr(),
                    out.slot.data_ptr(), out.next_tokens.data_ptr(), w.fallback_seed)
    P = lambda x: C.c_void_p(x.data_ptr())
    timed_out = 0
    for _ in range(5):  # a few calls: each must return; most give up somewhere
        rc = L.ssd_verify(P(t), P(d), None, ssd.DTYPE_BF16, w.B, w.K, w.V, P(tok), P(u), w.T, P(F), None, 0,
                          w.C, w.budget, P(out.n_accepted), P(out.bonus), P(out.out_tokens), P(out.accept_prob),
                          P(out.residual_mass), C.byref(cs), P(out.status), ws.ptr(), ws.nbytes,
                          C.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0
        torch.cuda.synchronize()
        st = out.status.cpu().numpy()
        tmo = (st & ssd.ROW_DEVICE_TIMEOUT) != 0
        # a row whose wait gave up carries the void-row outputs the row's
        # finish writes (a unit's own a_j may still land after it)
        assert np.all(out.n_accepted.cpu().numpy()[tmo] == -1)
        assert np.all(out.bonus.cpu().numpy()[tmo] == -1)
        assert np.all(out.hit.cpu().numpy()[tmo] == 0)
        assert np.all(out.slot.cpu().numpy()[tmo] == -1)
        err = C.c_int32(0)
        assert L.ssd_read_device_error(ws.ptr(), w.B, w.K, w.V, ssd.DTYPE_BF16,
                                       C.c_void_p(torch.cuda.current_stream().cuda_stream), C.byref(err)) == 0
        if tmo.any():
            assert err.value == SSD_ERR_TIMEOUT
        timed_out += int(tmo.sum())
        ws.reset()
    assert timed_out > 0, "no wait ran out at a 200 ns limit"
    # the normal library on the reset workspace: the oracle's answer again
    gpu = ssd.ssd_verify(t, d, tok, u, w.T, F=F, C_coef=w.C, budget=w.budget, cache=True,
                         fallback_seed=w.fallback_seed, workspace=ws)
    torch.cuda.synchronize()
    res = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in gpu.__dict__.items()}
    compare(case, res, case.run_oracle())
    assert ws.device_error() == 0
