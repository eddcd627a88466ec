"""The C ABI library builds, loads without a GPU, exports every symbol that
include/ssd.h declares, and rejects bad arguments on the host (no launch)."""
import ctypes as C
import os
import re

import pytest

from speculative_decoding_verify_ssd_b200 import binding as ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "ssd.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for must in ("ssd_verify", "ssd_fanout_plan", "ssd_saguaro_reweight", "ssd_cache_build",
                 "ssd_cache_lookup", "ssd_workspace_bytes", "ssd_status_string", "ssd_version"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ssd.load()
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} missing from libssd.so"


def test_status_strings_and_version():
    assert "sm_100a" in ssd.version()
    for code in range(8):
        assert ssd.status_string(code)


def test_workspace_size_formula():
    n = ssd.workspace_bytes(64, 6, 128256, ssd.DTYPE_BF16)
    # at least one slice partial (>= 1056 bytes) per (row, position) unit
    assert n % 256 == 0 and n >= 64 * 7 * 1056
    assert ssd.workspace_bytes(64, 6, 128256, ssd.DTYPE_BF16) <= ssd.workspace_bytes(64, 6, 262144, ssd.DTYPE_BF16)
    L = ssd.load()
    assert L.ssd_workspace_bytes(1, 0, 10, 1) == 0
    assert L.ssd_workspace_bytes(1, 2, 0, 1) == 0
    assert L.ssd_workspace_bytes(1, 2, 10, 9) == 0


def test_host_validation_without_gpu():
    L = ssd.load()
    null = None
    # bad dtype, bad K, negative B, T < 0: rejected before any CUDA call
    # target, draft, draft_next, dtype, B, K, V, tokens, uniforms, T, F, alpha, mode, C, budget,
    # n_accepted, bonus, out_tokens, accept_prob, residual_mass, cache, status, ws, ws_bytes, stream
    args = [null, null, null, 7, 4, 2, 100, null, null, C.c_float(1.0), null, null, 0, C.c_float(0.5), 0,
            null, null, null, null, null, null, null, null, 0, null]
    assert L.ssd_verify(*args) == 2          # dtype
    args[3] = 1
    args[5] = 0
    assert L.ssd_verify(*args) == 1          # K = 0
    args[5] = 2
    args[4] = -1
    assert L.ssd_verify(*args) == 1          # B < 0
    args[4] = 4
    args[9] = C.c_float(-1.0)
    assert L.ssd_verify(*args) == 1          # T < 0
    args[9] = C.c_float(1.0)
    args[4] = 0
    assert L.ssd_verify(*args) == 0          # B = 0: nothing to do
    assert L.ssd_fanout_plan(null, 4, 2, 10000, 0, null, null) == 1
    assert L.ssd_fanout_plan(null, 0, 2, 10, 0, null, null) == 0
    assert L.ssd_cache_lookup(null, null, 3, 0, 4, null, null, null, 0, 10, null, null, null, null) == 1
    assert L.ssd_saguaro_reweight(null, 1, 2, 2, 10, C.c_float(1.0), null, C.c_float(2.0), 4, null, 0,
                                  null, null, null, null, null, null, null, null, 0, null) == 1


def test_oracle_and_product_share_no_source():
    prod = os.path.join(ROOT, "speculative_decoding_verify_ssd_b200")
    for dirpath, _, files in os.walk(prod):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "oracle.c" not in text and "liboracle" not in text, f
