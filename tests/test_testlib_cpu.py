"""The parity comparison itself, on the CPU: compare() must accept every
outcome an exact evaluation can give at a near-tie and reject the rest.
The oracle's own outputs stand in for the device's, so no GPU is needed."""
import numpy as np
import pytest

import oracle
from speculative_decoding_verify_ssd_b200 import synth

from ssd_testlib import NEAR_TIE, Case, _flip_uniform, compare


def _as_device(orc):
    """Oracle outputs renamed and typed as the binding returns them."""
    return dict(n_accepted=orc["n_accepted"].copy(), bonus=orc["bonus"].copy(),
                out_tokens=orc["out_tokens"].copy(), accept_prob=orc["accept_prob"].astype(np.float32),
                residual_mass=orc["residual_mass"].astype(np.float32), status=orc["status"].copy(),
                cache_offsets=orc["offsets"].copy(), cache_tokens=orc["cache_tokens"].copy(),
                hit=orc["hit"].copy(), slot=orc["slot"].copy(), next_tokens=orc["next_tokens"].copy())


@pytest.fixture(scope="module")
def case():
    w = synth.WORKLOADS["zipf_b16_k5_v32000_bf16"].replace(B=12, V=4096)
    c = Case(w)
    return c, c.run_oracle()


def test_exact_outputs_pass(case):
    c, orc = case
    compare(c, _as_device(orc), orc)


def test_bonus_outside_the_window_fails(case):
    c, orc = case
    dev = _as_device(orc)
    b = int(np.argmax(orc["bonus_margin"]))
    assert orc["bonus_margin"][b] >= NEAR_TIE and orc["bonus_lo"][b] == orc["bonus_hi"][b]
    dev["bonus"][b] = (dev["bonus"][b] + 1) % c.w.V
    dev["out_tokens"][b, dev["n_accepted"][b]] = dev["bonus"][b]
    with pytest.raises(AssertionError):
        compare(c, dev, orc)


def test_bonus_inside_a_wide_window_passes():
    # Zipf rows over a large vocabulary hold much residual mass on tokens far
    # below 1e-5 each, so some draws have windows of many tokens
    w = synth.WORKLOADS["zipf_b64_k6_v128256_bf16"].replace(B=16)
    c = Case(w)
    orc = c.run_oracle()
    wide = np.nonzero(orc["bonus_hi"] > orc["bonus_lo"])[0]
    assert wide.size, "no wide window in this case"
    dev = _as_device(orc)
    b = int(wide[0])
    alt = int(orc["bonus_hi"][b] if orc["bonus"][b] != orc["bonus_hi"][b] else orc["bonus_lo"][b])
    dev["bonus"][b] = alt
    dev["out_tokens"][b, dev["n_accepted"][b]] = alt
    # hit / slot / next must follow the device's own bonus
    lo, hi = orc["offsets"][b, dev["n_accepted"][b]], orc["offsets"][b, dev["n_accepted"][b] + 1]
    seg = list(orc["cache_tokens"][b, lo:hi])
    if alt in seg:
        dev["hit"][b], dev["slot"][b] = 1, lo + seg.index(alt)
        dev["next_tokens"][b] = -1
    else:
        dev["hit"][b], dev["slot"][b] = 0, -1
        dev["next_tokens"][b] = [oracle.fallback_token(w.fallback_seed, b, i, w.V) for i in range(w.K)]
    dev["residual_mass"][b] = orc["residual_mass"][b]
    compare(c, dev, orc)


def test_accept_tie_taken_the_other_way_passes(case):
    c, orc = case
    b, j = 3, 0
    a = float(orc["accept_prob"][b, j])
    assert 0.0 < a < 1.0
    # put u_j within a grid step of a_j on the accepting side
    c2 = Case(c.w, tokens=c.tokens)
    c2.g = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in c.g.items()}
    u = np.float32(a)
    if float(u) >= a:
        u = np.nextafter(u, np.float32(0))
    c2.g["uniforms"][b, j] = u
    orc2 = c2.run_oracle()
    assert orc2["accept_margin"][b] < NEAR_TIE and orc2["n_accepted"][b] >= 1
    # the device rejected there instead: exactly the oracle's flipped outcome
    c3 = Case(c.w, tokens=c.tokens)
    c3.g = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in c2.g.items()}
    c3.g["uniforms"][b, j] = _flip_uniform(a, accepted=True)
    dev = _as_device(orc2)
    flipped = _as_device(c3.run_oracle())
    for k in dev:
        if k not in ("cache_offsets", "cache_tokens", "accept_prob"):
            dev[k][b] = flipped[k][b]
    assert dev["n_accepted"][b] == 0
    compare(c2, dev, orc2)
    # an outcome that is neither is refused
    dev["n_accepted"][b] = 2
    with pytest.raises(AssertionError):
        compare(c2, dev, orc2)
