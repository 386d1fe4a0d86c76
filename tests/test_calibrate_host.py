"""The library's host-side factor selection (sskip_calibrate_factor, no CUDA
call) on critical values from the fp64 closed form, checked against skip
counts of the CPU oracle at the returned factor."""
import math

import numpy as np
import pytest

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from brute_force import decode_critical_factors, prefill_critical_factors
from synth import DecodeWorkload, PrefillWorkload


def _w(**kw):
    base = dict(name="t", B=1, Hq=2, Hkv=1, L=512, d=32, causal=True, Br=64, Bc=64, tsf=8.0,
                seed=23, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4, sink_gain=3.0)
    base.update(kw)
    return PrefillWorkload(**base)


@pytest.mark.parametrize("target", [0.05, 0.2, 0.3])
@pytest.mark.parametrize("kw", [dict(), dict(causal=False, L=333, Hq=4, Hkv=2, Br=128, Bc=128)])
def test_prefill_selection_hits_target_on_oracle(target, kw):
    w = _w(**kw)
    x = synth.prefill_inputs(w, "rms")
    crit = prefill_critical_factors(x["q"], x["k"], causal=w.causal, scale=w.scale, Br=w.Br,
                                    Bc=w.Bc)
    r = sk.sskip_calibrate_factor(crit.astype(np.float32), target, float(w.L))
    got = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale,
                         tsf=r["factor"], Br=w.Br, Bc=w.Bc, precision="f64")
    assert got["visited"] == r["visited"]
    assert got["skipped"] == round(r["achieved_ratio"] * r["visited"])
    assert r["achieved_ratio"] >= target
    # No smaller share reaches the target: one tile fewer would miss it.
    assert (got["skipped"] - 1) / got["visited"] < target or got["skipped"] == 0


def test_decode_selection_hits_target_on_oracle():
    w = DecodeWorkload(name="t", B=3, Hq=4, Hkv=2, d=32, Lmin=300, Lmax=600, Bc=64,
                       num_splits=2, tsf=8.0, seed=5)
    x = synth.decode_inputs(w, "rms")
    crit = decode_critical_factors(x["q"], x["kcache"], x["seqlens"], scale=w.scale, Bc=w.Bc,
                                   num_splits=w.num_splits)
    r = sk.sskip_calibrate_factor(crit.astype(np.float32), 0.3, float(x["seqlens"].min()))
    got = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=w.scale,
                        tsf=r["factor"], Bc=w.Bc, num_splits=w.num_splits, precision="f64")
    assert got["visited"] == r["visited"]
    assert got["skipped"] == round(r["achieved_ratio"] * r["visited"])
    assert r["achieved_ratio"] >= 0.3


def test_selection_edge_cases():
    c = np.array([np.nan, np.inf, 1.0, 2.0, 3.0, 3.0, -np.inf, 5.0], np.float32)
    assert sk.sskip_calibrate_factor(c, 0.0, 100.0)["factor"] == 0.0
    r = sk.sskip_calibrate_factor(c, 0.1, 100.0)       # only the -inf tile
    assert 0 < r["factor"] <= math.e and r["achieved_ratio"] == pytest.approx(1 / 7)
    r = sk.sskip_calibrate_factor(c, 0.3, 100.0)       # between 2 and 3
    assert math.log(r["factor"]) == pytest.approx(2.5) and r["achieved_ratio"] == pytest.approx(3 / 7)
    r = sk.sskip_calibrate_factor(c, 0.5, 100.0)       # tie at 3, capped by ln 100
    assert math.log(r["factor"]) == pytest.approx((3 + math.log(100)) / 2)
    assert r["achieved_ratio"] == pytest.approx(5 / 7)
    with pytest.raises(sk.SSkipError):
        sk.sskip_calibrate_factor(c, 0.9, 100.0)       # needs the +inf tile
    with pytest.raises(sk.SSkipError):
        sk.sskip_calibrate_factor(c, 0.8, 100.0)       # needs 5 > ln 100
    with pytest.raises(sk.SSkipError):
        sk.sskip_calibrate_factor(np.full(4, np.nan, np.float32), 0.5, 10.0)
