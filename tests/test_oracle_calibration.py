"""Pins of the calibration oracle (bisection on the factor over the CPU
oracle's skip counts) against the closed form: while t < 1 a tile is skipped
iff ln(tsf) exceeds its critical value max_r (m_local - prefix max) + ln L,
so the factor where the count first reaches k is exp of the k-th smallest
critical value (fp64 brute force, no tiled online softmax involved)."""
import math

import numpy as np
import pytest

import synth
from brute_force import decode_critical_factors, prefill_critical_factors
from oracle import calibrate
from synth import DecodeWorkload, PrefillWorkload


def small_prefill(**kw):
    base = dict(name="t", B=1, Hq=2, Hkv=1, L=512, d=32, causal=True, Br=64, Bc=64,
                tsf=8.0, seed=17, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                sink_gain=3.0)
    base.update(kw)
    return PrefillWorkload(**base)


def kth(crit, k):
    c = np.sort(crit[np.isfinite(crit)])
    return c[k - 1]


@pytest.mark.parametrize("target", [0.1, 0.3, 0.45])
@pytest.mark.parametrize("kw", [dict(), dict(causal=False, L=333, Hq=4, Hkv=2)])
def test_prefill_bisection_lands_on_closed_form_quantile(target, kw):
    w = small_prefill(**kw)
    x = synth.prefill_inputs(w, "rms")
    r = calibrate.calibrate_prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale,
                                    Br=w.Br, Bc=w.Bc, target_ratio=target, rtol=1e-7)
    crit = prefill_critical_factors(x["q"], x["k"], causal=w.causal, scale=w.scale, Br=w.Br,
                                    Bc=w.Bc)
    assert r["visited"] == int(np.isfinite(crit).sum() + np.isposinf(crit).sum())
    star = math.exp(kth(crit, r["k"]))
    assert r["lo"] <= star * (1 + 1e-9) and star <= r["hi"] * (1 + 1e-9), (r, star)
    assert r["k"] / r["visited"] >= target


@pytest.mark.parametrize("target", [0.2, 0.4])
def test_decode_bisection_lands_on_closed_form_quantile(target):
    w = DecodeWorkload(name="t", B=3, Hq=4, Hkv=2, d=32, Lmin=300, Lmax=600, Bc=64,
                       num_splits=2, tsf=8.0, seed=5, q_shift=0.5, hot_frac=0.15, hot_gain=2.0,
                       sink_keys=4, sink_gain=3.0)
    x = synth.decode_inputs(w, "rms")
    r = calibrate.calibrate_decode(x["q"], x["kcache"], x["vcache"], x["seqlens"],
                                   sm_scale=w.scale, Bc=w.Bc, num_splits=w.num_splits,
                                   target_ratio=target, rtol=1e-7)
    crit = decode_critical_factors(x["q"], x["kcache"], x["seqlens"], scale=w.scale, Bc=w.Bc,
                                   num_splits=w.num_splits)
    star = math.exp(kth(crit, r["k"]))
    assert r["lo"] <= star * (1 + 1e-9) and star <= r["hi"] * (1 + 1e-9), (r, star)


def test_bisection_rejects_unreachable_target():
    with pytest.raises(ValueError):
        calibrate.bisect_factor(lambda f: 3, 5, 1.0, 10.0)


def test_target_count():
    assert calibrate.target_count(0.5, 10) == 5
    assert calibrate.target_count(0.51, 10) == 6
    assert calibrate.target_count(0.0, 10) == 0
    assert calibrate.target_count(1.0, 10) == 10
