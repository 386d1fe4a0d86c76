"""Pin of the oracle's per-tile margin output (no GPU).

The oracle records, for every visited tile, the margin
min over valid rows of (ln t - (m_local - m_run)). A tile is skipped iff that
margin is positive (TensorRT-LLM Skip-Softmax article, "Skip Softmax 的三步走
算法" section, with t = threshold_scale_factor / L from its "实战演练" section).
The GPU parity tests use this margin to tell a near-tie decision flip (fp32
accumulation order) from a wrong vote, so it is pinned here against a closed
form computed without the oracle: while t < 1 no skipped tile can raise a
row's running maximum, so m_run before tile j is the prefix maximum of the
row's local maxima, and the margin equals ln(tsf) - c with
c = max_rows (m_local - prefix_max) + ln L, the critical value that
``brute_force.prefill_critical_factors`` / ``decode_critical_factors`` compute
in fp64 from the logits alone.

A sign error, a margin taken over the wrong rows (padding rows, one row, a
max instead of a min) or a wrong L in t changes these values and fails here.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from brute_force import decode_critical_factors, prefill_critical_factors
from synth import DecodeWorkload, PrefillWorkload


def _prefill_case(**kw):
    base = dict(name="m", B=1, Hq=2, Hkv=1, L=200, d=32, causal=True, Br=64, Bc=64,
                tsf=8.0, seed=11, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                sink_gain=3.0)
    base.update(kw)
    return PrefillWorkload(**base)


def _expected_margin(ln_tsf, crit):
    with np.errstate(invalid="ignore"):
        return ln_tsf - crit


PREFILL_CASES = [
    # causal, Br = Bc = 64, full tiles
    dict(causal=True, L=512, Br=64, Bc=64, tsf=100.0),
    # non-causal GQA with a ragged last query tile: 333 = 5 * 64 + 13, so the
    # last tile has 51 padding rows that must not enter the margin
    dict(causal=False, L=333, Br=64, Bc=64, tsf=30.0, Hq=4, Hkv=2),
    # Br = Bc = 128 with padding rows (333 = 2 * 128 + 77), causal, d = 64
    dict(causal=True, L=333, Br=128, Bc=128, tsf=20.0, d=64, Hq=2, Hkv=2),
    # a longer causal case at 128 with GQA
    dict(causal=True, L=700, Br=128, Bc=128, tsf=40.0, d=64, Hq=4, Hkv=1),
]


@pytest.mark.parametrize("kw", PREFILL_CASES)
@pytest.mark.parametrize("reading", ["rms", "lit"])
def test_prefill_margin_equals_closed_form(kw, reading):
    w = _prefill_case(**kw)
    assert w.tsf / w.L < 1
    x = synth.prefill_inputs(w, reading)
    crit = prefill_critical_factors(x["q"], x["k"], causal=w.causal, scale=w.scale, Br=w.Br,
                                    Bc=w.Bc)
    want = _expected_margin(math.log(w.tsf), crit)
    visited = ~np.isnan(crit)
    for precision, tol in (("f64", 1e-9), ("f32", 5e-5)):
        got = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale,
                             tsf=w.tsf, Br=w.Br, Bc=w.Bc, precision=precision, want_margin=True)
        m = got["tile_margin"].astype(np.float64)
        assert np.array_equal(got["tile_state"] > 0, visited)
        # infinite margins (a row that cannot pass: nothing kept before) match exactly
        inf = visited & np.isinf(want)
        assert np.array_equal(m[inf], want[inf])
        fin = visited & np.isfinite(want)
        assert fin.sum() > 0
        np.testing.assert_allclose(m[fin], want[fin], atol=tol, rtol=0)
        # and the margin decides the recorded state (away from exact ties)
        clear = fin & (np.abs(want) > 10 * tol)
        assert np.array_equal(got["tile_state"][clear] == 2, want[clear] > 0)


@pytest.mark.parametrize("G,splits", [(4, 4), (1, 3), (8, 2)])
def test_decode_margin_equals_closed_form(G, splits):
    Hkv = 2
    w = DecodeWorkload(name="m", B=3, Hq=G * Hkv, Hkv=Hkv, Lmax=700, Lmin=1, d=64, Bc=64,
                       num_splits=splits, tsf=6.0, seed=13)
    x = synth.decode_inputs(w, "rms", seqlens=np.array([700, 333, 65], np.int32))
    crit = decode_critical_factors(x["q"], x["kcache"], x["seqlens"], scale=w.scale, Bc=w.Bc,
                                   num_splits=w.num_splits)
    want = _expected_margin(math.log(w.tsf), crit)
    visited = ~np.isnan(crit)
    for precision, tol in (("f64", 1e-9), ("f32", 5e-5)):
        got = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=w.scale,
                            tsf=w.tsf, Bc=w.Bc, num_splits=w.num_splits, precision=precision,
                            want_margin=True)
        assert np.array_equal(got["tile_state"] > 0, visited)
        m = got["tile_margin"].astype(np.float64)
        inf = visited & np.isinf(want)
        assert inf.sum() > 0  # every split's first tile
        assert np.array_equal(m[inf], want[inf])
        fin = visited & np.isfinite(want)
        assert fin.sum() > 0 and (want[fin] > 0).sum() > 0
        np.testing.assert_allclose(m[fin], want[fin], atol=tol, rtol=0)
        clear = fin & (np.abs(want) > 10 * tol)
        assert np.array_equal(got["tile_state"][clear] == 2, want[clear] > 0)
