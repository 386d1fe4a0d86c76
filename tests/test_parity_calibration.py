"""GPU parity of the critical-value records (sskip_attn_prefill_vote's and
sskip_attn_decode_crit's tile_crit) and of threshold calibration.

The oracle's per-tile margin ln t - max_r (m_local - m_run) gives the
critical value c = ln(tsf) - margin at any factor below L; the GPU record must
match it (same +inf / NaN pattern, finite values within NEAR_TIE). The factor
the GPU calibration returns must then skip the target share of tiles on the
GPU and on the oracle alike.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from parity_helpers import COUNT_REL, CRIT_LOG, NEAR_TIE, note_flips, to_device
from synth import DecodeWorkload, PrefillWorkload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()


def small(**kw):
    base = dict(name="t", B=1, Hq=2, Hkv=1, L=1000, d=128, causal=True, Br=128, Bc=128,
                tsf=100.0, seed=41, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                sink_gain=3.0)
    base.update(kw)
    return PrefillWorkload(**base)


PREFILL_CASES = [
    small(),
    small(B=2, Hq=4, Hkv=2, L=700, d=64, causal=False),
    small(Hq=2, Hkv=2, L=333, d=64, Br=64, Bc=64),
]


def check_crit(gpu, ref):
    assert np.array_equal(np.isnan(gpu), np.isnan(ref)), "visit sets differ"
    assert np.array_equal(np.isposinf(gpu), np.isposinf(ref)), "first tiles differ"
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(gpu), fin)
    d = np.abs(gpu[fin].astype(np.float64) - ref[fin])
    assert d.max() < NEAR_TIE, d.max()
    CRIT_LOG.append({"compared": int(fin.sum()), "worst": float(d.max())})


def gpu_prefill_crit(w, x):
    q, k, v = to_device(x["q"]), to_device(x["k"]), to_device(x["v"])
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=q.device)
    crit = torch.empty((w.B, w.Hq, w.n_q, w.n_k), dtype=torch.float32, device=q.device)
    sk.sskip_attn_prefill_vote(q, k, v, o, lse, causal=w.causal, sm_scale=w.scale,
                               threshold_scale_factor=w.tsf, Br=w.Br, Bc=w.Bc, vote_rows=w.Br,
                               tile_crit=crit)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    return crit.cpu().numpy(), (q, k, v)


@pytest.mark.parametrize("reading", ["lit", "rms"])
@pytest.mark.parametrize("w", PREFILL_CASES, ids=lambda w: f"L{w.L}d{w.d}B{w.Br}{'c' if w.causal else 'n'}")
def test_prefill_crit_record(w, reading):
    x = synth.prefill_inputs(w, reading)
    g, _ = gpu_prefill_crit(w, x)
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale, tsf=1.0,
                         Br=w.Br, Bc=w.Bc, want_margin=True)
    ref = np.where(ora["tile_state"] == 0, np.nan, 0.0 - ora["tile_margin"].astype(np.float64))
    check_crit(g, ref)


@pytest.mark.parametrize("target", [0.25, 0.5])
def test_prefill_calibration_small(target):
    w = small(L=2000, Hq=4, Hkv=2)
    x = synth.prefill_inputs(w, "rms")
    q, k, v = to_device(x["q"]), to_device(x["k"]), to_device(x["v"])
    r = sk.calibrate_prefill(q, k, v, causal=w.causal, sm_scale=w.scale, target_ratio=target,
                             Br=w.Br, Bc=w.Bc)
    assert r["achieved_ratio"] >= target
    want = round(r["achieved_ratio"] * r["visited"])
    out = sk.prefill(q, k, v, causal=w.causal, sm_scale=w.scale,
                     threshold_scale_factor=r["factor"], Br=w.Br, Bc=w.Bc)
    c = out["counts"].cpu().tolist()
    assert c[1] == r["visited"] and c[0] == want
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale,
                         tsf=r["factor"], Br=w.Br, Bc=w.Bc)
    assert abs(ora["skipped"] - want) <= max(1, COUNT_REL * want)


def test_prefill_calibration_llama8b_16k():
    w = synth.LLAMA8B_PREFILL_16K
    x = synth.prefill_inputs(w, "rms")
    q, k, v = to_device(x["q"]), to_device(x["k"]), to_device(x["v"])
    r = sk.calibrate_prefill(q, k, v, causal=True, sm_scale=w.scale, target_ratio=0.5)
    out = sk.prefill(q, k, v, causal=True, sm_scale=w.scale, threshold_scale_factor=r["factor"])
    c = out["counts"].cpu().tolist()
    assert c[1] == r["visited"]
    assert c[0] / c[1] >= 0.5 and abs(c[0] - r["achieved_ratio"] * c[1]) <= max(1, 1e-4 * c[1])
    # Sampled query tiles agree with the oracle at the calibrated factor.
    units = np.array([(0, h, i) for h, i in ((0, 127), (9, 64), (31, 100))], np.int32)
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=True, sm_scale=w.scale, tsf=r["factor"],
                         Br=w.Br, Bc=w.Bc, units=units, want_margin=True)
    crit = r["tile_crit"]
    for n, (b, h, i) in enumerate(units):
        g_skip = crit[b, h, i] < math.log(r["factor"])
        o_skip = ora["tile_state"][n] == 2
        flips = g_skip[:i + 1] != o_skip[:i + 1]
        assert np.all(np.abs(ora["tile_margin"][n][:i + 1][flips]) < NEAR_TIE)
        note_flips(i + 1, ora["tile_margin"][n][:i + 1][flips])


def decode_case():
    return DecodeWorkload(name="t", B=4, Hq=8, Hkv=2, d=128, Lmin=900, Lmax=3000, Bc=64,
                          num_splits=4, tsf=50.0, seed=9)


def test_decode_crit_record_and_calibration():
    w = decode_case()
    x = synth.decode_inputs(w, "rms")
    q, kc, vc = to_device(x["q"]), to_device(x["kcache"]), to_device(x["vcache"])
    lens = torch.from_numpy(x["seqlens"]).cuda()
    r = sk.calibrate_decode(q, kc, vc, lens, sm_scale=w.scale, target_ratio=0.4, Bc=w.Bc,
                            num_splits=w.num_splits)
    ora = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=w.scale,
                        tsf=1.0, Bc=w.Bc, num_splits=w.num_splits, want_margin=True)
    ref = np.where(ora["tile_state"] == 0, np.nan, 0.0 - ora["tile_margin"].astype(np.float64))
    check_crit(r["tile_crit"], ref)
    out = sk.decode(q, kc, vc, lens, sm_scale=w.scale, threshold_scale_factor=r["factor"],
                    Bc=w.Bc, num_splits=w.num_splits)
    c = out["counts"].cpu().tolist()
    assert c[1] == r["visited"] and c[0] == round(r["achieved_ratio"] * r["visited"])
    assert r["achieved_ratio"] >= 0.4


def test_decode_calibration_b64():
    w = synth.DECODE_B64_32K
    x = synth.decode_inputs(w, "rms")
    q, kc, vc = to_device(x["q"]), to_device(x["kcache"]), to_device(x["vcache"])
    lens = torch.from_numpy(x["seqlens"]).cuda()
    r = sk.calibrate_decode(q, kc, vc, lens, sm_scale=w.scale, target_ratio=0.5, Bc=w.Bc,
                            num_splits=w.num_splits)
    out = sk.decode(q, kc, vc, lens, sm_scale=w.scale, threshold_scale_factor=r["factor"],
                    Bc=w.Bc, num_splits=w.num_splits)
    c = out["counts"].cpu().tolist()
    assert c[1] == r["visited"] and c[0] / c[1] >= 0.5
    assert abs(c[0] - r["achieved_ratio"] * c[1]) <= max(1, 1e-4 * c[1])
