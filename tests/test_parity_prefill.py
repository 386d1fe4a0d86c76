"""GPU parity of the prefill kernel against the CPU oracle (through the C ABI).

Small cases span several tiles and a ragged tail and are compared in full;
the full-size workloads run in the launch configuration the benchmark times
and are compared on a seeded sample of whole query tiles the oracle computes
one by one (query tiles are independent), plus totals that hold at any size.
"""
import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from parity_helpers import (bf16_host, check_counts, check_rows, check_tiles, to_device,
                            unit_restricted_reference)
from synth import PrefillWorkload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()
    assert sk.lib().sskip_device_supported(torch.cuda.current_device()) == sk.SSKIP_OK


def run_gpu(w, x, tsf=None, dev=None):
    q, k, v = dev if dev is not None else (to_device(x["q"]), to_device(x["k"]), to_device(x["v"]))
    out = sk.prefill(q, k, v, causal=w.causal, sm_scale=w.scale,
                     threshold_scale_factor=w.tsf if tsf is None else tsf, Br=w.Br, Bc=w.Bc,
                     with_tiles=True)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    counts = out["counts"].cpu().numpy()
    return {"o": bf16_host(out["o"]), "lse": out["lse"].cpu().numpy(),
            "tile_state": out["tile_state"].cpu().numpy(), "skipped": int(counts[0]),
            "visited": int(counts[1])}


def compare_units(w, x, g, ora, units):
    """Compare GPU outputs with per-unit oracle outputs for (b, hq, i) units."""
    flips = 0
    for n, (b, hq, i) in enumerate(units):
        r0, r1 = i * w.Br, min(w.L, (i + 1) * w.Br)
        st_g = g["tile_state"][b, hq, i]
        diff = check_tiles(st_g, ora["tile_state"][n], ora["tile_margin"][n])
        if diff.any():
            flips += int(diff.sum())
            o_ref, lse_ref = unit_restricted_reference(x, w, b, hq, i, np.nonzero(st_g == 1)[0])
        else:
            o_ref, lse_ref = ora["o"][n, :r1 - r0], ora["lse"][n, :r1 - r0]
        check_rows(g["o"][b, hq, r0:r1], g["lse"][b, hq, r0:r1], o_ref, lse_ref,
                   what=f"unit {(b, hq, i)}")
    return flips


def small(**kw):
    base = dict(name="t", B=1, Hq=2, Hkv=1, L=1000, d=128, causal=True, Br=128, Bc=128, tsf=100.0,
                seed=21, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4, sink_gain=3.0)
    base.update(kw)
    return PrefillWorkload(**base)


SMALL_CASES = [
    small(),
    small(B=2, Hq=4, Hkv=2, L=700, d=64, causal=False, tsf=60.0),
    small(Hq=2, Hkv=2, L=333, d=64, Br=64, Bc=64, tsf=30.0),
    small(Hq=4, Hkv=1, L=450, d=128, causal=False, Br=64, Bc=64, tsf=30.0),
    small(Hq=1, Hkv=1, L=40, tsf=10.0),                   # L < Bc
    small(Hq=1, Hkv=1, L=1, d=64, Br=64, Bc=64, tsf=10.0),  # one row
    small(Hq=8, Hkv=1, L=512, tsf=0.0),                   # dense control, G = 8
    small(Hq=2, Hkv=2, L=640, tsf=1e6),                   # t >= 1
    small(B=3, Hq=2, Hkv=2, L=129, d=64, causal=False, Br=64, Bc=64, tsf=5.0),
]


@pytest.mark.parametrize("reading", ["lit", "rms"])
@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: f"L{w.L}d{w.d}B{w.Br}{'c' if w.causal else 'n'}G{w.Hq // w.Hkv}t{w.tsf:g}")
def test_prefill_small_full_compare(w, reading):
    x = synth.prefill_inputs(w, reading)
    g = run_gpu(w, x)
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale, tsf=w.tsf,
                         Br=w.Br, Bc=w.Bc, want_margin=True)
    check_counts(g["skipped"], ora["skipped"], g["visited"], ora["visited"])
    units = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.n_q)]
    per_unit = {"o": ora["o"], "lse": ora["lse"]}
    # reshape the full-layout oracle output into per-unit arrays
    n_q = w.n_q
    o_pad = np.zeros((w.B, w.Hq, n_q * w.Br, w.d), np.float32)
    l_pad = np.zeros((w.B, w.Hq, n_q * w.Br), np.float32)
    o_pad[:, :, :w.L] = per_unit["o"]
    l_pad[:, :, :w.L] = per_unit["lse"]
    ou = {"o": o_pad.reshape(w.B * w.Hq * n_q, w.Br, w.d),
          "lse": l_pad.reshape(-1, w.Br),
          "tile_state": ora["tile_state"].reshape(-1, w.n_k),
          "tile_margin": ora["tile_margin"].reshape(-1, w.n_k)}
    compare_units(w, x, g, ou, units)
    if w.tsf == 0:
        assert g["skipped"] == 0


@pytest.mark.parametrize("reading", ["lit", "rms"])
def test_tiny_prefill_workload(reading):
    w = synth.TINY_PREFILL
    x = synth.prefill_inputs(w, reading)
    g = run_gpu(w, x)
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=True, sm_scale=w.scale, tsf=w.tsf,
                         Br=w.Br, Bc=w.Bc, want_margin=True)
    check_counts(g["skipped"], ora["skipped"], g["visited"], ora["visited"])
    check_tiles(g["tile_state"], ora["tile_state"], ora["tile_margin"])
    check_rows(g["o"], g["lse"], ora["o"], ora["lse"], what="tiny")
    if reading == "rms":
        assert g["skipped"] > 0


def sample_units(w, n, seed):
    rng = np.random.default_rng(seed)
    i_vals = np.unique(np.concatenate([[0, w.n_q - 1], np.linspace(0, w.n_q - 1, n).astype(int)]))
    units = []
    for i in i_vals:
        units.append((int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(i)))
    return units


def full_size_check(w, reading, n_units, tsf=None, x=None, dev=None):
    x = synth.prefill_inputs(w, reading) if x is None else x
    g = run_gpu(w, x, tsf=tsf, dev=dev)
    tsf = w.tsf if tsf is None else tsf
    units = sample_units(w, n_units, seed=w.seed)
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale, tsf=tsf,
                         Br=w.Br, Bc=w.Bc, units=np.array(units, np.int32), want_margin=True)
    compare_units(w, x, g, ora, units)
    # Totals that hold at any size.
    n = w.n_q
    want_visited = w.B * w.Hq * (n * (n + 1) // 2 if w.causal else n * w.n_k)
    assert g["visited"] == want_visited
    st = g["tile_state"]
    assert int((st == 2).sum()) == g["skipped"] and int((st > 0).sum()) == g["visited"]
    assert np.all(st[..., 0] == 1)  # the first tile of every row is kept
    if tsf == 0:
        assert g["skipped"] == 0
    return g


@pytest.mark.parametrize("reading", ["lit", "rms"])
def test_llama8b_prefill_16k(reading):
    full_size_check(synth.LLAMA8B_PREFILL_16K, reading, n_units=24)


def test_videodit_prefill():
    full_size_check(synth.VIDEO_DIT_PREFILL, "lit", n_units=12)


@pytest.mark.parametrize("reading", ["lit", "rms"])
def test_llama70b_prefill_128k_sweep(reading):
    # The 128K workload at every factor of its sweep, in the launch the
    # benchmark times; 32 query tiles spread over the diagonal (plus both ends)
    # are compared with the oracle at each factor.
    w = synth.LLAMA70B_PREFILL_128K
    x = synth.prefill_inputs(w, reading)
    dev = (to_device(x["q"]), to_device(x["k"]), to_device(x["v"]))
    for tsf in synth.LLAMA70B_TSF_SWEEP:
        full_size_check(w, reading, n_units=32, tsf=tsf, x=x, dev=dev)
