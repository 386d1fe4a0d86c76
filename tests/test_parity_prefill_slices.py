"""GPU parity of the warp-granular vote (32-row slices, the SpargeAttn
article's "稀疏 Warp 在线 Softmax" granularity) against the CPU oracle, through
sskip_attn_prefill_vote.

Small cases are compared in full; the 16K Llama-8B-shaped workload runs at
full size and is compared on sampled query tiles. A slice decision may differ
from the oracle's only at a near-tie of that slice's fp64 margin; a unit with
such a flip is compared with fp64 attention restricted, row by row, to the
GPU's own kept (slice, tile) pairs.
"""
import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from parity_helpers import (COUNT_REL, NEAR_TIE, bf16_host, check_counts, check_rows, note_flips,
                            to_device, unit_slice_margins, unit_slice_restricted_reference)
from synth import PrefillWorkload

pytestmark = pytest.mark.gpu

R = 32


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()


def run_gpu(w, x, vote_rows=R, tsf=None):
    q, k, v = to_device(x["q"]), to_device(x["k"]), to_device(x["v"])
    out = sk.prefill(q, k, v, causal=w.causal, sm_scale=w.scale,
                     threshold_scale_factor=w.tsf if tsf is None else tsf, Br=w.Br, Bc=w.Bc,
                     with_tiles=True, vote_rows=vote_rows)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    c = out["counts"].cpu().numpy()
    return {"o": bf16_host(out["o"]), "lse": out["lse"].cpu().numpy(),
            "tile_state": out["tile_state"].cpu().numpy(),
            "slice_mask": out["slice_mask"].cpu().numpy(),
            "skipped": int(c[0]), "visited": int(c[1]),
            "slices_skipped": int(c[2]), "slices_visited": int(c[3])}


def compare_units(w, x, g, ora, units, tsf):
    """ora: per-unit oracle outputs (o [n,Br,d], lse [n,Br], slice_mask [n,n_k])."""
    flips = 0
    for n, (b, hq, i) in enumerate(units):
        r0, r1 = i * w.Br, min(w.L, (i + 1) * w.Br)
        sm_g = g["slice_mask"][b, hq, i]
        sm_o = ora["slice_mask"][n]
        assert np.array_equal(sm_g == 0, sm_o == 0), f"visit sets differ in {(b, hq, i)}"
        diff_bits = (sm_g ^ sm_o) & 0x7F
        flipped = []
        if diff_bits.any():
            marg = unit_slice_margins(x, w, b, hq, i, R, tsf)
            for j in np.nonzero(diff_bits)[0]:
                for s in range(w.Br // R):
                    if diff_bits[j] >> s & 1:
                        assert abs(marg[s, j]) < NEAR_TIE, (b, hq, i, j, s, marg[s, j])
                        flipped.append(marg[s, j])
                        flips += 1
        note_flips(int((sm_o != 0).sum()) * (w.Br // R), flipped)
        if diff_bits.any():
            o_ref, lse_ref = unit_slice_restricted_reference(x, w, b, hq, i, sm_g, R)
        else:
            o_ref, lse_ref = ora["o"][n, :r1 - r0], ora["lse"][n, :r1 - r0]
        check_rows(g["o"][b, hq, r0:r1], g["lse"][b, hq, r0:r1], o_ref, lse_ref,
                   what=f"unit {(b, hq, i)}")
    return flips


def small(**kw):
    base = dict(name="t", B=1, Hq=2, Hkv=1, L=1000, d=128, causal=True, Br=128, Bc=128,
                tsf=100.0, seed=33, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                sink_gain=3.0)
    base.update(kw)
    return PrefillWorkload(**base)


SMALL_CASES = [
    small(),
    small(B=2, Hq=4, Hkv=2, L=700, d=64, causal=False, tsf=60.0),
    small(Hq=2, Hkv=2, L=333, d=64, Br=64, Bc=64, tsf=30.0),
    small(Hq=4, Hkv=1, L=450, d=128, causal=False, Br=64, Bc=64, tsf=30.0),
    small(Hq=1, Hkv=1, L=40, tsf=10.0),                     # L < Bc: padding slices
    small(Hq=1, Hkv=1, L=77, d=64, Br=64, Bc=64, tsf=10.0),  # ragged, one padding slice
    small(Hq=4, Hkv=1, L=512, tsf=0.0),                     # dense control
]


def per_unit_oracle(w, x, tsf):
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale, tsf=tsf,
                         Br=w.Br, Bc=w.Bc, vote_rows=R)
    n_q = w.n_q
    o_pad = np.zeros((w.B, w.Hq, n_q * w.Br, w.d), np.float32)
    l_pad = np.zeros((w.B, w.Hq, n_q * w.Br), np.float32)
    o_pad[:, :, :w.L] = ora["o"]
    l_pad[:, :, :w.L] = ora["lse"]
    ou = {"o": o_pad.reshape(-1, w.Br, w.d), "lse": l_pad.reshape(-1, w.Br),
          "slice_mask": ora["slice_mask"].reshape(-1, w.n_k)}
    return ora, ou


@pytest.mark.parametrize("reading", ["lit", "rms"])
@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: f"L{w.L}d{w.d}B{w.Br}{'c' if w.causal else 'n'}t{w.tsf:g}")
def test_slice_vote_small_full_compare(w, reading):
    x = synth.prefill_inputs(w, reading)
    g = run_gpu(w, x)
    ora, ou = per_unit_oracle(w, x, w.tsf)
    check_counts(g["skipped"], ora["skipped"], g["visited"], ora["visited"])
    assert g["slices_visited"] == ora["slices_visited"]
    assert abs(g["slices_skipped"] - ora["slices_skipped"]) <= COUNT_REL * ora["slices_skipped"]
    units = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.n_q)]
    compare_units(w, x, g, ou, units, w.tsf)
    # The slice record agrees with the counters and with the block record.
    n_sl = w.Br // R
    full = 0x80 | ((1 << n_sl) - 1)
    sm, st = g["slice_mask"], g["tile_state"]
    assert np.array_equal(sm == 0, st == 0)
    assert np.array_equal(sm == full, st == 2)
    if w.tsf == 0:
        assert g["slices_skipped"] == 0 and g["skipped"] == 0


def test_slice_vote_block_decisions_match_block_vote():
    # While t < 1 both granularities take the same block decisions.
    w = synth.LLAMA8B_PREFILL_16K.replace(Hq=8, Hkv=2, L=4096)
    x = synth.prefill_inputs(w, "rms")
    g_sl = run_gpu(w, x)
    g_bl = run_gpu(w, x, vote_rows=w.Br)
    flips = g_sl["tile_state"] != g_bl["tile_state"]
    assert flips.sum() <= max(1, COUNT_REL * g_bl["skipped"])
    assert g_bl["slices_skipped"] == g_bl["skipped"] and g_bl["slices_visited"] == g_bl["visited"]
    assert g_sl["slices_skipped"] >= 4 * g_sl["skipped"]
    assert g_sl["slices_skipped"] > 4 * g_sl["skipped"], "the slice vote must add skips here"


@pytest.mark.parametrize("reading", ["lit", "rms"])
def test_slice_vote_llama8b_16k_sampled(reading):
    w = synth.LLAMA8B_PREFILL_16K
    x = synth.prefill_inputs(w, reading)
    g = run_gpu(w, x)
    rng = np.random.default_rng(5)
    i_vals = np.unique(np.concatenate([[0, w.n_q - 1], np.linspace(0, w.n_q - 1, 16).astype(int)]))
    units = [(0, int(rng.integers(w.Hq)), int(i)) for i in i_vals]
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=True, sm_scale=w.scale, tsf=w.tsf,
                         Br=w.Br, Bc=w.Bc, vote_rows=R, units=np.array(units, np.int32))
    compare_units(w, x, g, ora, units, w.tsf)
    n = w.n_q
    assert g["visited"] == w.Hq * n * (n + 1) // 2
    assert g["slices_visited"] == 4 * g["visited"]
    assert int((g["tile_state"] == 2).sum()) == g["skipped"]
