"""Pins for the CPU oracle (no GPU).

The oracle is checked against things other than itself: fp64 brute-force
dense attention, dense attention restricted to the kept tiles, the prefix-max
closed form of the skip set, invariants (V = 1 gives O = 1, unit row sums),
hand-built planted cases whose decision is fixed by construction, the
threshold t = threshold_scale_factor / L at the exact switching point, and the
pages' own configuration numbers.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth
from brute_force import (decode_dense, decode_prefix_max_states, dense_attention,
                         prefix_max_row_passes, prefix_max_states, restricted_attention,
                         slice_masks, slice_restricted_attention)
from synth import PrefillWorkload, DecodeWorkload, bf16_bits, bf16_to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_prefill(**kw):
    base = dict(name="t", B=1, Hq=2, Hkv=1, L=200, d=32, causal=True, Br=64, Bc=64,
                tsf=8.0, seed=7, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                sink_gain=3.0)
    base.update(kw)
    return PrefillWorkload(**base)


def run_prefill(w, x, precision="f32", tsf=None, **kw):
    return oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale,
                          tsf=w.tsf if tsf is None else tsf, Br=w.Br, Bc=w.Bc,
                          precision=precision, **kw)


# --------------------------------------------------------------------------
# tsf = 0 reproduces dense softmax attention (plug-and-play: no retraining).
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", [
    dict(Hq=1, Hkv=1, L=256, d=16, Br=64, Bc=64),
    dict(Hq=4, Hkv=2, L=200, d=64, Br=64, Bc=64),       # GQA, ragged tail
    dict(Hq=2, Hkv=2, L=300, d=32, Br=128, Bc=128),     # ragged tail at 128
    dict(Hq=2, Hkv=1, L=40, d=16, Br=64, Bc=64),        # L < Bc
])
@pytest.mark.parametrize("precision", ["f32", "f64"])
def test_tsf0_equals_dense(causal, shape, precision):
    w = small_prefill(causal=causal, tsf=0.0, **shape)
    x = synth.prefill_inputs(w, "rms")
    got = run_prefill(w, x, precision)
    O, lse = dense_attention(x["q"], x["k"], x["v"], causal=causal, scale=w.scale)
    tol = 2e-5 if precision == "f32" else 1e-11
    assert got["skipped"] == 0
    np.testing.assert_allclose(got["o"], O, atol=tol, rtol=0)
    np.testing.assert_allclose(got["lse"], lse, atol=tol, rtol=0)


def test_visited_tile_count_closed_form():
    # causal with Br = Bc visits n_q (n_q + 1) / 2 tiles per head.
    w = small_prefill(L=1000, Br=64, Bc=64, Hq=3, Hkv=1)
    got = run_prefill(w, synth.prefill_inputs(w, "lit"))
    n = -(-1000 // 64)
    assert got["visited"] == 3 * n * (n + 1) // 2
    w2 = w.replace(causal=False)
    got2 = run_prefill(w2, synth.prefill_inputs(w2, "lit"))
    assert got2["visited"] == 3 * n * n


# --------------------------------------------------------------------------
# Skip semantics: output = dense attention restricted to the kept tiles.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("precision", ["f32", "f64"])
@pytest.mark.parametrize("kw", [
    dict(causal=True, L=512, Br=64, Bc=64, tsf=100.0),
    dict(causal=False, L=333, Br=64, Bc=64, tsf=30.0, Hq=4, Hkv=2),
    dict(causal=True, L=700, Br=128, Bc=128, tsf=40.0, d=64),
])
def test_output_equals_restricted_dense(precision, kw):
    w = small_prefill(**kw)
    x = synth.prefill_inputs(w, "rms")
    got = run_prefill(w, x, precision)
    assert 0 < got["skipped"] < got["visited"], "case must exercise both branches"
    O, lse = restricted_attention(x["q"], x["k"], x["v"], got["tile_state"], causal=w.causal,
                                  scale=w.scale, Br=w.Br, Bc=w.Bc)
    tol = 3e-5 if precision == "f32" else 1e-11
    np.testing.assert_allclose(got["o"], O, atol=tol, rtol=0)
    np.testing.assert_allclose(got["lse"], lse, atol=tol, rtol=0)


@pytest.mark.parametrize("kw", [
    dict(causal=True, L=512, Br=64, Bc=64, tsf=100.0),
    dict(causal=False, L=333, Br=64, Bc=64, tsf=30.0, Hq=4, Hkv=2),
    dict(causal=True, L=1000, Br=128, Bc=128, tsf=100.0, d=64, Hq=2),
    dict(causal=True, L=1024, Br=64, Bc=64, tsf=100.0, d=64, Hq=1, q_shift=1.0,
         hot_frac=0.1, hot_gain=4.0, sink_keys=0, sink_gain=0.0),
])
def test_skip_set_equals_prefix_max_closed_form(kw):
    w = small_prefill(**kw)
    assert w.tsf / w.L < 1
    x = synth.prefill_inputs(w, "rms")
    got = run_prefill(w, x, "f64")
    want = prefix_max_states(x["q"], x["k"], causal=w.causal, scale=w.scale, tsf=w.tsf,
                             Br=w.Br, Bc=w.Bc)
    assert (want == 2).sum() > 0
    np.testing.assert_array_equal(got["tile_state"], want)
    # fp32 oracle: identical except at near-ties of the margin.
    got32 = run_prefill(w, x, "f32", want_margin=True)
    diff = got32["tile_state"] != want
    assert np.all(np.abs(got32["tile_margin"][diff]) < 1e-4)
    assert diff.sum() <= max(1, int(0.005 * got32["visited"]))


def test_v_all_ones_gives_ones():
    # O = sum_k p_k * 1 / sum_k p_k = 1 whatever is skipped: pins the shared
    # alpha rescale of the numerator and of the row sum.
    w = small_prefill(L=384, tsf=20.0, Hq=2, Hkv=2)
    x = synth.prefill_inputs(w, "rms")
    x["v"] = np.full_like(x["v"], bf16_bits(np.float32([1.0]))[0])
    got = run_prefill(w, x, "f32")
    assert got["skipped"] > 0
    np.testing.assert_allclose(got["o"], 1.0, atol=2e-6)


def test_row_sums_are_one_with_one_hot_values():
    # V = identity: O[r] is the restricted softmax row itself; its sum is 1.
    w = small_prefill(L=64, d=64, Br=16, Bc=16, Hq=1, Hkv=1, causal=True, tsf=2.0)
    x = synth.prefill_inputs(w, "rms")
    x["v"] = bf16_bits(np.eye(64, dtype=np.float32))[None, None]
    got = run_prefill(w, x, "f64")
    assert got["skipped"] > 0
    P = got["o"][0, 0]
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-12)
    # Keys of skipped tiles carry exactly zero probability.
    st = got["tile_state"][0, 0]
    for i in range(st.shape[0]):
        for j in range(st.shape[1]):
            if st[i, j] == 2:
                assert np.all(P[i * 16:(i + 1) * 16, j * 16:(j + 1) * 16] == 0)


# --------------------------------------------------------------------------
# Hand-built planted case: decisions fixed by construction.
# --------------------------------------------------------------------------
def planted_case():
    """d = 16, Bc = Br = 16, L = 64, non-causal, scale = 1/4, all q rows = 4 e0.
    Tile 0 holds key 0 = 8 e0 (logit 8). Tile 1 holds key 16 = 7 e0 (logit 7,
    one below the max: mildly low). Tile 2 keys = -8 e0 (logit -8: 16 below).
    Tile 3 keys = 0 (logit 0: 8 below). Other keys of tiles 0, 1 are zero."""
    d, L = 16, 64
    q = np.zeros((1, 1, L, d), np.float32)
    q[..., 0] = 4.0
    k = np.zeros((1, 1, L, d), np.float32)
    k[0, 0, 0, 0] = 8.0
    k[0, 0, 16, 0] = 7.0
    k[0, 0, 32:48, 0] = -8.0
    rng = np.random.default_rng(3)
    v = rng.standard_normal((1, 1, L, d)).astype(np.float32)
    return {"q": bf16_bits(q), "k": bf16_bits(k), "v": bf16_bits(v)}


@pytest.mark.parametrize("precision", ["f32", "f64"])
def test_planted_far_below_tile_is_skipped(precision):
    x = planted_case()
    # ln t = -4: tile 1 (gap 1) kept, tile 2 (gap 16) and tile 3 (gap 8) skipped.
    tsf = 64 * math.exp(-4.0)
    got = oracle.prefill(x["q"], x["k"], x["v"], causal=False, sm_scale=0.25, tsf=tsf,
                         Br=16, Bc=16, precision=precision)
    assert got["tile_state"].shape == (1, 1, 4, 4)
    for i in range(4):
        assert list(got["tile_state"][0, 0, i]) == [1, 1, 2, 2]
    assert got["skipped"] == 8 and got["visited"] == 16
    # Kept keys are exactly tiles 0 and 1; compare with the closed form.
    st = got["tile_state"]
    O, lse = restricted_attention(x["q"], x["k"], x["v"], st, causal=False, scale=0.25,
                                  Br=16, Bc=16)
    np.testing.assert_allclose(got["o"], O, atol=1e-5)
    # lse by hand: one key at 8, one at 7, 30 keys at 0.
    want_lse = math.log(math.exp(8) + math.exp(7) + 30.0)
    np.testing.assert_allclose(got["lse"], want_lse, atol=1e-5)


def test_threshold_is_scale_factor_over_L_in_natural_log():
    # Tile 1's local max sits exactly g = 3 below tile 0's (logits 8 and 5,
    # built from exact bf16 values). It is skipped iff e^{-3} < t = tsf / L,
    # i.e. iff tsf > L e^{-3}. A missing 1/L, a log2 for ln or an unscaled
    # logit moves this switching point.
    d, L = 16, 32
    q = np.zeros((1, 1, L, d), np.float32)
    q[..., 0] = 4.0
    k = np.zeros((1, 1, L, d), np.float32)
    k[0, 0, 0, 0] = 8.0
    k[0, 0, 16, 0] = 5.0
    v = np.ones((1, 1, L, d), np.float32)
    x = {"q": bf16_bits(q), "k": bf16_bits(k), "v": bf16_bits(v)}
    switch = L * math.exp(-3.0)
    for precision in ("f32", "f64"):
        lo = oracle.prefill(x["q"], x["k"], x["v"], causal=False, sm_scale=0.25,
                            tsf=switch * (1 - 1e-4), Br=16, Bc=16, precision=precision)
        hi = oracle.prefill(x["q"], x["k"], x["v"], causal=False, sm_scale=0.25,
                            tsf=switch * (1 + 1e-4), Br=16, Bc=16, precision=precision)
        assert list(lo["tile_state"][0, 0, 0]) == [1, 1]
        assert list(hi["tile_state"][0, 0, 0]) == [1, 2]


def test_first_tile_never_skipped_and_tsf0_never_skips():
    w = small_prefill(L=512, tsf=1e6)  # t >= 1: everything after tile 0 may pass
    x = synth.prefill_inputs(w, "rms")
    got = run_prefill(w, x, "f64")
    assert np.all(got["tile_state"][..., :, 0] == 1)
    got0 = run_prefill(w, x, "f64", tsf=0.0)
    assert got0["skipped"] == 0


def test_skip_count_monotone_in_threshold():
    w = small_prefill(L=768, Hq=2, Hkv=1)
    x = synth.prefill_inputs(w, "rms")
    counts = [run_prefill(w, x, "f64", tsf=t)["skipped"] for t in (0.0, 1.0, 4.0, 16.0, 64.0)]
    assert counts == sorted(counts) and counts[-1] > 0


def test_pages_threshold_numbers():
    g = json.load(open(os.path.join(GOLDEN, "pages_threshold.json")))
    # t = threshold_scale_factor / L for the pages' factors at the workloads' L.
    for tsf, L in ((g["threshold_scale_factor"]["prefill"], 16384),
                   (g["threshold_scale_factor"]["decode"], 32768)):
        t = tsf / L
        # A planted gap just above / below ln(1/t) flips the decision.
        d = 16
        q = np.zeros((1, 1, 32, d), np.float32)
        q[..., 0] = 4.0
        k = np.zeros((1, 1, 32, d), np.float32)
        k[0, 0, 0, 0] = 8.0
        k[0, 0, 16, 0] = 5.0
        x = {"q": bf16_bits(q), "k": bf16_bits(k), "v": bf16_bits(np.ones_like(q))}
        # gap 3 vs ln(1/t): scale tsf so that the call's own L = 32 sees the same t.
        tsf_call = t * 32
        got = oracle.prefill(x["q"], x["k"], x["v"], causal=False, sm_scale=0.25,
                             tsf=tsf_call, Br=16, Bc=16, precision="f64")
        want = 2 if math.exp(-3.0) < t else 1
        assert got["tile_state"][0, 0, 0, 1] == want
    # The premise: exp(-100) is negligible next to exp(-1).
    a, b = g["premise_exponents"]
    assert math.exp(a) / math.exp(b) < 1e-40


# --------------------------------------------------------------------------
# GQA head mapping: query head hq reads kv head hq // G.
# --------------------------------------------------------------------------
def test_gqa_equals_replicated_mha():
    w = small_prefill(Hq=8, Hkv=2, L=300, tsf=16.0)
    x = synth.prefill_inputs(w, "rms")
    gqa = run_prefill(w, x, "f32")
    G = w.Hq // w.Hkv
    wm = w.replace(Hkv=w.Hq)
    xm = {"q": x["q"], "k": np.repeat(x["k"], G, axis=1), "v": np.repeat(x["v"], G, axis=1)}
    mha = run_prefill(wm, xm, "f32")
    np.testing.assert_array_equal(gqa["o"], mha["o"])
    np.testing.assert_array_equal(gqa["lse"], mha["lse"])
    np.testing.assert_array_equal(gqa["tile_state"], mha["tile_state"])
    assert gqa["skipped"] > 0


def test_units_subset_matches_full_run():
    w = small_prefill(Hq=4, Hkv=2, L=500, tsf=16.0, B=2)
    x = synth.prefill_inputs(w, "rms")
    full = run_prefill(w, x, "f32")
    units = np.array([[1, 3, 7], [0, 0, 0], [1, 1, 3]], np.int32)
    sub = run_prefill(w, x, "f32", units=units)
    for n, (b, h, i) in enumerate(units):
        r0, r1 = i * w.Br, min(w.L, (i + 1) * w.Br)
        np.testing.assert_array_equal(sub["o"][n, :r1 - r0], full["o"][b, h, r0:r1])
        np.testing.assert_array_equal(sub["lse"][n, :r1 - r0], full["lse"][b, h, r0:r1])
        np.testing.assert_array_equal(sub["tile_state"][n], full["tile_state"][b, h, i])


# --------------------------------------------------------------------------
# Decode: split layout, joint GQA vote, LSE merge.
# --------------------------------------------------------------------------
def small_decode(**kw):
    base = dict(name="td", B=3, Hq=8, Hkv=2, Lmax=300, Lmin=1, d=32, Bc=16, num_splits=4,
                tsf=4.0, seed=11)
    base.update(kw)
    return DecodeWorkload(**base)


def run_decode(w, x, precision="f32", **kw):
    args = dict(sm_scale=w.scale, tsf=w.tsf, Bc=w.Bc, num_splits=w.num_splits,
                precision=precision)
    args.update(kw)
    return oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], **args)


SEQLENS = np.array([300, 17, 129], np.int32)


@pytest.mark.parametrize("splits", [1, 4, 16])
@pytest.mark.parametrize("precision", ["f32", "f64"])
def test_decode_tsf0_equals_dense(splits, precision):
    w = small_decode(tsf=0.0, num_splits=splits)
    x = synth.decode_inputs(w, "rms", seqlens=SEQLENS)
    got = run_decode(w, x, precision)
    O, lse = decode_dense(x["q"], x["kcache"], x["vcache"], x["seqlens"], scale=w.scale)
    tol = 2e-5 if precision == "f32" else 1e-11
    assert got["skipped"] == 0
    np.testing.assert_allclose(got["o"], O, atol=tol, rtol=0)
    np.testing.assert_allclose(got["lse"], lse, atol=tol, rtol=0)


def test_decode_split_count_invariance_at_tsf0():
    w = small_decode(tsf=0.0, Lmax=2048, B=2)
    x = synth.decode_inputs(w, "rms", seqlens=np.array([2048, 1500], np.int32))
    a = run_decode(w, x, num_splits=1)
    b = run_decode(w, x, num_splits=16)
    np.testing.assert_allclose(a["o"], b["o"], atol=1e-5)
    np.testing.assert_allclose(a["lse"], b["lse"], atol=1e-5)


@pytest.mark.parametrize("splits", [1, 4, 16])
def test_decode_restricted_dense_and_prefix_max(splits):
    w = small_decode(num_splits=splits, tsf=4.0)
    x = synth.decode_inputs(w, "rms", seqlens=SEQLENS)
    got = run_decode(w, x, "f64", want_partials=True)
    assert 0 < got["skipped"] < got["visited"]
    want = decode_prefix_max_states(x["q"], x["kcache"], x["seqlens"], scale=w.scale,
                                    tsf=w.tsf, Bc=w.Bc, num_splits=splits)
    np.testing.assert_array_equal(got["tile_state"], want)
    O, lse = decode_dense(x["q"], x["kcache"], x["vcache"], x["seqlens"], scale=w.scale,
                          tile_state=got["tile_state"], Bc=w.Bc)
    np.testing.assert_allclose(got["o"], O, atol=1e-11)
    np.testing.assert_allclose(got["lse"], lse, atol=1e-11)
    # Empty splits (L_b = 17 gives 2 tiles) carry lse = -inf and O = 0.
    n_k = -(-17 // w.Bc)
    c = -(-n_k // splits)
    empty = [s for s in range(splits) if s * c >= n_k]
    for s in empty:
        assert np.all(got["lse_part"][1, :, s] == -np.inf)
        assert np.all(got["o_part"][1, :, s] == 0)


def test_decode_threshold_uses_each_sequence_length():
    # Same cache content, two lengths: t_b = tsf / L_b differs per sequence.
    d, Bc = 16, 16
    q = np.zeros((2, 1, d), np.float32)
    q[..., 0] = 4.0
    kc = np.zeros((2, 1, 64, d), np.float32)
    kc[:, 0, 0, 0] = 8.0
    kc[:, 0, 16, 0] = 5.0   # gap 3 below the max
    x = {"q": bf16_bits(q), "kcache": bf16_bits(kc), "vcache": bf16_bits(np.ones_like(kc)),
         "seqlens": np.array([32, 64], np.int32)}
    # tsf between 32 e^-3 and 64 e^-3: t_0 = tsf/32 > e^-3 (skip), t_1 = tsf/64 < e^-3.
    tsf = 48 * math.exp(-3.0)
    got = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=0.25, tsf=tsf,
                        Bc=Bc, num_splits=1, precision="f64")
    assert got["tile_state"][0, 0, 1] == 2
    assert got["tile_state"][1, 0, 1] == 1


def test_decode_joint_vote_needs_every_head():
    # Two heads share a kv head. Head 0 finds tile 1 far below its max, head 1
    # finds tile 1 at its max: the joint vote keeps the tile.
    d, Bc = 16, 16
    q = np.zeros((1, 2, d), np.float32)
    q[0, 0, 0] = 4.0
    q[0, 1, 1] = 4.0
    kc = np.zeros((1, 1, 32, d), np.float32)
    kc[0, 0, 0, 0] = 8.0     # head 0 max in tile 0
    kc[0, 0, 16, 1] = 8.0    # head 1 max in tile 1
    x = {"q": bf16_bits(q), "kcache": bf16_bits(kc), "vcache": bf16_bits(np.ones_like(kc)),
         "seqlens": np.array([32], np.int32)}
    got = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=0.25,
                        tsf=32 * math.exp(-1.0), Bc=Bc, num_splits=1, precision="f64")
    assert list(got["tile_state"][0, 0]) == [1, 1]
    q1 = q.copy()
    q1[0, 1] = q[0, 0]
    x["q"] = bf16_bits(q1)
    got = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=0.25,
                        tsf=32 * math.exp(-1.0), Bc=Bc, num_splits=1, precision="f64")
    assert list(got["tile_state"][0, 0]) == [1, 2]


def test_oracle_rejects_bad_arguments():
    w = small_prefill()
    x = synth.prefill_inputs(w, "lit")
    with pytest.raises(ValueError):
        oracle.prefill(x["q"], x["k"][:, :1, :10], x["v"], causal=True, sm_scale=1, tsf=1,
                       Br=64, Bc=64)
    with pytest.raises(ValueError):
        oracle.prefill(x["q"], x["k"], x["v"], causal=True, sm_scale=1, tsf=-1, Br=64, Bc=64)


# --------------------------------------------------------------------------
# Warp-granular vote (SpargeAttn article, "稀疏 Warp 在线 Softmax" stage:
# the local-vs-global maximum test per warp): slices of R rows vote alone.
# --------------------------------------------------------------------------
SLICE_CASES = [
    dict(causal=True, L=512, Br=128, Bc=128, tsf=60.0, d=32, R=32),
    dict(causal=True, L=700, Br=128, Bc=128, tsf=40.0, d=64, R=32, Hq=4, Hkv=2),
    dict(causal=False, L=333, Br=64, Bc=64, tsf=30.0, R=32, Hq=2, Hkv=1),
    dict(causal=True, L=448, Br=128, Bc=128, tsf=50.0, d=32, R=64),
]


def _slice_case(kw):
    kw = dict(kw)
    R = kw.pop("R")
    w = small_prefill(**kw)
    return w, R, synth.prefill_inputs(w, "rms")


@pytest.mark.parametrize("kw", SLICE_CASES)
def test_slice_votes_equal_prefix_max_closed_form(kw):
    w, R, x = _slice_case(kw)
    assert w.tsf / w.L < 1
    got = run_prefill(w, x, "f64", vote_rows=R)
    passes, visited = prefix_max_row_passes(x["q"], x["k"], causal=w.causal, scale=w.scale,
                                            tsf=w.tsf, Br=w.Br, Bc=w.Bc)
    want = slice_masks(passes, visited, L=w.L, Br=w.Br, R=R)
    np.testing.assert_array_equal(got["slice_mask"], want)
    # The block decision is the AND of the slices (every slice bit set).
    full = np.uint8(0x80 | ((1 << (w.Br // R)) - 1))
    np.testing.assert_array_equal(got["tile_state"] == 2, want == full)
    # Slices that vote to skip while their block is kept: the variant's gain.
    assert np.any((want != full) & (want & 0x7F != 0) & (want != 0)), "case must hit partial skips"


@pytest.mark.parametrize("precision", ["f32", "f64"])
@pytest.mark.parametrize("kw", SLICE_CASES)
def test_slice_vote_output_equals_row_restricted_dense(kw, precision):
    w, R, x = _slice_case(kw)
    got = run_prefill(w, x, precision, vote_rows=R)
    O, lse = slice_restricted_attention(x["q"], x["k"], x["v"], got["slice_mask"],
                                        causal=w.causal, scale=w.scale, Br=w.Br, Bc=w.Bc, R=R)
    tol = 3e-5 if precision == "f32" else 1e-11
    np.testing.assert_allclose(got["o"], O, atol=tol, rtol=0)
    np.testing.assert_allclose(got["lse"], lse, atol=tol, rtol=0)


@pytest.mark.parametrize("kw", SLICE_CASES)
def test_slice_vote_keeps_block_decisions_and_counts(kw):
    # While t < 1 a passing row never moves its maximum, so the running maxima
    # and hence the block decisions are the same under both granularities.
    w, R, x = _slice_case(kw)
    blk = run_prefill(w, x, "f64")
    sl = run_prefill(w, x, "f64", vote_rows=R)
    np.testing.assert_array_equal(blk["tile_state"], sl["tile_state"])
    assert (blk["skipped"], blk["visited"]) == (sl["skipped"], sl["visited"])
    n_sl = w.Br // R
    mask = sl["slice_mask"]
    bits = np.unpackbits(mask[..., None], axis=-1)[..., -n_sl:].sum()
    # Counters: slices holding a valid row. Bits of empty (padding) slices are set
    # but not counted.
    n_q = -(-w.L // w.Br)
    rows_last = w.L - (n_q - 1) * w.Br
    empty_last = n_sl - (-(-rows_last // R))
    vis_last = int((mask[:, :, -1, :] != 0).sum())
    assert sl["slices_visited"] == n_sl * sl["visited"] - empty_last * vis_last
    assert sl["slices_skipped"] == bits - empty_last * vis_last
    assert sl["slices_skipped"] >= n_sl * sl["skipped"] - empty_last * vis_last
    # vote_rows = Br: one slice per tile, same counts as the blocks.
    assert (blk["slices_skipped"], blk["slices_visited"]) == (blk["skipped"], blk["visited"])


def test_slice_vote_planted_case():
    # 32 query rows, Br = 32, R = 16, Bc = 16, non-causal, scale 1/4.
    # Rows 0-15 (slice 0) have q = 4 e0, rows 16-31 (slice 1) q = 4 e1.
    # Key tile 0: key 0 = 8 e0 + 8 e1 (logit 8 for every row).
    # Key tile 1: key 16 = 7.5 e1 and key 17 = 0: slice 0 sees max logit 0
    #   (gap 8: passes at ln t = -4), slice 1 sees 7.5 (gap 0.5: fails).
    # The block is kept, slice 0 skips it, slice 1 keeps it.
    d, L = 16, 32
    q = np.zeros((1, 1, L, d), np.float32)
    q[0, 0, :16, 0] = 4.0
    q[0, 0, 16:, 1] = 4.0
    k = np.zeros((1, 1, L, d), np.float32)
    k[0, 0, 0, 0] = 8.0
    k[0, 0, 0, 1] = 8.0
    k[0, 0, 16, 1] = 7.5
    v = np.ones((1, 1, L, d), np.float32)
    v[0, 0, 16:, :] = 3.0
    x = {"q": bf16_bits(q), "k": bf16_bits(k), "v": bf16_bits(v)}
    tsf = L * math.exp(-4.0)
    for precision in ("f32", "f64"):
        got = oracle.prefill(x["q"], x["k"], x["v"], causal=False, sm_scale=0.25, tsf=tsf,
                             Br=32, Bc=16, vote_rows=16, precision=precision)
        assert list(got["tile_state"][0, 0, 0]) == [1, 1]
        assert list(got["slice_mask"][0, 0, 0]) == [0x80, 0x80 | 0b01]
        assert (got["slices_skipped"], got["slices_visited"]) == (1, 4)
        # slice 0: only tile 0 -> all V = 1 -> O = 1; lse = ln(e^8 + 15).
        np.testing.assert_allclose(got["o"][0, 0, :16], 1.0, atol=1e-6)
        np.testing.assert_allclose(got["lse"][0, 0, :16], math.log(math.exp(8) + 15), atol=1e-5)
        # slice 1: tile 0 (one key at 8, 15 at 0; V = 1) + tile 1 (one key at
        # 7.5, 15 at 0; V = 3).
        num = math.exp(8) + 15 + 3 * (math.exp(7.5) + 15)
        den = math.exp(8) + 15 + math.exp(7.5) + 15
        np.testing.assert_allclose(got["o"][0, 0, 16:], num / den, rtol=1e-5)
        np.testing.assert_allclose(got["lse"][0, 0, 16:], math.log(den), atol=1e-5)
        blk = oracle.prefill(x["q"], x["k"], x["v"], causal=False, sm_scale=0.25, tsf=tsf,
                             Br=32, Bc=16, precision=precision)
        np.testing.assert_allclose(blk["o"][0, 0, :16],
                                   (math.exp(8) + 15 + 3 * 16) / (math.exp(8) + 15 + 16),
                                   rtol=1e-5)


def test_slice_vote_rejects_bad_rows():
    w = small_prefill(L=128, Br=64, Bc=64)
    x = synth.prefill_inputs(w, "lit")
    for R in (0, 48, 65, 8):   # not a divisor, too large, or more than 7 slices
        with pytest.raises(ValueError):
            run_prefill(w, x, vote_rows=R)
