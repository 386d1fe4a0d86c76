"""GPU parity of the split-KV decode kernels against the CPU oracle (C ABI)."""
import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from parity_helpers import bf16_host, check_counts, check_rows, check_tiles, to_device
from brute_force import decode_dense
from synth import DecodeWorkload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()


def run_gpu(w, x, tsf=None, splits=None):
    q = to_device(x["q"])
    kc, vc = to_device(x["kcache"]), to_device(x["vcache"])
    lens = torch.from_numpy(x["seqlens"]).cuda()
    out = sk.decode(q, kc, vc, lens, sm_scale=w.scale,
                    threshold_scale_factor=w.tsf if tsf is None else tsf, Bc=w.Bc,
                    num_splits=w.num_splits if splits is None else splits, with_tiles=True)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    c = out["counts"].cpu().numpy()
    return {"o": bf16_host(out["o"]), "lse": out["lse"].cpu().numpy(),
            "tile_state": out["tile_state"].cpu().numpy(), "skipped": int(c[0]),
            "visited": int(c[1])}


def compare(w, x, g, ora):
    check_counts(g["skipped"], ora["skipped"], g["visited"], ora["visited"])
    diff = check_tiles(g["tile_state"], ora["tile_state"], ora["tile_margin"])
    flipped = np.nonzero(diff.any(axis=2))
    ok = np.ones((w.B, w.Hq), bool)
    G = w.Hq // w.Hkv
    for b, h in zip(*flipped):
        ok[b, h * G:(h + 1) * G] = False
    check_rows(g["o"][ok], g["lse"][ok], ora["o"][ok], ora["lse"][ok], what="decode")
    if (~ok).any():
        # near-tie flips: the GPU result must be attention over its own kept tiles
        o_ref, lse_ref = decode_dense(x["q"], x["kcache"], x["vcache"], x["seqlens"],
                                      scale=w.scale, tile_state=g["tile_state"], Bc=w.Bc)
        check_rows(g["o"][~ok], g["lse"][~ok], o_ref[~ok], lse_ref[~ok], what="decode flips")


def small(**kw):
    base = dict(name="td", B=3, Hq=8, Hkv=2, Lmax=300, Lmin=1, d=128, Bc=64, num_splits=4,
                tsf=4.0, seed=31)
    base.update(kw)
    return DecodeWorkload(**base)


SEQLENS = np.array([300, 17, 129], np.int32)


@pytest.mark.parametrize("reading", ["lit", "rms"])
@pytest.mark.parametrize("w", [
    small(), small(num_splits=1), small(num_splits=16), small(d=64),
    small(Hq=2, Hkv=2), small(Hq=4, Hkv=2, d=64), small(Hq=16, Hkv=2),
    small(tsf=0.0), small(tsf=1e5), small(Lmax=1000, num_splits=64),
], ids=lambda w: f"d{w.d}G{w.Hq // w.Hkv}S{w.num_splits}t{w.tsf:g}L{w.Lmax}")
def test_decode_small(w, reading):
    x = synth.decode_inputs(w, reading, seqlens=SEQLENS if w.Lmax == 300 else
                            np.array([1000, 1, 640], np.int32))
    g = run_gpu(w, x)
    ora = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=w.scale,
                        tsf=w.tsf, Bc=w.Bc, num_splits=w.num_splits, want_margin=True)
    compare(w, x, g, ora)
    if w.tsf == 0:
        assert g["skipped"] == 0


@pytest.mark.parametrize("reading", ["lit", "rms"])
def test_decode_full_workload(reading):
    w = synth.DECODE_B64_32K
    x = synth.decode_inputs(w, reading)
    g = run_gpu(w, x)
    ora = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=w.scale,
                        tsf=w.tsf, Bc=w.Bc, num_splits=w.num_splits, want_margin=True)
    compare(w, x, g, ora)
    n_k = -(-x["seqlens"].astype(np.int64) // w.Bc)
    assert g["visited"] == int(n_k.sum()) * w.Hkv
