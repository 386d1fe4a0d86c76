"""GPU checks of the serving-step call: each phase runs with its own factor,
and the step equals the two separate calls bit for bit (and so the oracle)."""
import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from parity_helpers import bf16_host, check_counts, check_rows, to_device
from synth import DecodeWorkload, PrefillWorkload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()


def make_case():
    pw = PrefillWorkload(name="p", B=1, Hq=8, Hkv=2, L=1000, d=128, causal=True, Br=128, Bc=128,
                         tsf=0.0, seed=61, q_shift=0.5, hot_frac=0.15, hot_gain=2.0,
                         sink_keys=4, sink_gain=3.0)
    dw = DecodeWorkload(name="d", B=4, Hq=8, Hkv=2, d=128, Lmin=900, Lmax=3000, Bc=64,
                        num_splits=4, tsf=0.0, seed=62)
    px = synth.prefill_inputs(pw, "rms")
    dx = synth.decode_inputs(dw, "rms")
    P = {"q": to_device(px["q"]), "k": to_device(px["k"]), "v": to_device(px["v"])}
    P["o"] = torch.empty_like(P["q"])
    P["lse"] = torch.empty((pw.B, pw.Hq, pw.L), dtype=torch.float32, device="cuda")
    P["count"] = torch.zeros(2, dtype=torch.int64, device="cuda")
    D = {"q": to_device(dx["q"]), "kcache": to_device(dx["kcache"]),
         "vcache": to_device(dx["vcache"]), "seqlens": torch.from_numpy(dx["seqlens"]).cuda()}
    D["o"] = torch.empty_like(D["q"])
    D["lse"] = torch.empty((dw.B, dw.Hq), dtype=torch.float32, device="cuda")
    D["workspace"] = torch.empty(sk.sskip_attn_decode_workspace_size(dw.B, dw.Hq, dw.d,
                                                                     dw.num_splits),
                                 dtype=torch.uint8, device="cuda")
    D["count"] = torch.zeros(2, dtype=torch.int64, device="cuda")
    return pw, dw, px, dx, P, D


def run_step(pw, dw, P, D, factors):
    sk.sskip_attn_step(threshold_scale_factor=factors, sm_scale=pw.scale, prefill=P, decode=D,
                       Br=pw.Br, Bc=pw.Bc, causal=pw.causal, num_splits=dw.num_splits)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    return P["count"].cpu().tolist(), D["count"].cpu().tolist()


def test_each_phase_gets_its_own_factor():
    pw, dw, px, dx, P, D = make_case()
    cp, cd = run_step(pw, dw, P, D, {"prefill": 100.0, "decode": 0.0})
    assert cp[0] > 0 and cd[0] == 0
    cp, cd = run_step(pw, dw, P, D, {"prefill": 0.0, "decode": 50.0})
    assert cp[0] == 0 and cd[0] > 0
    cp2, cd2 = run_step(pw, dw, P, D, 50.0)  # one number: both phases
    assert cd2 == cd and cp2[0] > 0


def test_step_equals_separate_calls_and_the_oracle():
    pw, dw, px, dx, P, D = make_case()
    factors = {"prefill": 100.0, "decode": 50.0}
    cp, cd = run_step(pw, dw, P, D, factors)
    o_step, lse_step = P["o"].clone(), P["lse"].clone()
    do_step, dlse_step = D["o"].clone(), D["lse"].clone()
    sep_p = sk.prefill(P["q"], P["k"], P["v"], causal=True, sm_scale=pw.scale,
                       threshold_scale_factor=100.0, Br=pw.Br, Bc=pw.Bc)
    sep_d = sk.decode(D["q"], D["kcache"], D["vcache"], D["seqlens"], sm_scale=dw.scale,
                      threshold_scale_factor=50.0, Bc=dw.Bc, num_splits=dw.num_splits)
    torch.cuda.synchronize()
    assert torch.equal(o_step, sep_p["o"]) and torch.equal(lse_step, sep_p["lse"])
    assert torch.equal(do_step, sep_d["o"]) and torch.equal(dlse_step, sep_d["lse"])
    ora_p = oracle.prefill(px["q"], px["k"], px["v"], causal=True, sm_scale=pw.scale, tsf=100.0,
                           Br=pw.Br, Bc=pw.Bc)
    check_counts(cp[0], ora_p["skipped"], cp[1], ora_p["visited"])
    check_rows(bf16_host(o_step), lse_step.cpu().numpy(), ora_p["o"], ora_p["lse"], what="prefill")
    ora_d = oracle.decode(dx["q"], dx["kcache"], dx["vcache"], dx["seqlens"], sm_scale=dw.scale,
                          tsf=50.0, Bc=dw.Bc, num_splits=dw.num_splits)
    check_counts(cd[0], ora_d["skipped"], cd[1], ora_d["visited"])
    check_rows(bf16_host(do_step), dlse_step.cpu().numpy(), ora_d["o"], ora_d["lse"], what="decode")


def test_step_with_one_phase_only():
    pw, dw, px, dx, P, D = make_case()
    sk.sskip_attn_step(threshold_scale_factor=50.0, sm_scale=dw.scale, decode=D,
                       num_splits=dw.num_splits)
    torch.cuda.synchronize()
    assert D["count"].cpu().tolist()[0] > 0


def test_step_replayed_from_a_cuda_graph_equals_eager():
    pw, dw, px, dx, P, D = make_case()
    factors = {"prefill": 100.0, "decode": 50.0}
    run_step(pw, dw, P, D, factors)
    eager = [P["o"].clone(), P["lse"].clone(), D["o"].clone(), D["lse"].clone(),
             P["count"].clone(), D["count"].clone()]
    for t in (P["o"], D["o"]):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside capture (attributes, descriptors)
        sk.sskip_attn_step(threshold_scale_factor=factors, sm_scale=pw.scale, prefill=P,
                           decode=D, num_splits=dw.num_splits)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        sk.sskip_attn_step(threshold_scale_factor=factors, sm_scale=pw.scale, prefill=P,
                           decode=D, num_splits=dw.num_splits)
    for t in (P["o"], D["o"], P["count"], D["count"]):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    got = [P["o"], P["lse"], D["o"], D["lse"], P["count"], D["count"]]
    for a, b in zip(got, eager):
        assert torch.equal(a, b)
    del g
