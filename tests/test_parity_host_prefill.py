"""GPU checks of the host-buffer prefill and decode (sskip_attn_prefill_host,
sskip_attn_decode_host): for every way of cutting the kv heads into groups,
pinned or pageable host memory, their outputs and skip counts are
bit-identical to the one-shot device call, and on one case each they are
compared with the CPU oracle directly."""
import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from brute_force import decode_dense
from parity_helpers import check_counts, check_rows, check_tiles, compare_prefill_units, to_device
from synth import PrefillWorkload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()


def host_bf16(bits, pin):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pin else t.clone()


@pytest.mark.parametrize("kv_per_chunk", [0, 1, 3, 8])
@pytest.mark.parametrize("pin", [True, False])
@pytest.mark.parametrize("w", [
    PrefillWorkload(name="h", B=2, Hq=8, Hkv=4, L=700, d=128, causal=True, Br=128, Bc=128,
                    tsf=60.0, seed=71, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                    sink_gain=3.0),
    PrefillWorkload(name="h", B=1, Hq=6, Hkv=3, L=333, d=64, causal=False, Br=64, Bc=64,
                    tsf=30.0, seed=72, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                    sink_gain=3.0),
], ids=["gqa_causal_d128", "noncausal_d64_br64"])
def test_host_prefill_equals_device_call(w, pin, kv_per_chunk):
    x = synth.prefill_inputs(w, "rms")
    q, k, v = to_device(x["q"]), to_device(x["k"]), to_device(x["v"])
    ref = sk.prefill(q, k, v, causal=w.causal, sm_scale=w.scale, threshold_scale_factor=w.tsf,
                     Br=w.Br, Bc=w.Bc)
    host = {n: host_bf16(x[n], pin) for n in ("q", "k", "v")}
    host["o"] = torch.empty_like(host["q"])
    host["lse"] = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32)
    if pin:
        host["o"], host["lse"] = host["o"].pin_memory(), host["lse"].pin_memory()
    dev = {n: torch.empty_like(t, device="cuda") for n, t in host.items()}
    cnt = torch.zeros(2, dtype=torch.int64, device="cuda")
    sk.sskip_attn_prefill_host(host, dev, causal=w.causal, sm_scale=w.scale,
                               threshold_scale_factor=w.tsf, Br=w.Br, Bc=w.Bc,
                               kv_per_chunk=kv_per_chunk, skip_count=cnt)
    torch.cuda.current_stream().synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    assert torch.equal(host["o"], ref["o"].cpu())
    assert torch.equal(host["lse"], ref["lse"].cpu())
    assert cnt.cpu().tolist() == ref["counts"].cpu().tolist()
    assert ref["counts"].cpu().tolist()[0] > 0


def test_host_prefill_against_oracle():
    # The workload as written (literal reading): the host path's copies and
    # chunking are what this checks; its skip path is covered above by the
    # bit-identity with the device call on the rms reading.
    w = PrefillWorkload(name="h", B=2, Hq=8, Hkv=4, L=700, d=128, causal=True, Br=128, Bc=128,
                        tsf=60.0, seed=76, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                        sink_gain=3.0)
    x = synth.prefill_inputs(w, "lit")
    host = {n: host_bf16(x[n], True) for n in ("q", "k", "v")}
    host["o"] = torch.empty_like(host["q"]).pin_memory()
    host["lse"] = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32).pin_memory()
    dev = {n: torch.empty_like(t, device="cuda") for n, t in host.items()}
    cnt = torch.zeros(2, dtype=torch.int64, device="cuda")
    sk.sskip_attn_prefill_host(host, dev, causal=w.causal, sm_scale=w.scale,
                               threshold_scale_factor=w.tsf, Br=w.Br, Bc=w.Bc, kv_per_chunk=1,
                               skip_count=cnt)
    torch.cuda.current_stream().synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    # The host call records no tiles; the device call's record (bit-identical
    # run) tells which units flipped a near-tie decision.
    rec = sk.prefill(to_device(x["q"]), to_device(x["k"]), to_device(x["v"]), causal=w.causal,
                     sm_scale=w.scale, threshold_scale_factor=w.tsf, Br=w.Br, Bc=w.Bc,
                     with_tiles=True)
    units = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.n_q)]
    ora = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale, tsf=w.tsf,
                         Br=w.Br, Bc=w.Bc, units=np.array(units, np.int32), want_margin=True)
    c = cnt.cpu().tolist()
    check_counts(c[0], ora["skipped"], c[1], ora["visited"])
    g = {"o": host["o"].float().numpy(), "lse": host["lse"].numpy(),
         "tile_state": rec["tile_state"].cpu().numpy()}
    compare_prefill_units(w, x, g, ora, units)


def test_host_prefill_twice_in_a_row_reuses_the_staging_buffers():
    w = PrefillWorkload(name="h", B=1, Hq=4, Hkv=2, L=512, d=128, causal=True, Br=128, Bc=128,
                        tsf=60.0, seed=73)
    outs = []
    for seed in (73, 74):
        x = synth.prefill_inputs(w.replace(seed=seed), "rms")
        host = {n: host_bf16(x[n], True) for n in ("q", "k", "v")}
        host["o"] = torch.empty_like(host["q"]).pin_memory()
        host["lse"] = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32).pin_memory()
        if not outs:
            dev = {n: torch.empty_like(t, device="cuda") for n, t in host.items()}
        sk.sskip_attn_prefill_host(host, dev, causal=True, sm_scale=w.scale,
                                   threshold_scale_factor=w.tsf, kv_per_chunk=1)
        ref = sk.prefill(to_device(x["q"]), to_device(x["k"]), to_device(x["v"]), causal=True,
                         sm_scale=w.scale, threshold_scale_factor=w.tsf)
        torch.cuda.synchronize()
        assert torch.equal(host["o"], ref["o"].cpu())
        outs.append(host["o"])
    assert not torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("pin", [True, False])
def test_host_decode_equals_device_call(pin):
    from synth import DecodeWorkload
    w = DecodeWorkload(name="hd", B=5, Hq=8, Hkv=2, d=128, Lmin=200, Lmax=1500, Bc=64,
                       num_splits=4, tsf=40.0, seed=75)
    x = synth.decode_inputs(w, "rms")
    kc, vc = to_device(x["kcache"]), to_device(x["vcache"])
    lens = torch.from_numpy(x["seqlens"]).cuda()
    q = to_device(x["q"])
    ref = sk.decode(q, kc, vc, lens, sm_scale=w.scale, threshold_scale_factor=w.tsf, Bc=w.Bc,
                    num_splits=w.num_splits)
    host = {"q": host_bf16(x["q"], pin), "seqlens": torch.from_numpy(x["seqlens"]).clone(),
            "o": torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16),
            "lse": torch.empty((w.B, w.Hq), dtype=torch.float32)}
    if pin:
        host = {n: t.pin_memory() for n, t in host.items()}
    dev = {n: torch.empty_like(t, device="cuda") for n, t in host.items()}
    ws = torch.empty(sk.sskip_attn_decode_workspace_size(w.B, w.Hq, w.d, w.num_splits),
                     dtype=torch.uint8, device="cuda")
    cnt = torch.zeros(2, dtype=torch.int64, device="cuda")
    sk.sskip_attn_decode_host(host, dev, kc, vc, sm_scale=w.scale, threshold_scale_factor=w.tsf,
                              Bc=w.Bc, num_splits=w.num_splits, workspace=ws, skip_count=cnt)
    torch.cuda.current_stream().synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    assert torch.equal(host["o"], ref["o"].cpu()) and torch.equal(host["lse"], ref["lse"].cpu())
    assert cnt.cpu().tolist() == ref["counts"].cpu().tolist() and cnt.cpu().tolist()[0] > 0
    if not pin:
        return
    # Direct comparison with the oracle (near-tie flips, if any, against fp64
    # attention over the GPU's own kept tiles).
    rec = sk.decode(q, kc, vc, lens, sm_scale=w.scale, threshold_scale_factor=w.tsf, Bc=w.Bc,
                    num_splits=w.num_splits, with_tiles=True)
    ora = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=w.scale,
                        tsf=w.tsf, Bc=w.Bc, num_splits=w.num_splits, want_margin=True)
    c = cnt.cpu().tolist()
    check_counts(c[0], ora["skipped"], c[1], ora["visited"])
    st = rec["tile_state"].cpu().numpy()
    diff = check_tiles(st, ora["tile_state"], ora["tile_margin"])
    o_h, lse_h = host["o"].float().numpy(), host["lse"].numpy()
    if diff.any():
        o_ref, lse_ref = decode_dense(x["q"], x["kcache"], x["vcache"], x["seqlens"],
                                      scale=w.scale, tile_state=st, Bc=w.Bc)
    else:
        o_ref, lse_ref = ora["o"], ora["lse"]
    check_rows(o_h, lse_h, o_ref, lse_ref, what="decode host")
