"""The debug build (libsskip_attn_debug.so) on the GPU: the same kernels with
device-side checks of tile, ring and record indices, the stand-in for a
memory checker. On valid inputs of every kernel configuration no check may
fail (status stays SSKIP_OK) and every output must be bit-identical to the
release build's, which the parity tests compare with the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import synth
from parity_helpers import to_device
from synth import DecodeWorkload, PrefillWorkload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()


def same_bits(a, b):
    """Bitwise equality (the records hold NaN for tiles never visited)."""
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def run_prefill(L, w, x, vote_rows):
    q, k, v = to_device(x["q"]), to_device(x["k"]), to_device(x["v"])
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device="cuda")
    cnt = torch.zeros(4, dtype=torch.int64, device="cuda")
    rec = (w.B, w.Hq, w.n_q, w.n_k)
    st = torch.empty(rec, dtype=torch.uint8, device="cuda")
    sm = torch.empty(rec, dtype=torch.uint8, device="cuda")
    cr = torch.empty(rec, dtype=torch.float32, device="cuda")
    rc = L.sskip_attn_prefill_vote(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), w.B, w.Hq, w.Hkv,
                                   w.L, w.d, int(w.causal), ctypes.c_float(w.scale),
                                   ctypes.c_float(w.tsf), w.Br, w.Bc, vote_rows, _ptr(cnt),
                                   _ptr(st), _ptr(sm), _ptr(cr), None)
    assert rc == sk.SSKIP_OK
    rc2 = L.sskip_attn_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), w.B, w.Hq,
                                  w.Hkv, w.L, w.d, int(w.causal), ctypes.c_float(w.scale),
                                  ctypes.c_float(w.tsf), w.Br, w.Bc, _ptr(cnt), _ptr(st), None)
    assert rc2 == sk.SSKIP_OK
    torch.cuda.synchronize()
    return {"o": o.cpu(), "lse": lse.cpu(), "cnt": cnt.cpu(), "st": st.cpu(), "sm": sm.cpu(),
            "cr": cr.cpu()}


def small(**kw):
    base = dict(name="dbg", B=1, Hq=4, Hkv=2, L=700, d=128, causal=True, Br=128, Bc=128,
                tsf=60.0, seed=81, q_shift=0.5, hot_frac=0.15, hot_gain=2.0, sink_keys=4,
                sink_gain=3.0)
    base.update(kw)
    return PrefillWorkload(**base)


@pytest.mark.parametrize("w", [
    small(),                                               # d128, two S buffers
    small(d=64, causal=False, B=2, Hq=2, Hkv=2, L=333),    # d64, three S buffers
    small(Br=64, Bc=64, L=129),                            # Br = 64 stacked tiles
    small(d=64, Br=64, Bc=64, L=1, Hq=1, Hkv=1),           # one row
], ids=["d128", "d64_triple", "br64", "one_row"])
def test_debug_prefill_matches_release(w):
    x = synth.prefill_inputs(w, "rms")
    rel = run_prefill(sk.lib(), w, x, 32)
    assert sk.lib().sskip_get_status(None) == sk.SSKIP_OK
    dbg = run_prefill(sk.debug_lib(), w, x, 32)
    assert sk.debug_lib().sskip_get_status(None) == sk.SSKIP_OK
    for n in rel:
        assert same_bits(rel[n], dbg[n]), n


def run_decode(L, w, x):
    q, kc, vc = to_device(x["q"]), to_device(x["kcache"]), to_device(x["vcache"])
    lens = torch.from_numpy(x["seqlens"]).cuda()
    o = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(sk.sskip_attn_decode_workspace_size(w.B, w.Hq, w.d, w.num_splits),
                     dtype=torch.uint8, device="cuda")
    cnt = torch.zeros(2, dtype=torch.int64, device="cuda")
    st = torch.empty((w.B, w.Hkv, -(-w.Lmax // w.Bc)), dtype=torch.uint8, device="cuda")
    cr = torch.empty(st.shape, dtype=torch.float32, device="cuda")
    rc = L.sskip_attn_decode_crit(_ptr(q), _ptr(kc), _ptr(vc), _ptr(lens), _ptr(o), _ptr(lse),
                                  w.B, w.Hq, w.Hkv, w.Lmax, w.d, ctypes.c_float(w.scale),
                                  ctypes.c_float(w.tsf), w.Bc, w.num_splits, _ptr(ws),
                                  ws.numel(), _ptr(cnt), _ptr(st), _ptr(cr), None)
    assert rc == sk.SSKIP_OK
    torch.cuda.synchronize()
    return {"o": o.view(torch.int16).cpu(), "lse": lse.cpu(), "cnt": cnt.cpu(), "st": st.cpu(),
            "cr": cr.cpu()}


@pytest.mark.parametrize("G,splits", [(4, 4), (8, 16), (1, 1)])
def test_debug_decode_matches_release(G, splits):
    w = DecodeWorkload(name="dbg", B=3, Hq=2 * G, Hkv=2, Lmax=700, Lmin=1, d=128, Bc=64,
                       num_splits=splits, tsf=4.0, seed=83)
    x = synth.decode_inputs(w, "rms", seqlens=np.array([700, 65, 1], np.int32))
    rel = run_decode(sk.lib(), w, x)
    assert sk.lib().sskip_get_status(None) == sk.SSKIP_OK
    dbg = run_decode(sk.debug_lib(), w, x)
    assert sk.debug_lib().sskip_get_status(None) == sk.SSKIP_OK
    for n in rel:
        assert same_bits(rel[n], dbg[n]), n
