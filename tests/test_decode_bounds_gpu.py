"""Device-side check of the decode sequence lengths.

seqlens lives in device memory, so the host cannot validate it. The decode
kernel accepts 1 <= seqlens[b] <= Lmax; a length outside that range is
latched as SSKIP_ERR_INVALID_ARG in the device status word and clamped into
[0, Lmax] before any index is formed, so every copy stays inside the
sequence's [Lmax, d] cache slab and every record index stays inside its row.
A clamped length of 0 leaves every split empty: O = 0 and lse = -inf. The
other sequences of the batch are unaffected and still match the oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import oracle
import synth
from parity_helpers import bf16_host, check_rows, to_device
from synth import DecodeWorkload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert torch.cuda.is_available()


W = DecodeWorkload(name="bounds", B=3, Hq=8, Hkv=2, Lmax=256, Lmin=1, d=128, Bc=64,
                   num_splits=4, tsf=4.0, seed=91)


@pytest.mark.parametrize("bad_len,as_len", [(256 + 300, 256), (0, 0), (-7, 0)])
def test_out_of_range_length_is_latched_and_clamped(bad_len, as_len):
    x = synth.decode_inputs(W, "rms", seqlens=np.array([256, 100, 37], np.int32))
    lens = torch.tensor([bad_len, 100, 37], dtype=torch.int32, device="cuda")
    assert sk.sskip_get_status() == sk.SSKIP_OK
    out = sk.decode(to_device(x["q"]), to_device(x["kcache"]), to_device(x["vcache"]), lens,
                    sm_scale=W.scale, threshold_scale_factor=W.tsf, Bc=W.Bc,
                    num_splits=W.num_splits, with_tiles=True)
    torch.cuda.synchronize()
    assert sk.sskip_get_status() == sk.SSKIP_ERR_INVALID_ARG
    assert sk.sskip_get_status() == sk.SSKIP_OK  # reading clears it
    o, lse = bf16_host(out["o"]), out["lse"].cpu().numpy()
    st = out["tile_state"].cpu().numpy()
    n_k = -(-as_len // W.Bc)
    assert np.all(st[0, :, :n_k] > 0) and np.all(st[0, :, n_k:] == 0)
    if as_len == 0:
        assert np.all(o[0] == 0) and np.all(lse[0] == -np.inf)
        rows = slice(1, 3)
        ref = oracle.decode(x["q"][1:], x["kcache"][1:], x["vcache"][1:], x["seqlens"][1:],
                            sm_scale=W.scale, tsf=W.tsf, Bc=W.Bc, num_splits=W.num_splits)
    else:  # ran as a sequence of length Lmax
        rows = slice(0, 3)
        ref = oracle.decode(x["q"], x["kcache"], x["vcache"], x["seqlens"], sm_scale=W.scale,
                            tsf=W.tsf, Bc=W.Bc, num_splits=W.num_splits)
    check_rows(o[rows], lse[rows], ref["o"], ref["lse"], what="clamped batch")
