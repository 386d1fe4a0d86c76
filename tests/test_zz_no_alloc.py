"""The decode entry point that allocates nothing (sskip_attn_decode_noalloc).

Some callers of this library cannot allocate device memory -- embedded
runtimes without a device allocator, plugins whose host framework owns every
allocation, serving loops that forbid allocation after start-up. For them the
split-KV decode keeps its partial results in the library's own fixed device
array instead of a caller-provided workspace. These tests call it through the
C ABI and check it against sskip_attn_decode on the same inputs, twice in a
row (the shared array keeps the previous call's contents, which must not leak
into the next result).

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_long_tiled_b200 as sk
import synth
from parity_helpers import LSE_ABS, MAX_ABS, MEAN_ABS, to_device


def _call_noalloc(lib, x, w, o, lse, counts, stream):
    return lib.sskip_attn_decode_noalloc(
        ctypes.c_void_p(x["q"].data_ptr()), ctypes.c_void_p(x["kc"].data_ptr()),
        ctypes.c_void_p(x["vc"].data_ptr()), ctypes.c_void_p(x["lens"].data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        w.B, w.Hq, w.Hkv, w.Lmax, w.d, ctypes.c_float(w.scale), ctypes.c_float(w.tsf),
        w.Bc, w.num_splits, ctypes.c_void_p(counts.data_ptr()), stream)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    from block_sparse_long_tiled_b200 import build
    build.build()
    lib = sk.lib()
    fake = ctypes.c_void_p(1 << 20)
    # 256 x 64 heads x 64 splits x (128 + 1) floats is far above 32 MiB.
    assert sk.sskip_attn_decode_workspace_size(256, 64, 128, 64) > sk.DECODE_NOALLOC_SCRATCH_BYTES
    rc = lib.sskip_attn_decode_noalloc(fake, fake, fake, fake, fake, fake, 256, 64, 8, 1024, 128,
                                       0.088, 1.0, 64, 64, None, None)
    assert rc == sk.SSKIP_ERR_UNSUPPORTED
    rc = lib.sskip_attn_decode_noalloc(fake, fake, fake, fake, fake, fake, 0, 64, 8, 1024, 128,
                                       0.088, 1.0, 64, 16, None, None)
    assert rc == sk.SSKIP_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_matches_decode_on_two_calls_in_a_row():
    from block_sparse_long_tiled_b200 import build
    build.build()
    lib = sk.lib()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    cases = [
        (synth.DecodeWorkload(name="na1", B=4, Hq=32, Hkv=8, Lmax=4096, Lmin=1, d=128, Bc=64,
                              num_splits=16, tsf=500.0, seed=41), "rms",
         np.array([4096, 1000, 3333, 64], np.int32)),
        (synth.DecodeWorkload(name="na2", B=3, Hq=16, Hkv=4, Lmax=2048, Lmin=1, d=64, Bc=64,
                              num_splits=8, tsf=50.0, seed=42), "lit",
         np.array([17, 2048, 900], np.int32)),
    ]
    for w, reading, lens in cases:
        h = synth.decode_inputs(w, reading, seqlens=lens)
        x = {"q": to_device(h["q"]), "kc": to_device(h["kcache"]), "vc": to_device(h["vcache"]),
             "lens": torch.from_numpy(h["seqlens"]).to(dev)}
        assert sk.sskip_attn_decode_workspace_size(w.B, w.Hq, w.d, w.num_splits) <= \
            sk.DECODE_NOALLOC_SCRATCH_BYTES
        ref = sk.decode(x["q"], x["kc"], x["vc"], x["lens"], sm_scale=w.scale,
                        threshold_scale_factor=w.tsf, Bc=w.Bc, num_splits=w.num_splits)
        o = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
        counts = torch.zeros(2, dtype=torch.int64, device=dev)
        before = torch.cuda.memory_allocated(dev)
        rc = _call_noalloc(lib, x, w, o, lse, counts, ctypes.c_void_p(stream.cuda_stream))
        assert rc == sk.SSKIP_OK, sk.status_string(rc)
        assert sk.sskip_get_status(stream) == sk.SSKIP_OK
        assert torch.cuda.memory_allocated(dev) == before
        d = (o.float() - ref["o"].float()).abs()
        assert float(d.max()) <= MAX_ABS and float(d.mean()) <= MEAN_ABS
        assert float((lse - ref["lse"]).abs().max()) <= LSE_ABS
        assert counts.tolist() == ref["counts"].tolist()
