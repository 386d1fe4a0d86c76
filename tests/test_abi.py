"""C-ABI checks that need no GPU: the library loads, exports every function
include/sskip_attn.h declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

import block_sparse_long_tiled_b200 as sk
from block_sparse_long_tiled_b200 import build as sk_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sskip_attn.h")


@pytest.fixture(scope="module")
def lib():
    sk_build.build()
    return sk.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(sskip_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_expected_api():
    names = header_functions()
    assert "sskip_attn_prefill" in names and "sskip_attn_decode" in names
    assert set(names) == set(sk.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    assert lib.sskip_version() == 100


def test_debug_library_exports_the_same_api(lib):
    dbg = sk.debug_lib()
    for name in header_functions():
        assert hasattr(dbg, name), name
    assert dbg.sskip_version() == lib.sskip_version()
    assert dbg.sskip_status_string(sk.SSKIP_ERR_DEVICE_CHECK).decode().startswith("device-side index")


def test_status_strings(lib):
    assert sk.status_string(0) == "ok"
    assert "timed out" in sk.status_string(4)
    assert "debug build" in sk.status_string(5)
    assert sk.status_string(99) == "unknown status"


def test_decode_workspace_size(lib):
    B, Hq, d, S = 64, 32, 128, 16
    rows = B * Hq * S
    want = ((rows * d * 4 + 255) // 256) * 256 + ((rows * 4 + 255) // 256) * 256
    assert sk.sskip_attn_decode_workspace_size(B, Hq, d, S) == want
    assert sk.sskip_attn_decode_workspace_size(0, Hq, d, S) == 0


FAKE = ctypes.c_void_p(1 << 20)      # 16-byte aligned, never dereferenced
FAKE_ODD = ctypes.c_void_p((1 << 20) + 8)


def prefill_call(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=1, L=128, d=128,
                 causal=1, scale=0.088, tsf=10.0, Br=128, Bc=128, counts=None):
    return lib.sskip_attn_prefill(q, k, v, o, lse, B, Hq, Hkv, L, d, causal, scale, tsf, Br, Bc,
                                  counts, None)


def test_prefill_argument_validation(lib):
    assert prefill_call(lib, q=None) == sk.SSKIP_ERR_INVALID_ARG
    assert prefill_call(lib, k=FAKE_ODD) == sk.SSKIP_ERR_INVALID_ARG
    assert prefill_call(lib, L=0) == sk.SSKIP_ERR_INVALID_ARG
    assert prefill_call(lib, Hq=3, Hkv=2) == sk.SSKIP_ERR_INVALID_ARG
    assert prefill_call(lib, tsf=-1.0) == sk.SSKIP_ERR_INVALID_ARG
    assert prefill_call(lib, tsf=float("inf")) == sk.SSKIP_ERR_INVALID_ARG
    assert prefill_call(lib, scale=0.0) == sk.SSKIP_ERR_INVALID_ARG
    assert prefill_call(lib, d=96) == sk.SSKIP_ERR_UNSUPPORTED
    assert prefill_call(lib, Br=64, Bc=128) == sk.SSKIP_ERR_UNSUPPORTED
    assert prefill_call(lib, counts=ctypes.c_void_p((1 << 20) + 4)) == sk.SSKIP_ERR_INVALID_ARG


def decode_call(lib, q=FAKE, ws=FAKE, ws_bytes=1 << 30, B=2, Hq=8, Hkv=2, Lmax=256, d=128,
                Bc=64, S=4, tsf=5.0, seqlens=FAKE):
    return lib.sskip_attn_decode(q, FAKE, FAKE, seqlens, FAKE, FAKE, B, Hq, Hkv, Lmax, d, 0.088,
                                 tsf, Bc, S, ws, ws_bytes, None, None)


def test_decode_argument_validation(lib):
    assert decode_call(lib, q=None) == sk.SSKIP_ERR_INVALID_ARG
    assert decode_call(lib, ws=None) == sk.SSKIP_ERR_INVALID_ARG
    assert decode_call(lib, ws=ctypes.c_void_p((1 << 20) + 16)) == sk.SSKIP_ERR_INVALID_ARG
    assert decode_call(lib, ws_bytes=16) == sk.SSKIP_ERR_INVALID_ARG
    assert decode_call(lib, Hq=6, Hkv=4) == sk.SSKIP_ERR_INVALID_ARG
    assert decode_call(lib, tsf=-2.0) == sk.SSKIP_ERR_INVALID_ARG
    assert decode_call(lib, Bc=128) == sk.SSKIP_ERR_UNSUPPORTED
    assert decode_call(lib, Hq=24, Hkv=2) == sk.SSKIP_ERR_UNSUPPORTED   # G = 12
    assert decode_call(lib, S=65) == sk.SSKIP_ERR_UNSUPPORTED
    assert decode_call(lib, d=32) == sk.SSKIP_ERR_UNSUPPORTED


def test_watchdog_selftest_rejects_bad_limits(lib):
    assert lib.sskip_selftest_watchdog(0, None) == sk.SSKIP_ERR_INVALID_ARG
    assert lib.sskip_selftest_watchdog(3_000_000, None) == sk.SSKIP_ERR_INVALID_ARG


def test_product_path_has_no_oracle_dependency():
    # The CUDA binding and its sources never reach the CPU oracle.
    pkg = os.path.join(ROOT, "block_sparse_long_tiled_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "sskip_oracle" not in src, f


def test_vote_record_and_host_entry_validation(lib):
    P = ctypes.c_void_p
    odd4 = P((1 << 20) + 2)  # not 4-byte aligned
    # sskip_attn_prefill_vote: vote_rows must be Br or 32; records 4-byte aligned.
    f = lib.sskip_attn_prefill_vote
    args = [FAKE] * 5 + [1, 2, 1, 128, 128, 1, ctypes.c_float(0.088), ctypes.c_float(10.0), 128, 128]
    assert f(*args, 48, None, None, None, None, None) == sk.SSKIP_ERR_UNSUPPORTED
    assert f(*args, 64, None, None, None, None, None) == sk.SSKIP_ERR_UNSUPPORTED
    assert f(*args, 32, None, None, None, odd4, None) == sk.SSKIP_ERR_INVALID_ARG
    # sskip_attn_decode_crit: misaligned record.
    g = lib.sskip_attn_decode_crit
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 2, 256, 128, ctypes.c_float(0.088),
             ctypes.c_float(5.0), 64, 4, FAKE, 1 << 30, None, None, odd4, None) == \
        sk.SSKIP_ERR_INVALID_ARG
    # sskip_attn_prefill_host: pointers, shapes and d are checked before any CUDA call.
    h = lib.sskip_attn_prefill_host
    tail = [ctypes.c_float(0.088), ctypes.c_float(10.0), 128, 128]
    assert h(*([None] + [FAKE] * 9), 1, 2, 1, 128, 128, 1, *tail, 0, None, None) == \
        sk.SSKIP_ERR_INVALID_ARG
    assert h(*([FAKE] * 10), 1, 3, 2, 128, 128, 1, *tail, 0, None, None) == \
        sk.SSKIP_ERR_INVALID_ARG
    assert h(*([FAKE] * 10), 1, 2, 1, 128, 128, 1, *tail, -1, None, None) == \
        sk.SSKIP_ERR_INVALID_ARG
    assert h(*([FAKE] * 10), 1, 2, 1, 128, 96, 1, *tail, 0, None, None) == \
        sk.SSKIP_ERR_UNSUPPORTED
    # sskip_attn_decode_host: host and staging pointers.
    dh = lib.sskip_attn_decode_host
    assert dh(*([None] + [FAKE] * 9), 2, 8, 2, 256, 128, ctypes.c_float(0.088),
              ctypes.c_float(5.0), 64, 4, FAKE, 1 << 30, None, None) == sk.SSKIP_ERR_INVALID_ARG
    # sskip_permute_rows: in place, row size and index alignment.
    pr = lib.sskip_permute_rows
    assert pr(FAKE, FAKE, FAKE, 2, 64, 128, 0, None) == sk.SSKIP_ERR_INVALID_ARG
    assert pr(FAKE, P(1 << 21), FAKE, 2, 64, 6, 0, None) == sk.SSKIP_ERR_INVALID_ARG
    assert pr(FAKE, P(1 << 21), odd4, 2, 64, 128, 0, None) == sk.SSKIP_ERR_INVALID_ARG
    assert pr(FAKE, P(1 << 21), FAKE, 0, 64, 128, 0, None) == sk.SSKIP_ERR_INVALID_ARG
    # sskip_attn_step: at least one phase.
    st = lib.sskip_attn_step
    assert st(*([None] * 5), 0, 0, 1, 128, 128, None, *([None] * 6), 0, 0, 4, None, 0, None,
              8, 2, 128, ctypes.c_float(0.088), ctypes.c_float(1000.0), ctypes.c_float(500.0),
              None) == sk.SSKIP_ERR_INVALID_ARG
    # sskip_calibrate_factor: bad ratio.
    cf = lib.sskip_calibrate_factor
    d = ctypes.c_double()
    import numpy as np
    c = np.zeros(4, np.float32)
    assert cf(c.ctypes.data_as(P), 4, ctypes.c_double(1.5), ctypes.c_double(10.0),
              ctypes.byref(d), None, None) == sk.SSKIP_ERR_INVALID_ARG
