"""Skip-Softmax tiled attention on B200 (sm_100a).

Thin Python binding of libsskip_attn.so (C ABI in include/sskip_attn.h). The
functions below only marshal torch tensors into the C calls of the same names:
every step of the computation runs in the library's CUDA kernels. There is no
CPU fallback; a missing library is an error.

The method (TensorRT-LLM Skip-Softmax article, "Skip Softmax 的三步走算法"
section): per attention tile, compare the tile's local maximum logit with the
running maximum and, when every row sits more than ln(1/t) below it, skip the
tile's softmax, its P.V and its V load; t = threshold_scale_factor / L
("实战演练" section).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsskip_attn.so")

SSKIP_OK, SSKIP_ERR_INVALID_ARG, SSKIP_ERR_UNSUPPORTED, SSKIP_ERR_CUDA, SSKIP_ERR_TIMEOUT = range(5)

EXPORTS = ("sskip_version", "sskip_status_string", "sskip_device_supported",
           "sskip_attn_prefill", "sskip_attn_prefill_ex", "sskip_attn_prefill_vote",
           "sskip_attn_decode_workspace_size",
           "sskip_attn_decode", "sskip_attn_decode_ex", "sskip_attn_decode_noalloc",
           "sskip_get_status", "sskip_selftest_watchdog")

# Size of the library's fixed decode scratch (see sskip_attn_decode_noalloc).
DECODE_NOALLOC_SCRATCH_BYTES = 32 << 20


class SSkipError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsskip_attn.so (build it first with block_sparse_long_tiled_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_long_tiled_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.sskip_version.restype = I
        L.sskip_version.argtypes = []
        L.sskip_status_string.restype = ctypes.c_char_p
        L.sskip_status_string.argtypes = [I]
        L.sskip_device_supported.restype = I
        L.sskip_device_supported.argtypes = [I]
        pre = [P, P, P, P, P, I, I, I, I, I, I, F, F, I, I, P]
        L.sskip_attn_prefill.restype = I
        L.sskip_attn_prefill.argtypes = pre + [P]
        L.sskip_attn_prefill_ex.restype = I
        L.sskip_attn_prefill_ex.argtypes = pre[:-1] + [P, P, P]
        L.sskip_attn_prefill_vote.restype = I
        L.sskip_attn_prefill_vote.argtypes = pre[:-1] + [I, P, P, P, P]
        L.sskip_attn_decode_workspace_size.restype = Z
        L.sskip_attn_decode_workspace_size.argtypes = [I, I, I, I]
        dec = [P, P, P, P, P, P, I, I, I, I, I, F, F, I, I, P, Z, P]
        L.sskip_attn_decode.restype = I
        L.sskip_attn_decode.argtypes = dec + [P]
        L.sskip_attn_decode_ex.restype = I
        L.sskip_attn_decode_ex.argtypes = dec + [P, P]
        L.sskip_attn_decode_noalloc.restype = I
        L.sskip_attn_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, F, I, I, P, P]
        L.sskip_get_status.restype = I
        L.sskip_get_status.argtypes = [P]
        L.sskip_selftest_watchdog.restype = I
        L.sskip_selftest_watchdog.argtypes = [ctypes.c_uint, P]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().sskip_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, what: str):
    if rc != SSKIP_OK:
        raise SSkipError(rc, what)


def _bf16_view(t):
    # bf16 tensors, or raw bf16 bits stored as int16/uint16, are passed as is.
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected bf16 storage, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t


def sskip_attn_prefill(q, k, v, o, lse, *, causal: bool, sm_scale: float,
                       threshold_scale_factor: float, Br: int = 128, Bc: int = 128,
                       skip_count=None, tile_state=None, stream=None) -> None:
    """Marshal q/k/v [B,H,L,d] bf16, o [B,Hq,L,d] bf16, lse [B,Hq,L] fp32,
    skip_count int64[2] (optional), tile_state uint8 (optional) into
    sskip_attn_prefill_ex."""
    for t in (q, k, v, o):
        _bf16_view(t)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    rc = lib().sskip_attn_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv,
                                     L, d, int(bool(causal)), float(sm_scale),
                                     float(threshold_scale_factor), int(Br), int(Bc),
                                     _ptr(skip_count), _ptr(tile_state), _stream(stream))
    _check(rc, "sskip_attn_prefill")


def sskip_attn_prefill_vote(q, k, v, o, lse, *, causal: bool, sm_scale: float,
                            threshold_scale_factor: float, Br: int = 128, Bc: int = 128,
                            vote_rows: int = 32, counts=None, tile_state=None, slice_mask=None,
                            stream=None) -> None:
    """Marshal the prefill tensors plus vote_rows, counts int64[4] (optional),
    tile_state and slice_mask uint8 (optional) into sskip_attn_prefill_vote."""
    for t in (q, k, v, o):
        _bf16_view(t)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    rc = lib().sskip_attn_prefill_vote(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                                       Hkv, L, d, int(bool(causal)), float(sm_scale),
                                       float(threshold_scale_factor), int(Br), int(Bc),
                                       int(vote_rows), _ptr(counts), _ptr(tile_state),
                                       _ptr(slice_mask), _stream(stream))
    _check(rc, "sskip_attn_prefill_vote")


def sskip_attn_decode_workspace_size(B: int, Hq: int, d: int, num_splits: int) -> int:
    return int(lib().sskip_attn_decode_workspace_size(B, Hq, d, num_splits))


def sskip_attn_decode(q, kcache, vcache, seqlens, o, lse, *, sm_scale: float,
                      threshold_scale_factor: float, Bc: int = 64, num_splits: int = 16,
                      workspace=None, skip_count=None, tile_state=None, stream=None) -> None:
    """Marshal q [B,Hq,d], caches [B,Hkv,Lmax,d] bf16, seqlens [B] int32,
    o [B,Hq,d] bf16, lse [B,Hq] fp32 and a uint8 workspace into sskip_attn_decode_ex."""
    for t in (q, kcache, vcache, o):
        _bf16_view(t)
    B, Hq, d = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().sskip_attn_decode_ex(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(o),
                                    _ptr(lse), B, Hq, Hkv, Lmax, d, float(sm_scale),
                                    float(threshold_scale_factor), int(Bc), int(num_splits),
                                    _ptr(workspace), ws_bytes, _ptr(skip_count), _ptr(tile_state),
                                    _stream(stream))
    _check(rc, "sskip_attn_decode")


def sskip_attn_decode_noalloc(q, kcache, vcache, seqlens, o, lse, *, sm_scale: float,
                              threshold_scale_factor: float, Bc: int = 64, num_splits: int = 16,
                              skip_count=None, stream=None) -> None:
    """Marshal the same tensors as sskip_attn_decode, minus the workspace, into
    sskip_attn_decode_noalloc: for callers that cannot allocate device memory,
    the library's own fixed scratch array (DECODE_NOALLOC_SCRATCH_BYTES) holds
    the split partials. Calls that overlap on the GPU race on that array."""
    for t in (q, kcache, vcache, o):
        _bf16_view(t)
    B, Hq, d = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    rc = lib().sskip_attn_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens),
                                         _ptr(o), _ptr(lse), B, Hq, Hkv, Lmax, d, float(sm_scale),
                                         float(threshold_scale_factor), int(Bc), int(num_splits),
                                         _ptr(skip_count), _stream(stream))
    _check(rc, "sskip_attn_decode_noalloc")


def sskip_get_status(stream=None) -> int:
    return int(lib().sskip_get_status(_stream(stream)))


def sskip_selftest_watchdog(limit_us: int, stream=None) -> None:
    _check(lib().sskip_selftest_watchdog(int(limit_us), _stream(stream)), "sskip_selftest_watchdog")


# -------------------------------------------------------------- conveniences
def prefill(q, k, v, *, causal: bool, sm_scale: float, threshold_scale_factor: float,
            Br: int = 128, Bc: int = 128, with_tiles: bool = False, vote_rows: int | None = None,
            stream=None) -> dict:
    """Allocate outputs with torch and run sskip_attn_prefill on q's device;
    with ``vote_rows`` (Br or 32), run sskip_attn_prefill_vote instead and
    also return the four counters and the slice record."""
    B, Hq, L, d = q.shape
    o = torch.empty((B, Hq, L, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    tiles = None
    rec_shape = (B, Hq, -(-L // Br), -(-L // Bc))
    if with_tiles:
        tiles = torch.empty(rec_shape, dtype=torch.uint8, device=q.device)
    if vote_rows is None:
        counts = torch.zeros(2, dtype=torch.int64, device=q.device)
        sskip_attn_prefill(q, k, v, o, lse, causal=causal, sm_scale=sm_scale,
                           threshold_scale_factor=threshold_scale_factor, Br=Br, Bc=Bc,
                           skip_count=counts, tile_state=tiles, stream=stream)
        return {"o": o, "lse": lse, "counts": counts, "tile_state": tiles}
    counts = torch.zeros(4, dtype=torch.int64, device=q.device)
    smask = torch.empty(rec_shape, dtype=torch.uint8, device=q.device) if with_tiles else None
    sskip_attn_prefill_vote(q, k, v, o, lse, causal=causal, sm_scale=sm_scale,
                            threshold_scale_factor=threshold_scale_factor, Br=Br, Bc=Bc,
                            vote_rows=vote_rows, counts=counts, tile_state=tiles,
                            slice_mask=smask, stream=stream)
    return {"o": o, "lse": lse, "counts": counts, "tile_state": tiles, "slice_mask": smask}


def decode(q, kcache, vcache, seqlens, *, sm_scale: float, threshold_scale_factor: float,
           Bc: int = 64, num_splits: int = 16, with_tiles: bool = False, stream=None) -> dict:
    """Allocate outputs and workspace with torch and run sskip_attn_decode."""
    B, Hq, d = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    o = torch.empty((B, Hq, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws = torch.empty(sskip_attn_decode_workspace_size(B, Hq, d, num_splits), dtype=torch.uint8,
                     device=q.device)
    counts = torch.zeros(2, dtype=torch.int64, device=q.device)
    tiles = None
    if with_tiles:
        tiles = torch.empty((B, Hkv, -(-Lmax // Bc)), dtype=torch.uint8, device=q.device)
    sskip_attn_decode(q, kcache, vcache, seqlens, o, lse, sm_scale=sm_scale,
                      threshold_scale_factor=threshold_scale_factor, Bc=Bc, num_splits=num_splits,
                      workspace=ws, skip_count=counts, tile_state=tiles, stream=stream)
    return {"o": o, "lse": lse, "counts": counts, "tile_state": tiles}
