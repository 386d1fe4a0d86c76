"""Skip-Softmax tiled attention on B200 (sm_100a).

Thin Python binding of libsskip_attn.so (C ABI in include/sskip_attn.h). The
sskip_* functions below only marshal torch tensors into the C calls of the
same names, and the conveniences after them only allocate outputs and chain
those calls: every step of the computation runs in the library, in its CUDA
kernels or, for the two host-side steps (the calibration's factor selection
and the Hilbert order), in its C++. There is no CPU fallback; a missing
library is an error.

The method (TensorRT-LLM Skip-Softmax article, "Skip Softmax 的三步走算法"
section): per attention tile, compare the tile's local maximum logit with the
running maximum and, when every row sits more than ln(1/t) below it, skip the
tile's softmax, its P.V and its V load; t = threshold_scale_factor / L
("实战演练" section).
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsskip_attn.so")

(SSKIP_OK, SSKIP_ERR_INVALID_ARG, SSKIP_ERR_UNSUPPORTED, SSKIP_ERR_CUDA, SSKIP_ERR_TIMEOUT,
 SSKIP_ERR_DEVICE_CHECK) = range(6)
LIB_DEBUG_PATH = os.path.join(_PKG, "libsskip_attn_debug.so")

EXPORTS = ("sskip_version", "sskip_status_string", "sskip_device_supported",
           "sskip_attn_prefill", "sskip_attn_prefill_ex", "sskip_attn_prefill_vote",
           "sskip_attn_decode_workspace_size",
           "sskip_attn_decode", "sskip_attn_decode_ex", "sskip_attn_decode_crit",
           "sskip_attn_decode_noalloc", "sskip_calibrate_factor", "sskip_hilbert3d_order",
           "sskip_permute_rows", "sskip_attn_step", "sskip_attn_prefill_host",
           "sskip_attn_decode_host",
           "sskip_get_status", "sskip_selftest_watchdog")

# Size of the library's fixed decode scratch (see sskip_attn_decode_noalloc).
DECODE_NOALLOC_SCRATCH_BYTES = 32 << 20


class SSkipError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None
_lib_debug = None


def lib() -> ctypes.CDLL:
    """Load libsskip_attn.so (build it first with block_sparse_long_tiled_b200.build)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


def debug_lib() -> ctypes.CDLL:
    """Load libsskip_attn_debug.so: the same C ABI with device-side index
    checks (a failed one latches SSKIP_ERR_DEVICE_CHECK). Its status word is
    its own: read it with debug_lib().sskip_get_status."""
    global _lib_debug
    if _lib_debug is None:
        _lib_debug = _load(LIB_DEBUG_PATH)
    return _lib_debug


def _load(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m block_sparse_long_tiled_b200.build`")
    L = ctypes.CDLL(path)
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
    L.sskip_attn_prefill_vote.argtypes = pre[:-1] + [I, P, P, P, P, P]
    L.sskip_attn_decode_workspace_size.restype = Z
    L.sskip_attn_decode_workspace_size.argtypes = [I, I, I, I]
    dec = [P, P, P, P, P, P, I, I, I, I, I, F, F, I, I, P, Z, P]
    L.sskip_attn_decode.restype = I
    L.sskip_attn_decode.argtypes = dec + [P]
    L.sskip_attn_decode_ex.restype = I
    L.sskip_attn_decode_ex.argtypes = dec + [P, P]
    L.sskip_attn_decode_crit.restype = I
    L.sskip_attn_decode_crit.argtypes = dec + [P, P, P]
    D = ctypes.c_double
    L.sskip_calibrate_factor.restype = I
    L.sskip_calibrate_factor.argtypes = [P, Z, D, D, P, P, P]
    L.sskip_hilbert3d_order.restype = I
    L.sskip_hilbert3d_order.argtypes = [I, I, I, I, P]
    L.sskip_permute_rows.restype = I
    L.sskip_permute_rows.argtypes = [P, P, P, ctypes.c_longlong, I, I, I, P]
    L.sskip_attn_prefill_host.restype = I
    L.sskip_attn_prefill_host.argtypes = [P] * 10 + [I, I, I, I, I, I, F, F, I, I, I, P, P]
    L.sskip_attn_decode_host.restype = I
    L.sskip_attn_decode_host.argtypes = [P] * 10 + [I, I, I, I, I, F, F, I, I, P, Z, P, P]
    L.sskip_attn_step.restype = I
    L.sskip_attn_step.argtypes = ([P, P, P, P, P, I, I, I, I, I, P] +
                                  [P, P, P, P, P, P, I, I, I, P, Z, P] +
                                  [I, I, I, F, F, F, P])
    L.sskip_attn_decode_noalloc.restype = I
    L.sskip_attn_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, F, I, I, P, P]
    L.sskip_get_status.restype = I
    L.sskip_get_status.argtypes = [P]
    L.sskip_selftest_watchdog.restype = I
    L.sskip_selftest_watchdog.argtypes = [ctypes.c_uint, P]
    return L


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


def _bf16_view(t, cuda: bool = True):
    # bf16 tensors, or raw bf16 bits stored as int16/uint16, are passed as is.
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected bf16 storage, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    if t.is_cuda != cuda:
        raise ValueError(f"expected a {'CUDA' if cuda else 'host'} tensor")
    return t


def _dev(t, dtype, what: str, cuda: bool = True):
    """Check an optional non-bf16 argument: dtype, device side, contiguity."""
    if t is None:
        return t
    if t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if t.is_cuda != cuda:
        raise ValueError(f"{what} must be a {'CUDA' if cuda else 'host'} tensor")
    return t


def _check_counts(t, n: int):
    # Counters are unsigned 64-bit on the device; int64 storage of them is accepted.
    if t is not None:
        _dev(t, torch.int64, "skip_count")
        if t.numel() < n:
            raise ValueError(f"skip_count needs {n} entries")


def _alloc_on(stream):
    """Allocate on the stream a convenience launches on, so that buffers freed
    when it returns are reused only after that stream's work."""
    if stream is None:
        return contextlib.nullcontext()
    if not isinstance(stream, torch.cuda.Stream):
        stream = torch.cuda.ExternalStream(int(stream))
    return torch.cuda.stream(stream)


def sskip_attn_prefill(q, k, v, o, lse, *, causal: bool, sm_scale: float,
                       threshold_scale_factor: float, Br: int = 128, Bc: int = 128,
                       skip_count=None, tile_state=None, stream=None) -> None:
    """Marshal q/k/v [B,H,L,d] bf16, o [B,Hq,L,d] bf16, lse [B,Hq,L] fp32,
    skip_count int64[2] (optional), tile_state uint8 (optional) into
    sskip_attn_prefill_ex."""
    for t in (q, k, v, o):
        _bf16_view(t)
    _dev(lse, torch.float32, "lse")
    _dev(tile_state, torch.uint8, "tile_state")
    _check_counts(skip_count, 2)
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
                            tile_crit=None, stream=None) -> None:
    """Marshal the prefill tensors plus vote_rows, counts int64[4] (optional),
    tile_state and slice_mask uint8 and tile_crit fp32 (optional) into
    sskip_attn_prefill_vote."""
    for t in (q, k, v, o):
        _bf16_view(t)
    _dev(lse, torch.float32, "lse")
    _dev(tile_state, torch.uint8, "tile_state")
    _dev(slice_mask, torch.uint8, "slice_mask")
    _dev(tile_crit, torch.float32, "tile_crit")
    _check_counts(counts, 4)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    rc = lib().sskip_attn_prefill_vote(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                                       Hkv, L, d, int(bool(causal)), float(sm_scale),
                                       float(threshold_scale_factor), int(Br), int(Bc),
                                       int(vote_rows), _ptr(counts), _ptr(tile_state),
                                       _ptr(slice_mask), _ptr(tile_crit), _stream(stream))
    _check(rc, "sskip_attn_prefill_vote")


def sskip_attn_prefill_host(host: dict, dev: dict, *, causal: bool, sm_scale: float,
                            threshold_scale_factor: float, Br: int = 128, Bc: int = 128,
                            kv_per_chunk: int = 0, skip_count=None, stream=None) -> None:
    """Marshal host tensors (q, k, v, o, lse; pinned for overlap) and device
    staging tensors of the same shapes into sskip_attn_prefill_host."""
    for n in ("q", "k", "v", "o"):
        _bf16_view(host[n], cuda=False)
        _bf16_view(dev[n])
    _dev(host["lse"], torch.float32, "host lse", cuda=False)
    _dev(dev["lse"], torch.float32, "lse")
    _check_counts(skip_count, 2)
    B, Hq, L, d = host["q"].shape
    Hkv = host["k"].shape[1]
    rc = lib().sskip_attn_prefill_host(*(_ptr(host[n]) for n in ("q", "k", "v", "o", "lse")),
                                       *(_ptr(dev[n]) for n in ("q", "k", "v", "o", "lse")),
                                       B, Hq, Hkv, L, d, int(bool(causal)), float(sm_scale),
                                       float(threshold_scale_factor), int(Br), int(Bc),
                                       int(kv_per_chunk), _ptr(skip_count), _stream(stream))
    _check(rc, "sskip_attn_prefill_host")


def sskip_attn_decode_host(host: dict, dev: dict, kcache, vcache, *, sm_scale: float,
                           threshold_scale_factor: float, Bc: int = 64, num_splits: int = 16,
                           workspace=None, skip_count=None, stream=None) -> None:
    """Marshal host q, seqlens, o, lse (pinned for async copies), their device
    staging buffers and the device-resident caches into sskip_attn_decode_host."""
    for n in ("q", "o"):
        _bf16_view(host[n], cuda=False)
        _bf16_view(dev[n])
    for t in (kcache, vcache):
        _bf16_view(t)
    _dev(host["seqlens"], torch.int32, "host seqlens", cuda=False)
    _dev(dev["seqlens"], torch.int32, "seqlens")
    _dev(host["lse"], torch.float32, "host lse", cuda=False)
    _dev(dev["lse"], torch.float32, "lse")
    _check_counts(skip_count, 2)
    B, Hq, d = host["q"].shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().sskip_attn_decode_host(*(_ptr(host[n]) for n in ("q", "seqlens", "o", "lse")),
                                      *(_ptr(dev[n]) for n in ("q", "seqlens", "o", "lse")),
                                      _ptr(kcache), _ptr(vcache), B, Hq, Hkv, Lmax, d,
                                      float(sm_scale), float(threshold_scale_factor), int(Bc),
                                      int(num_splits), _ptr(workspace), ws_bytes,
                                      _ptr(skip_count), _stream(stream))
    _check(rc, "sskip_attn_decode_host")


def _check_decode_args(q, kcache, vcache, seqlens, o, lse, skip_count):
    for t in (q, kcache, vcache, o):
        _bf16_view(t)
    # int32 lengths on the device: an int64 tensor would be read as pairs of
    # 32-bit words, i.e. wrong lengths.
    _dev(seqlens, torch.int32, "seqlens")
    _dev(lse, torch.float32, "lse")
    _check_counts(skip_count, 2)


def sskip_attn_decode_workspace_size(B: int, Hq: int, d: int, num_splits: int) -> int:
    return int(lib().sskip_attn_decode_workspace_size(B, Hq, d, num_splits))


def sskip_attn_decode(q, kcache, vcache, seqlens, o, lse, *, sm_scale: float,
                      threshold_scale_factor: float, Bc: int = 64, num_splits: int = 16,
                      workspace=None, skip_count=None, tile_state=None, stream=None) -> None:
    """Marshal q [B,Hq,d], caches [B,Hkv,Lmax,d] bf16, seqlens [B] int32,
    o [B,Hq,d] bf16, lse [B,Hq] fp32 and a uint8 workspace into sskip_attn_decode_ex."""
    _check_decode_args(q, kcache, vcache, seqlens, o, lse, skip_count)
    _dev(tile_state, torch.uint8, "tile_state")
    B, Hq, d = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().sskip_attn_decode_ex(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(o),
                                    _ptr(lse), B, Hq, Hkv, Lmax, d, float(sm_scale),
                                    float(threshold_scale_factor), int(Bc), int(num_splits),
                                    _ptr(workspace), ws_bytes, _ptr(skip_count), _ptr(tile_state),
                                    _stream(stream))
    _check(rc, "sskip_attn_decode")


def sskip_attn_decode_crit(q, kcache, vcache, seqlens, o, lse, *, sm_scale: float,
                           threshold_scale_factor: float, Bc: int = 64, num_splits: int = 16,
                           workspace=None, skip_count=None, tile_state=None, tile_crit=None,
                           stream=None) -> None:
    """sskip_attn_decode plus the fp32 critical-value record tile_crit
    [B, Hkv, ceil(Lmax/Bc)] (sskip_attn_decode_crit)."""
    _check_decode_args(q, kcache, vcache, seqlens, o, lse, skip_count)
    _dev(tile_state, torch.uint8, "tile_state")
    _dev(tile_crit, torch.float32, "tile_crit")
    B, Hq, d = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().sskip_attn_decode_crit(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens),
                                      _ptr(o), _ptr(lse), B, Hq, Hkv, Lmax, d, float(sm_scale),
                                      float(threshold_scale_factor), int(Bc), int(num_splits),
                                      _ptr(workspace), ws_bytes, _ptr(skip_count),
                                      _ptr(tile_state), _ptr(tile_crit), _stream(stream))
    _check(rc, "sskip_attn_decode_crit")


def sskip_calibrate_factor(tile_crit_host, target_ratio: float, max_factor: float) -> dict:
    """Marshal a host fp32 critical-value record into sskip_calibrate_factor."""
    import numpy as np
    a = np.ascontiguousarray(np.asarray(tile_crit_host, dtype=np.float32)).reshape(-1)
    f, r = ctypes.c_double(0.0), ctypes.c_double(0.0)
    v = ctypes.c_longlong(0)
    rc = lib().sskip_calibrate_factor(a.ctypes.data_as(ctypes.c_void_p), a.size,
                                      float(target_ratio), float(max_factor), ctypes.byref(f),
                                      ctypes.byref(r), ctypes.byref(v))
    _check(rc, "sskip_calibrate_factor")
    return {"factor": f.value, "achieved_ratio": r.value, "visited": v.value}


def sskip_attn_decode_noalloc(q, kcache, vcache, seqlens, o, lse, *, sm_scale: float,
                              threshold_scale_factor: float, Bc: int = 64, num_splits: int = 16,
                              skip_count=None, stream=None) -> None:
    """Marshal the same tensors as sskip_attn_decode, minus the workspace, into
    sskip_attn_decode_noalloc: for callers that cannot allocate device memory,
    the library's own fixed scratch array (DECODE_NOALLOC_SCRATCH_BYTES) holds
    the split partials. Calls that overlap on the GPU race on that array."""
    _check_decode_args(q, kcache, vcache, seqlens, o, lse, skip_count)
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
    rec_shape = (B, Hq, -(-L // Br), -(-L // Bc))
    with _alloc_on(stream):
        o = torch.empty((B, Hq, L, d), dtype=q.dtype, device=q.device)
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
        tiles = torch.empty(rec_shape, dtype=torch.uint8, device=q.device) if with_tiles else None
        counts = torch.zeros(2 if vote_rows is None else 4, dtype=torch.int64, device=q.device)
        smask = (torch.empty(rec_shape, dtype=torch.uint8, device=q.device)
                 if with_tiles and vote_rows is not None else None)
    if vote_rows is None:
        sskip_attn_prefill(q, k, v, o, lse, causal=causal, sm_scale=sm_scale,
                           threshold_scale_factor=threshold_scale_factor, Br=Br, Bc=Bc,
                           skip_count=counts, tile_state=tiles, stream=stream)
        return {"o": o, "lse": lse, "counts": counts, "tile_state": tiles}
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
    with _alloc_on(stream):
        o = torch.empty((B, Hq, d), dtype=q.dtype, device=q.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        ws = torch.empty(sskip_attn_decode_workspace_size(B, Hq, d, num_splits),
                         dtype=torch.uint8, device=q.device)
        counts = torch.zeros(2, dtype=torch.int64, device=q.device)
        tiles = (torch.empty((B, Hkv, -(-Lmax // Bc)), dtype=torch.uint8, device=q.device)
                 if with_tiles else None)
    sskip_attn_decode(q, kcache, vcache, seqlens, o, lse, sm_scale=sm_scale,
                      threshold_scale_factor=threshold_scale_factor, Bc=Bc, num_splits=num_splits,
                      workspace=ws, skip_count=counts, tile_state=tiles, stream=stream)
    return {"o": o, "lse": lse, "counts": counts, "tile_state": tiles}


def calibrate_prefill(q, k, v, *, causal: bool, sm_scale: float, target_ratio: float,
                      Br: int = 128, Bc: int = 128, stream=None) -> dict:
    """One prefill pass (factor 0) with the critical-value record on the GPU,
    then the host selection of the factor that skips target_ratio of the
    tiles. Returns factor, achieved_ratio, visited and the record."""
    B, Hq, L, d = q.shape
    with _alloc_on(stream):
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
        crit = torch.empty((B, Hq, -(-L // Br), -(-L // Bc)), dtype=torch.float32,
                           device=q.device)
    sskip_attn_prefill_vote(q, k, v, o, lse, causal=causal, sm_scale=sm_scale,
                            threshold_scale_factor=0.0, Br=Br, Bc=Bc, vote_rows=Br,
                            tile_crit=crit, stream=stream)
    host = crit.cpu().numpy()
    out = sskip_calibrate_factor(host, target_ratio, float(L))
    out["tile_crit"] = host
    return out


def calibrate_decode(q, kcache, vcache, seqlens, *, sm_scale: float, target_ratio: float,
                     Bc: int = 64, num_splits: int = 16, stream=None) -> dict:
    """Decode counterpart of calibrate_prefill (the cap is the shortest
    sequence, so every t_b = factor / seqlens[b] stays below 1)."""
    B, Hq, d = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    with _alloc_on(stream):
        o = torch.empty((B, Hq, d), dtype=q.dtype, device=q.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        ws = torch.empty(sskip_attn_decode_workspace_size(B, Hq, d, num_splits),
                         dtype=torch.uint8, device=q.device)
        crit = torch.empty((B, Hkv, -(-Lmax // Bc)), dtype=torch.float32, device=q.device)
    sskip_attn_decode_crit(q, kcache, vcache, seqlens, o, lse, sm_scale=sm_scale,
                           threshold_scale_factor=0.0, Bc=Bc, num_splits=num_splits,
                           workspace=ws, tile_crit=crit, stream=stream)
    host = crit.cpu().numpy()
    out = sskip_calibrate_factor(host, target_ratio, float(seqlens.min().item()))
    out["tile_crit"] = host
    return out


def sskip_hilbert3d_order(T: int, H: int, W: int, L: int):
    """Host int32 numpy [L]: raster index of the token at each position of the
    3-D Hilbert order (sskip_hilbert3d_order)."""
    import numpy as np
    perm = np.empty(L, np.int32)
    _check(lib().sskip_hilbert3d_order(int(T), int(H), int(W), int(L),
                                       perm.ctypes.data_as(ctypes.c_void_p)),
           "sskip_hilbert3d_order")
    return perm


def sskip_permute_rows(src, dst, idx, *, scatter: bool, stream=None) -> None:
    """Marshal src/dst [..., L, row] (contiguous, same shape) and idx int32 [L]
    into sskip_permute_rows; n_mats = product of the leading dims."""
    if src.shape != dst.shape or not (src.is_contiguous() and dst.is_contiguous()):
        raise ValueError("src and dst must be contiguous and of one shape")
    L = src.shape[-2]
    row_bytes = src.shape[-1] * src.element_size()
    n_mats = src.numel() // (L * src.shape[-1])
    _check(lib().sskip_permute_rows(_ptr(src), _ptr(dst), _ptr(idx), n_mats, L, row_bytes,
                                    int(bool(scatter)), _stream(stream)), "sskip_permute_rows")


def prefill_reordered(q, k, v, perm, *, sm_scale: float, threshold_scale_factor: float,
                      Br: int = 128, Bc: int = 128, vote_rows: int | None = None,
                      with_tiles: bool = False, stream=None) -> dict:
    """Non-causal prefill in the token order `perm` (device int32 [L], e.g.
    the Hilbert order): gather Q, K, V, run the kernel, scatter O and lse back
    to the original order. Every step runs in the library's kernels; the tile
    record, if asked for, is in the reordered frame."""
    with _alloc_on(stream):
        qp, kp, vp = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for a, b in ((q, qp), (k, kp), (v, vp)):
        sskip_permute_rows(a, b, perm, scatter=False, stream=stream)
    out = prefill(qp, kp, vp, causal=False, sm_scale=sm_scale,
                  threshold_scale_factor=threshold_scale_factor, Br=Br, Bc=Bc,
                  with_tiles=with_tiles, vote_rows=vote_rows, stream=stream)
    with _alloc_on(stream):
        o = torch.empty_like(out["o"])
        lse = torch.empty_like(out["lse"])
    sskip_permute_rows(out["o"], o, perm, scatter=True, stream=stream)
    sskip_permute_rows(out["lse"].unsqueeze(-1), lse.unsqueeze(-1), perm, scatter=True,
                       stream=stream)
    out.update(o=o, lse=lse)
    return out


def phase_factors(threshold_scale_factor) -> tuple[float, float]:
    """(prefill, decode) factors from one number or a {"prefill", "decode"}
    mapping, the two forms the TensorRT-LLM configuration accepts."""
    if isinstance(threshold_scale_factor, dict):
        extra = set(threshold_scale_factor) - {"prefill", "decode"}
        if extra or len(threshold_scale_factor) != 2:
            raise ValueError("threshold_scale_factor needs exactly the keys 'prefill' and 'decode'")
        return float(threshold_scale_factor["prefill"]), float(threshold_scale_factor["decode"])
    f = float(threshold_scale_factor)
    return f, f


def sskip_attn_step(*, threshold_scale_factor, sm_scale: float, prefill=None, decode=None,
                    Br: int = 128, Bc: int = 128, causal: bool = True, num_splits: int = 16,
                    stream=None) -> None:
    """Marshal one serving step into sskip_attn_step.

    prefill: dict q, k, v, o, lse (and optional count int64[2]) or None;
    decode: dict q, kcache, vcache, seqlens, o, lse, workspace (optional count)
    or None; threshold_scale_factor: a number or {"prefill": a, "decode": b}."""
    tp, td = phase_factors(threshold_scale_factor)
    if prefill is None and decode is None:
        raise ValueError("a step needs a prefill or a decode batch")
    ref = (prefill or decode)["q"]
    Hq = ref.shape[1]
    d = ref.shape[-1]
    if prefill is not None:
        for n in ("q", "k", "v", "o"):
            _bf16_view(prefill[n])
        Bp, _, L, _ = prefill["q"].shape
        Hkv = prefill["k"].shape[1]
    else:
        Bp, L = 0, 0
    if decode is not None:
        for n in ("q", "kcache", "vcache", "o"):
            _bf16_view(decode[n])
        Bd = decode["q"].shape[0]
        Hkv_d, Lmax = decode["kcache"].shape[1], decode["kcache"].shape[2]
        if prefill is not None and (Hkv_d != Hkv or decode["q"].shape[1] != Hq
                                    or decode["q"].shape[-1] != d):
            raise ValueError("both phases must come from one layer (Hq, Hkv, d)")
        Hkv = Hkv_d
        ws = decode["workspace"]
        ws_bytes = ws.numel() * ws.element_size()
    else:
        Bd, Lmax, ws, ws_bytes = 0, 0, None, 0
    P = prefill or {}
    D = decode or {}
    rc = lib().sskip_attn_step(_ptr(P.get("q")), _ptr(P.get("k")), _ptr(P.get("v")),
                               _ptr(P.get("o")), _ptr(P.get("lse")), Bp, L, int(bool(causal)),
                               int(Br), int(Bc), _ptr(P.get("count")), _ptr(D.get("q")),
                               _ptr(D.get("kcache")), _ptr(D.get("vcache")),
                               _ptr(D.get("seqlens")), _ptr(D.get("o")), _ptr(D.get("lse")), Bd,
                               Lmax, int(num_splits), _ptr(ws), ws_bytes, _ptr(D.get("count")),
                               Hq, Hkv, d, float(sm_scale), tp, td, _stream(stream))
    _check(rc, "sskip_attn_step")
