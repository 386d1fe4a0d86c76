"""CPU oracle for Skip-Softmax tiled attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, the smoke check in ``__graft_entry__`` and the CPU-baseline leg
of ``bench.py`` may import this package. The CUDA library never calls it and
shares no code with it.

The arithmetic is plain C (``sskip_oracle.c`` / ``sskip_oracle_impl.h``): the
tiled online softmax with the Skip-Softmax block test of the TensorRT-LLM
Skip-Softmax article ("Skip Softmax 的三步走算法" section), with the threshold
t = threshold_scale_factor / L ("实战演练" section). It runs in fp32 (the
precision the method's spec fixes for its oracle) or fp64.

Pins: ``tests/test_oracle_pins.py`` checks it against fp64 brute-force dense
attention (tsf = 0), dense attention restricted to the kept key tiles, the
prefix-max closed form of the skip set, unit row sums, planted skip cases,
GQA-vs-replicated-MHA, and split-count invariance of the decode merge.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = [os.path.join(_HERE, "sskip_oracle.c"), os.path.join(_HERE, "sskip_oracle_impl.h")]
_LIB_PATH = os.path.join(_HERE, "_build", "libsskip_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into oracle/_build/libsskip_oracle.so."""
    stale = (not os.path.exists(_LIB_PATH)) or any(
        os.path.getmtime(s) > os.path.getmtime(_LIB_PATH) for s in _SRC)
    if force or stale:
        os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-std=c11",
                               "-D_GNU_SOURCE", _SRC[0], "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        for suf in ("_f32", "_f64"):
            f = getattr(lib, "sskip_oracle_prefill" + suf)
            f.restype = I
            f.argtypes = [P, P, P, I, I, I, I, I, I, D, D, I, I, I, P, I, P, P, P, P, P, P, I]
            g = getattr(lib, "sskip_oracle_decode" + suf)
            g.restype = I
            g.argtypes = [P, P, P, P, I, I, I, I, I, D, D, I, I, P, P, P, P, P, P, P, I]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are raw bf16 bits (uint16)")
    return a


def default_threads() -> int:
    return os.cpu_count() or 1


def prefill(q, k, v, *, causal: bool, sm_scale: float, tsf: float, Br: int, Bc: int,
            units=None, precision: str = "f32", nthreads: int | None = None,
            want_margin: bool = False, vote_rows: int | None = None) -> dict:
    """Skip-Softmax prefill on bf16 bits q [B,Hq,L,d], k/v [B,Hkv,L,d].

    ``units``: optional int array of (b, hq, i) query-tile units; when given,
    outputs are per unit: o [n,Br,d], lse [n,Br], tile_state [n,n_k].
    Otherwise o [B,Hq,L,d], lse [B,Hq,L], tile_state [B,Hq,n_q,n_k].
    tile_state: 0 = not visited, 1 = kept, 2 = skipped.

    ``vote_rows``: rows per vote (default Br, the block vote). A smaller
    divisor of Br cuts each query tile into slices that vote alone (the
    warp-granular variant); ``slice_mask`` then records per tile 0 (not
    visited) or 0x80 | the bitmask of slices that skipped it, and
    ``slices_skipped`` / ``slices_visited`` count slices holding a valid row.
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape:
        raise ValueError("shape mismatch")
    n_q, n_k = -(-L // Br), -(-L // Bc)
    real = np.float32 if precision == "f32" else np.float64
    if units is not None:
        units = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 3))
        n = units.shape[0]
    else:
        n = B * Hq * n_q
    o = np.empty((n, Br, d), real)
    lse = np.empty((n, Br), real)
    counts = np.zeros(4, np.int64)
    state = np.empty((n, n_k), np.int8)
    smask = np.empty((n, n_k), np.uint8)
    margin = np.empty((n, n_k), real) if want_margin else None
    fn = getattr(_load(), "sskip_oracle_prefill_" + precision)
    rc = fn(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, L, d, int(causal), float(sm_scale),
            float(tsf), Br, Bc, int(Br if vote_rows is None else vote_rows), _ptr(units), n, _ptr(o), _ptr(lse),
            _ptr(counts), _ptr(state), _ptr(smask), _ptr(margin),
            int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    out = {"skipped": int(counts[0]), "visited": int(counts[1]),
           "slices_skipped": int(counts[2]), "slices_visited": int(counts[3])}
    if units is None:
        out["o"] = o.reshape(B, Hq, n_q * Br, d)[:, :, :L]
        out["lse"] = lse.reshape(B, Hq, n_q * Br)[:, :, :L]
        out["tile_state"] = state.reshape(B, Hq, n_q, n_k)
        out["slice_mask"] = smask.reshape(B, Hq, n_q, n_k)
        if margin is not None:
            out["tile_margin"] = margin.reshape(B, Hq, n_q, n_k)
    else:
        out.update(o=o, lse=lse, tile_state=state, slice_mask=smask)
        if margin is not None:
            out["tile_margin"] = margin
    return out


def decode(q, kcache, vcache, seqlens, *, sm_scale: float, tsf: float, Bc: int,
           num_splits: int, precision: str = "f32", nthreads: int | None = None,
           want_partials: bool = False, want_margin: bool = False) -> dict:
    """Split-KV Skip-Softmax decode: q [B,Hq,d], caches [B,Hkv,Lmax,d] (bf16
    bits), seqlens [B] int32. Returns o [B,Hq,d], lse [B,Hq] and the tile
    states [B,Hkv,ceil(Lmax/Bc)] of the joint (per kv head) votes."""
    q, kcache, vcache = _u16(q), _u16(kcache), _u16(vcache)
    seqlens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B, Hq, d = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    if kcache.shape != (B, Hkv, Lmax, d) or vcache.shape != kcache.shape or seqlens.shape != (B,):
        raise ValueError("shape mismatch")
    real = np.float32 if precision == "f32" else np.float64
    n_k_max = -(-Lmax // Bc)
    o = np.empty((B, Hq, d), real)
    lse = np.empty((B, Hq), real)
    o_part = np.empty((B, Hq, num_splits, d), real) if want_partials else None
    lse_part = np.empty((B, Hq, num_splits), real) if want_partials else None
    counts = np.zeros(2, np.int64)
    state = np.empty((B, Hkv, n_k_max), np.int8)
    margin = np.empty((B, Hkv, n_k_max), real) if want_margin else None
    fn = getattr(_load(), "sskip_oracle_decode_" + precision)
    rc = fn(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), B, Hq, Hkv, Lmax, d,
            float(sm_scale), float(tsf), Bc, num_splits, _ptr(o), _ptr(lse), _ptr(o_part),
            _ptr(lse_part), _ptr(counts), _ptr(state), _ptr(margin),
            int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    out = {"o": o, "lse": lse, "skipped": int(counts[0]), "visited": int(counts[1]),
           "tile_state": state}
    if want_partials:
        out.update(o_part=o_part, lse_part=lse_part)
    if margin is not None:
        out["tile_margin"] = margin
    return out
