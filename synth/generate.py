"""Seeded input generators shared by the CPU oracle and the CUDA path.

Only input preparation lives here: seeded normal draws, the planted direction,
the video raster fields, and the fp32 -> bf16 round-to-nearest-even packing of
the result. None of the attention arithmetic is here.

Every random stream is a numpy Philox (counter-based) generator keyed by
``(seed, tensor tag, batch, head)``, so a tensor can be generated head by head
on any number of threads and always comes out bit-identical.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .workloads import DecodeWorkload, PrefillWorkload

TAG_Q, TAG_K, TAG_V, TAG_U, TAG_HOT, TAG_LEN = 1, 2, 3, 4, 5, 6
TAG_FIELD_Q, TAG_FIELD_K = 7, 8


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence(list(key))))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return raw bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits to fp32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_half_up(x: float) -> int:
    return int(math.floor(x + 0.5))


def unit_direction(seed: int, d: int, reading: str) -> np.ndarray:
    """The planted direction u: unit norm ("lit") or norm sqrt(d) ("rms")."""
    if reading not in ("lit", "rms"):
        raise ValueError(f"unknown reading {reading!r}")
    u = _rng(seed, TAG_U).standard_normal(d)
    u = u / np.linalg.norm(u)
    if reading == "rms":
        u = u * math.sqrt(d)
    return u.astype(np.float32)


def hot_tiles(seed: int, b: int, kvh: int, n_tiles: int, frac: float) -> np.ndarray:
    """round(frac * n_tiles) distinct key-tile indices for one (batch, kv head)."""
    n_hot = round_half_up(frac * n_tiles)
    if n_hot <= 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(_rng(seed, TAG_HOT, b, kvh).choice(n_tiles, size=n_hot, replace=False))


def _parallel(fn, items):
    items = list(items)
    if len(items) == 1:
        fn(items[0])
        return
    with ThreadPoolExecutor(_threads()) as ex:
        for _ in ex.map(fn, items):
            pass


def _normal_bf16(out: np.ndarray, seed: int, tag: int, rows=None, post=None):
    """Fill out[b, h] (uint16 bf16 bits, shape [B,H,R,d]) with N(0,1) per (b, h).

    ``rows(b)`` limits generation to the first rows of each head (the rest stays
    zero); ``post(b, h, x)`` modifies the fp32 block before rounding."""
    B, H, R, d = out.shape

    def one(bh):
        b, h = bh
        n = R if rows is None else rows(b)
        x = _rng(seed, tag, b, h).standard_normal((n, d), dtype=np.float32)
        if post is not None:
            post(b, h, x)
        out[b, h, :n] = bf16_bits(x)

    _parallel(one, [(b, h) for b in range(B) for h in range(H)])


def _video_coords(grid, L: int) -> np.ndarray:
    T, Hh, W = grid
    n = np.arange(L)
    t = n // (Hh * W)
    h = (n // W) % Hh
    w = n % W
    return np.stack([t / T, h / Hh, w / W], axis=1)  # (L, 3) float64


def _video_field(seed: int, tag: int, b: int, h: int, coords: np.ndarray, d: int,
                 terms: int, noise: float) -> np.ndarray:
    """Per channel: sum of `terms` unit-amplitude sinusoids over (t, h, w) with
    integer frequencies in {0,1,2}^3 and uniform phases, plus noise*N(0,1)."""
    rng = _rng(seed, tag, b, h)
    freq = rng.integers(0, 3, size=(d * terms, 3)).astype(np.float64)
    phase = rng.uniform(0.0, 2.0 * math.pi, size=(d * terms,))
    arg = (2.0 * math.pi) * (coords @ freq.T) + phase  # (L, d*terms)
    field = np.sin(arg).reshape(coords.shape[0], d, terms).sum(axis=2)
    field += noise * rng.standard_normal((coords.shape[0], d))
    return field.astype(np.float32)


def prefill_inputs(w: PrefillWorkload, reading: str = "lit") -> dict:
    """q [B,Hq,L,d], k and v [B,Hkv,L,d] as uint16 bf16 bits (contiguous)."""
    q = np.zeros((w.B, w.Hq, w.L, w.d), dtype=np.uint16)
    k = np.zeros((w.B, w.Hkv, w.L, w.d), dtype=np.uint16)
    v = np.zeros((w.B, w.Hkv, w.L, w.d), dtype=np.uint16)
    _normal_bf16(v, w.seed, TAG_V)
    if w.kind == "video":
        coords = _video_coords(w.video_grid, w.L)
        for arr, tag in ((q, TAG_FIELD_Q), (k, TAG_FIELD_K)):
            H = arr.shape[1]

            def one(bh, arr=arr, tag=tag):
                b, h = bh
                arr[b, h] = bf16_bits(_video_field(w.seed, tag, b, h, coords, w.d,
                                                   w.video_terms, w.video_noise))

            _parallel(one, [(b, h) for b in range(w.B) for h in range(H)])
        return {"q": q, "k": k, "v": v, "hot": {}}

    u = unit_direction(w.seed, w.d, reading)
    hot = {(b, h): hot_tiles(w.seed, b, h, w.n_k, w.hot_frac)
           for b in range(w.B) for h in range(w.Hkv)}

    def plant_k(b, h, x):
        if w.sink_keys:
            x[:w.sink_keys] += w.sink_gain * u
        for j in hot[(b, h)]:
            x[j * w.Bc:(j + 1) * w.Bc] += w.hot_gain * u

    def plant_q(b, h, x):
        if w.q_shift:
            x += w.q_shift * u

    _normal_bf16(q, w.seed, TAG_Q, post=plant_q)
    _normal_bf16(k, w.seed, TAG_K, post=plant_k)
    return {"q": q, "k": k, "v": v, "hot": hot}


def decode_seqlens(w: DecodeWorkload) -> np.ndarray:
    return _rng(w.seed, TAG_LEN).integers(w.Lmin, w.Lmax, size=w.B, endpoint=True).astype(np.int32)


def decode_inputs(w: DecodeWorkload, reading: str = "lit", seqlens=None) -> dict:
    """q [B,Hq,d]; kcache, vcache [B,Hkv,Lmax,d] (rows >= seqlens[b] are zero);
    seqlens [B] int32. All bf16 tensors as uint16 bits."""
    lens = decode_seqlens(w) if seqlens is None else np.asarray(seqlens, dtype=np.int32)
    if lens.shape != (w.B,) or lens.min() < 1 or lens.max() > w.Lmax:
        raise ValueError("seqlens must be [B] with 1 <= L_b <= Lmax")
    u = unit_direction(w.seed, w.d, reading)
    hot = {(b, h): hot_tiles(w.seed, b, h, -(-int(lens[b]) // w.Bc), w.hot_frac)
           for b in range(w.B) for h in range(w.Hkv)}
    q = np.zeros((w.B, w.Hq, 1, w.d), dtype=np.uint16)
    kc = np.zeros((w.B, w.Hkv, w.Lmax, w.d), dtype=np.uint16)
    vc = np.zeros((w.B, w.Hkv, w.Lmax, w.d), dtype=np.uint16)

    def plant_k(b, h, x):
        if w.sink_keys:
            x[:w.sink_keys] += w.sink_gain * u
        for j in hot[(b, h)]:
            x[j * w.Bc:(j + 1) * w.Bc] += w.hot_gain * u

    def plant_q(b, h, x):
        x += w.q_shift * u

    rows = lambda b: int(lens[b])
    _normal_bf16(q, w.seed, TAG_Q, post=plant_q)
    _normal_bf16(kc, w.seed, TAG_K, rows=rows, post=plant_k)
    _normal_bf16(vc, w.seed, TAG_V, rows=rows)
    return {"q": q.reshape(w.B, w.Hq, w.d), "kcache": kc, "vcache": vc,
            "seqlens": lens, "hot": hot}
