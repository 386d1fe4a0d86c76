"""fp64 brute-force references that pin the CPU oracle.

Each function is a textbook definition or a closed form derived from the
Skip-Softmax rule (TensorRT-LLM Skip-Softmax article, "Skip Softmax 的三步走算法"
section); none of them runs the tiled online softmax the oracle runs.

* ``dense_attention``      -- softmax(scale * Q K^T) V over all visible keys.
* ``restricted_attention`` -- the same, over the keys of the kept tiles only.
  Skipping a block removes it from the softmax numerator and denominator, so
  the method's output equals dense attention restricted to kept keys.
* ``prefix_max_states``    -- the skip set in closed form. For t < 1 a skipped
  block has m_local < m_run + ln t < m_run, so it can never raise the running
  maximum: m_run before block j equals the prefix maximum of the earlier blocks'
  local maxima whether or not they were skipped.
"""
from __future__ import annotations

import math

import numpy as np

from synth import bf16_to_f32


def _f64(bits):
    return bf16_to_f32(bits).astype(np.float64)


def logits(q_bits, k_bits, scale):
    """[B,Hq,L,d] x [B,Hkv,L,d] -> scaled logits [B,Hq,L,L] in fp64."""
    q, k = _f64(q_bits), _f64(k_bits)
    G = q.shape[1] // k.shape[1]
    k = np.repeat(k, G, axis=1)
    return scale * np.einsum("bhrd,bhcd->bhrc", q, k)


def causal_mask(L):
    r = np.arange(L)[:, None]
    c = np.arange(L)[None, :]
    return c <= r


def masked_softmax_attention(S, v_bits, allowed):
    """softmax over `allowed` keys of S [B,H,L,L], times V [B,Hkv,L,d]; fp64."""
    v = _f64(v_bits)
    G = S.shape[1] // v.shape[1]
    v = np.repeat(v, G, axis=1)
    S = np.where(allowed, S, -np.inf)
    m = S.max(axis=-1, keepdims=True)
    P = np.where(allowed, np.exp(S - m), 0.0)
    l = P.sum(axis=-1, keepdims=True)
    O = np.einsum("bhrc,bhcd->bhrd", P, v) / l
    lse = (m + np.log(l))[..., 0]
    return O, lse


def dense_attention(q_bits, k_bits, v_bits, *, causal, scale):
    S = logits(q_bits, k_bits, scale)
    L = S.shape[-1]
    allowed = np.broadcast_to(causal_mask(L) if causal else np.ones((L, L), bool), S.shape)
    return masked_softmax_attention(S, v_bits, allowed)


def kept_key_mask(tile_state, L, Br, Bc, causal):
    """tile_state [B,Hq,n_q,n_k] (1 = kept) -> allowed [B,Hq,L,L]."""
    rows_tile = np.arange(L) // Br
    keys_tile = np.arange(L) // Bc
    kept = tile_state == 1
    allowed = kept[:, :, rows_tile][:, :, :, keys_tile]
    if causal:
        allowed = allowed & causal_mask(L)
    return allowed


def restricted_attention(q_bits, k_bits, v_bits, tile_state, *, causal, scale, Br, Bc):
    S = logits(q_bits, k_bits, scale)
    L = S.shape[-1]
    return masked_softmax_attention(S, v_bits, kept_key_mask(tile_state, L, Br, Bc, causal))


def prefix_max_states(q_bits, k_bits, *, causal, scale, tsf, Br, Bc):
    """Closed-form skip set (valid for t = tsf/L < 1): 1 kept, 2 skipped, 0 unvisited."""
    S = logits(q_bits, k_bits, scale)
    B, H, L, _ = S.shape
    n_q, n_k = -(-L // Br), -(-L // Bc)
    ln_t = math.log(tsf / L) if tsf > 0 else -math.inf
    if causal:
        S = np.where(causal_mask(L), S, -np.inf)
    states = np.zeros((B, H, n_q, n_k), np.int8)
    for i in range(n_q):
        r0, r1 = i * Br, min(L, (i + 1) * Br)
        j_max = min(n_k - 1, ((i + 1) * Br - 1) // Bc) if causal else n_k - 1
        m_loc = np.stack([S[:, :, r0:r1, j * Bc:min(L, (j + 1) * Bc)].max(axis=-1)
                          for j in range(j_max + 1)], axis=-1)  # [B,H,rows,j]
        prefix = np.full(m_loc.shape[:-1], -np.inf)
        for j in range(j_max + 1):
            ml = m_loc[..., j]
            with np.errstate(invalid="ignore"):
                passes = np.where(ml == -np.inf, ln_t > -np.inf,
                                  np.where(prefix == -np.inf, False, (ml - prefix) < ln_t))
            skip = passes.all(axis=-1)
            states[:, :, i, j] = np.where(skip, 2, 1)
            prefix = np.maximum(prefix, ml)
    return states


def decode_logits(q_bits, k_bits, Lb, scale):
    """q [G,d], k [L,d] of one (batch, kv head) -> [G, Lb] fp64."""
    return scale * (_f64(q_bits) @ _f64(k_bits[:Lb]).T)


def decode_dense(q_bits, kc_bits, vc_bits, seqlens, *, scale, tile_state=None, Bc=None):
    """Dense (or kept-tile restricted) decode attention in fp64: o [B,Hq,d], lse [B,Hq]."""
    B, Hq, d = q_bits.shape
    Hkv = kc_bits.shape[1]
    G = Hq // Hkv
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        Lb = int(seqlens[b])
        for h in range(Hkv):
            S = decode_logits(q_bits[b, h * G:(h + 1) * G], kc_bits[b, h], Lb, scale)
            allowed = np.ones(Lb, bool)
            if tile_state is not None:
                allowed = tile_state[b, h][np.arange(Lb) // Bc] == 1
            S = np.where(allowed[None, :], S, -np.inf)
            m = S.max(axis=1, keepdims=True)
            P = np.exp(S - m)
            l = P.sum(axis=1, keepdims=True)
            o[b, h * G:(h + 1) * G] = (P @ _f64(vc_bits[b, h, :Lb])) / l
            lse[b, h * G:(h + 1) * G] = (m + np.log(l))[:, 0]
    return o, lse


def decode_prefix_max_states(q_bits, kc_bits, seqlens, *, scale, tsf, Bc, num_splits):
    """Closed-form joint skip set per (batch, kv head), split by split (t < 1)."""
    B, Hq, d = q_bits.shape
    Hkv, Lmax = kc_bits.shape[1], kc_bits.shape[2]
    G = Hq // Hkv
    states = np.zeros((B, Hkv, -(-Lmax // Bc)), np.int8)
    for b in range(B):
        Lb = int(seqlens[b])
        ln_t = math.log(tsf / Lb) if tsf > 0 else -math.inf
        n_k = -(-Lb // Bc)
        c = -(-n_k // num_splits)
        for h in range(Hkv):
            S = decode_logits(q_bits[b, h * G:(h + 1) * G], kc_bits[b, h], Lb, scale)
            m_loc = np.stack([S[:, j * Bc:min(Lb, (j + 1) * Bc)].max(axis=1) for j in range(n_k)], 1)
            for s in range(num_splits):
                prefix = np.full(G, -np.inf)
                for j in range(s * c, min((s + 1) * c, n_k)):
                    ml = m_loc[:, j]
                    passes = np.where(prefix == -np.inf, False, (ml - prefix) < ln_t)
                    states[b, h, j] = 2 if passes.all() else 1
                    prefix = np.maximum(prefix, ml)
    return states


def prefix_max_row_passes(q_bits, k_bits, *, causal, scale, tsf, Br, Bc):
    """Closed-form vote of every row on every tile its query tile visits (t < 1).

    Returns (passes [B,H,L,n_k] bool, visited [n_q,n_k] bool). Same argument as
    ``prefix_max_states``: while t < 1 no passing block can raise a row's
    running maximum, so the maximum before block j is the prefix maximum of the
    row's local maxima over blocks 0..j-1, whatever its slice decided.
    """
    S = logits(q_bits, k_bits, scale)
    B, H, L, _ = S.shape
    n_q, n_k = -(-L // Br), -(-L // Bc)
    ln_t = math.log(tsf / L) if tsf > 0 else -math.inf
    if causal:
        S = np.where(causal_mask(L), S, -np.inf)
    m_loc = np.stack([S[..., j * Bc:min(L, (j + 1) * Bc)].max(axis=-1) for j in range(n_k)],
                     axis=-1)  # [B,H,L,n_k]
    passes = np.zeros((B, H, L, n_k), bool)
    visited = np.zeros((n_q, n_k), bool)
    prefix = np.full((B, H, L), -np.inf)
    for j in range(n_k):
        ml = m_loc[..., j]
        with np.errstate(invalid="ignore"):
            passes[..., j] = np.where(ml == -np.inf, ln_t > -np.inf,
                                      np.where(prefix == -np.inf, False, (ml - prefix) < ln_t))
        prefix = np.maximum(prefix, ml)
    for i in range(n_q):
        j_max = min(n_k - 1, ((i + 1) * Br - 1) // Bc) if causal else n_k - 1
        visited[i, :j_max + 1] = True
    return passes, visited


def slice_masks(passes, visited, *, L, Br, R):
    """Per (b, h, query tile, key tile): 0 if not visited, else 0x80 | bitmask
    of the R-row slices whose every valid row passes (a slice with no valid
    row passes vacuously)."""
    B, H, _, n_k = passes.shape
    n_q = visited.shape[0]
    out = np.zeros((B, H, n_q, n_k), np.uint8)
    for i in range(n_q):
        for j in range(n_k):
            if not visited[i, j]:
                continue
            m = 0x80
            for s in range(Br // R):
                r0, r1 = i * Br + s * R, min(L, i * Br + (s + 1) * R)
                m_s = np.ones((B, H), bool) if r0 >= r1 else passes[:, :, r0:r1, j].all(axis=-1)
                out[:, :, i, j] |= np.where(m_s, 1 << s, 0).astype(np.uint8)
            out[:, :, i, j] |= m
    return out


def slice_kept_key_mask(slice_mask, L, Br, Bc, R, causal):
    """slice_mask [B,H,n_q,n_k] -> allowed [B,H,L,L]: row r sees the keys of
    tile j iff its query tile visited j and r's slice did not skip it."""
    r = np.arange(L)
    bit = ((r % Br) // R).astype(np.uint8)
    sm = slice_mask[:, :, r // Br]                       # [B,H,L,n_k]
    kept_tile = (sm & 0x80).astype(bool) & ~((sm >> bit[None, None, :, None]) & 1).astype(bool)
    allowed = kept_tile[..., np.arange(L) // Bc]
    if causal:
        allowed = allowed & causal_mask(L)
    return allowed


def slice_restricted_attention(q_bits, k_bits, v_bits, slice_mask, *, causal, scale, Br, Bc, R):
    S = logits(q_bits, k_bits, scale)
    L = S.shape[-1]
    return masked_softmax_attention(S, v_bits,
                                    slice_kept_key_mask(slice_mask, L, Br, Bc, R, causal))


def prefill_critical_factors(q_bits, k_bits, *, causal, scale, Br, Bc):
    """ln of the smallest threshold_scale_factor at which each visited tile is
    skipped, in closed form (t < 1): the tile is skipped iff every valid row
    has m_local - prefix_max < ln(tsf / L), i.e. iff
    ln tsf > max_r (m_local - prefix_max) + ln L. +inf for a tile no factor
    below L skips (the first tile). Returns [B, H, n_q, n_k] with NaN where
    the tile is not visited."""
    S = logits(q_bits, k_bits, scale)
    B, H, L, _ = S.shape
    n_q, n_k = -(-L // Br), -(-L // Bc)
    if causal:
        S = np.where(causal_mask(L), S, -np.inf)
    out = np.full((B, H, n_q, n_k), np.nan)
    for i in range(n_q):
        r0, r1 = i * Br, min(L, (i + 1) * Br)
        j_max = min(n_k - 1, ((i + 1) * Br - 1) // Bc) if causal else n_k - 1
        prefix = np.full((B, H, r1 - r0), -np.inf)
        for j in range(j_max + 1):
            ml = S[:, :, r0:r1, j * Bc:min(L, (j + 1) * Bc)].max(axis=-1)
            with np.errstate(invalid="ignore"):
                gap = np.where(ml == -np.inf, -np.inf,
                               np.where(prefix == -np.inf, np.inf, ml - prefix))
            out[:, :, i, j] = gap.max(axis=-1) + math.log(L)
            prefix = np.maximum(prefix, ml)
    return out


def decode_critical_factors(q_bits, kc_bits, seqlens, *, scale, Bc, num_splits):
    """Decode version: joint vote of the G heads, per-split running maximum,
    t_b = tsf / L_b. [B, Hkv, ceil(Lmax/Bc)], NaN beyond each sequence."""
    B, Hq, d = q_bits.shape
    Hkv, Lmax = kc_bits.shape[1], kc_bits.shape[2]
    G = Hq // Hkv
    out = np.full((B, Hkv, -(-Lmax // Bc)), np.nan)
    for b in range(B):
        Lb = int(seqlens[b])
        n_k = -(-Lb // Bc)
        c = -(-n_k // num_splits)
        for h in range(Hkv):
            S = decode_logits(q_bits[b, h * G:(h + 1) * G], kc_bits[b, h], Lb, scale)
            m_loc = np.stack([S[:, j * Bc:min(Lb, (j + 1) * Bc)].max(axis=1) for j in range(n_k)], 1)
            for s in range(num_splits):
                prefix = np.full(G, -np.inf)
                for j in range(s * c, min((s + 1) * c, n_k)):
                    ml = m_loc[:, j]
                    gap = np.where(prefix == -np.inf, np.inf, ml - prefix)
                    out[b, h, j] = gap.max() + math.log(Lb)
                    prefix = np.maximum(prefix, ml)
    return out
