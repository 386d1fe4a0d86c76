"""Threshold calibration oracle -- TEST INFRASTRUCTURE ONLY.

The Model Optimizer attention-sparsity tutorial (step 4, "用 RULER 校准找到最优
稀疏阈值") calibrates Skip-Softmax by running the model on calibration
samples, collecting the attention statistics and searching for the threshold
that reaches a target sparsity ratio; the TensorRT-LLM article ("实战演练"
closing paragraph) names the same goal: give a target sparsity, get the
threshold factor. Calibration data here are the seeded synthetic workloads.

This oracle is the plain search: bisection on ln(threshold_scale_factor),
each probe a full run of the CPU oracle (``oracle.prefill`` /
``oracle.decode``) read back only through its skip counter. The skip count is
a non-decreasing step function of the factor while t < 1, so for a target
count k the bisection narrows the step where the count first reaches k:
it returns (lo, hi) with count(lo) < k <= count(hi) and hi / lo <= 1 + rtol.
"""
from __future__ import annotations

import math

from . import decode as _decode
from . import prefill as _prefill


def target_count(target_ratio: float, visited: int) -> int:
    """Smallest skipped-tile count whose ratio reaches the target."""
    return min(visited, max(0, math.ceil(target_ratio * visited - 1e-9)))


def bisect_factor(count_at, k: int, lo: float, hi: float, rtol: float = 1e-6,
                  max_iter: int = 200) -> tuple[float, float, int]:
    """Bisection in log space on a non-decreasing step function count_at(f).

    Requires count_at(lo) < k <= count_at(hi). Returns (lo, hi, probes)."""
    c_lo, c_hi = count_at(lo), count_at(hi)
    if not (c_lo < k <= c_hi):
        raise ValueError(f"bracket does not contain the target: {c_lo} < {k} <= {c_hi} fails")
    n = 2
    while hi / lo > 1.0 + rtol and n < max_iter:
        mid = math.sqrt(lo * hi)
        if count_at(mid) >= k:
            hi = mid
        else:
            lo = mid
        n += 1
    return lo, hi, n


def calibrate_prefill(q, k, v, *, causal: bool, sm_scale: float, Br: int, Bc: int,
                      target_ratio: float, lo: float = 1e-6, hi: float | None = None,
                      rtol: float = 1e-6, precision: str = "f64", nthreads=None) -> dict:
    """Bisection for the prefill factor reaching `target_ratio` of skipped
    tiles (upper end of the bracket kept below L, i.e. t < 1)."""
    L = q.shape[2]
    hi = hi if hi is not None else L * (1 - 1e-9)

    def count_at(f):
        return _prefill(q, k, v, causal=causal, sm_scale=sm_scale, tsf=f, Br=Br, Bc=Bc,
                        precision=precision, nthreads=nthreads)["skipped"]

    visited = _prefill(q, k, v, causal=causal, sm_scale=sm_scale, tsf=0.0, Br=Br, Bc=Bc,
                       precision=precision, nthreads=nthreads)["visited"]
    kk = target_count(target_ratio, visited)
    a, b, n = bisect_factor(count_at, kk, lo, hi, rtol)
    return {"lo": a, "hi": b, "k": kk, "visited": visited, "probes": n}


def calibrate_decode(q, kcache, vcache, seqlens, *, sm_scale: float, Bc: int, num_splits: int,
                     target_ratio: float, lo: float = 1e-6, hi: float | None = None,
                     rtol: float = 1e-6, precision: str = "f64", nthreads=None) -> dict:
    """Bisection for the decode factor (t_b = factor / seqlens[b]); the
    bracket stays below the shortest sequence so every t_b < 1."""
    hi = hi if hi is not None else float(min(seqlens)) * (1 - 1e-9)

    def run(f):
        return _decode(q, kcache, vcache, seqlens, sm_scale=sm_scale, tsf=f, Bc=Bc,
                       num_splits=num_splits, precision=precision, nthreads=nthreads)

    visited = run(0.0)["visited"]
    kk = target_count(target_ratio, visited)
    a, b, n = bisect_factor(lambda f: run(f)["skipped"], kk, lo, hi, rtol)
    return {"lo": a, "hi": b, "k": kk, "visited": visited, "probes": n}
