"""Synthetic workload definitions for Skip-Softmax tiled attention.

These describe shapes, tile sizes, thresholds and the planted structure of the
seeded inputs. They hold no attention arithmetic: the same definitions feed the
CPU oracle (test infrastructure) and the CUDA path.

The shapes stand in for the models the TensorRT-LLM Skip-Softmax article
measures ("Skip Softmax 带来了哪些实战好处" section: Llama 3.3 70B at 128K,
Llama 3.1 8B at 16K) and for the video-DiT token grids of the SpargeAttn page
(Table 1: CogvideoX 17K). No item of any dataset or benchmark suite is used;
every input is drawn from a seeded generator.

Two readings of the planted direction ``u`` exist:

* ``"lit"``  -- ``|u| = 1`` exactly as the workload text states;
* ``"rms"``  -- ``|u| = sqrt(d)``, the same per-component scale as the N(0,1)
  noise, so that planted tiles dominate the logits.
"""
from __future__ import annotations

import dataclasses
import math

READINGS = ("lit", "rms")


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    causal: bool
    Br: int
    Bc: int
    tsf: float            # threshold_scale_factor; t = tsf / L
    seed: int
    kind: str = "planted"  # "planted" or "video"
    q_shift: float = 0.0   # every query row += q_shift * u
    hot_frac: float = 0.0  # fraction of key tiles (per batch, kv head) planted
    hot_gain: float = 0.0  # keys of planted tiles += hot_gain * u
    sink_keys: int = 0     # first keys += sink_gain * u
    sink_gain: float = 0.0
    video_grid: tuple = ()  # (T, H, W) raster for kind == "video"
    video_terms: int = 0
    video_noise: float = 0.0
    sm_scale: float = 0.0  # 0 -> 1/sqrt(d)

    @property
    def scale(self) -> float:
        return self.sm_scale if self.sm_scale > 0 else 1.0 / math.sqrt(self.d)

    @property
    def n_q(self) -> int:
        return -(-self.L // self.Br)

    @property
    def n_k(self) -> int:
        return -(-self.L // self.Bc)

    def replace(self, **kw) -> "PrefillWorkload":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lmax: int
    Lmin: int
    d: int
    Bc: int
    num_splits: int
    tsf: float
    seed: int
    q_shift: float = 0.5
    hot_frac: float = 0.15
    hot_gain: float = 2.0
    sink_keys: int = 4
    sink_gain: float = 3.0
    sm_scale: float = 0.0

    @property
    def scale(self) -> float:
        return self.sm_scale if self.sm_scale > 0 else 1.0 / math.sqrt(self.d)

    def replace(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


# Tiny causal prefill: one head, 16 tiles of 64; 10 % of key tiles get +4u.
TINY_PREFILL = PrefillWorkload(
    name="prefill_tiny_L1024_d64", B=1, Hq=1, Hkv=1, L=1024, d=64, causal=True,
    Br=64, Bc=64, tsf=100.0, seed=1000, q_shift=1.0, hot_frac=0.10, hot_gain=4.0,
    sm_scale=1.0 / 8.0)

# Llama-3.1-8B-shaped GQA prefill at 16K.
LLAMA8B_PREFILL_16K = PrefillWorkload(
    name="prefill_llama8b_L16384_Hq32_Hkv8_d128", B=1, Hq=32, Hkv=8, L=16384, d=128,
    causal=True, Br=128, Bc=128, tsf=1000.0, seed=1001, q_shift=0.5, hot_frac=0.15,
    hot_gain=2.0, sink_keys=4, sink_gain=3.0)

# Llama-3.3-70B-layer-shaped prefill at 128K; the threshold is swept.
LLAMA70B_PREFILL_128K = PrefillWorkload(
    name="prefill_llama70b_L131072_Hq64_Hkv8_d128", B=1, Hq=64, Hkv=8, L=131072, d=128,
    causal=True, Br=128, Bc=128, tsf=1000.0, seed=1002, q_shift=0.5, hot_frac=0.15,
    hot_gain=2.0, sink_keys=4, sink_gain=3.0)
LLAMA70B_TSF_SWEEP = (0.0, 100.0, 1000.0, 5000.0)

# Batched GQA decode over a contiguous KV cache, lengths uniform in [16K, 32K].
DECODE_B64_32K = DecodeWorkload(
    name="decode_B64_Hq32_Hkv8_d128_L16K-32K", B=64, Hq=32, Hkv=8, Lmax=32768,
    Lmin=16384, d=128, Bc=64, num_splits=16, tsf=500.0, seed=1003)

# Non-causal video-DiT-shaped MHA prefill on a 13 x 32 x 43 token raster.
# 13*32*43 = 17888 grid positions; L = 17776 keeps the first 17776 of them in
# t-major raster order.
VIDEO_DIT_PREFILL = PrefillWorkload(
    name="prefill_videodit_B2_H48_L17776_d64_noncausal", B=2, Hq=48, Hkv=48, L=17776,
    d=64, causal=False, Br=128, Bc=128, tsf=1000.0, seed=1004, kind="video",
    video_grid=(13, 32, 43), video_terms=8, video_noise=0.3)

PREFILL_WORKLOADS = {w.name: w for w in (TINY_PREFILL, LLAMA8B_PREFILL_16K,
                                         LLAMA70B_PREFILL_128K, VIDEO_DIT_PREFILL)}
DECODE_WORKLOADS = {DECODE_B64_32K.name: DECODE_B64_32K}
