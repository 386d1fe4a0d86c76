"""Seeded synthetic inputs for Skip-Softmax tiled attention.

This package is shared by the CPU oracle (test infrastructure) and the CUDA
path. It generates inputs only and contains none of the attention arithmetic.
"""
from .generate import (bf16_bits, bf16_to_f32, decode_inputs, decode_seqlens,
                       hot_tiles, prefill_inputs, round_half_up, unit_direction)
from .workloads import (DECODE_B64_32K, DECODE_WORKLOADS, LLAMA8B_PREFILL_16K,
                        LLAMA70B_PREFILL_128K, LLAMA70B_TSF_SWEEP, PREFILL_WORKLOADS,
                        READINGS, TINY_PREFILL, VIDEO_DIT_PREFILL, DecodeWorkload,
                        PrefillWorkload)
