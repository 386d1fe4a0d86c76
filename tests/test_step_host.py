"""Host logic of the serving-step call: the factor may be one number or a
{prefill, decode} pair (TensorRT-LLM article, "实战演练")."""
import pytest

import block_sparse_long_tiled_b200 as sk


def test_phase_factors_forms():
    assert sk.phase_factors(1000) == (1000.0, 1000.0)
    assert sk.phase_factors({"prefill": 1000.0, "decode": 500.0}) == (1000.0, 500.0)
    for bad in ({"prefill": 1.0}, {"prefill": 1.0, "decode": 2.0, "x": 3.0}, {"pre": 1, "dec": 2}):
        with pytest.raises(ValueError):
            sk.phase_factors(bad)


def test_step_needs_a_batch():
    with pytest.raises(ValueError):
        sk.sskip_attn_step(threshold_scale_factor=1.0, sm_scale=0.1)
