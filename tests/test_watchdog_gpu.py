"""The bounded-wait watchdog on the GPU: a kernel waits on an mbarrier that
nothing completes; the wait runs out, latches SSKIP_ERR_TIMEOUT and returns,
and the context stays usable. No fault, trap or hang is involved."""
import pytest
import torch

import block_sparse_long_tiled_b200 as sk

pytestmark = pytest.mark.gpu


def test_watchdog_times_out_and_context_survives():
    from block_sparse_long_tiled_b200 import build
    build.build()
    assert sk.sskip_get_status() == sk.SSKIP_OK
    sk.sskip_selftest_watchdog(20_000)  # 20 ms limit
    assert sk.sskip_get_status() == sk.SSKIP_ERR_TIMEOUT
    assert sk.sskip_get_status() == sk.SSKIP_OK  # reading clears it
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0
