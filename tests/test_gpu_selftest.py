"""Bounded device waits: a wait on an mbarrier that nothing completes gives up
after its limit, records its site and lets the kernel return; the host reads
USP_ERR_TIMEOUT and the context stays usable."""
import pytest
import torch

from long_context_exact_tma_b200 import api
from long_context_exact_tma_b200 import binding as B_

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives(cuda):
    ws = api.workspace(256, cuda)
    B_.usp_selftest_wait_timeout(ws, ws.numel(), 20_000_000)  # 20 ms
    rc, site = B_.usp_workspace_status(ws)
    assert rc == B_.USP_ERR_TIMEOUT and site == 0x7E57
    rc, site = B_.usp_workspace_status(ws)  # cleared by the read
    assert rc == B_.USP_OK and site == 0
    x = torch.ones(1024, device=cuda)
    assert float(x.sum()) == 1024.0
