"""Device-side failure reporting without faulting the GPU.

A bounded wait that nothing satisfies gives up after its budget, reports
MOE_ERR_TIMEOUT in the status word, and the context stays usable.
"""
import time

import pytest
import torch

import mixture_experts_layer_44_b200 as M

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_the_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    M.moe_probe_wait_timeout(status, 20_000)          # 20 ms budget
    assert M.moe_read_status(status) == M.MOE_ERR_TIMEOUT
    assert time.time() - t0 < 5
    # the context is still usable: a router call afterwards works
    x = torch.randn(4, 64, device="cuda")
    W = torch.randn(8, 64, device="cuda")
    logits = torch.empty(4, 8, device="cuda")
    ids = torch.empty(4, 2, dtype=torch.int32, device="cuda")
    w = torch.empty(4, 2, device="cuda")
    M.moe_route(x, W, None, 2, True, logits, ids, w)
    torch.cuda.synchronize()
    torch.testing.assert_close(logits, x @ W.T, rtol=1e-5, atol=1e-5)


def test_status_stays_zero_on_a_clean_run():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert M.moe_read_status(status) == 0
