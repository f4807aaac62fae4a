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


def test_grouped_gemm_abort_path_runs_and_the_context_survives():
    """A 1 us main-loop budget makes the GEMM's ordinary waits run out: it must
    report MOE_ERR_TIMEOUT, drain what it issued and leave the context usable
    (the next call, at the default budget, is correct)."""
    import numpy as np
    import oracle.moe_oracle as O
    from tests.gpu_util import rel
    g = torch.Generator().manual_seed(3)
    counts = [700, 0, 1300, 33, 900, 2048, 5, 640]
    E, H, I = len(counts), 1024, 512
    offs = torch.tensor(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))
    N = int(offs[-1])
    x = torch.randn(N, H, generator=g).to(torch.bfloat16)
    w13 = (torch.randn(E, 2 * I, H, generator=g) / H ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(E, H, I, generator=g) / I ** 0.5).to(torch.bfloat16)
    pw = torch.rand(N, generator=g)
    dx, do, dp, d13, d2 = (t.cuda() for t in (x, offs, pw, w13, w2))
    h = torch.empty(N, I, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(N, H, device="cuda")
    ws = torch.zeros(M.moe_experts_workspace_bytes(N, H, I, E, M.MOE_BF16), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    M.moe_test_set_wait_budget_ns(1000)
    try:
        M.moe_experts(dx, do, dp, d13, d2, h, y, ws=ws, status=status)
        torch.cuda.synchronize()
    finally:
        M.moe_test_set_wait_budget_ns(0)
    assert M.moe_read_status(status) == M.MOE_ERR_TIMEOUT
    assert time.time() - t0 < 10
    # the same context, default budget, fresh workspace: correct again
    ws.zero_()
    status.zero_()
    M.moe_experts(dx, do, dp, d13, d2, h, y, ws=ws, status=status)
    torch.cuda.synchronize()
    assert M.moe_read_status(status) == 0
    ho, yo = O.experts(x, offs.numpy(), pw, w13, w2)
    assert rel(y.cpu(), yo) <= 2e-2


def test_tensor_core_router_abort_path_runs_and_the_context_survives():
    """The same for the tensor-core router, whose CTAs must still pass both
    cluster barriers after a wait ran out."""
    x = torch.randn(4096, 4096, device="cuda").to(torch.bfloat16)
    W = (torch.randn(64, 4096, device="cuda") / 64).to(torch.bfloat16)
    logits = torch.empty(4096, 64, device="cuda")
    ids = torch.empty(4096, 2, dtype=torch.int32, device="cuda")
    w = torch.empty(4096, 2, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    seen = 0
    M.moe_test_set_wait_budget_ns(1000)
    try:
        for _ in range(5):                 # a 1 us budget runs out on the first loads
            status.zero_()
            M.moe_route(x, W, None, 2, True, logits, ids, w, status=status)
            torch.cuda.synchronize()
            seen = M.moe_read_status(status)
            if seen == M.MOE_ERR_TIMEOUT:
                break
    finally:
        M.moe_test_set_wait_budget_ns(0)
    assert seen == M.MOE_ERR_TIMEOUT
    status.zero_()
    M.moe_route(x, W, None, 2, True, logits, ids, w, status=status)
    torch.cuda.synchronize()
    assert M.moe_read_status(status) == 0
    torch.testing.assert_close(logits, x.float() @ W.float().T, rtol=1e-4, atol=1e-3)


def test_wait_budget_hook_rejects_bad_values():
    with pytest.raises(M.MoEError):
        M.moe_test_set_wait_budget_ns(10)
    with pytest.raises(M.MoEError):
        M.moe_test_set_wait_budget_ns(3 * 10 ** 9)
    M.moe_test_set_wait_budget_ns(0)
