"""Merger parity: GPU moe_combine against the oracle's combine().

y_packed and the shared output come as fp16 or fp32 (the oracle reads the
same values); the only roundings on the GPU are the fp32 sum of k (+1) terms
and one final rounding to the output type, so the bound is per element:
|gpu - oracle| <= 2^-8 |oracle| + 1e-6 rms for a bf16 output, 1e-6 |oracle| +
1e-6 rms for an fp32 output.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_44_b200 as M
import oracle.moe_oracle as O
from tests.gpu_util import DEV, dev

pytestmark = pytest.mark.gpu


def _run(y, inv_perm, T, k, shared=None, sg=None, out_dtype=torch.float32):
    H = y.shape[1]
    out = torch.full((T, H), 77.0, dtype=out_dtype, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    M.moe_combine(dev(y), dev(inv_perm), T, k, out, dev(shared), dev(sg), status=status)
    torch.cuda.synchronize()
    return out.cpu(), int(status.item())


def _bound(got, want, dtype):
    g = O.to_f64(got)
    rms = np.sqrt(np.mean(want * want))
    rtol = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-6
    assert (np.abs(g - want) <= rtol * np.abs(want) + 1e-6 * rms).all()


@pytest.mark.parametrize("T,k,H", [(1, 1, 8), (64, 2, 128), (333, 8, 2048), (4096, 2, 4096),
                                   (32, 4, 2048), (7, 3, 72)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("y_dtype", [torch.float32, torch.float16])
def test_combine(T, k, H, dtype, y_dtype):
    rng = np.random.default_rng(T + k)
    N = T * k
    y = torch.randn(N, H, generator=torch.Generator().manual_seed(N)).to(y_dtype)
    inv = torch.tensor(rng.permutation(N), dtype=torch.int32)
    out, st = _run(y, inv, T, k, out_dtype=dtype)
    assert st == 0
    _bound(out, O.combine(y, inv.numpy(), T, k), dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("y_dtype", [torch.float32, torch.float16])
def test_combine_with_shared_expert_gate(dtype, y_dtype):
    g = torch.Generator().manual_seed(9)
    T, k, H = 50, 4, 256
    y = torch.randn(T * k, H, generator=g).to(y_dtype)
    inv = torch.randperm(T * k, generator=g).to(torch.int32)
    sh = torch.randn(T, H, generator=g).to(y_dtype)
    sg = torch.randn(T, generator=g) * 3
    out, st = _run(y, inv, T, k, sh, sg, out_dtype=dtype)
    assert st == 0
    _bound(out, O.combine(y, inv.numpy(), T, k, sh, sg), dtype)


def test_combine_bad_inverse_permutation_is_reported_and_skipped():
    y = torch.randn(8, 64)
    inv = torch.tensor([0, 1, 2, -1, 4, 99, 6, 7], dtype=torch.int32)
    out, st = _run(y, inv, 4, 2)
    assert st == M.MOE_ERR_BAD_INDEX
    np.testing.assert_allclose(out[1].numpy(), y[2].numpy(), rtol=1e-6)   # j=1 skipped
    np.testing.assert_allclose(out[2].numpy(), y[4].numpy(), rtol=1e-6)   # j=1 skipped
    np.testing.assert_allclose(out[0].numpy(), (y[0] + y[1]).numpy(), rtol=1e-6)
