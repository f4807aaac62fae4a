"""The comparison rules the GPU parity tests use, checked on the CPU."""
import numpy as np
import torch

import oracle.moe_oracle as O
from tests.gpu_util import bf16_half_ulp, err_bf16_out, err_stored, f16_half_ulp


def test_half_ulp_bounds_a_correct_bf16_rounding():
    rng = np.random.default_rng(0)
    # fp32 values rounded once to bf16, as the kernels store them
    a = (rng.standard_normal(100000) * 10.0 ** rng.integers(-3, 4, size=100000)).astype(np.float32)
    r = torch.tensor(a).to(torch.bfloat16).double().numpy()
    a = a.astype(np.float64)
    assert (np.abs(r - a) <= bf16_half_ulp(a) * (1 + 1e-12)).all()
    # and it is tight: some value needs (almost) the whole half ulp
    assert (np.abs(r - a) / bf16_half_ulp(a)).max() > 0.99


def test_exactly_rounded_output_scores_zero_but_not_on_the_plain_bound():
    rng = np.random.default_rng(1)
    want = rng.standard_normal((512, 4096)).astype(np.float32).astype(np.float64)
    got = torch.tensor(want).float().to(torch.bfloat16)
    assert err_bf16_out(got, want) == 0.0
    assert O.rel_err_rms(got, want) > 1e-2            # why the allowance exists
    # one element off by 3e-2 rms beyond its rounding is caught
    bad = got.clone()
    bad[7, 9] = float(bad[7, 9]) + 0.03 * np.sqrt(np.mean(want * want)) + 0.2
    assert err_bf16_out(bad, want) > 2e-2


def test_exactly_rounded_swiglu_hidden_fails_the_plain_bound():
    # The expert hidden h = silu(x W1^T) * (x W3^T) is a product of two
    # correlated normals: heavy-tailed (max / rms ~ 18 here), so the bf16
    # store alone moves its largest elements by several percent of the rms.
    # That is why h (a bf16 tensor) is compared beyond its own rounding.
    rng = np.random.default_rng(3)
    H, I, N = 1024, 256, 2048
    x = rng.standard_normal((N, H))
    w13 = rng.standard_normal((2 * I, H)) / np.sqrt(H)
    h = O.expert_hidden(x, w13, I)
    # rounded as the kernels store it: an fp32 value, rounded once to bf16 (the
    # fp64 -> fp32 step can push a value onto a bf16 midpoint: ~1e-8 excess)
    r = torch.tensor(h).float().to(torch.bfloat16)
    assert O.rel_err_rms(r, h) > 2e-2
    assert err_bf16_out(r, h) <= 1e-6


def test_half_ulp_bounds_a_correct_fp16_rounding():
    rng = np.random.default_rng(4)
    # fp32 values inside the fp16 range (normal and subnormal), rounded once
    a = (rng.standard_normal(100000) * 10.0 ** rng.integers(-7, 4, size=100000)).astype(np.float32)
    r = torch.tensor(a).to(torch.float16).double().numpy()
    a = a.astype(np.float64)
    assert (np.abs(r - a) <= f16_half_ulp(a) * (1 + 1e-12)).all()
    assert (np.abs(r - a) / f16_half_ulp(a)).max() > 0.99
    # eight times finer than bf16 for normal values
    n = np.abs(a) > 2.0 ** -14
    np.testing.assert_allclose(bf16_half_ulp(a[n]) / f16_half_ulp(a[n]), 8.0)


def test_err_stored_reads_the_type_of_the_tensor():
    rng = np.random.default_rng(5)
    want = rng.standard_normal((256, 512)).astype(np.float32).astype(np.float64)
    for dt in (torch.bfloat16, torch.float16):
        got = torch.tensor(want).float().to(dt)
        assert err_stored(got, want) == 0.0
        bad = got.clone()
        bad[3, 4] = float(bad[3, 4]) + 0.05
        assert err_stored(bad, want) > 0.04
    # fp32: the plain bound
    got = torch.tensor(want).float()
    assert err_stored(got, want) == O.rel_err_rms(got, want)
