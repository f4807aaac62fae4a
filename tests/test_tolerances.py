"""The comparison rules the GPU parity tests use, checked on the CPU."""
import numpy as np
import torch

import oracle.moe_oracle as O
from tests.gpu_util import bf16_half_ulp, err_bf16_out


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
