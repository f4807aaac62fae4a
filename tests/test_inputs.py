"""The seeded workload generator: determinism, shapes, distributions, load skew."""
import math

import numpy as np
import torch

import oracle as O
from moe_inputs import CONFIGS, LayerConfig, make_layer, make_tokens


def test_deterministic_and_seed_sensitive():
    cfg = CONFIGS["tiny_f32"]
    a = make_layer(cfg, seed=0)
    b = make_layer(cfg, seed=0)
    c = make_layer(cfg, seed=1)
    for key in ("x", "W_gate", "w13", "w2"):
        assert torch.equal(a[key], b[key])
        assert not torch.equal(a[key], c[key])


def test_shapes_dtypes_and_w13_is_w1_then_w3():
    cfg = LayerConfig("t", T=5, H=16, E=3, k=2, I=8, dtype="bf16", renormalize=False, shared_I=12)
    p = make_layer(cfg, seed=3)
    assert p["x"].shape == (5, 16) and p["x"].dtype == torch.bfloat16
    assert p["W_gate"].shape == (3, 16)
    assert p["w13"].shape == (3, 16, 16) and p["w2"].shape == (3, 16, 8)
    assert p["w13s"].shape == (24, 16) and p["w2s"].shape == (16, 12) and p["w_sg"].shape == (16,)
    # Re-draw w1 / w3 in the documented order and check the fused layout.
    g = torch.Generator().manual_seed(3)
    torch.randn(5, 16, generator=g)
    torch.randn(3, 16, generator=g)
    w1 = [torch.randn(8, 16, generator=g) / 4 for _ in range(3)]
    w3 = [torch.randn(8, 16, generator=g) / 4 for _ in range(3)]
    for e in range(3):
        assert torch.equal(p["w13"][e, :8], w1[e].to(torch.bfloat16))
        assert torch.equal(p["w13"][e, 8:], w3[e].to(torch.bfloat16))


def test_weight_scales_follow_fan_in():
    cfg = LayerConfig("t", T=256, H=256, E=4, k=2, I=512, dtype="f32", renormalize=True)
    p = make_layer(cfg, seed=0)
    assert abs(p["x"].std().item() - 1.0) < 0.02
    assert abs(p["w13"].std().item() * math.sqrt(256) - 1.0) < 0.02
    assert abs(p["w2"].std().item() * math.sqrt(512) - 1.0) < 0.02


def test_make_tokens_is_a_fresh_batch():
    cfg = CONFIGS["tiny_f32"]
    assert torch.equal(make_tokens(cfg, 5), make_tokens(cfg, 5))
    assert not torch.equal(make_tokens(cfg, 5), make_tokens(cfg, 6))


def _realised_counts(cfg, seed=0):
    """Route a reduced-width stand-in of ``cfg`` with the oracle (H=256 keeps it fast;
    the logit variance is 1 at any H)."""
    small = LayerConfig("z", T=cfg.T, H=256, E=cfg.E, k=cfg.k, I=8, dtype="f32",
                        renormalize=cfg.renormalize, zipf_s=cfg.zipf_s, empty_tail=cfg.empty_tail)
    p = make_layer(small, seed)
    _, ids, _ = O.route(p["x"], p["W_gate"], p["bias"], cfg.k, cfg.renormalize)
    return np.bincount(ids.ravel(), minlength=cfg.E), p["bias"].numpy()


def test_zipf_bias_gives_skewed_load_with_slope_near_minus_s():
    for name in ("builder_bf16", "qwen3_t16384"):
        cfg = CONFIGS[name]
        counts, bias = _realised_counts(cfg)
        live = bias > -29
        order = np.argsort(-bias[live])                  # by Zipf rank
        c = counts[live][order].astype(float)
        ranks = np.arange(1, len(c) + 1)
        m = c > 0
        slope = np.polyfit(np.log(ranks[m]), np.log(c[m]), 1)[0]
        assert abs(slope + cfg.zipf_s) < 0.3, (name, slope)
        assert counts[~live].sum() == 0                  # forced-empty experts get nothing
        assert (~live).sum() == cfg.empty_tail
