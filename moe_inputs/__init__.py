"""Seeded synthetic inputs for one Mixture-of-Experts layer.

This module is shared by the fp64 oracle (``oracle/``), the GPU tests and the
benchmark.  It holds random draws and the shape table only: no routing,
dispatch, expert or merge arithmetic lives here, so neither side can inherit a
mistake in the method from it.

Workloads (the layer shapes the pages' sources imply):

* ``tiny_f32``      -- T=64, H=128, E=8, k=2, I=256, all fp32, renormalised.
* ``builder_bf16``  -- the runtime's explicit-layer example (hidden 4096,
  64 experts, top-2; DWDP README, "How To Use", ``build_reference``), I=1408,
  T=4096, bf16, renormalised, Zipf(1.0)-skewed expert load.
* ``qwen15_t32`` / ``qwen15_t8192`` -- Qwen1.5-MoE-A2.7B-shaped layer (the
  model the DWDP README benchmarks and its adapter targets): H=2048, E=60,
  k=4, I=1408, softmax top-k WITHOUT renormalisation, plus one always-on
  shared SwiGLU expert (I_s=5632) scaled by a sigmoid gate.
* ``qwen3_t16384``  -- Qwen3-30B-A3B-shaped layer (128 experts, as the
  modelexpress refit test's coverage note counts): H=2048, E=128, k=8, I=768,
  renormalised, Zipf(1.1) load with the 8 least popular experts given no
  tokens at all.
* ``decode_t1`` / ``decode_t8`` / ``decode_t64`` -- decode-bound large-expert
  layer: H=4096, E=8, k=2, I=14336, renormalised.

Recipe (every workload): a CPU ``torch.Generator`` seeded with ``seed`` draws,
in this order, fp32 normals for x[T,H]; W_gate[E,H]; w1[e] ([I,H]) for each
expert e in turn; w3[e] ([I,H]) likewise; w2[e] ([H,I]) likewise; then, for
the shared expert, w1s[I_s,H], w3s[I_s,H], w2s[H,I_s], w_sg[H]; and last the
Zipf rank permutation.  x ~ N(0,1); every weight ~ N(0, 1/fan_in) with
fan_in = H for W_gate, w1, w3, w1s, w3s and w_sg and fan_in = I (I_s) for w2
(w2s).  bf16 workloads round each fp32 draw to bf16 (round to nearest even).
The fused gate/up buffer is ``w13[e] = cat(w1[e], w3[e])`` along rows, gate
(w1) in rows [0, I) and up (w3) in rows [I, 2I), the layout the modelexpress
refit test pins for ``w13_weight`` (shape [E, 2*I, H]).

Zipf load: a seeded permutation gives each expert a rank r(e) in 1..E, the
target share is q_r proportional to r**-s, and the router bias is
b_e = 0.5 * ln(q_r(e)), stored as fp32.  With x ~ N(0,1) and W_gate ~
N(0,1/H) the router logits have unit variance, and under that noise a bias of
half the log-share gives a realised load whose log-log slope against rank is
close to -s; the realised histogram is recorded by the benchmark rather than
assumed.  ``empty_tail`` experts (the highest ranks) get b_e = -30, which no
unit-variance logit overcomes, so they receive no tokens.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = ["LayerConfig", "CONFIGS", "make_layer", "make_tokens", "layer_nbytes"]


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    dtype: str                      # "f32" or "bf16"
    renormalize: bool
    zipf_s: Optional[float] = None  # router-bias skew; None = no bias
    empty_tail: int = 0             # experts forced to receive no tokens
    shared_I: Optional[int] = None  # always-on shared SwiGLU expert

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_tokens(self, T: int) -> "LayerConfig":
        return dataclasses.replace(self, T=T)


CONFIGS = {
    c.name: c
    for c in [
        LayerConfig("tiny_f32", T=64, H=128, E=8, k=2, I=256, dtype="f32", renormalize=True),
        LayerConfig("builder_bf16", T=4096, H=4096, E=64, k=2, I=1408, dtype="bf16",
                    renormalize=True, zipf_s=1.0),
        LayerConfig("qwen15_t32", T=32, H=2048, E=60, k=4, I=1408, dtype="bf16",
                    renormalize=False, shared_I=5632),
        LayerConfig("qwen15_t8192", T=8192, H=2048, E=60, k=4, I=1408, dtype="bf16",
                    renormalize=False, shared_I=5632),
        LayerConfig("qwen3_t16384", T=16384, H=2048, E=128, k=8, I=768, dtype="bf16",
                    renormalize=True, zipf_s=1.1, empty_tail=8),
        LayerConfig("decode_t1", T=1, H=4096, E=8, k=2, I=14336, dtype="bf16", renormalize=True),
        LayerConfig("decode_t8", T=8, H=4096, E=8, k=2, I=14336, dtype="bf16", renormalize=True),
        LayerConfig("decode_t64", T=64, H=4096, E=8, k=2, I=14336, dtype="bf16", renormalize=True),
    ]
}


def _normal(gen: torch.Generator, shape, std: float, dtype: torch.dtype) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t if dtype == torch.float32 else t.to(dtype)


def _stacked(gen, E, rows, cols, std, dtype) -> torch.Tensor:
    """E matrices [rows, cols] drawn one after another into one [E, rows, cols] tensor."""
    out = torch.empty(E, rows, cols, dtype=dtype)
    for e in range(E):
        out[e].copy_(_normal(gen, (rows, cols), std, dtype))
    return out


def make_layer(cfg: LayerConfig, seed: int = 0) -> dict:
    """Draw every tensor of one layer instance on the CPU (see module docstring).

    Returns a dict of CPU tensors: ``x [T,H]``, ``W_gate [E,H]``, ``bias [E] f32``
    or None, ``w13 [E,2I,H]``, ``w2 [E,H,I]`` and, when the workload has a
    shared expert, ``w13s [2I_s,H]``, ``w2s [H,I_s]``, ``w_sg [H]`` (else None).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    dt = cfg.torch_dtype
    T, H, E, I = cfg.T, cfg.H, cfg.E, cfg.I
    x = _normal(gen, (T, H), 1.0, dt)
    W_gate = _normal(gen, (E, H), 1.0 / math.sqrt(H), dt)
    w1 = _stacked(gen, E, I, H, 1.0 / math.sqrt(H), dt)
    w3 = _stacked(gen, E, I, H, 1.0 / math.sqrt(H), dt)
    w13 = torch.cat([w1, w3], dim=1)
    del w1, w3
    w2 = _stacked(gen, E, H, I, 1.0 / math.sqrt(I), dt)
    w13s = w2s = w_sg = None
    if cfg.shared_I:
        Is = cfg.shared_I
        w1s = _normal(gen, (Is, H), 1.0 / math.sqrt(H), dt)
        w3s = _normal(gen, (Is, H), 1.0 / math.sqrt(H), dt)
        w13s = torch.cat([w1s, w3s], dim=0)
        del w1s, w3s
        w2s = _normal(gen, (H, Is), 1.0 / math.sqrt(Is), dt)
        w_sg = _normal(gen, (H,), 1.0 / math.sqrt(H), dt)
    bias = None
    if cfg.zipf_s is not None:
        rank = torch.randperm(E, generator=gen) + 1          # r(e) in 1..E
        r = rank.to(torch.float64)
        q = r.pow(-cfg.zipf_s)
        q = q / q.sum()
        b = 0.5 * torch.log(q)
        if cfg.empty_tail:
            b[rank > E - cfg.empty_tail] = -30.0
        bias = b.to(torch.float32)
    return dict(x=x, W_gate=W_gate, bias=bias, w13=w13, w2=w2,
                w13s=w13s, w2s=w2s, w_sg=w_sg)


def make_tokens(cfg: LayerConfig, seed: int) -> torch.Tensor:
    """A fresh activation batch x[T,H] ~ N(0,1) for replica ``seed`` (weights unchanged)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return _normal(gen, (cfg.T, cfg.H), 1.0, cfg.torch_dtype)


def layer_nbytes(cfg: LayerConfig) -> int:
    """Bytes of all weights of one layer instance (for memory planning only)."""
    es = 4 if cfg.dtype == "f32" else 2
    n = cfg.E * cfg.H + 3 * cfg.E * cfg.H * cfg.I
    if cfg.shared_I:
        n += 3 * cfg.H * cfg.shared_I + cfg.H
    return n * es
