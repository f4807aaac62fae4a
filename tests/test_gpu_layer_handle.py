"""The layer handle (moe_layer_create / moe_layer_forward / moe_layer_forward_host).

* moe_layer_forward runs the same kernels in the same order as the four stage
  calls: its output equals theirs bit for bit (and so inherits their parity
  with the oracle, tested in test_gpu_layer.py);
* moe_layer_forward_host, called for several steps in a row with different
  host batches (uploads, layers and downloads overlapping across steps),
  gives every step exactly the output of moe_layer_forward on that batch;
* the device status word stays clear.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_44_b200 as M
import oracle.moe_oracle as O
from moe_inputs import CONFIGS, LayerConfig, make_layer, make_tokens
from tests.gpu_util import params_to

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("name,groups", [("tiny_f32", (1, 1)), ("builder_bf16", (1, 1)),
                                         ("qwen15_t32", (1, 1)), ("decode_t8", (1, 1)),
                                         ("grouped", (8, 3))])
def test_layer_handle(name, groups):
    cfg = CONFIGS.get(name) or LayerConfig("grouped", T=200, H=512, E=64, k=6, I=192,
                                           dtype="bf16", renormalize=True)
    p = make_layer(cfg, seed=0)
    dp = params_to(p)
    buf = M.MoELayerBuffers(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.torch_dtype,
                            shared_I=cfg.shared_I)
    ref = M.moe_layer_forward(dp["x"], dp, cfg.k, cfg.renormalize, buf, n_groups=groups[0],
                              topk_groups=groups[1]).clone()
    L = M.MoELayer(dp, cfg.T, cfg.k, cfg.renormalize, n_groups=groups[0], topk_groups=groups[1])
    out = torch.empty_like(ref)
    L.forward(dp["x"], out)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out), _bits(ref))
    ids = L.buffer("ids", (cfg.T, cfg.k), torch.int32).cpu()
    assert torch.equal(ids, buf.ids.cpu())
    # pipelined host steps, each with its own batch
    steps = 5
    xs = [make_tokens(cfg, seed=100 + i).pin_memory() for i in range(steps)]
    outs = [torch.empty(cfg.T, cfg.H, dtype=cfg.torch_dtype).pin_memory() for _ in range(steps)]
    for i in range(steps):
        L.forward_host(xs[i], outs[i])
    L.join()
    torch.cuda.synchronize()
    assert L.status() == 0
    for i in range(steps):
        want = torch.empty_like(ref)
        L.forward(xs[i].cuda(), want)
        torch.cuda.synchronize()
        assert torch.equal(_bits(outs[i]), _bits(want.cpu())), i
    L.close()


def test_layer_handle_against_the_oracle_on_host_buffers():
    cfg = LayerConfig("h", T=96, H=256, E=8, k=2, I=128, dtype="bf16", renormalize=True,
                      shared_I=128)
    p = make_layer(cfg, seed=7)
    dp = params_to(p)
    L = M.MoELayer(dp, cfg.T, cfg.k, cfg.renormalize)
    xh = p["x"].pin_memory()
    oh = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
    L.forward_host(xh, oh)
    L.join()
    torch.cuda.synchronize()
    ids = L.buffer("ids", (cfg.T, cfg.k), torch.int32).cpu().numpy()
    l64 = O.router_logits(p["x"], p["W_gate"], None)
    want = O.moe_forward_tokens(p, np.arange(cfg.T), ids, O.routing_weights(l64, ids, True))
    from tests.gpu_util import err_bf16_out
    assert err_bf16_out(oh, want) <= 2e-2


@pytest.mark.parametrize("name", ["qwen15_t32", "decode_t1"])
def test_layer_handle_with_fp32_packed_outputs(name):
    # y_f32: y_packed (and the shared expert's output) kept in fp32, as the
    # Python chain does with MoELayerBuffers(y_f32=True): the same bits
    cfg = CONFIGS[name]
    p = make_layer(cfg, seed=3)
    dp = params_to(p)
    buf = M.MoELayerBuffers(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.torch_dtype,
                            shared_I=cfg.shared_I, y_f32=True)
    assert buf.y_packed.dtype == torch.float32
    ref = M.moe_layer_forward(dp["x"], dp, cfg.k, cfg.renormalize, buf).clone()
    L = M.MoELayer(dp, cfg.T, cfg.k, cfg.renormalize, y_f32=True)
    out = torch.empty_like(ref)
    L.forward(dp["x"], out)
    torch.cuda.synchronize()
    assert L.status() == 0
    assert torch.equal(_bits(out), _bits(ref))
    y = L.buffer("y_packed", (cfg.T * cfg.k, cfg.H), torch.float32)
    assert torch.equal(y, buf.y_packed)
    L.close()
