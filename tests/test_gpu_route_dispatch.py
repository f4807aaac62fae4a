"""One-launch router + dispatcher (moe_route_dispatch) for decode batches.

Its outputs must be bit-identical to moe_route_grouped followed by
moe_dispatch on the same arguments (same routing arithmetic, same stable
order), and through them match the oracle: ids re-derived from the GPU's
logits, the dispatch tables from the oracle's stable counting sort, x_packed
byte-identical to x gathered by packed_tok.  The ticket word must be back at
zero after every call, so that back-to-back calls on one counter stay right.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_44_b200 as M
import oracle.moe_oracle as O
from moe_inputs import LayerConfig, make_layer
from tests.gpu_util import DEV, dev, rel

pytestmark = pytest.mark.gpu

KEYS = ("logits", "ids", "w", "counts", "offsets", "perm", "inv_perm", "packed_tok", "packed_w",
        "x_packed")


def _bufs(T, H, E, k, dtype):
    N = T * k
    i32 = dict(dtype=torch.int32, device=DEV)
    return dict(logits=torch.full((T, E), -7.0, device=DEV),
                ids=torch.full((T, k), -7, **i32), w=torch.full((T, k), -7.0, device=DEV),
                counts=torch.full((E,), -7, **i32), offsets=torch.full((E + 1,), -7, **i32),
                perm=torch.full((N,), -7, **i32), inv_perm=torch.full((N,), -7, **i32),
                packed_tok=torch.full((N,), -7, **i32),
                packed_w=torch.full((N,), -7.0, device=DEV),
                x_packed=torch.zeros(N, H, dtype=dtype, device=DEV),
                status=torch.zeros(1, **i32))


def _fused(x, W, b, k, renorm, G=1, Mg=1, counter=None):
    T, H = x.shape
    E = W.shape[0]
    o = _bufs(T, H, E, k, x.dtype)
    counter = torch.zeros(1, dtype=torch.int32, device=DEV) if counter is None else counter
    M.moe_route_dispatch(x, W, b, k, renorm, o["logits"], o["ids"], o["w"], o["counts"],
                         o["offsets"], o["perm"], o["inv_perm"], o["packed_tok"], o["packed_w"],
                         o["x_packed"], counter, status=o["status"], n_groups=G, topk_groups=Mg)
    torch.cuda.synchronize()
    assert int(counter[0]) == 0, "the ticket word must be back at zero"
    return {key: v.cpu() for key, v in o.items()}


def _separate(x, W, b, k, renorm, G=1, Mg=1):
    T, H = x.shape
    E = W.shape[0]
    o = _bufs(T, H, E, k, x.dtype)
    M.moe_route_grouped(x, W, b, k, renorm, G, Mg, o["logits"], o["ids"], o["w"],
                        status=o["status"])
    ws = torch.empty(M.moe_dispatch_workspace_bytes(T, k, E), dtype=torch.uint8, device=DEV)
    M.moe_dispatch(o["ids"], o["w"], x, E, o["counts"], o["offsets"], o["perm"], o["inv_perm"],
                   o["packed_tok"], o["packed_w"], o["x_packed"], ws, o["status"])
    torch.cuda.synchronize()
    return {key: v.cpu() for key, v in o.items()}


def _same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def _check(cfg, seed, G=1, Mg=1, bias=True):
    p = make_layer(cfg, seed=seed)
    x, W = dev(p["x"]), dev(p["W_gate"])
    b = dev(p["bias"]) if bias else None
    g = _fused(x, W, b, cfg.k, cfg.renormalize, G, Mg)
    s = _separate(x, W, b, cfg.k, cfg.renormalize, G, Mg)
    assert int(g["status"][0]) == 0 and int(s["status"][0]) == 0
    for key in KEYS:
        assert _same_bits(g[key], s[key]), f"{key} differs from the two-call chain"
    _against_oracle(g, p, cfg, G, Mg, bias)
    return g


def _against_oracle(g, p, cfg, G=1, Mg=1, bias=True):
    # routing from the GPU's logits, then the oracle's counting sort
    assert rel(g["logits"], O.router_logits(p["x"], p["W_gate"], p["bias"] if bias else None)) \
        <= 1e-5
    ids_o, w_o = O.route_from_logits(g["logits"], cfg.k, cfg.renormalize, G, Mg)
    np.testing.assert_array_equal(g["ids"].numpy(), ids_o)
    np.testing.assert_allclose(g["w"].numpy(), w_o, rtol=1e-5, atol=0)
    o = O.dispatch(g["ids"].numpy(), g["w"].numpy().astype(np.float64), cfg.E)
    for key in ("counts", "offsets", "perm", "inv_perm", "packed_tok"):
        np.testing.assert_array_equal(g[key].numpy(), o[key], err_msg=key)
    np.testing.assert_array_equal(g["packed_w"].numpy(), g["w"].numpy().reshape(-1)[o["perm"]])
    assert _same_bits(g["x_packed"], p["x"][torch.as_tensor(o["packed_tok"])])


@pytest.mark.parametrize("T,H,E,k", [(1, 4096, 8, 2), (8, 4096, 8, 2), (3, 96, 1, 1),
                                     (5, 72, 3, 2), (17, 2048, 60, 4), (64, 2048, 60, 4),
                                     (64, 128, 64, 8), (33, 256, 16, 8), (64, 4096, 8, 2)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_route_dispatch_matches_two_calls(T, H, E, k, dtype):
    # (64, 4096, 8, 2) in bf16 gathers 1 MiB: the rows go to the multi-CTA
    # gather kernel after the fused launch; the other shapes gather in-kernel
    cfg = LayerConfig("rd", T=T, H=H, E=E, k=k, I=8, dtype=dtype, renormalize=(E % 2 == 0))
    _check(cfg, seed=T * 7 + E)


@pytest.mark.parametrize("E,k,G,Mg", [(8, 2, 4, 2), (64, 6, 8, 3), (60, 4, 6, 2), (32, 4, 32, 4)])
def test_route_dispatch_grouped(E, k, G, Mg):
    cfg = LayerConfig("rdg", T=40, H=256, E=E, k=k, I=8, dtype="bf16", renormalize=True)
    g = _check(cfg, seed=E + G, G=G, Mg=Mg, bias=False)
    assert max(len(set((r // (E // G)).tolist())) for r in g["ids"].numpy()) <= Mg


def test_route_dispatch_back_to_back_on_one_counter():
    # five calls on one stream share the ticket word; each must see it at zero
    cfg = LayerConfig("rdb", T=24, H=512, E=16, k=4, I=8, dtype="bf16", renormalize=True)
    counter = torch.zeros(1, dtype=torch.int32, device=DEV)
    for seed in range(5):
        p = make_layer(cfg, seed=100 + seed)
        x, W = dev(p["x"]), dev(p["W_gate"])
        g = _fused(x, W, dev(p["bias"]), cfg.k, True, counter=counter)
        s = _separate(x, W, dev(p["bias"]), cfg.k, True)
        for key in KEYS:
            assert _same_bits(g[key], s[key]), f"call {seed}: {key} differs"


def test_route_dispatch_rejects_large_shapes():
    x = torch.zeros(65, 64, dtype=torch.bfloat16, device=DEV)
    W = torch.zeros(8, 64, dtype=torch.bfloat16, device=DEV)
    o = _bufs(65, 64, 8, 2, torch.bfloat16)
    counter = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(M.MoEError, match="T must be in"):
        M.moe_route_dispatch(x, W, None, 2, True, o["logits"], o["ids"], o["w"], o["counts"],
                             o["offsets"], o["perm"], o["inv_perm"], o["packed_tok"],
                             o["packed_w"], o["x_packed"], counter)


@pytest.mark.parametrize("T,H,E,k,dtype", [(32, 2048, 60, 4, "bf16"), (1, 4096, 8, 2, "bf16"),
                                           (5, 72, 3, 2, "f32"), (64, 256, 63, 8, "bf16"),
                                           (17, 512, 15, 4, "f32")])
def test_route_dispatch_with_the_shared_gate(T, H, E, k, dtype):
    # the shared expert's gate row rides along as row E: the routed outputs
    # match the oracle as without it (and are bit-identical to the launch
    # without it when E + 1 rows keep the same power-of-two row block, so
    # that every dot product is split into the same slices), and the gate
    # logit is x . w_sg
    cfg = LayerConfig("rdsg", T=T, H=H, E=E, k=k, I=8, dtype=dtype, renormalize=(E % 2 == 0))
    p = make_layer(cfg, seed=T + E)
    x, W, b = dev(p["x"]), dev(p["W_gate"]), dev(p["bias"])
    g = torch.Generator().manual_seed(E)
    w_sg = (torch.randn(H, generator=g) / H ** 0.5).to(p["x"].dtype)
    plain = _fused(x, W, b, k, cfg.renormalize)
    o = _bufs(T, H, E, k, x.dtype)
    sg = torch.full((T,), -7.0, device=DEV)
    counter = torch.zeros(1, dtype=torch.int32, device=DEV)
    M.moe_route_dispatch(x, W, b, k, cfg.renormalize, o["logits"], o["ids"], o["w"], o["counts"],
                         o["offsets"], o["perm"], o["inv_perm"], o["packed_tok"], o["packed_w"],
                         o["x_packed"], counter, status=o["status"], w_gate_shared=dev(w_sg),
                         shared_gate_logit=sg)
    torch.cuda.synchronize()
    assert int(counter[0]) == 0 and int(o["status"][0]) == 0
    gated = {key: v.cpu() for key, v in o.items()}
    _against_oracle(gated, p, cfg)
    pow2 = lambda n: 1 << max(0, (n - 1).bit_length())
    if pow2(E + 1) == pow2(E):
        for key in KEYS:
            assert _same_bits(gated[key], plain[key]), f"{key} changed with the gate row"
    ref = p["x"].double() @ w_sg.double()
    assert rel(sg.cpu(), ref) <= 1e-5


def test_route_dispatch_gate_needs_a_free_row():
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    W = torch.zeros(64, 64, dtype=torch.bfloat16, device=DEV)
    o = _bufs(4, 64, 64, 2, torch.bfloat16)
    counter = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(M.MoEError, match="E must be"):
        M.moe_route_dispatch(x, W, None, 2, True, o["logits"], o["ids"], o["w"], o["counts"],
                             o["offsets"], o["perm"], o["inv_perm"], o["packed_tok"],
                             o["packed_w"], o["x_packed"], counter,
                             w_gate_shared=torch.zeros(64, dtype=torch.bfloat16, device=DEV),
                             shared_gate_logit=torch.zeros(4, device=DEV))
