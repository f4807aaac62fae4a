"""Router parity: GPU moe_route against the fp64 oracle.

Logits (fp32) within 1e-5 of the oracle's fp64 logits (relative to their
RMS).  Given the GPU's own logits, the oracle's top-k ids must match bit for
bit and its weights within 1e-5 relative, element by element.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_44_b200 as M
import oracle.moe_oracle as O
from moe_inputs import CONFIGS, LayerConfig, make_layer
from tests.gpu_util import DEV, dev, rel

pytestmark = pytest.mark.gpu


def _run(x, W, b, k, renorm):
    T, E = x.shape[0], W.shape[0]
    logits = torch.empty(T, E, device=DEV)
    ids = torch.empty(T, max(k, 1), dtype=torch.int32, device=DEV)
    w = torch.empty(T, max(k, 1), device=DEV)
    M.moe_route(dev(x), dev(W), dev(b), k, renorm, logits, ids if k else None, w if k else None)
    torch.cuda.synchronize()
    return logits.cpu(), ids.cpu()[:, :k], w.cpu()[:, :k]


def _check(x, W, b, k, renorm, logit_tol=1e-5):
    logits, ids, w = _run(x, W, b, k, renorm)
    l64 = O.router_logits(x, W, b)
    assert rel(logits, l64) <= logit_tol
    if k == 0:
        return
    ids_o, w_o = O.route_from_logits(logits, k, renorm)
    np.testing.assert_array_equal(ids.numpy(), ids_o)
    np.testing.assert_allclose(w.numpy(), w_o, rtol=1e-5, atol=0)


@pytest.mark.parametrize("name", ["tiny_f32", "builder_bf16", "qwen15_t32", "qwen3_t16384",
                                  "decode_t1", "decode_t64"])
def test_route_configs(name):
    cfg = CONFIGS[name]
    # Router-only draw: the expert weights are not needed here, so draw a
    # narrow layer with the same T, H, E, k and bias recipe.
    small = LayerConfig("r", T=cfg.T, H=cfg.H, E=cfg.E, k=cfg.k, I=8, dtype=cfg.dtype,
                        renormalize=cfg.renormalize, zipf_s=cfg.zipf_s, empty_tail=cfg.empty_tail)
    p = make_layer(small, seed=0)
    _check(p["x"], p["W_gate"], p["bias"], cfg.k, cfg.renormalize)


@pytest.mark.parametrize("E,k", [(1, 1), (3, 2), (8, 8), (60, 4), (64, 2), (65, 3), (128, 8),
                                 (200, 5), (256, 8)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("H", [72, 96])
@pytest.mark.parametrize("T", [7, 131])       # one-CTA-per-token path / cluster path
def test_route_shapes(E, k, dtype, H, T):
    cfg = LayerConfig("r", T=T, H=H, E=E, k=k, I=8, dtype=dtype, renormalize=(E % 2 == 0))
    p = make_layer(cfg, seed=E + k)
    _check(p["x"], p["W_gate"], None, k, cfg.renormalize)


def test_route_with_bias_and_no_renorm():
    rng = np.random.default_rng(5)
    x = torch.randn(77, 256, generator=torch.Generator().manual_seed(1))
    W = torch.randn(40, 256, generator=torch.Generator().manual_seed(2)) / 16
    b = torch.tensor(rng.standard_normal(40), dtype=torch.float32)
    _check(x, W, b, 6, False)


def test_route_ties_go_to_lower_expert_id():
    # Duplicate W_gate rows give bit-identical logits: the lower id must win.
    g = torch.Generator().manual_seed(3)
    x = torch.randn(50, 64, generator=g)
    W = torch.randn(16, 64, generator=g)
    W[9] = W[2]
    W[12] = W[2]
    W[5] = W[14]
    logits, ids, _ = _run(x, W, None, 4, True)
    assert torch.equal(logits[:, 9], logits[:, 2]) and torch.equal(logits[:, 12], logits[:, 2])
    ids_o, _ = O.route_from_logits(logits, 4, True)
    np.testing.assert_array_equal(ids.numpy(), ids_o)
    for t in range(50):
        row = ids[t].tolist()
        if 9 in row or 12 in row:
            assert 2 in row and row.index(2) < row.index(9 if 9 in row else 12)
    # All-equal logits: ids are 0..k-1 in order, weights uniform.
    logits, ids, w = _run(torch.zeros(3, 64), torch.randn(10, 64, generator=g), None, 3, True)
    assert ids.tolist() == [[0, 1, 2]] * 3
    np.testing.assert_allclose(w.numpy(), 1 / 3, rtol=1e-6)


def test_route_logits_only_for_a_shared_gate():
    g = torch.Generator().manual_seed(4)
    x = torch.randn(33, 128, generator=g).to(torch.bfloat16)
    wsg = (torch.randn(1, 128, generator=g) / 11).to(torch.bfloat16)
    _check(x, wsg, None, 0, False)


def test_route_k_equals_E_is_the_full_softmax():
    g = torch.Generator().manual_seed(6)
    x = torch.randn(20, 64, generator=g)
    W = torch.randn(8, 64, generator=g) / 8
    logits, ids, w = _run(x, W, None, 8, False)
    full = torch.zeros(20, 8)
    full.scatter_(1, ids.long(), w)
    np.testing.assert_allclose(full.numpy(), O.softmax_rows(O.to_f64(logits)), rtol=1e-5)


@pytest.mark.parametrize("T,H,E,k", [
    (4096, 4096, 64, 2),     # 32 token tiles x clusters of 4 H-slices
    (1024, 4096, 64, 2),     # 8 tiles x clusters of 8
    (300, 256, 128, 8),      # ragged last tile, 4 H-blocks of 64, two accumulator chains
    (129, 2048, 256, 8),     # 256 experts: one accumulator chain, 2 tiles
    (65, 64, 1, 1),          # a single H-block and a single expert
    (200, 8, 33, 3),         # H shorter than one 64-column block
    (8192, 2048, 60, 4),     # Qwen1.5-MoE-A2.7B prefill routing
])
def test_route_tensor_core_shapes(T, H, E, k):
    # bf16 batches above 64 tokens take the tensor-core router
    cfg = LayerConfig("r", T=T, H=H, E=E, k=k, I=8, dtype="bf16", renormalize=True)
    p = make_layer(cfg, seed=T + E)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    logits = torch.empty(T, E, device=DEV)
    ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, device=DEV)
    M.moe_route(dev(p["x"]), dev(p["W_gate"]), None, k, True, logits, ids, w, status=status)
    logits2 = torch.empty_like(logits)
    M.moe_route(dev(p["x"]), dev(p["W_gate"]), None, k, True, logits2, ids, w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(logits, logits2)              # deterministic
    l64 = O.router_logits(p["x"], p["W_gate"], None)
    assert rel(logits.cpu(), l64) <= 1e-5
    ids_o, w_o = O.route_from_logits(logits.cpu(), k, True)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_o)
    np.testing.assert_allclose(w.cpu().numpy(), w_o, rtol=1e-5, atol=0)


def test_route_ties_on_the_tensor_core_path():
    g = torch.Generator().manual_seed(8)
    x = torch.randn(200, 256, generator=g).to(torch.bfloat16)
    W = (torch.randn(100, 256, generator=g) / 16).to(torch.bfloat16)
    W[70] = W[3]
    W[99] = W[3]
    logits, ids, _ = _run(x, W, None, 5, True)
    assert torch.equal(logits[:, 70], logits[:, 3]) and torch.equal(logits[:, 99], logits[:, 3])
    ids_o, _ = O.route_from_logits(logits, 5, True)
    np.testing.assert_array_equal(ids.numpy(), ids_o)
    logits, ids, w = _run(torch.zeros(130, 64, dtype=torch.bfloat16),
                          torch.randn(80, 64, generator=g).to(torch.bfloat16), None, 4, True)
    assert ids.tolist() == [[0, 1, 2, 3]] * 130
    np.testing.assert_allclose(w.numpy(), 0.25, rtol=1e-6)


# ------------------------------------------------ group-limited router ---

def _run_grouped(x, W, b, k, renorm, G, M):
    T, E = x.shape[0], W.shape[0]
    logits = torch.empty(T, E, device=DEV)
    ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, device=DEV)
    M_ = M
    import mixture_experts_layer_44_b200 as MM
    MM.moe_route_grouped(dev(x), dev(W), dev(b), k, renorm, G, M_, logits, ids, w)
    torch.cuda.synchronize()
    return logits.cpu(), ids.cpu(), w.cpu()


@pytest.mark.parametrize("E,k,G,Mg", [(8, 2, 4, 2), (64, 6, 8, 3), (60, 4, 6, 2), (128, 8, 8, 4),
                                      (256, 8, 8, 4), (32, 4, 32, 4), (64, 2, 2, 1)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [7, 131])       # one-CTA-per-token path / cluster or tensor-core path
def test_route_grouped_shapes(E, k, G, Mg, dtype, T):
    cfg = LayerConfig("g", T=T, H=96, E=E, k=k, I=8, dtype=dtype, renormalize=(E % 3 != 0))
    p = make_layer(cfg, seed=E + G)
    logits, ids, w = _run_grouped(p["x"], p["W_gate"], None, k, cfg.renormalize, G, Mg)
    l64 = O.router_logits(p["x"], p["W_gate"], None)
    assert rel(logits, l64) <= 1e-5
    ids_o, w_o = O.route_from_logits(logits, k, cfg.renormalize, G, Mg)
    np.testing.assert_array_equal(ids.numpy(), ids_o)
    np.testing.assert_allclose(w.numpy(), w_o, rtol=1e-5, atol=0)
    assert max(len(set((r // (E // G)).tolist())) for r in ids.numpy()) <= Mg


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [64, 200])      # small-batch path / cluster or tensor-core path
def test_route_grouped_ties_between_groups(dtype, T):
    # groups of 4 over 16 experts; experts 1, 6 and 13 share one W_gate row, so
    # groups 0, 1 and 3 tie whenever that row wins its group
    cfg = LayerConfig("gt", T=T, H=64, E=16, k=3, I=8, dtype=dtype, renormalize=True)
    p = make_layer(cfg, seed=99)
    W = p["W_gate"].clone()
    W[1] *= 4                   # the shared row wins for every token with a positive score
    W[6] = W[1]
    W[13] = W[1]
    logits, ids, w = _run_grouped(p["x"], W, None, 3, True, 4, 2)
    ids_o, w_o = O.route_from_logits(logits, 3, True, 4, 2)
    np.testing.assert_array_equal(ids.numpy(), ids_o)
    np.testing.assert_allclose(w.numpy(), w_o, rtol=1e-5, atol=0)
    # the tie really happens and goes to the lower groups
    l = logits.numpy()
    tied = (l[:, 1] == l[:, 6]) & (l[:, 1] == l[:, 13]) & (l[:, 1] == l.max(axis=1))
    assert tied.sum() > 0
    assert all(set(r.tolist()) >= {1, 6} for r in ids.numpy()[tied])


def test_grouped_routing_through_the_whole_layer():
    cfg = LayerConfig("g_layer", T=300, H=512, E=64, k=6, I=256, dtype="bf16", renormalize=True)
    p = make_layer(cfg, seed=5)
    dp = {k_: (dev(v) if v is not None else None) for k_, v in p.items()}
    import mixture_experts_layer_44_b200 as MM
    buf = MM.MoELayerBuffers(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, torch.bfloat16)
    out = MM.moe_layer_forward(dp["x"], dp, cfg.k, True, buf, n_groups=8, topk_groups=3)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    ids = buf.ids.cpu().numpy()
    ids_o, _ = O.route_from_logits(buf.logits.cpu(), cfg.k, True, 8, 3)
    np.testing.assert_array_equal(ids, ids_o)
    l64 = O.router_logits(p["x"], p["W_gate"], None)
    w64 = O.routing_weights(l64, ids, True)
    want = O.moe_forward_tokens(p, np.arange(cfg.T), ids, w64)
    from tests.gpu_util import err_bf16_out
    assert err_bf16_out(out.cpu(), want) <= 2e-2


# moe_route_gated: the shared expert's gate logit x . w_sg in the router's own
# launch (row E of the small router; the idle warps of the tensor-core router,
# from the staged x tiles), or a second launch (fp32 above 64 tokens).  The
# routed outputs meet the oracle as moe_route's do (and are bit-identical to
# moe_route's where the gate leaves the router's row block unchanged); the
# gate logit is within 1e-5 of x . w_sg in fp64.
def _pow2(n):
    return 1 << max(0, (n - 1).bit_length())


@pytest.mark.parametrize("T,H,E,k,dtype", [
    (32, 2048, 60, 4, "bf16"),      # small router, row block 64 either way
    (8192, 2048, 60, 4, "bf16"),    # Qwen1.5 prefill: tensor-core router, column E of 64
    (300, 200, 64, 2, "bf16"),      # E + 1 = 65: a wider block; H ends in a partial k-block
    (131, 96, 8, 2, "bf16"),        # E = 8: 32 columns either way
    (257, 4096, 255, 8, "bf16"),    # the last padding column of the 256-column block
    (200, 96, 60, 4, "f32"),        # fp32 above 64 tokens: a second launch
    (7, 72, 3, 2, "f32"),
])
def test_route_gated(T, H, E, k, dtype):
    cfg = LayerConfig("rg", T=T, H=H, E=E, k=k, I=8, dtype=dtype, renormalize=(E % 2 == 0))
    p = make_layer(cfg, seed=T + E)
    g = torch.Generator().manual_seed(H)
    w_sg = (torch.randn(H, generator=g) / H ** 0.5).to(p["x"].dtype)
    logits = torch.empty(T, E, device=DEV)
    ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, device=DEV)
    sg = torch.full((T,), -7.0, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    M.moe_route_gated(dev(p["x"]), dev(p["W_gate"]), None, dev(w_sg), k, cfg.renormalize, logits,
                      ids, w, sg, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    logits, ids, w, sg = logits.cpu(), ids.cpu(), w.cpu(), sg.cpu()
    assert rel(logits, O.router_logits(p["x"], p["W_gate"], None)) <= 1e-5
    ids_o, w_o = O.route_from_logits(logits, k, cfg.renormalize)
    np.testing.assert_array_equal(ids.numpy(), ids_o)
    np.testing.assert_allclose(w.numpy(), w_o, rtol=1e-5, atol=0)
    assert rel(sg, p["x"].double() @ w_sg.double()) <= 1e-5
    same_block = (_pow2(E + 1) == _pow2(E)) if T <= 64 else \
        (max(32, _pow2(E + 1)) == max(32, _pow2(E)))
    if same_block and not (dtype == "f32" and T > 64):
        l2, i2, w2 = _run(p["x"], p["W_gate"], None, k, cfg.renormalize)
        assert torch.equal(logits, l2) and torch.equal(ids, i2) and torch.equal(w, w2)


def test_route_gated_random_shapes():
    # seeded random shapes over both launches the gate rides in (T <= 64 small
    # router, tensor-core router above), H tails included
    rng = np.random.default_rng(11)
    for _ in range(24):
        T = int(rng.choice([1, 5, 33, 64, 65, 129, 257, 1000]))
        E = int(rng.integers(1, 256))
        k = int(rng.integers(1, min(E, 8) + 1))
        H = 8 * int(rng.integers(1, 257))
        cfg = LayerConfig("rgr", T=T, H=H, E=E, k=k, I=8, dtype="bf16", renormalize=True)
        p = make_layer(cfg, seed=T * 1000 + E)
        w_sg = (torch.randn(H, generator=torch.Generator().manual_seed(H)) / H ** 0.5).to(
            torch.bfloat16)
        logits = torch.empty(T, E, device=DEV)
        ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
        w = torch.empty(T, k, device=DEV)
        sg = torch.full((T,), -7.0, device=DEV)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        M.moe_route_gated(dev(p["x"]), dev(p["W_gate"]), None, dev(w_sg), k, True, logits, ids,
                          w, sg, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, (T, E, k, H)
        assert rel(logits.cpu(), O.router_logits(p["x"], p["W_gate"], None)) <= 1e-5, (T, E, H)
        ids_o, _ = O.route_from_logits(logits.cpu(), k, True)
        np.testing.assert_array_equal(ids.cpu().numpy(), ids_o)
        assert rel(sg.cpu(), p["x"].double() @ w_sg.double()) <= 1e-5, (T, E, k, H)
