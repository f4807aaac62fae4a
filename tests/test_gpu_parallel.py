"""Parity of the expert-parallel, tensor-parallel and all-to-all pieces on one GPU.

* moe_ep_partition (metrale's build_ep_routing_table on the device): every
  worked example of the page's tests module, and large random tables, bit
  for bit against the oracle's ep_partition;
* moe_ep_owner / moe_ep_pack_ids: bit for bit against the oracle's expert
  ownership;
* moe_gather over an expert range, moe_combine_range, moe_finalize: against
  their definitions;
* whole layers split over R ranks, the ranks run one after the other on the
  one GPU (each rank's kernels are independent of the others'; the
  collective between them is emulated by adding the fp32 partials, or by
  moving the exchanged rows, in the test): the result against the oracle's
  unsharded layer, every token, and each rank's partial against the
  oracle's partial of that rank on a sample of tokens.
"""
import json
import os

import numpy as np
import pytest
import torch

import mixture_experts_layer_44_b200 as M
import mixture_experts_layer_44_b200.sharded as S
import oracle.moe_oracle as O
from moe_inputs import CONFIGS, LayerConfig, make_layer, make_tokens
from tests.gpu_util import DEV, TOL, dev, err_bf16_out, params_to, rand_ids, rel

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
KEYS = ("local_token_indices", "local_expert_ids", "local_weights", "remote_token_indices",
        "remote_expert_ids", "remote_weights")


def _partition(indices, weights, T, k, lo, hi):
    n = T * k
    ids = torch.tensor(np.asarray(indices, dtype=np.int64).astype(np.int32), device=DEV)
    w = torch.tensor(np.asarray(weights, dtype=np.float32), device=DEV)
    out = {key: torch.full((max(n, 1),), -9, dtype=torch.float32 if "weights" in key
                           else torch.int32, device=DEV) for key in KEYS}
    counts = torch.full((2,), -9, dtype=torch.int32, device=DEV)
    ws = torch.empty(max(16, M.moe_ep_partition_workspace_bytes(T, k)), dtype=torch.uint8,
                     device=DEV)
    M.moe_ep_partition(ids, w, T, k, lo, hi, *(out[key] for key in KEYS), counts, ws)
    torch.cuda.synchronize()
    c = counts.cpu().tolist()
    res = {"local_count": c[0], "remote_count": c[1]}
    for key in KEYS:
        m = c[0] if key.startswith("local") else c[1]
        res[key] = out[key][:m].cpu()
    return res


def test_ep_partition_reproduces_the_pages_worked_examples():
    g = json.load(open(os.path.join(GOLDEN, "ep_dispatch_buckets.json")))
    for case in g["cases"]:
        got = _partition(case["indices"], case["weights"], case["num_tokens"], case["top_k"],
                         case["local_start"], case["local_end"])
        want = O.ep_partition(case["indices"], np.float32(case["weights"]), case["num_tokens"],
                              case["top_k"], case["local_start"], case["local_end"])
        ex = case["expect"]
        for side in ("local", "remote"):
            assert got[f"{side}_count"] == len(want[f"{side}_token_indices"]), case["name"]
            if f"{side}_count" in ex:
                assert got[f"{side}_count"] == ex[f"{side}_count"], case["name"]
        for key in KEYS:
            if "weights" in key:
                np.testing.assert_array_equal(got[key].numpy(),
                                              np.asarray(want[key], dtype=np.float32))
            else:
                assert got[key].tolist() == [int(v) for v in want[key]], (case["name"], key)
            if key in ex:
                if "weights" in key:
                    np.testing.assert_array_equal(got[key].numpy(),
                                                  np.asarray(ex[key], dtype=np.float32))
                else:
                    assert got[key].tolist() == ex[key], (case["name"], key)


@pytest.mark.parametrize("T,k,lo,hi", [(1, 1, 0, 1), (7, 3, 2, 5), (1024, 2, 0, 32),
                                       (4096, 8, 96, 128), (16384, 8, 17, 91),
                                       (3000, 5, 0, 0), (2049, 1, 0, 512)])
def test_ep_partition_random_tables(T, k, lo, hi):
    rng = np.random.default_rng(T + k + lo)
    ids = rng.integers(0, 128, size=(T, k))
    ids[rng.random((T, k)) < 0.01] = 1000                # ids beyond every range: remote
    w = rng.random((T, k)).astype(np.float32)
    got = _partition(ids.reshape(-1), w.reshape(-1), T, k, lo, hi)
    want = O.ep_partition(ids.reshape(-1).tolist(), w.reshape(-1), T, k, lo, hi)
    assert got["local_count"] + got["remote_count"] == T * k
    for key in KEYS:
        if "weights" in key:
            np.testing.assert_array_equal(got[key].numpy(), np.asarray(want[key], np.float32))
        else:
            np.testing.assert_array_equal(got[key].numpy(), np.asarray(want[key]))


def test_ep_owner_and_local_ids_are_exact():
    rng = np.random.default_rng(5)
    for E, world, T, k in [(8, 2, 33, 2), (60, 4, 500, 4), (128, 7, 3000, 8), (5, 5, 9, 5)]:
        ids = rand_ids(rng, T, k, E)
        owner = torch.empty(T, k, dtype=torch.int32, device=DEV)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        M.moe_ep_owner(dev(ids), E, world, owner, status=st)
        want = O.expert_owner(ids.numpy(), E, world)
        np.testing.assert_array_equal(owner.cpu().numpy(), want)
        # dispatch by owner, then each send row's expert id local to its owner
        buf = M.MoELayerBuffers(T, 64, world, k, 8, torch.bfloat16)
        x = torch.randn(T, 64, device=DEV).to(torch.bfloat16)
        w = torch.rand(T, k, device=DEV)
        M.moe_dispatch(owner, w, x, world, buf.counts, buf.offsets, buf.perm, buf.inv_perm,
                       buf.packed_tok, buf.packed_w, buf.x_packed, buf.ws, st)
        local = torch.full((T * k,), -5, dtype=torch.int32, device=DEV)
        M.moe_ep_pack_ids(dev(ids), buf.perm, buf.offsets, E, world, local)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        d = O.dispatch(want, w.cpu().numpy().astype(np.float64), world)
        np.testing.assert_array_equal(buf.perm.cpu().numpy(), d["perm"])
        flat = ids.numpy().reshape(-1)[d["perm"]]
        starts = np.array([a for a, _ in O.expert_ranges(E, world)])
        np.testing.assert_array_equal(local.cpu().numpy(), flat - starts[want.reshape(-1)[d["perm"]]])


def test_gather_range_combine_range_and_finalize():
    rng = np.random.default_rng(9)
    T, k, E, H = 700, 4, 16, 256
    ids = rand_ids(rng, T, k, E)
    w = torch.tensor(rng.random((T, k)), dtype=torch.float32)
    x = torch.randn(T, H).to(torch.bfloat16)
    buf = M.MoELayerBuffers(T, H, E, k, 64, torch.bfloat16)
    M.moe_dispatch(dev(ids), dev(w), None, E, buf.counts, buf.offsets, buf.perm, buf.inv_perm,
                   buf.packed_tok, buf.packed_w, buf.x_packed, buf.ws, buf.status)
    buf.x_packed.fill_(3.0)
    lo, hi = 5, 11
    M.moe_gather(dev(x), buf.packed_tok, buf.offsets, lo, hi, buf.x_packed, status=buf.status)
    y = torch.randn(T * k, H, device=DEV)
    part = torch.empty(T, H, device=DEV)
    M.moe_combine_range(y, buf.inv_perm, buf.offsets, lo, hi, T, k, part, status=buf.status)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    M.moe_finalize(part, out)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    offs = buf.offsets.cpu().numpy()
    a, b = offs[lo], offs[hi]
    tok = buf.packed_tok.cpu().long()
    xp = buf.x_packed.cpu()
    assert torch.equal(xp[a:b].view(torch.int16), x[tok[a:b]].view(torch.int16))
    assert (xp[:a].float() == 3.0).all() and (xp[b:].float() == 3.0).all()
    # masked merge: assignments whose expert is in [lo, hi), in j order
    ip = buf.inv_perm.cpu().numpy().reshape(T, k)
    yc = O.to_f64(y)
    want = np.zeros((T, H))
    idn = ids.numpy()
    for j in range(k):
        m = (idn[:, j] >= lo) & (idn[:, j] < hi)
        want[m] += yc[ip[m, j]]
    assert rel(part, want) <= TOL["f32"]
    # one rounding: exactly torch's round-to-nearest-even conversion of the fp32 sum
    assert torch.equal(out.cpu().view(torch.int16), part.cpu().to(torch.bfloat16).view(torch.int16))


# ------------------------------------------------------------ layers ---

SMALL = {
    "ep_small": LayerConfig("ep_small", T=384, H=512, E=16, k=4, I=256, dtype="bf16",
                            renormalize=True, zipf_s=1.0),
    "ep_small_shared": LayerConfig("ep_small_shared", T=96, H=512, E=12, k=4, I=192,
                                   dtype="bf16", renormalize=False, shared_I=384),
}


def _oracle_full(cfg, p, ids):
    l64 = O.router_logits(p["x"], p["W_gate"], p["bias"])
    w64 = O.routing_weights(l64, ids, cfg.renormalize)
    return O.moe_forward_tokens(p, np.arange(cfg.T), ids, w64), w64


@pytest.mark.parametrize("name,world", [("ep_small", 1), ("ep_small", 3), ("ep_small_shared", 4),
                                        ("decode_t8", 2), ("qwen3_t16384", 8),
                                        ("builder_bf16", 4)])
def test_expert_parallel_layer(name, world):
    cfg = SMALL.get(name) or CONFIGS[name]
    p = make_layer(cfg, seed=0)
    dp = params_to(p)
    parts, ids_seen = [], None
    for r in range(world):
        lo, hi = S.expert_range(cfg.E, world, r)
        local = S.ep_local_params(dp, lo, hi, run_shared=(r == 0))
        buf = S.ShardedBuffers(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.torch_dtype,
                               shared_I=cfg.shared_I if r == 0 else None)
        S.moe_layer_partial_ep(dp["x"], local, lo, hi, cfg.k, cfg.renormalize, buf)
        torch.cuda.synchronize()
        assert int(buf.status.item()) == 0
        ids = buf.ids.cpu().numpy()
        if ids_seen is None:
            ids_seen = ids
        np.testing.assert_array_equal(ids, ids_seen)       # every rank routes alike
        parts.append((lo, hi, buf.partial.clone()))
        del buf, local
    acc = torch.zeros(cfg.T, cfg.H, device=DEV)
    for _, _, part in parts:                                # the all-reduce, in rank order
        acc += part
    out = torch.empty(cfg.T, cfg.H, dtype=cfg.torch_dtype, device=DEV)
    M.moe_finalize(acc, out)
    torch.cuda.synchronize()
    l64 = O.router_logits(p["x"], p["W_gate"], p["bias"])
    rng = np.random.default_rng(world)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], rng.choice(cfg.T, min(cfg.T, 16), False)]))
    w64 = O.routing_weights(l64[toks], ids_seen[toks], cfg.renormalize)
    want = O.moe_forward_tokens(p, toks, ids_seen[toks], w64)
    sel = torch.as_tensor(toks)
    assert rel(acc.cpu()[sel], want) <= TOL["bf16"]
    assert err_bf16_out(out.cpu()[sel], want) <= TOL["bf16"]
    for r, (lo, hi, part) in enumerate(parts):
        want_r = O.moe_forward_tokens_ep(p, toks, ids_seen[toks], w64, lo, hi, with_shared=(r == 0))
        scale = float(np.sqrt(np.mean(want ** 2)))
        assert float(np.abs(O.to_f64(part.cpu()[sel]) - want_r).max()) / scale <= TOL["bf16"]
    # every token against the single-GPU layer (both bf16: beyond one rounding)
    buf1 = M.MoELayerBuffers(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.torch_dtype,
                             shared_I=cfg.shared_I)
    one = M.moe_layer_forward(dp["x"], dp, cfg.k, cfg.renormalize, buf1)
    torch.cuda.synchronize()
    assert err_bf16_out(out.cpu(), O.to_f64(one.cpu())) <= TOL["bf16"]


TP_CASES = [("ep_small", 2), ("ep_small_shared", 3), ("decode_t64", 4), ("qwen3_t16384", 2),
            ("qwen15_t32", 2), ("builder_bf16", 2)]


@pytest.mark.parametrize("name,tp", TP_CASES)
def test_tensor_parallel_layer(name, tp):
    cfg = SMALL.get(name) or CONFIGS[name]
    p = make_layer(cfg, seed=0)
    dp = params_to(p)
    acc = torch.zeros(cfg.T, cfg.H, device=DEV)
    parts, ids_seen = [], None
    for r in range(tp):
        sh = S.tp_shard_params(dp, r, tp)
        buf = S.ShardedBuffers(cfg.T, cfg.H, cfg.E, cfg.k, cfg.I // tp, cfg.torch_dtype,
                               shared_I=cfg.shared_I // tp if cfg.shared_I else None)
        S.moe_layer_partial_tp(dp["x"], sh, cfg.k, cfg.renormalize, buf)
        torch.cuda.synchronize()
        assert int(buf.status.item()) == 0
        ids = buf.ids.cpu().numpy()
        if ids_seen is None:
            ids_seen = ids
        np.testing.assert_array_equal(ids, ids_seen)
        acc += buf.partial
        parts.append(buf.partial.clone())
        del buf, sh
    out = torch.empty(cfg.T, cfg.H, dtype=cfg.torch_dtype, device=DEV)
    M.moe_finalize(acc, out)
    torch.cuda.synchronize()
    l64 = O.router_logits(p["x"], p["W_gate"], p["bias"])
    rng = np.random.default_rng(tp)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], rng.choice(cfg.T, min(cfg.T, 16), False)]))
    w64 = O.routing_weights(l64[toks], ids_seen[toks], cfg.renormalize)
    want = O.moe_forward_tokens(p, toks, ids_seen[toks], w64)
    sel = torch.as_tensor(toks)
    assert rel(acc.cpu()[sel], want) <= TOL["bf16"]
    assert err_bf16_out(out.cpu()[sel], want) <= TOL["bf16"]
    scale = float(np.sqrt(np.mean(want ** 2)))
    for r, part in enumerate(parts):
        want_r = O.moe_forward_tokens_tp(p, toks, ids_seen[toks], w64, r, tp)
        assert float(np.abs(O.to_f64(part.cpu()[sel]) - want_r).max()) / scale <= TOL["bf16"]


@pytest.mark.parametrize("name,world", [("ep_small", 2), ("ep_small_shared", 3),
                                        ("qwen3_t16384", 4)])
def test_all_to_all_layer(name, world):
    base = SMALL.get(name) or CONFIGS[name]
    # each rank has its own tokens: the workload's batch split in world parts
    T_r = base.T // world
    cfg = LayerConfig(base.name, T=T_r * world, H=base.H, E=base.E, k=base.k, I=base.I,
                      dtype=base.dtype, renormalize=base.renormalize, zipf_s=base.zipf_s,
                      empty_tail=base.empty_tail, shared_I=base.shared_I)
    p = make_layer(cfg, seed=0)
    dp = params_to(p)
    xs = [dp["x"][r * T_r:(r + 1) * T_r].contiguous() for r in range(world)]
    locs, bufs, sends = [], [], []
    for r in range(world):
        lo, hi = S.expert_range(cfg.E, world, r)
        locs.append(dict(S.ep_local_params(dp, lo, hi, run_shared=False),
                         **({"w13s": dp["w13s"], "w2s": dp["w2s"], "w_sg": dp["w_sg"]}
                            if cfg.shared_I else {})))
        bufs.append(S.A2ABuffers(T_r, cfg.H, cfg.E, cfg.k, world, cfg.torch_dtype,
                                 shared_I=cfg.shared_I))
        counts, xs_, eid, w = S.a2a_send(xs[r], locs[r], cfg.k, cfg.renormalize, bufs[r])
        torch.cuda.synchronize()
        c = counts.cpu().tolist()
        offs = np.concatenate([[0], np.cumsum(c)])
        sends.append((c, offs, xs_, eid, w))
    # the exchange: rank q receives, in source-rank order, what each rank sent it
    ys = []
    for q in range(world):
        parts = [(s[2][s[1][q]:s[1][q + 1]], s[3][s[1][q]:s[1][q + 1]], s[4][s[1][q]:s[1][q + 1]])
                 for s in sends]
        xr = torch.cat([a for a, _, _ in parts])
        er = torch.cat([b for _, b, _ in parts])
        wr = torch.cat([c for _, _, c in parts])
        ys.append((S.a2a_experts(xr, er, wr, locs[q], bufs[q]), [len(a) for a, _, _ in parts]))
        torch.cuda.synchronize()
    outs = []
    for r in range(world):
        # back to rank r: its rows from every owner q, in owner order
        back = torch.cat([ys[q][0][sum(ys[q][1][:r]):sum(ys[q][1][:r + 1])] for q in range(world)])
        outs.append(S.a2a_merge(xs[r], back, locs[r], cfg.k, bufs[r]).clone())
        torch.cuda.synchronize()
        assert int(bufs[r].route.status.item()) == 0
    out = torch.cat(outs).cpu()
    ids = torch.cat([b.route.ids for b in bufs]).cpu().numpy()
    l64 = O.router_logits(p["x"], p["W_gate"], p["bias"])
    rng = np.random.default_rng(world)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], rng.choice(cfg.T, min(cfg.T, 16), False)]))
    w64 = O.routing_weights(l64[toks], ids[toks], cfg.renormalize)
    want = O.moe_forward_tokens(p, toks, ids[toks], w64)
    assert err_bf16_out(out[torch.as_tensor(toks)], want) <= TOL["bf16"]
    # every token against the single-GPU layer on each rank's batch (both bf16:
    # compared beyond one rounding; the merge here adds fp32 rows, the layer fp16 ones)
    for r in range(world):
        b1 = M.MoELayerBuffers(T_r, cfg.H, cfg.E, cfg.k, cfg.I, cfg.torch_dtype,
                               shared_I=cfg.shared_I)
        one = M.moe_layer_forward(xs[r], dp, cfg.k, cfg.renormalize, b1)
        torch.cuda.synchronize()
        assert err_bf16_out(outs[r].cpu(), O.to_f64(one.cpu())) <= TOL["bf16"]


@pytest.mark.parametrize("I", [192, 704])
def test_experts_with_I_a_multiple_of_64_only(I):
    # the tensor-parallel slices of I = 1408 (Qwen1.5-MoE-A2.7B, the builder) are 704
    g = torch.Generator().manual_seed(I)
    counts = [0, 130, 5, 300]
    E, H = len(counts), 512
    offs = torch.tensor(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))
    N = int(offs[-1])
    x = torch.randn(N, H, generator=g).to(torch.bfloat16)
    w13 = (torch.randn(E, 2 * I, H, generator=g) / H ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(E, H, I, generator=g) / I ** 0.5).to(torch.bfloat16)
    pw = torch.rand(N, generator=g)
    for with_ws in (True, False):
        h = torch.full((N + 1, I), 1536.0, dtype=torch.bfloat16, device=DEV)
        y = torch.full((N + 1, H), 1536.0, device=DEV)
        ws = torch.zeros(M.moe_experts_workspace_bytes(N, H, I, E, M.MOE_BF16), dtype=torch.uint8,
                         device=DEV) if with_ws else None
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        M.moe_experts(dev(torch.cat([x, x[:1]])), dev(offs), dev(torch.cat([pw, pw[:1]])),
                      dev(w13), dev(w2), h, y, ws=ws, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        ho, yo = O.experts(x, offs.numpy(), pw, w13, w2)
        assert err_bf16_out(h.cpu()[:N], ho) <= TOL["bf16"]
        assert rel(y.cpu()[:N], yo) <= TOL["bf16"]
        # nothing written past I in any row, nor past the last row
        assert (h.cpu()[N].float() == 1536.0).all() and (y.cpu()[N] == 1536.0).all()
