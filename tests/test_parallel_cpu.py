"""Multi-rank host logic of the sharded layers on CPU (gloo, 2 and 3 ranks).

The rank-local arithmetic here is the oracle's (the library's kernels need a
GPU); what is under test is the library's host side: the expert ranges, the
tensor-parallel weight slices, and the collectives the sharded layers use
between ranks -- the all-reduce of the partial outputs, the exchange of
counts and the uneven all-to-all of token rows and of the outputs coming
back.  Every rank's result must equal the unsharded oracle layer.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import mixture_experts_layer_44_b200.sharded as S
import oracle.moe_oracle as O
from moe_inputs import LayerConfig, make_layer

CFG = LayerConfig("cpu_ranks", T=24, H=32, E=6, k=3, I=16, dtype="f32", renormalize=True,
                  zipf_s=1.0)
CFG_SHARED = LayerConfig("cpu_ranks_shared", T=18, H=32, E=6, k=2, I=16, dtype="f32",
                         renormalize=False, shared_I=24)


@pytest.mark.parametrize("E,world", [(8, 1), (8, 3), (60, 4), (64, 8), (128, 7)])
def test_expert_range_is_the_oracles(E, world):
    assert [S.expert_range(E, world, r) for r in range(world)] == O.expert_ranges(E, world)
    with pytest.raises(ValueError):
        S.expert_range(E, E + 1, 0)


@pytest.mark.parametrize("tp", [1, 2, 4])
def test_tp_shard_params_are_the_oracles_slices(tp):
    p = make_layer(CFG_SHARED, seed=3)
    for r in range(tp):
        sh = S.tp_shard_params(p, r, tp)
        for e in range(CFG_SHARED.E):
            slot, w2r = O.tp_slice(p["w13"][e], p["w2"][e], r, tp)
            np.testing.assert_array_equal(O.to_f64(sh["w13"][e]), slot)
            np.testing.assert_array_equal(O.to_f64(sh["w2"][e]), w2r)
        slot, w2r = O.tp_slice(p["w13s"], p["w2s"], r, tp)
        np.testing.assert_array_equal(O.to_f64(sh["w13s"]), slot)
        np.testing.assert_array_equal(O.to_f64(sh["w2s"]), w2r)
        assert sh["w13"].is_contiguous() and sh["w2"].is_contiguous()


def test_ep_local_params_hold_the_ranks_experts_only():
    p = make_layer(CFG_SHARED, seed=4)
    loc = S.ep_local_params(p, 2, 5, run_shared=False)
    assert torch.equal(loc["w13"], p["w13"][2:5]) and torch.equal(loc["w2"], p["w2"][2:5])
    assert "w13s" not in loc and torch.equal(loc["W_gate"], p["W_gate"])
    assert "w13s" in S.ep_local_params(p, 0, 2, run_shared=True)


def _route(cfg, p, x):
    l = O.router_logits(x, p["W_gate"], p["bias"])
    ids = O.topk_experts(l, cfg.k)
    return ids, O.routing_weights(l, ids, cfg.renormalize)


def _worker(rank, world, port, mode, cfg_name, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = CFG if cfg_name == "plain" else CFG_SHARED
        p = make_layer(cfg, seed=0)
        T = cfg.T
        if mode in ("ep", "tp"):
            ids, w = _route(cfg, p, p["x"])
            toks = np.arange(T)
            want = O.moe_forward_tokens(p, toks, ids, w)
            if mode == "ep":
                lo, hi = S.expert_range(cfg.E, world, rank)
                part = O.moe_forward_tokens_ep(p, toks, ids, w, lo, hi, with_shared=(rank == 0))
            else:
                part = O.moe_forward_tokens_tp(p, toks, ids, w, rank, world)
            t = torch.tensor(part)
            S.allreduce_sum_(t)
            q.put((rank, O.rel_err_rms(t, want)))
        else:
            # all-to-all: rank r owns tokens [r*T/world, (r+1)*T/world) and experts
            # expert_range(E, world, r)
            tr = T // world
            x = p["x"][rank * tr:(rank + 1) * tr]
            ids, w = _route(cfg, p, x)
            owner = O.expert_owner(ids, cfg.E, world)
            d = O.dispatch(owner, w, world)               # send order: by owner, then f
            sc = torch.tensor(d["counts"], dtype=torch.int64)
            rc = S.exchange_counts(sc)
            flat_ids = ids.reshape(-1)[d["perm"]]
            starts = np.array([a for a, _ in O.expert_ranges(cfg.E, world)])
            send_x = torch.tensor(O.to_f64(x)[d["packed_tok"]])
            send_e = torch.tensor(flat_ids - starts[owner.reshape(-1)[d["perm"]]], dtype=torch.int64)
            send_w = torch.tensor(d["packed_w"])
            rx = S.all_to_all_rows(send_x, sc.tolist(), rc.tolist())
            re = S.all_to_all_rows(send_e, sc.tolist(), rc.tolist())
            rw = S.all_to_all_rows(send_w, sc.tolist(), rc.tolist())
            lo, hi = S.expert_range(cfg.E, world, rank)
            I = p["w13"].shape[1] // 2
            y = torch.zeros(rx.shape[0], cfg.H, dtype=torch.float64)
            for i in range(rx.shape[0]):
                e = lo + int(re[i])
                assert lo <= e < hi
                y[i] = float(rw[i]) * torch.tensor(
                    O.expert_output(rx[i:i + 1].numpy(), p["w13"][e], p["w2"][e], I)[0])
            back = S.all_to_all_rows(y, rc.tolist(), sc.tolist())
            sg = shared = None
            if p.get("w13s") is not None:
                shared = O.shared_expert(x, p["w13s"], p["w2s"])
                sg = O.shared_gate_logit(x, p["w_sg"])
            out = O.combine(back, d["inv_perm"], tr, cfg.k, shared, sg)
            want = O.moe_forward_tokens(dict(p, x=x), np.arange(tr), ids, w)
            q.put((rank, O.rel_err_rms(out, want)))
    finally:
        dist.destroy_process_group()


def _run(world, mode, cfg_name):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() * 7 + world * 31 + len(mode) * 3 + len(cfg_name)) % 2000
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, cfg_name, q))
             for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=180)
        assert pr.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, err in res:
        assert err <= 1e-12, (mode, cfg_name, rank, err)


@pytest.mark.parametrize("mode", ["ep", "tp", "a2a"])
@pytest.mark.parametrize("cfg_name", ["plain", "shared"])
def test_two_gloo_ranks_reproduce_the_unsharded_layer(mode, cfg_name):
    _run(2, mode, cfg_name)


def test_three_gloo_ranks_all_to_all():
    _run(3, "a2a", "plain")
