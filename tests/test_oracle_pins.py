"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a value the pages print, a closed form, an
invariant, a textbook special case computed with library routines, or brute
force on tiny inputs.  No GPU.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.moe_oracle as O
from moe_inputs import CONFIGS, make_layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_layer(rng, T, H, E, k, I, shared_I=None, bias=False):
    p = dict(
        x=rng.standard_normal((T, H)),
        W_gate=rng.standard_normal((E, H)) / math.sqrt(H),
        bias=(rng.standard_normal(E) if bias else None),
        w13=rng.standard_normal((E, 2 * I, H)) / math.sqrt(H),
        w2=rng.standard_normal((E, H, I)) / math.sqrt(I),
        w13s=None, w2s=None, w_sg=None,
    )
    if shared_I:
        p["w13s"] = rng.standard_normal((2 * shared_I, H)) / math.sqrt(H)
        p["w2s"] = rng.standard_normal((H, shared_I)) / math.sqrt(shared_I)
        p["w_sg"] = rng.standard_normal(H) / math.sqrt(H)
    return p


def _swiglu_mlp_torch(x, w13_e, w2_e):
    """Textbook SwiGLU MLP with torch library ops: linear(silu(linear(x, W1)) * linear(x, W3), W2)."""
    x = torch.as_tensor(x, dtype=torch.float64)
    w13_e = torch.as_tensor(w13_e, dtype=torch.float64)
    I = w13_e.shape[0] // 2
    g = F.linear(x, w13_e[:I])
    u = F.linear(x, w13_e[I:])
    return F.linear(F.silu(g) * u, torch.as_tensor(w2_e, dtype=torch.float64)).numpy()


# ------------------------------------------------------------ router pins ---

def test_logits_bias_and_orientation_brute_force():
    rng = np.random.default_rng(1)
    T, H, E = 3, 5, 4
    x = rng.standard_normal((T, H))
    W = rng.standard_normal((E, H))
    b = rng.standard_normal(E)
    l = O.router_logits(x, W, b)
    for t in range(T):
        for e in range(E):
            s = 0.0
            for h in range(H):
                s += x[t, h] * W[e, h]
            assert abs(l[t, e] - (s + b[e])) < 1e-12


def test_softmax_matches_library_and_closed_form():
    import scipy.special
    rng = np.random.default_rng(2)
    l = rng.standard_normal((7, 9)) * 5
    np.testing.assert_allclose(O.softmax_rows(l), scipy.special.softmax(l, axis=1), rtol=1e-13)
    # Two experts: p_max = sigmoid(l_max - l_min).
    l2 = np.array([[0.3, -1.2]])
    assert abs(O.softmax_rows(l2)[0, 0] - 1 / (1 + math.exp(-1.5))) < 1e-15
    # Large logits: the max shift keeps it finite.
    big = np.array([[1000.0, 999.0]])
    assert np.isfinite(O.softmax_rows(big)).all()


def _brute_topk(row, k):
    E = len(row)
    best = None
    for sub in itertools.combinations(range(E), k):
        key = (sum(row[e] for e in sub), tuple(-e for e in sub))
        if best is None or key > best[0]:
            best = (key, sub)
    chosen = list(best[1])
    return sorted(chosen, key=lambda e: (-row[e], e))


@pytest.mark.parametrize("E,k", [(1, 1), (3, 1), (4, 2), (5, 3), (6, 6), (7, 4)])
def test_topk_brute_force_random(E, k):
    rng = np.random.default_rng(10 + E * 7 + k)
    l = rng.standard_normal((25, E))
    ids = O.topk_experts(l, k)
    for t in range(l.shape[0]):
        assert list(ids[t]) == _brute_topk(l[t], k)


def test_topk_ties_go_to_lower_expert_id():
    # Deliberate duplicates: equal logits must select (and list first) the lower id.
    l = np.array([[1.0, 3.0, 3.0, 2.0],
                  [2.0, 2.0, 2.0, 2.0],
                  [0.0, 5.0, 0.0, 5.0],
                  [-1.0, -1.0, 4.0, -1.0]])
    assert O.topk_experts(l, 1).tolist() == [[1], [0], [1], [2]]
    assert O.topk_experts(l, 2).tolist() == [[1, 2], [0, 1], [1, 3], [2, 0]]
    assert O.topk_experts(l, 3).tolist() == [[1, 2, 3], [0, 1, 2], [1, 3, 0], [2, 0, 1]]
    for t in range(l.shape[0]):
        for k in range(1, 5):
            assert O.topk_experts(l[t:t + 1], k)[0].tolist() == _brute_topk(l[t], k)


def test_weights_renormalised_sum_to_one_and_unrenormalised_are_probs():
    rng = np.random.default_rng(3)
    l = rng.standard_normal((50, 12)) * 2
    ids = O.topk_experts(l, 3)
    w = O.routing_weights(l, ids, True)
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12)
    # Renormalised weights equal the softmax over the k selected logits.
    sel = np.take_along_axis(l, ids, axis=1)
    np.testing.assert_allclose(w, O.softmax_rows(sel), rtol=1e-13)
    wn = O.routing_weights(l, ids, False)
    p = O.softmax_rows(l)
    assert np.array_equal(wn, np.take_along_axis(p, ids, axis=1))
    assert (wn.sum(1) <= 1 + 1e-15).all()
    # Ordered by descending logit -> descending weight.
    assert (np.diff(w, axis=1) <= 0).all()


def test_k_equals_E_gives_full_softmax():
    rng = np.random.default_rng(4)
    l = rng.standard_normal((10, 6))
    ids = O.topk_experts(l, 6)
    for ren in (True, False):
        w = O.routing_weights(l, ids, ren)
        full = np.zeros_like(l)
        np.put_along_axis(full, ids, w, axis=1)
        np.testing.assert_allclose(full, O.softmax_rows(l), rtol=1e-13)


# ---------------------------------------------------------- dispatch pins ---

def _check_dispatch_invariants(ids, w, E, d):
    T, k = ids.shape
    N = T * k
    flat = ids.reshape(N)
    assert d["counts"].sum() == N
    np.testing.assert_array_equal(d["counts"], np.bincount(flat, minlength=E))
    assert d["offsets"][0] == 0 and d["offsets"][E] == N
    np.testing.assert_array_equal(np.diff(d["offsets"]), d["counts"])
    np.testing.assert_array_equal(d["perm"][d["inv_perm"]], np.arange(N))
    np.testing.assert_array_equal(d["inv_perm"][d["perm"]], np.arange(N))
    for e in range(E):
        a, b = d["offsets"][e], d["offsets"][e + 1]
        seg = d["perm"][a:b]
        assert (np.diff(seg) > 0).all()
        assert (flat[seg] == e).all()
    assert (d["packed_tok"] * k <= d["perm"]).all()
    assert (d["perm"] < d["packed_tok"] * k + k).all()
    np.testing.assert_array_equal(d["packed_w"], np.asarray(w).reshape(N)[d["perm"]])


@pytest.mark.parametrize("seed", range(12))
def test_dispatch_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    T = int(rng.integers(1, 7))
    E = int(rng.integers(1, 6))
    k = int(rng.integers(1, min(E, 3) + 1))
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    w = rng.random((T, k))
    d = O.dispatch(ids, w, E)
    _check_dispatch_invariants(ids, w, E, d)
    N = T * k
    flat = ids.reshape(N)
    order = sorted(range(N), key=lambda f: (flat[f], f))   # O(N log N) library sort by (e, f)
    np.testing.assert_array_equal(d["perm"], order)


def test_dispatch_invariants_larger_and_empty_experts():
    rng = np.random.default_rng(7)
    T, E, k = 300, 16, 4
    ids = np.stack([rng.choice(np.arange(0, E, 2), size=k, replace=False) for _ in range(T)])
    w = rng.random((T, k))
    d = O.dispatch(ids, w, E)
    _check_dispatch_invariants(ids, w, E, d)
    assert (d["counts"][1::2] == 0).all()


def _load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_ep_partition_reproduces_the_pages_worked_examples():
    g = _load_golden("ep_dispatch_buckets.json")
    for case in g["cases"]:
        b = O.ep_partition(case["indices"], case["weights"], case["num_tokens"], case["top_k"],
                           case["local_start"], case["local_end"])
        ex = case["expect"]
        if "local_count" in ex:
            assert len(b["local_token_indices"]) == ex["local_count"], case["name"]
        if "remote_count" in ex:
            assert len(b["remote_token_indices"]) == ex["remote_count"], case["name"]
        if "total_count" in ex:
            assert len(b["local_token_indices"]) + len(b["remote_token_indices"]) == ex["total_count"]
        for key in ("local_token_indices", "local_expert_ids", "local_weights",
                    "remote_token_indices", "remote_expert_ids", "remote_weights"):
            if key in ex:
                assert b[key] == ex[key], (case["name"], key)
    for case in g["length_mismatch"]:
        with pytest.raises(ValueError, match=case["message"]):
            O.ep_partition(case["indices"], case["weights"], case["num_tokens"], case["top_k"], 0, 256)


def test_dispatch_order_agrees_with_the_pages_bucket_order():
    """Within one expert, the expert-major range lists assignments in the order
    the worked examples' buckets keep (given order = ascending t*k + j)."""
    g = _load_golden("ep_dispatch_buckets.json")
    for case in g["cases"]:
        T, k = case["num_tokens"], case["top_k"]
        idx = np.array(case["indices"]).reshape(T, k)
        w = np.array(case["weights"]).reshape(T, k)
        E = int(idx.max()) + 1
        d = O.dispatch(idx, w, E)
        for side in ("local", "remote"):
            b = O.ep_partition(case["indices"], case["weights"], T, k,
                               case["local_start"], case["local_end"])
            for e in set(b[f"{side}_expert_ids"]):
                sel = [i for i, x in enumerate(b[f"{side}_expert_ids"]) if x == e]
                want_tok = [b[f"{side}_token_indices"][i] for i in sel]
                want_w = [b[f"{side}_weights"][i] for i in sel]
                a, z = d["offsets"][e], d["offsets"][e + 1]
                assert d["packed_tok"][a:z].tolist() == want_tok
                assert d["packed_w"][a:z].tolist() == pytest.approx(want_w, abs=0)


# ------------------------------------------------------- w13 layout pin ---

def test_w13_up_half_offset_matches_the_refit_test():
    g = _load_golden("w13_layout.json")
    I = g["INTER"] // g["TP_SIZE"]
    H = g["HIDDEN"]
    E = g["LOCAL_EXPERTS"]
    buf = np.arange(E * 2 * I * H, dtype=np.float32).reshape(E, 2 * I, H)
    gate, up = O.w13_halves(buf[g["expert"]], I)
    assert int(up[0, 0]) * g["elsize"] == g["expected_dst_bytes"]
    assert up.size * g["elsize"] == g["pulled_bytes"]
    assert int(gate[0, 0]) * g["elsize"] == g["expert"] * 2 * I * H * g["elsize"]


# ------------------------------------------------- experts / merge pins ---

def test_single_expert_layer_is_a_dense_swiglu_mlp():
    rng = np.random.default_rng(11)
    p = _rand_layer(rng, T=9, H=16, E=1, k=1, I=24)
    r = O.moe_forward(p, k=1, renormalize=True)
    np.testing.assert_allclose(r["w"], 1.0)
    want = _swiglu_mlp_torch(p["x"], p["w13"][0], p["w2"][0])
    np.testing.assert_allclose(r["out"], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("renorm", [True, False])
def test_k_equals_E_identical_experts_is_the_dense_mlp(renorm):
    rng = np.random.default_rng(12)
    p = _rand_layer(rng, T=7, H=16, E=4, k=4, I=8)
    p["w13"][:] = p["w13"][0]
    p["w2"][:] = p["w2"][0]
    r = O.moe_forward(p, k=4, renormalize=renorm)
    want = _swiglu_mlp_torch(p["x"], p["w13"][0], p["w2"][0])
    np.testing.assert_allclose(r["out"], want, rtol=1e-11, atol=1e-12)


def test_staged_equals_direct_form():
    rng = np.random.default_rng(13)
    p = _rand_layer(rng, T=40, H=16, E=6, k=2, I=12, shared_I=20, bias=True)
    for ren in (True, False):
        r = O.moe_forward(p, k=2, renormalize=ren)
        d = O.moe_forward_tokens(p, np.arange(40), r["ids"], r["w"])
        np.testing.assert_allclose(r["out"], d, rtol=1e-12, atol=1e-12)


def test_brute_force_triple_loops():
    rng = np.random.default_rng(14)
    T, H, E, k, I = 2, 4, 3, 2, 8
    p = _rand_layer(rng, T, H, E, k, I, bias=True)
    r = O.moe_forward(p, k=k, renormalize=True)
    x, Wg, b, w13, w2 = p["x"], p["W_gate"], p["bias"], p["w13"], p["w2"]
    for t in range(T):
        l = [sum(x[t, h] * Wg[e, h] for h in range(H)) + b[e] for e in range(E)]
        order = sorted(range(E), key=lambda e: (-l[e], e))[:k]
        ex = [math.exp(l[e] - max(l)) for e in order]
        wts = [v / sum(ex) for v in ex]
        out = [0.0] * H
        for e, wt in zip(order, wts):
            hid = []
            for i in range(I):
                g = sum(w13[e, i, h] * x[t, h] for h in range(H))
                u = sum(w13[e, I + i, h] * x[t, h] for h in range(H))
                hid.append(g / (1 + math.exp(-g)) * u)
            for h in range(H):
                out[h] += wt * sum(w2[e, h, i] * hid[i] for i in range(I))
        np.testing.assert_allclose(r["out"][t], out, rtol=1e-12, atol=1e-13)
        assert r["ids"][t].tolist() == order


def test_shared_expert_and_sigmoid_gate():
    rng = np.random.default_rng(15)
    p = _rand_layer(rng, T=5, H=8, E=3, k=1, I=4, shared_I=6)
    r = O.moe_forward(p, k=1, renormalize=False)
    base = dict(p, w13s=None, w2s=None, w_sg=None)
    r0 = O.moe_forward(base, k=1, renormalize=False)
    s = _swiglu_mlp_torch(p["x"], p["w13s"], p["w2s"])
    g = torch.sigmoid(torch.as_tensor(p["x"] @ p["w_sg"])).numpy()
    np.testing.assert_allclose(r["out"] - r0["out"], g[:, None] * s, rtol=1e-11, atol=1e-13)


def test_combine_with_identity_permutation_is_a_row_sum():
    rng = np.random.default_rng(16)
    T, k, H = 6, 3, 5
    y = rng.standard_normal((T * k, H))
    out = O.combine(y, np.arange(T * k), T, k)
    np.testing.assert_allclose(out, y.reshape(T, k, H).sum(1), rtol=1e-14)


def test_rel_err_rms_definition():
    want = np.array([3.0, -4.0])           # rms = sqrt(12.5)
    got = np.array([3.5, -4.0])
    assert abs(O.rel_err_rms(got, want) - 0.5 / math.sqrt(12.5)) < 1e-15


# -------------------------------------------------- workload generator ---

def test_tiny_workload_end_to_end_invariants():
    cfg = CONFIGS["tiny_f32"]
    p = make_layer(cfg, seed=0)
    r = O.moe_forward(p, cfg.k, cfg.renormalize)
    _check_dispatch_invariants(r["ids"], r["w"], cfg.E, r)
    np.testing.assert_allclose(r["w"].sum(1), 1.0, atol=1e-12)
    d = O.moe_forward_tokens(p, np.arange(cfg.T), r["ids"], r["w"])
    np.testing.assert_allclose(r["out"], d, rtol=1e-12, atol=1e-12)
