"""Pins of the oracle's expert- and tensor-parallel forms (CPU).

* expert ownership: every expert on exactly one rank, the same owner as a
  library search (numpy.searchsorted over the range starts);
* the tensor-parallel slice of w13: the worked example of the modelexpress
  refit test (rank 0 of 2, INTER = 8, HIDDEN = 4, fp32: expert 1's w3 slice
  lands at byte 192 of the fused destination and 64 bytes are pulled, from
  the start of the source);
* the ranks' partial outputs add up to the unsharded layer (masked-local
  expert parallelism, tensor parallelism), within fp64 rounding.
"""
import json
import os

import numpy as np
import pytest

import oracle.moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _layer(rng, T, H, E, k, I, shared_I=None):
    p = {"x": rng.standard_normal((T, H)),
         "W_gate": rng.standard_normal((E, H)) / np.sqrt(H), "bias": None,
         "w13": rng.standard_normal((E, 2 * I, H)) / np.sqrt(H),
         "w2": rng.standard_normal((E, H, I)) / np.sqrt(I), "w13s": None, "w2s": None,
         "w_sg": None}
    if shared_I:
        p["w13s"] = rng.standard_normal((2 * shared_I, H)) / np.sqrt(H)
        p["w2s"] = rng.standard_normal((H, shared_I)) / np.sqrt(shared_I)
        p["w_sg"] = rng.standard_normal(H) / np.sqrt(H)
    return p


@pytest.mark.parametrize("E,world", [(8, 1), (8, 3), (60, 4), (64, 8), (128, 7), (5, 5)])
def test_expert_ranges_partition_the_experts(E, world):
    ranges = O.expert_ranges(E, world)
    covered = np.concatenate([np.arange(a, b) for a, b in ranges])
    np.testing.assert_array_equal(covered, np.arange(E))
    sizes = [b - a for a, b in ranges]
    assert min(sizes) >= E // world and max(sizes) <= -(-E // world)
    owner = O.expert_owner(np.arange(E), E, world)
    starts = np.array([a for a, _ in ranges])
    np.testing.assert_array_equal(owner, np.searchsorted(starts, np.arange(E), side="right") - 1)


def test_tp_slice_reproduces_the_refit_tests_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "w13_layout.json")))
    H, INTER, TP, LOCAL = g["HIDDEN"], g["INTER"], g["TP_SIZE"], g["LOCAL_EXPERTS"]
    it = INTER // TP
    rng = np.random.default_rng(0)
    # per-expert HF sources (gate_proj = w1, up_proj = w3), each [INTER, HIDDEN]
    w1 = rng.standard_normal((LOCAL, INTER, H)).astype(np.float32)
    w3 = rng.standard_normal((LOCAL, INTER, H)).astype(np.float32)
    w2 = rng.standard_normal((LOCAL, H, INTER)).astype(np.float32)
    dest = np.stack([O.tp_slice(np.concatenate([w1[e], w3[e]]), w2[e], 0, TP)[0]
                     for e in range(LOCAL)]).astype(np.float32)
    assert dest.shape == (LOCAL, 2 * it, H)
    flat = dest.reshape(-1)
    e, es = g["expert"], g["elsize"]
    start = g["expected_dst_bytes"] // es
    # expert 1's w3 slice starts at byte 192 of the fused destination ...
    np.testing.assert_array_equal(flat[start:start + it * H], w3[e, 0:it].reshape(-1))
    # ... is exactly this rank's rows (64 bytes, read from the start of the source)
    assert it * H * es == g["pulled_bytes"]
    # and expert 1's w1 slice sits just below it, the low half of its slot
    low = e * 2 * it * H
    np.testing.assert_array_equal(flat[low:low + it * H], w1[e, 0:it].reshape(-1))


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("shared", [False, True])
def test_masked_local_partials_add_up_to_the_layer(world, shared):
    rng = np.random.default_rng(world)
    T, H, E, k, I = 13, 16, 8, 3, 12
    p = _layer(rng, T, H, E, k, I, shared_I=8 if shared else None)
    l, ids, w = O.route(p["x"], p["W_gate"], None, k, True)
    toks = np.arange(T)
    want = O.moe_forward_tokens(p, toks, ids, w)
    parts = [O.moe_forward_tokens_ep(p, toks, ids, w, a, b, with_shared=(q == 0))
             for q, (a, b) in enumerate(O.expert_ranges(E, world))]
    assert O.rel_err_rms(sum(parts), want) <= 1e-12
    if world > 1:
        # a rank alone is not the layer: the split really drops the other experts
        assert O.rel_err_rms(parts[-1], want) > 1e-3


@pytest.mark.parametrize("tp", [1, 2, 4])
@pytest.mark.parametrize("shared", [False, True])
def test_tensor_parallel_partials_add_up_to_the_layer(tp, shared):
    rng = np.random.default_rng(10 + tp)
    T, H, E, k, I = 11, 16, 6, 2, 16
    p = _layer(rng, T, H, E, k, I, shared_I=8 if shared else None)
    l, ids, w = O.route(p["x"], p["W_gate"], None, k, False)
    toks = np.arange(T)
    want = O.moe_forward_tokens(p, toks, ids, w)
    parts = [O.moe_forward_tokens_tp(p, toks, ids, w, r, tp) for r in range(tp)]
    assert O.rel_err_rms(sum(parts), want) <= 1e-12
    if tp > 1:
        assert O.rel_err_rms(parts[0], want) > 1e-3


def test_tp_slice_of_every_rank_tiles_w13_and_w2():
    rng = np.random.default_rng(3)
    I, H, tp = 12, 5, 3
    w13 = rng.standard_normal((2 * I, H))
    w2 = rng.standard_normal((H, I))
    slots = [O.tp_slice(w13, w2, r, tp) for r in range(tp)]
    it = I // tp
    np.testing.assert_array_equal(np.concatenate([s[0][:it] for s in slots]), w13[:I])
    np.testing.assert_array_equal(np.concatenate([s[0][it:] for s in slots]), w13[I:])
    np.testing.assert_array_equal(np.concatenate([s[1] for s in slots], axis=1), w2)
