"""Plant plausible mistakes in the oracle (CPU only) and check that a pin fails.

Each mutation swaps one oracle function for a subtly wrong version and runs the
pin that should catch it; the test passes when the pin raises.
"""
import numpy as np
import pytest

import oracle.moe_oracle as M
import tests.test_oracle_pins as P


def _fails(fn, *args, **kw):
    try:
        fn(*args, **kw)
    except (AssertionError, ValueError, IndexError):
        return True
    return False


def test_swapped_w13_halves_is_caught(monkeypatch):
    monkeypatch.setattr(M, "w13_halves", lambda w, I: (w[I:2 * I], w[:I]))
    assert _fails(P.test_single_expert_layer_is_a_dense_swiglu_mlp)
    assert _fails(P.test_w13_up_half_offset_matches_the_refit_test)


def test_wrong_silu_sign_is_caught(monkeypatch):
    monkeypatch.setattr(M, "silu", lambda z: z / (1.0 + np.exp(z)))
    assert _fails(P.test_single_expert_layer_is_a_dense_swiglu_mlp)
    assert _fails(P.test_brute_force_triple_loops)


def test_untransposed_w2_is_caught(monkeypatch):
    def bad(x_rows, w13_e, w2_e, I):
        return M.expert_hidden(x_rows, w13_e, I) @ M.to_f64(w2_e)      # missing .T
    monkeypatch.setattr(M, "expert_output", bad)
    assert _fails(P.test_staged_equals_direct_form)


def test_tie_break_to_higher_id_is_caught(monkeypatch):
    def bad(l, k):
        order = np.argsort(-l[:, ::-1], axis=1, kind="stable")
        return (l.shape[1] - 1 - order)[:, :k]
    monkeypatch.setattr(M, "topk_experts", bad)
    assert _fails(P.test_topk_ties_go_to_lower_expert_id)


def test_ascending_selection_is_caught(monkeypatch):
    monkeypatch.setattr(M, "topk_experts", lambda l, k: np.argsort(l, axis=1, kind="stable")[:, :k])
    assert _fails(P.test_topk_brute_force_random, 5, 3)


def test_missing_renormalisation_is_caught(monkeypatch):
    orig = M.routing_weights
    monkeypatch.setattr(M, "routing_weights", lambda l, ids, ren: orig(l, ids, False))
    assert _fails(P.test_weights_renormalised_sum_to_one_and_unrenormalised_are_probs)
    assert _fails(P.test_brute_force_triple_loops)


def test_dropped_bias_is_caught(monkeypatch):
    monkeypatch.setattr(M, "router_logits", lambda x, W, b=None: M.to_f64(x) @ M.to_f64(W).T)
    assert _fails(P.test_logits_bias_and_orientation_brute_force)


def test_unstable_dispatch_is_caught(monkeypatch):
    orig = M.dispatch

    def bad(ids, w, E):
        d = orig(ids, w, E)
        # reverse the order inside every expert range
        perm = d["perm"].copy()
        for e in range(E):
            a, b = d["offsets"][e], d["offsets"][e + 1]
            perm[a:b] = perm[a:b][::-1]
        k = np.asarray(ids).shape[1]
        inv = np.empty_like(perm)
        inv[perm] = np.arange(len(perm))
        d.update(perm=perm, inv_perm=inv, packed_tok=perm // k,
                 packed_w=np.asarray(w, dtype=np.float64).reshape(-1)[perm])
        return d
    monkeypatch.setattr(M, "dispatch", bad)
    # (The pages' worked examples never route two assignments to one expert, so
    # only the brute-force pin sees the order inside an expert.)
    assert any(_fails(P.test_dispatch_brute_force_tiny, s) for s in range(12))


def test_wrong_merge_index_is_caught(monkeypatch):
    def bad(y_packed, inv_perm, T, k, shared=None, shared_gate=None):
        y = M.to_f64(y_packed)
        ip = np.asarray(inv_perm)
        out = np.zeros((T, y.shape[1]))
        for j in range(k):
            out += y[ip[np.arange(T) + j * T]]          # column-major flat index
        return out
    monkeypatch.setattr(M, "combine", bad)
    assert _fails(P.test_staged_equals_direct_form)


def test_routing_weight_applied_twice_is_caught(monkeypatch):
    orig = M.experts

    def bad(x_packed, offsets, packed_w, w13, w2):
        h, y = orig(x_packed, offsets, packed_w, w13, w2)
        pw = np.ones(len(y)) if packed_w is None else M.to_f64(packed_w)
        return h, y * pw[:, None]
    monkeypatch.setattr(M, "experts", bad)
    assert _fails(P.test_staged_equals_direct_form)
    assert _fails(P.test_k_equals_E_identical_experts_is_the_dense_mlp, True)


@pytest.mark.parametrize("bad_gate", ["no_sigmoid", "minus"])
def test_wrong_shared_gate_is_caught(monkeypatch, bad_gate):
    orig = M.combine

    def bad(y_packed, inv_perm, T, k, shared=None, shared_gate=None):
        if shared is not None:
            sg = M.to_f64(shared_gate)
            # sigmoid(g) = 1/(1+exp(-g)); feed a logit that yields the wrong factor
            sg = np.log(np.maximum(sg, 1e-300)) if bad_gate == "no_sigmoid" else -sg
            shared_gate = sg
        return orig(y_packed, inv_perm, T, k, shared, shared_gate)
    monkeypatch.setattr(M, "combine", bad)
    assert _fails(P.test_shared_expert_and_sigmoid_gate)


# --------------------------- the sharded forms and group-limited selection ---

import tests.test_oracle_grouped as G          # noqa: E402
import tests.test_oracle_parallel as PP        # noqa: E402


def test_group_scored_by_its_worst_expert_is_caught(monkeypatch):
    def bad(l, k, n_groups, topk_groups):
        T, E = l.shape
        gs = E // n_groups
        out = np.empty((T, k), dtype=np.int64)
        for t in range(T):
            score = [min(l[t, g * gs:(g + 1) * gs]) for g in range(n_groups)]    # min, not max
            groups = sorted(range(n_groups), key=lambda g: (-score[g], g))[:topk_groups]
            cand = sorted((e for g in groups for e in range(g * gs, (g + 1) * gs)),
                          key=lambda e: (-l[t, e], e))
            out[t] = cand[:k]
        return out
    monkeypatch.setattr(M, "topk_experts_grouped", bad)
    assert _fails(G.test_brute_force_on_tiny_layers, 8, 3, 4, 2)
    assert _fails(G.test_a_case_where_group_limiting_changes_the_choice)


def test_group_ties_to_the_higher_group_are_caught(monkeypatch):
    orig = M.topk_experts_grouped

    def bad(l, k, n_groups, topk_groups):
        E = l.shape[1]
        gs = E // n_groups
        flip = np.concatenate([np.arange((n_groups - 1 - g) * gs, (n_groups - g) * gs)
                               for g in range(n_groups)])
        got = orig(l[:, flip], k, n_groups, topk_groups)        # groups numbered backwards
        return flip[got]
    monkeypatch.setattr(M, "topk_experts_grouped", bad)
    assert _fails(G.test_equal_group_scores_keep_the_lower_group)


def test_tp_slice_with_swapped_members_is_caught(monkeypatch):
    orig = M.tp_slice

    def bad(w13_e, w2_e, rank, tp):
        slot, w2r = orig(w13_e, w2_e, rank, tp)
        it = slot.shape[0] // 2
        return np.concatenate([slot[it:], slot[:it]]), w2r         # w3 low, w1 high
    monkeypatch.setattr(M, "tp_slice", bad)
    assert _fails(PP.test_tp_slice_reproduces_the_refit_tests_worked_example)
    assert _fails(PP.test_tensor_parallel_partials_add_up_to_the_layer, 2, False)


def test_tp_slice_from_the_wrong_rank_is_caught(monkeypatch):
    orig = M.tp_slice
    monkeypatch.setattr(M, "tp_slice", lambda a, b, rank, tp: orig(a, b, (rank + 1) % tp, tp))
    assert _fails(PP.test_tp_slice_of_every_rank_tiles_w13_and_w2) or \
        _fails(PP.test_tensor_parallel_partials_add_up_to_the_layer, 2, True)
    assert _fails(PP.test_tp_slice_reproduces_the_refit_tests_worked_example)


def test_expert_range_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(M, "expert_ranges",
                        lambda E, world: [(E * q // world, E * (q + 1) // world + (q == 0))
                                          for q in range(world)])
    assert _fails(PP.test_expert_ranges_partition_the_experts, 8, 3)
    assert _fails(PP.test_masked_local_partials_add_up_to_the_layer, 3, False)
