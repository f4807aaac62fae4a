"""Pins of the oracle's group-limited top-k (CPU).

The pages name the router (diffulex.moe.topk, GroupLimitedTopKRouter: "router
with group-limited expert selection") without its rule; the oracle takes the
plainest reading (groups of consecutive experts, a group scored by its best
logit, the best `topk_groups` groups kept, top-k among their experts).  The
pins below fix that reading without re-running the oracle's own steps:
special cases that reduce to plain top-k, a brute-force search under an
independently worded eligibility rule, a hand-worked case where the two
routers differ, and ties between groups.
"""
import itertools

import numpy as np
import pytest

import oracle.moe_oracle as O


@pytest.mark.parametrize("E,k,G", [(8, 2, 1), (16, 4, 1), (64, 8, 1)])
def test_one_group_is_plain_topk(E, k, G):
    l = np.random.default_rng(E).standard_normal((50, E))
    np.testing.assert_array_equal(O.topk_experts_grouped(l, k, G, 1), O.topk_experts(l, k))


@pytest.mark.parametrize("E,k,G", [(8, 2, 4), (16, 4, 8), (256, 8, 8)])
def test_keeping_every_group_is_plain_topk(E, k, G):
    l = np.random.default_rng(E + G).standard_normal((40, E))
    np.testing.assert_array_equal(O.topk_experts_grouped(l, k, G, G), O.topk_experts(l, k))


@pytest.mark.parametrize("E,k,M", [(8, 2, 2), (8, 3, 5), (12, 4, 4)])
def test_groups_of_one_expert_with_enough_groups_is_plain_topk(E, k, M):
    l = np.random.default_rng(E * k).standard_normal((40, E))
    np.testing.assert_array_equal(O.topk_experts_grouped(l, k, E, M), O.topk_experts(l, k))


def _brute(l_row, k, G, M):
    E = len(l_row)
    gs = E // G
    score = [max(l_row[g * gs:(g + 1) * gs]) for g in range(G)]
    # group g is eligible when fewer than M groups beat it (a higher score, or
    # an equal score and a lower id)
    ok = [sum(1 for h in range(G) if score[h] > score[g] or (score[h] == score[g] and h < g)) < M
          for g in range(G)]
    elig = [e for e in range(E) if ok[e // gs]]
    best = None
    for sub in itertools.combinations(elig, k):
        key = sorted(((-l_row[e], e) for e in sub))
        if best is None or key < best:
            best = key
    return [e for _, e in best]


@pytest.mark.parametrize("E,k,G,M", [(6, 2, 3, 1), (8, 3, 4, 2), (8, 2, 2, 1), (9, 3, 3, 2)])
def test_brute_force_on_tiny_layers(E, k, G, M):
    rng = np.random.default_rng(E + 10 * k + 100 * G + 1000 * M)
    l = rng.standard_normal((60, E))
    l[::7, :] = np.round(l[::7, :])             # rows with ties
    got = O.topk_experts_grouped(l, k, G, M)
    for t in range(l.shape[0]):
        assert got[t].tolist() == _brute(l[t], k, G, M)


def test_selection_stays_inside_the_kept_groups():
    rng = np.random.default_rng(3)
    E, G, M, k = 256, 8, 4, 8
    l = rng.standard_normal((200, E))
    ids = O.topk_experts_grouped(l, k, G, M)
    for t in range(l.shape[0]):
        assert len(set(ids[t] // (E // G))) <= M
        assert len(set(ids[t].tolist())) == k


def test_a_case_where_group_limiting_changes_the_choice():
    # groups {0,1} {2,3} {4,5}: best logits 0.9, 0.1, 0.88 -> with one group
    # kept, the two experts of group 0 win although expert 4 beats expert 1
    l = np.array([[0.9, 0.85, 0.1, 0.1, 0.88, 0.0]])
    assert O.topk_experts_grouped(l, 2, 3, 1).tolist() == [[0, 1]]
    assert O.topk_experts(l, 2).tolist() == [[0, 4]]
    assert O.topk_experts_grouped(l, 2, 3, 2).tolist() == [[0, 4]]


def test_equal_group_scores_keep_the_lower_group():
    l = np.array([[0.5, 0.1, 0.0, 0.5, 0.2, 0.3]])      # groups of 2: scores 0.5, 0.5, 0.3
    assert O.topk_experts_grouped(l, 2, 3, 1).tolist() == [[0, 1]]
    assert O.topk_experts_grouped(l, 2, 3, 2).tolist() == [[0, 3]]
