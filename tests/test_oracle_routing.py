"""Pins for the oracle's router selection, gates and permutation.

Selection reading (not fixed by the pages): top-K by logit with ties to the
lower expert index; gates = softmax over all N experts, restricted to the K
chosen and renormalised. Expert counts per token come from the pages' shapes
(128 experts / 6 active on the jiwasawa Nano page; 512 / 22 on the greeksharifa
page, section 2.2 "LatentMoE").
"""
import itertools

import numpy as np
import pytest

from oracle import lmoe_oracle as O


@pytest.mark.parametrize("N,K", [(4, 1), (5, 2), (6, 3), (8, 3), (7, 7)])
def test_topk_matches_subset_enumeration_integer_ties(N, K):
    rng = np.random.default_rng(N * 10 + K)
    logits = rng.integers(-2, 3, size=(40, N)).astype(np.float64)   # many exact ties
    idx, _ = O.route_topk(logits, K)
    for t in range(logits.shape[0]):
        assert list(idx[t]) == O.brute_force_topk(list(logits[t]), K)


def test_topk_matches_subset_enumeration_random():
    rng = np.random.default_rng(11)
    logits = rng.standard_normal((60, 8))
    idx, _ = O.route_topk(logits, 3)
    for t in range(60):
        assert list(idx[t]) == O.brute_force_topk(list(logits[t]), 3)


def test_tie_goes_to_lower_index():
    logits = np.array([[0.0, 1.0, 1.0, 1.0, 0.5]])
    idx, g = O.route_topk(logits, 2)
    assert list(idx[0]) == [1, 2]
    assert np.allclose(g, 0.5, atol=0, rtol=0) or np.allclose(g, 0.5)


def test_k_distinct_experts_and_gates_sum_to_one():
    rng = np.random.default_rng(12)
    logits = rng.standard_normal((200, 32)) * 3
    idx, g = O.route_topk(logits, 6)
    for t in range(200):
        assert len(set(idx[t])) == 6
    assert np.all(np.abs(g.sum(axis=1) - 1.0) <= 1e-12)
    assert np.all(g > 0)
    # gates descend with the selection order (softmax is monotone)
    assert np.all(np.diff(g, axis=1) <= 1e-15)


def test_renormalised_gates_equal_softmax_over_selected():
    rng = np.random.default_rng(13)
    logits = rng.standard_normal((50, 16)) * 4
    idx, g = O.route_topk(logits, 4)
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    ref = np.exp(sel - sel.max(axis=1, keepdims=True))
    ref /= ref.sum(axis=1, keepdims=True)
    assert np.max(np.abs(g - ref)) <= 1e-15


def test_k_equals_one_gate_is_one():
    rng = np.random.default_rng(14)
    logits = rng.standard_normal((30, 8))
    idx, g = O.route_topk(logits, 1)
    assert np.array_equal(idx[:, 0], np.argmax(logits, axis=1))
    assert np.all(g == 1.0)


def test_router_bias_shifts_selection():
    logits = np.zeros((1, 4))
    x = np.ones((1, 2))
    w = np.zeros((4, 2))
    b = np.array([0.0, 0.0, 3.0, 1.0])
    lg = O.router_logits(x, w, b)
    assert np.array_equal(lg, logits + b)
    idx, _ = O.route_topk(lg, 2)
    assert list(idx[0]) == [2, 3]


def test_near_tie_detection():
    logits = np.array([[3.0, 2.0, 2.0 - 1e-6, 0.0],      # K-th vs (K+1)-th: set ambiguous
                       [3.0, 2.0, 1.0, 0.0],             # clear
                       [3.0, 3.0 - 1e-6, 1.0, 0.0],      # order of the two chosen ambiguous
                       [3.0, 2.0, 1.0, 1.0 - 1e-7]])     # tie below the (K+1)-th: irrelevant
    flags = O.near_tie_tokens(logits, 2)
    assert list(flags) == [True, False, True, False]
    assert O.near_tie_tokens(np.array([[1.0, 1.0]]), 2)[0]    # K = N: only the order can tie
    assert O.near_tie_tokens(np.array([[1.0, 1.0 - 1e-9]]), 1)[0]


def _naive_permute(idx, N):
    T, K = idx.shape
    rows = []
    for e in range(N):
        for t in range(T):
            for k in range(K):
                if idx[t, k] == e:
                    rows.append(t * K + k)
    counts = [sum(1 for v in idx.reshape(-1) if v == e) for e in range(N)]
    return counts, rows


@pytest.mark.parametrize("T,N,K", [(1, 4, 2), (7, 5, 3), (33, 16, 4), (64, 32, 4)])
def test_permute_matches_naive_loop(T, N, K):
    rng = np.random.default_rng(T + N + K)
    idx = np.stack([rng.permutation(N)[:K] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm_src, inv_perm = O.permute(idx, N)
    c_ref, rows_ref = _naive_permute(idx, N)
    assert list(counts) == c_ref
    assert list(perm_src) == rows_ref
    assert offsets[0] == 0 and offsets[-1] == T * K
    assert np.all(np.diff(offsets) == counts)
    assert np.array_equal(inv_perm[perm_src], np.arange(T * K))
    assert np.array_equal(perm_src[inv_perm], np.arange(T * K))
    flat = idx.reshape(-1)
    for e in range(N):
        assert np.all(flat[perm_src[offsets[e]:offsets[e + 1]]] == e)


def test_permute_all_tokens_to_one_expert_and_empty_experts():
    idx = np.zeros((10, 1), dtype=np.int32) + 3
    counts, offsets, perm_src, inv_perm = O.permute(idx, 8)
    assert list(counts) == [0, 0, 0, 10, 0, 0, 0, 0]
    assert list(offsets) == [0, 0, 0, 0, 10, 10, 10, 10, 10]
    assert list(perm_src) == list(range(10))


def test_brute_force_enumerator_itself_on_known_case():
    # hand-checked: the two largest are 5 (idx 3) and the tied 4s at idx 0, 2 -> idx 0
    assert O.brute_force_topk([4.0, 1.0, 4.0, 5.0], 2) == [3, 0]
    assert O.brute_force_topk([1.0, 1.0, 1.0], 3) == [0, 1, 2]
    assert len(list(itertools.combinations(range(5), 2))) == 10
