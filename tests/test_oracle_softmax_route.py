"""Pins for the oracle's softmax baseline router and balance statistic
(oracle.route_softmax, oracle.balance_loss), checked against brute force,
a library softmax and closed forms rather than against themselves."""
import itertools

import numpy as np
import pytest
from scipy.special import softmax

import oracle


def _case(T, d, N, seed):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(T, d)), rng.normal(size=(N, d)) / np.sqrt(d)


@pytest.mark.parametrize("T,d,N,K", [(40, 16, 6, 2), (25, 8, 5, 3), (30, 12, 7, 1)])
def test_selection_is_best_subset_by_brute_force(T, d, N, K):
    """The selected experts are the K-subset with the largest total softmax
    probability, found by enumerating every subset."""
    x, R = _case(T, d, N, T + N)
    r = oracle.route_softmax(x, R, K)
    p = softmax(x @ R.T, axis=1)
    for t in range(T):
        best = max(itertools.combinations(range(N), K), key=lambda c: p[t, list(c)].sum())
        assert tuple(r["idx"][t]) == tuple(sorted(best))


def test_probabilities_match_library_softmax():
    x, R = _case(50, 32, 16, 3)
    r = oracle.route_softmax(x, R, 4)
    np.testing.assert_allclose(r["p"], softmax(x @ R.T, axis=1), rtol=1e-13, atol=0)
    np.testing.assert_allclose(r["prob_sum"], softmax(x @ R.T, axis=1).sum(axis=0), rtol=1e-12)
    assert r["counts"].sum() == 50 * 4


def test_gates_are_the_softmax_over_the_selected_logits():
    """gate_k = exp(z_k) / sum over the selected exp(z_j): the library softmax
    of the K selected logits alone."""
    x, R = _case(30, 20, 10, 5)
    r = oracle.route_softmax(x, R, 3)
    z = x @ R.T
    for t in range(30):
        np.testing.assert_allclose(r["gate"][t], softmax(z[t, r["idx"][t]]), rtol=1e-13)


def test_all_experts_selected_gives_the_probabilities():
    """K = N: every expert is chosen and the gates are the probabilities."""
    x, R = _case(20, 8, 5, 7)
    r = oracle.route_softmax(x, R, 5)
    assert np.all(r["idx"] == np.arange(5))
    np.testing.assert_allclose(r["gate"], softmax(x @ R.T, axis=1), rtol=1e-13)
    assert np.all(r["counts"] == 20)


def test_balance_loss_closed_forms():
    N, K, T = 8, 2, 64
    # uniform loads and uniform probabilities: L = 1
    counts = np.full(N, K * T // N)
    assert oracle.balance_loss(counts, np.full(N, T / N), T, K) == pytest.approx(1.0)
    # every token picks experts 0 and 1 with all probability on them: f = P = 1/2 there
    counts = np.zeros(N)
    counts[:2] = T
    prob = np.zeros(N)
    prob[:2] = T / 2
    assert oracle.balance_loss(counts, prob, T, K) == pytest.approx(N / 2)


def test_identical_experts_give_uniform_probabilities():
    """Identical router rows: p = 1/N for every token; lower index wins the
    tie, so every token picks experts 0..K-1 with equal gates."""
    rng = np.random.default_rng(11)
    x = rng.normal(size=(12, 6))
    R = np.tile(rng.normal(size=(1, 6)), (5, 1))
    r = oracle.route_softmax(x, R, 2)
    np.testing.assert_allclose(r["p"], 0.2, rtol=1e-14)
    assert np.all(r["idx"] == [0, 1])
    np.testing.assert_allclose(r["gate"], 0.5, rtol=1e-14)
    assert oracle.balance_loss(r["counts"], r["prob_sum"], 12, 2) == pytest.approx(
        5 * (0.5 * 0.2 + 0.5 * 0.2))


def test_concentrated_routing_approaches_n():
    """One expert whose router row dominates every token: probabilities near
    one-hot and all loads on it, so L -> N (for K = 1)."""
    rng = np.random.default_rng(2)
    x = np.abs(rng.normal(size=(16, 4))) + 1.0
    R = rng.normal(size=(6, 4)) * 0.01
    R[3] = 50.0
    r = oracle.route_softmax(x, R, 1)
    assert np.all(r["idx"][:, 0] == 3)
    assert oracle.balance_loss(r["counts"], r["prob_sum"], 16, 1) == pytest.approx(6.0, rel=1e-6)


def test_margins_brute_force():
    x, R = _case(30, 10, 9, 13)
    m = oracle.route_softmax_margins(x, R, 4)
    z = x @ R.T
    for t in range(30):
        v = sorted(z[t], reverse=True)
        assert m[t] == pytest.approx(v[3] - v[4], rel=1e-12, abs=1e-15)
    assert np.all(np.isinf(oracle.route_softmax_margins(x, R, 9)))
