"""Pins for the oracle's routing (CPU only).

Each test checks the oracle against something other than itself: a
hand-worked fixture, brute-force enumeration, closed forms, invariants the
pages fix, and special cases that reduce to plain top-K.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from synth import CONFIGS, gen

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _hand():
    with open(os.path.join(GOLD, "route_hand.json")) as fh:
        h = json.load(fh)
    lut = {"0": 0.0, "ln3": math.log(3), "-ln3": -math.log(3), "ln9": math.log(9),
           "-ln9": -math.log(9), "ln4": math.log(4)}
    x = np.array([[lut[v] for v in row] for row in h["x_logits"]])
    return h, x, np.eye(h["N"]), np.array(h["bias"])


def test_hand_worked_fixture():
    h, x, R, b = _hand()
    r = oracle.route(x, R, b, h["G"], h["topG"], h["K"])
    assert r["idx"].tolist() == h["idx"]
    want = np.array([[n / d for n, d in row] for row in h["gate_num_den"]])
    np.testing.assert_allclose(r["gate"], want, rtol=0, atol=1e-12)
    assert r["counts"].tolist() == h["counts"]
    r1 = oracle.route(x, R, b, 1, 1, h["K"])
    assert r1["idx"].tolist() == h["idx_without_group_limit"]
    b32 = b.astype(np.float32)
    nb = oracle.bias_update(b32, r["counts"], 2, h["K"], h["gamma"])
    assert np.sign(nb.astype(np.float64) - b32).astype(int).tolist() == h["bias_direction"]


def _random_case(rng, T, d, N):
    x = rng.standard_normal((T, d))
    R = rng.standard_normal((N, d)) / math.sqrt(d)
    b = rng.uniform(-0.05, 0.05, N)
    return x, R, b


def _brute_force_route(sb, G, topG, K):
    """Enumerate group subsets (score = best pair sum) and expert subsets."""
    N = sb.size
    gs = N // G
    def gscore(g):
        m = list(range(g * gs, (g + 1) * gs))
        if len(m) == 1:
            return sb[m[0]]
        return max(sb[a] + sb[c] for a, c in itertools.combinations(m, 2))
    gsc = [gscore(g) for g in range(G)]
    best_groups = max(itertools.combinations(range(G), topG), key=lambda S: sum(gsc[g] for g in S))
    allowed = [i for g in best_groups for i in range(g * gs, (g + 1) * gs)]
    best = max(itertools.combinations(allowed, K), key=lambda S: sum(sb[i] for i in S))
    return sorted(best)


@pytest.mark.parametrize("T,d,N,G,topG,K", [(40, 16, 16, 1, 1, 4), (40, 16, 16, 4, 2, 3),
                                             (30, 8, 12, 3, 2, 4), (30, 8, 8, 8, 3, 2)])
def test_brute_force_selection(T, d, N, G, topG, K):
    rng = np.random.default_rng(T * 1000 + N * 10 + G)
    x, R, b = _random_case(rng, T, d, N)
    r = oracle.route(x, R, b, G, topG, K)
    s = 1.0 / (1.0 + np.exp(-(x @ R.T)))
    for t in range(T):
        assert r["idx"][t].tolist() == _brute_force_route(s[t] + b, G, topG, K)


def test_brute_force_tiny_config():
    cfg = CONFIGS[0]
    x = gen.make_x(cfg)
    R = gen.make_router(cfg)
    b = gen.make_bias(cfg)
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    s = 1.0 / (1.0 + np.exp(-(x.astype(np.float64) @ R.astype(np.float64).T)))
    for t in range(cfg.T):
        assert r["idx"][t].tolist() == _brute_force_route(s[t] + b, cfg.G, cfg.topG, cfg.K)


@pytest.mark.parametrize("cfg_id", [0, 1])
def test_invariants(cfg_id):
    cfg = CONFIGS[cfg_id]
    x, R, b = gen.make_x(cfg), gen.make_router(cfg), gen.make_bias(cfg)
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    idx = r["idx"]
    assert idx.shape == (cfg.T, cfg.K)
    assert np.all(np.diff(idx, axis=1) > 0)             # K distinct, ascending
    assert np.all((idx >= 0) & (idx < cfg.N))
    groups = idx // (cfg.N // cfg.G)
    assert max(len(set(g)) for g in groups.tolist()) <= cfg.topG
    assert r["counts"].sum() == cfg.T * cfg.K
    assert np.all(r["gate"] >= 0)
    np.testing.assert_allclose(r["gate"].sum(axis=1), 1.0, rtol=0, atol=1e-12)
    # chosen experts lie in the groups with the best scores
    gsc = oracle.group_scores(r["sb"], cfg.G)
    kept = oracle.kept_groups(gsc, cfg.topG)
    for t in range(0, cfg.T, 97):
        assert set(groups[t].tolist()) <= set(kept[t].tolist())


def test_bias_moves_selection_not_gates():
    cfg = CONFIGS[1]
    x, R = gen.make_x(cfg)[:512], gen.make_router(cfg)
    b = np.zeros(cfg.N)
    b_big = np.linspace(-0.3, 0.3, cfg.N)
    r0 = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    r1 = oracle.route(x, R, b_big, cfg.G, cfg.topG, cfg.K)
    changed = np.any(r0["idx"] != r1["idx"], axis=1)
    assert changed.mean() > 0.5                          # the bias moves selection
    # gates are the un-biased scores renormalised over the chosen set
    s = r0["s"]
    sel = np.take_along_axis(s, r1["idx"], axis=1)
    np.testing.assert_array_equal(r1["gate"], sel / sel.sum(axis=1, keepdims=True))
    same = ~changed
    np.testing.assert_array_equal(r0["gate"][same], r1["gate"][same])


def test_special_cases():
    rng = np.random.default_rng(7)
    x, R, b = _random_case(rng, 64, 16, 16)
    # K = N selects every expert
    r = oracle.route(x, R, b, 1, 1, 16)
    assert np.all(r["idx"] == np.arange(16))
    # topG = G is no group limit
    np.testing.assert_array_equal(oracle.route(x, R, b, 4, 4, 3)["idx"],
                                  oracle.route(x, R, b, 1, 1, 3)["idx"])
    # b = 0 and no group limit is plain top-K of the sigmoid scores (= top-K of the logits)
    r = oracle.route(x, R, np.zeros(16), 1, 1, 5)
    plain = np.sort(np.argsort(-(x @ R.T), axis=1)[:, :5], axis=1)
    np.testing.assert_array_equal(r["idx"], plain)
    # a +10 bias forces an expert into every token's selection (with its group kept)
    bb = b.copy()
    bb[5] = 10.0
    r = oracle.route(x, R, bb, 4, 2, 3)
    assert np.all(np.any(r["idx"] == 5, axis=1))


def test_margins_brute_force():
    rng = np.random.default_rng(3)
    x, R, b = _random_case(rng, 20, 8, 12)
    G, topG, K = 3, 2, 3
    m = oracle.route_margins(x, R, b, G, topG, K)
    s = 1.0 / (1.0 + np.exp(-(x @ R.T)))
    sb = s + b
    for t in range(20):
        gsc = sorted((max(sb[t][a] + sb[t][c] for a, c in itertools.combinations(range(g * 4, g * 4 + 4), 2))
                      for g in range(G)), reverse=True)
        gm = gsc[topG - 1] - gsc[topG]
        sel = _brute_force_route(sb[t], G, topG, K)
        groups = sorted({i // 4 for i in sel})
        # kept groups are the top-scoring ones; allowed experts are theirs
        kept = oracle.kept_groups(oracle.group_scores(sb[t:t + 1], G), topG)[0]
        vals = sorted((sb[t][i] for g in kept for i in range(g * 4, g * 4 + 4)), reverse=True)
        em = vals[K - 1] - vals[K]
        assert set(groups) <= set(kept.tolist())
        assert m[t] == pytest.approx(min(gm, em), abs=1e-15)
