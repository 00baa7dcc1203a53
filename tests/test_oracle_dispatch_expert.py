"""Pins for the oracle's dispatch, expert FFN, combine and bias update (CPU)."""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import CONFIGS, gen


def test_dispatch_is_lexicographic_sort():
    rng = np.random.default_rng(0)
    T, N, K = 200, 16, 4
    idx = np.sort(np.stack([rng.choice(N, K, replace=False) for _ in range(T)]), axis=1)
    d = oracle.dispatch(idx, N)
    tok = np.repeat(np.arange(T), K)
    exp_ = idx.ravel()
    order = np.lexsort((tok, exp_))                   # by expert, then token
    np.testing.assert_array_equal(d["perm_tok"], tok[order])
    assert sorted(d["perm_tok"].tolist()) == sorted(tok.tolist())
    np.testing.assert_array_equal(d["offsets"], np.concatenate([[0], np.cumsum(np.bincount(exp_, minlength=N))]))
    for t in range(T):
        for k in range(K):
            r = d["slot"][t, k]
            assert d["perm_tok"][r] == t
            assert d["offsets"][idx[t, k]] <= r < d["offsets"][idx[t, k] + 1]


def _loop_expert(xrow, w1, w3, w2):
    """One SwiGLU expert written with explicit loops (tiny sizes only)."""
    f, dd = w1.shape
    h = []
    for j in range(f):
        a = sum(xrow[c] * w1[j, c] for c in range(dd))
        g = sum(xrow[c] * w3[j, c] for c in range(dd))
        h.append(a / (1.0 + math.exp(-a)) * g)
    return np.array([sum(h[j] * w2[r, j] for j in range(f)) for r in range(dd)])


def test_dense_brute_force_moe():
    """y = y_sh + sum_i G[t,i] E_i(x_t) with every expert run on every token
    and a dense gate matrix that is zero off the selection."""
    rng = np.random.default_rng(1)
    T, d, N, K, f, G, topG = 12, 10, 8, 3, 6, 4, 2
    x = rng.standard_normal((T, d))
    R = rng.standard_normal((N, d)) / math.sqrt(d)
    b = rng.uniform(-0.01, 0.01, N)
    W = [(rng.standard_normal((f, d)) / math.sqrt(d), rng.standard_normal((f, d)) / math.sqrt(d),
          rng.standard_normal((d, f)) / math.sqrt(f)) for _ in range(N + 1)]
    out = oracle.moe_forward(x, R, b, lambda e: W[e], G, topG, K)
    r = out["route"]
    Gd = np.zeros((T, N))
    for t in range(T):
        for k in range(K):
            Gd[t, r["idx"][t, k]] = r["gate"][t, k]
    for t in range(T):
        want = _loop_expert(x[t], *W[N])
        for i in range(N):
            want = want + Gd[t, i] * _loop_expert(x[t], *W[i])
        np.testing.assert_allclose(out["y"][t], want, rtol=0, atol=1e-12)


def test_silu_glu_special_case_matches_torch():
    """With W3 reading a constant-1 input coordinate, the SwiGLU expert is the
    textbook SiLU MLP y = silu(x W1^T) W2^T (torch's silu as the library routine)."""
    rng = np.random.default_rng(2)
    M, d, f = 9, 7, 5
    x = rng.standard_normal((M, d))
    x[:, -1] = 1.0
    w1 = rng.standard_normal((f, d))
    w3 = np.zeros((f, d))
    w3[:, -1] = 1.0
    w2 = rng.standard_normal((d, f))
    y = oracle.swiglu_expert(x, w1, w3, w2)
    want = torch.nn.functional.silu(torch.from_numpy(x) @ torch.from_numpy(w1).T) @ torch.from_numpy(w2).T
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-13, atol=1e-13)


def test_round_bf16_matches_torch_from_float32():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(50000) * 10.0 ** rng.integers(-30, 30, 50000),
                        [0.0, -0.0, 1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8]]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(v.astype(np.float64)), want)


def test_combine_weights_and_order():
    shared = np.array([[1.0, 2.0]])
    routed = {(0, 3): np.array([10.0, 0.0]), (0, 5): np.array([0.0, 100.0])}
    idx = np.array([[3, 5]])
    gate = np.array([[0.25, 0.75]])
    np.testing.assert_array_equal(oracle.combine(shared, routed, idx, gate, [0]), [[3.5, 77.0]])


def test_bias_update_closed_form():
    rng = np.random.default_rng(4)
    N, T, K = 64, 96, 6                                   # mean load T*K/N = 9
    b = rng.uniform(-0.01, 0.01, N).astype(np.float32)
    c = rng.integers(0, 20, N)
    c[:4] = 9                                             # exactly at the mean
    gamma = 0.001
    nb = oracle.bias_update(b, c, T, K, gamma)
    want = (b - np.float32(gamma) * np.sign(c - 9).astype(np.float32)).astype(np.float32)
    np.testing.assert_array_equal(nb, want)
    np.testing.assert_array_equal(nb[:4], b[:4])
    np.testing.assert_array_equal(oracle.bias_update(b, c, T, K, 0.0), b)
    assert nb.dtype == np.float32


def test_zipf_recipe_is_skewed():
    """The decode workload's router gives a heavy-headed expert popularity
    that follows the seeded rank order (Zipf-like), checked with the oracle."""
    cfg = CONFIGS[4]
    x, R = gen.make_x(cfg), gen.make_router(cfg)
    r = oracle.route(x, R, np.zeros(cfg.N), cfg.G, cfg.topG, cfg.K)
    _, rank, _ = gen.zipf_shift(cfg, 0)
    c = r["counts"]
    by_rank = c[np.argsort(rank)]
    assert by_rank[:2].min() > 0.8 * cfg.T                # the head is picked by most tokens
    assert c.max() / c.mean() > 8                          # far from uniform
    assert np.corrcoef(np.log1p(by_rank), -np.log(np.arange(1, cfg.N + 1)))[0, 1] > 0.8
