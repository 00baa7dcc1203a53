"""Pins for the oracle's layer backward (oracle.combine_backward,
route_backward, dispatch_backward, moe_backward).

The gradients are checked against central finite differences of the
oracle's own layer forward (oracle.moe_forward, pinned separately), with the
routing held fixed: the cases are drawn with every routing margin far above
the perturbation, and each perturbed forward is checked to select the same
experts.  Closed forms cover the gate normalisation (gates sum to one, so a
uniform gate gradient moves nothing) and top-1 routing."""
import numpy as np
import pytest

import oracle

EPS = 1e-6


def _case(seed, T=6, d=8, N=8, K=2, G=4, topG=2, f=5, min_margin=1e-3):
    rng = np.random.default_rng(seed)
    for _ in range(200):
        x = rng.normal(size=(T, d))
        R = rng.normal(size=(N, d)) / np.sqrt(d)
        b = rng.uniform(-0.01, 0.01, size=N)
        if oracle.route_margins(x, R, b, G, topG, K).min() > min_margin:
            break
    else:
        raise RuntimeError("no tie-free case")
    W = {e: [rng.normal(size=(f, d)) / np.sqrt(d), rng.normal(size=(f, d)) / np.sqrt(d),
             rng.normal(size=(d, f)) / np.sqrt(f)] for e in range(N + 1)}
    ybar = rng.normal(size=(T, d))
    return dict(x=x, R=R, b=b, W=W, ybar=ybar, G=G, topG=topG, K=K, N=N)


def _loss(c, x=None, R=None, W=None, idx_ref=None):
    x = c["x"] if x is None else x
    R = c["R"] if R is None else R
    W = c["W"] if W is None else W
    out = oracle.moe_forward(x, R, c["b"], lambda e: W[e], c["G"], c["topG"], c["K"])
    if idx_ref is not None:
        assert np.array_equal(out["route"]["idx"], idx_ref), "perturbation changed the routing"
    return float(np.sum(c["ybar"] * out["y"]))


def _backward(c):
    return oracle.moe_backward(c["x"], c["R"], c["b"], lambda e: c["W"][e], c["G"], c["topG"],
                               c["K"], c["ybar"])


@pytest.mark.parametrize("seed", [0, 1])
def test_dx_matches_finite_differences(seed):
    c = _case(seed)
    g = _backward(c)
    idx = g["route"]["idx"]
    num = np.empty_like(c["x"])
    for i in np.ndindex(*c["x"].shape):
        xp, xm = c["x"].copy(), c["x"].copy()
        xp[i] += EPS
        xm[i] -= EPS
        num[i] = (_loss(c, x=xp, idx_ref=idx) - _loss(c, x=xm, idx_ref=idx)) / (2 * EPS)
    np.testing.assert_allclose(g["dx"], num, rtol=1e-6, atol=1e-8)


def test_drouter_matches_finite_differences():
    c = _case(2)
    g = _backward(c)
    idx = g["route"]["idx"]
    num = np.empty_like(c["R"])
    for i in np.ndindex(*c["R"].shape):
        Rp, Rm = c["R"].copy(), c["R"].copy()
        Rp[i] += EPS
        Rm[i] -= EPS
        num[i] = (_loss(c, R=Rp, idx_ref=idx) - _loss(c, R=Rm, idx_ref=idx)) / (2 * EPS)
    np.testing.assert_allclose(g["drouter"], num, rtol=1e-6, atol=1e-8)
    # only experts some token selected receive a router gradient
    used = np.zeros(c["N"], dtype=bool)
    used[np.unique(idx)] = True
    assert np.all(g["drouter"][~used] == 0.0)


def test_expert_weight_gradients_match_finite_differences():
    c = _case(3, T=5, N=8, K=2)
    g = _backward(c)
    idx = g["route"]["idx"]
    rng = np.random.default_rng(9)
    for e in range(c["N"] + 1):
        for w in range(3):
            for _ in range(3):
                i = tuple(rng.integers(0, n) for n in c["W"][e][w].shape)
                Wp = {k: [m.copy() for m in v] for k, v in c["W"].items()}
                Wm = {k: [m.copy() for m in v] for k, v in c["W"].items()}
                Wp[e][w][i] += EPS
                Wm[e][w][i] -= EPS
                num = (_loss(c, W=Wp, idx_ref=idx) - _loss(c, W=Wm, idx_ref=idx)) / (2 * EPS)
                assert g["dw"][e][w][i] == pytest.approx(num, rel=1e-6, abs=1e-8)
    counts = np.bincount(idx.ravel(), minlength=c["N"])
    for e in np.flatnonzero(counts == 0):      # an idle expert has zero gradients
        assert all(np.all(m == 0.0) for m in g["dw"][e])


def test_combine_backward_is_the_derivative_of_combine():
    """combine is linear in the gates and in the routed outputs, so central
    differences are exact up to rounding."""
    rng = np.random.default_rng(4)
    T, K, N, d = 5, 3, 6, 7
    idx = np.sort(np.stack([rng.choice(N, K, replace=False) for _ in range(T)]), axis=1)
    slot = oracle.dispatch(idx, N)["slot"]
    gate = rng.uniform(0.1, 1.0, size=(T, K))
    y_perm = rng.normal(size=(T * K, d))
    shared = rng.normal(size=(T, d))
    dy = rng.normal(size=(T, d))

    def L(gt, yp):
        routed = {(t, int(idx[t, k])): yp[slot[t, k]] for t in range(T) for k in range(K)}
        return float(np.sum(dy * oracle.combine(shared, routed, idx, gt, np.arange(T))))

    cb = oracle.combine_backward(dy, y_perm, slot, gate)
    for t in range(T):
        for k in range(K):
            gp, gm = gate.copy(), gate.copy()
            gp[t, k] += 0.5
            gm[t, k] -= 0.5
            assert cb["dgate"][t, k] == pytest.approx(L(gp, y_perm) - L(gm, y_perm), rel=1e-12)
    for r in range(T * K):
        for j in range(d):
            yp, ym = y_perm.copy(), y_perm.copy()
            yp[r, j] += 0.5
            ym[r, j] -= 0.5
            assert cb["dy_perm"][r, j] == pytest.approx(L(gate, yp) - L(gate, ym), rel=1e-12,
                                                         abs=1e-14)


def test_uniform_gate_gradient_moves_nothing():
    """The gates always sum to one, so dgate = c * ones has no effect on the
    logits, the input or the router."""
    c = _case(5)
    idx = oracle.route(c["x"], c["R"], c["b"], c["G"], c["topG"], c["K"])["idx"]
    rb = oracle.route_backward(c["x"], c["R"], idx, np.full(idx.shape, 3.7))
    assert np.abs(rb["dz"]).max() < 1e-15
    assert np.abs(rb["dx"]).max() < 1e-14
    assert np.abs(rb["drouter"]).max() < 1e-14


def test_top1_routing_has_no_gate_gradient():
    """K = 1: the gate is s/s = 1 whatever the logit."""
    rng = np.random.default_rng(6)
    x, R = rng.normal(size=(9, 5)), rng.normal(size=(4, 5))
    idx = rng.integers(0, 4, size=(9, 1))
    rb = oracle.route_backward(x, R, idx, rng.normal(size=(9, 1)))
    np.testing.assert_array_equal(rb["gate"], 1.0)
    assert np.abs(rb["dz"]).max() < 1e-15


def test_route_backward_gates_match_the_forward():
    c = _case(7)
    r = oracle.route(c["x"], c["R"], c["b"], c["G"], c["topG"], c["K"])
    rb = oracle.route_backward(c["x"], c["R"], r["idx"], np.zeros(r["idx"].shape))
    np.testing.assert_allclose(rb["gate"], r["gate"], rtol=1e-14)
    np.testing.assert_allclose(rb["s"], np.take_along_axis(r["s"], r["idx"], axis=1), rtol=1e-14)


def test_dispatch_backward_returns_every_copy_once():
    """Each row of dx_perm belongs to exactly one (t, k), so the column sums of
    dx equal those of dx_shared + dx_perm + dx_route; and with one-hot rows the
    token that receives each row is the one DISPATCH copied it from."""
    rng = np.random.default_rng(8)
    T, K, N, d = 7, 3, 5, 4
    idx = np.sort(np.stack([rng.choice(N, K, replace=False) for _ in range(T)]), axis=1)
    dsp = oracle.dispatch(idx, N)
    dx_perm, dx_sh, dx_rt = (rng.normal(size=(T * K, d)), rng.normal(size=(T, d)),
                             rng.normal(size=(T, d)))
    dx = oracle.dispatch_backward(dx_perm, dx_sh, dsp["slot"], dx_rt)
    np.testing.assert_allclose(dx.sum(axis=0), dx_perm.sum(axis=0) + dx_sh.sum(axis=0)
                               + dx_rt.sum(axis=0), rtol=1e-12)
    for r in range(T * K):
        onehot = np.zeros((T * K, d))
        onehot[r, 0] = 1.0
        got = oracle.dispatch_backward(onehot, np.zeros((T, d)), dsp["slot"])
        assert got[dsp["perm_tok"][r], 0] == 1.0 and got[:, 0].sum() == 1.0
