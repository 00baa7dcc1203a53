"""Pins for the oracle's expert backward pass (oracle.swiglu_expert_backward):
central finite differences of the forward oracle, and special cases."""
import numpy as np
import pytest

import oracle


def _case(M, d, f, seed):
    rng = np.random.default_rng(seed)
    a = rng.normal(size=(M, d))
    w1, w3 = rng.normal(size=(f, d)) / np.sqrt(d), rng.normal(size=(f, d)) / np.sqrt(d)
    w2 = rng.normal(size=(d, f)) / np.sqrt(f)
    dy = rng.normal(size=(M, d))
    return a, w1, w3, w2, dy


def _loss(a, w1, w3, w2, dy):
    return float(np.sum(dy * oracle.swiglu_expert(a, w1, w3, w2)))


@pytest.mark.parametrize("M,d,f", [(3, 5, 4), (2, 8, 6)])
def test_gradients_match_central_differences(M, d, f):
    """Every entry of da, dW1, dW3 and dW2 against (L(p+e) - L(p-e)) / 2e of
    L = sum(dy * y), y from the forward oracle."""
    a, w1, w3, w2, dy = _case(M, d, f, M * 10 + d)
    r = oracle.swiglu_expert_backward(a, w1, w3, w2, dy)
    eps = 1e-6
    args = [a, w1, w3, w2]
    for which, key in enumerate(["da", "dw1", "dw3", "dw2"]):
        num = np.zeros_like(args[which])
        for ix in np.ndindex(*args[which].shape):
            p, m = [x.copy() for x in args], [x.copy() for x in args]
            p[which][ix] += eps
            m[which][ix] -= eps
            num[ix] = (_loss(*p, dy) - _loss(*m, dy)) / (2 * eps)
        np.testing.assert_allclose(r[key], num, rtol=1e-6, atol=1e-8, err_msg=key)


def test_zero_upstream_gradient_gives_zero():
    a, w1, w3, w2, dy = _case(4, 6, 5, 3)
    r = oracle.swiglu_expert_backward(a, w1, w3, w2, np.zeros_like(dy))
    for k in ("da", "dw1", "dw3", "dw2"):
        assert np.all(r[k] == 0.0)


def test_zero_up_projection_kills_the_gate_path():
    """W3 = 0: u = 0 and h = 0, so dg = 0, dW1 = 0, dW2 = 0; only the up path
    carries gradient: da = du W3 = 0 as well, while dW3 = du^T a is not zero."""
    a, w1, w3, w2, dy = _case(4, 6, 5, 4)
    r = oracle.swiglu_expert_backward(a, w1, np.zeros_like(w3), w2, dy)
    assert np.all(r["dg"] == 0) and np.all(r["dw1"] == 0) and np.all(r["dw2"] == 0)
    assert np.all(r["da"] == 0) and np.any(r["dw3"] != 0)


def test_rows_are_independent():
    """The input gradient of each row depends only on that row."""
    a, w1, w3, w2, dy = _case(5, 6, 4, 5)
    full = oracle.swiglu_expert_backward(a, w1, w3, w2, dy)["da"]
    for t in range(5):
        one = oracle.swiglu_expert_backward(a[t:t + 1], w1, w3, w2, dy[t:t + 1])["da"]
        np.testing.assert_allclose(one[0], full[t], rtol=1e-14, atol=1e-15)


def test_rounding_options_round_the_stated_values():
    a, w1, w3, w2, dy = _case(3, 8, 6, 6)
    r = oracle.swiglu_expert_backward(a, w1, w3, w2, dy, gu_round="bf16", dgu_round="bf16")
    for k in ("dg", "du"):
        np.testing.assert_array_equal(r[k], oracle.round_bf16(r[k]))
