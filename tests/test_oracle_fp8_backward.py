"""Pins for oracle.fp8_swiglu_expert_backward_dx, the FP8 input gradient of
one expert (E4M3 forward operands, E5M2 gradients).

With the quantisation switched off the same steps must give the exact
backward (pinned separately by finite differences), which checks the wiring:
which weight, which transpose, which rounding of g and u.  With it switched
on, the result must stay within the precision of the two formats, keep rows
independent (every scale belongs to one row), and map a zero gradient to an
exactly zero one."""
import numpy as np
import pytest

import oracle


def _case(seed, M=4, d=256, f=256):
    rng = np.random.default_rng(seed)
    a = oracle.round_bf16(rng.normal(size=(M, d)))
    w1 = oracle.round_bf16(rng.normal(size=(f, d)) / np.sqrt(d))
    w3 = oracle.round_bf16(rng.normal(size=(f, d)) / np.sqrt(d))
    w2 = oracle.round_bf16(rng.normal(size=(d, f)) / np.sqrt(f))
    dy = oracle.round_bf16(rng.normal(size=(M, d)) * 1e-2)
    return a, w1, w3, w2, dy


@pytest.mark.parametrize("seed", [0, 1])
def test_without_quantisation_it_is_the_exact_backward(seed):
    a, w1, w3, w2, dy = _case(seed)
    got = oracle.fp8_swiglu_expert_backward_dx(a, w1, w3, w2, dy, quant=False)
    want = oracle.swiglu_expert_backward(a, w1, w3, w2, dy, gu_round="bf16")
    np.testing.assert_allclose(got["da"], want["da"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(got["dg"], want["dg"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(got["du"], want["du"], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("seed", [2, 3])
def test_fp8_error_stays_within_the_formats_precision(seed):
    """E5M2 keeps 2 mantissa bits (half-step 2^-3 relative), E4M3 3 bits
    (2^-4); summed over 256-long contractions the errors average, so the
    gradient lands within 20% in norm, but it is not exact."""
    a, w1, w3, w2, dy = _case(seed)
    got = oracle.fp8_swiglu_expert_backward_dx(a, w1, w3, w2, dy)
    exact = oracle.swiglu_expert_backward(a, w1, w3, w2, dy)
    def rel(x, y):
        return np.linalg.norm(x - y) / np.linalg.norm(y)
    assert rel(got["dh"], exact["dh"]) <= 0.1
    assert rel(got["g"], a @ w1.T) <= 0.06
    assert 1e-3 <= rel(got["da"], exact["da"]) <= 0.2


def test_rows_are_independent():
    a, w1, w3, w2, dy = _case(4, M=6)
    whole = oracle.fp8_swiglu_expert_backward_dx(a, w1, w3, w2, dy)["da"]
    for r in range(6):
        one = oracle.fp8_swiglu_expert_backward_dx(a[r:r + 1], w1, w3, w2, dy[r:r + 1])["da"]
        np.testing.assert_array_equal(one[0], whole[r])


def test_zero_gradient_gives_exact_zero():
    a, w1, w3, w2, dy = _case(5)
    got = oracle.fp8_swiglu_expert_backward_dx(a, w1, w3, w2, np.zeros_like(dy))
    assert np.all(got["dh"] == 0.0) and np.all(got["da"] == 0.0)


def test_gradient_scale_invariance():
    """Scaling dy by a power of two scales every E5M2 tile scale by the same
    power and leaves the codes unchanged, so dh and da scale exactly."""
    a, w1, w3, w2, dy = _case(6)
    base = oracle.fp8_swiglu_expert_backward_dx(a, w1, w3, w2, dy)
    big = oracle.fp8_swiglu_expert_backward_dx(a, w1, w3, w2, dy * 2.0 ** 20)
    np.testing.assert_array_equal(big["dh"], base["dh"] * 2.0 ** 20)
    np.testing.assert_array_equal(big["da"], base["da"] * 2.0 ** 20)


def test_bf16_rounding_of_dg_du_is_the_stated_rounding():
    a, w1, w3, w2, dy = _case(7)
    got = oracle.fp8_swiglu_expert_backward_dx(a, w1, w3, w2, dy, quant=False, dgu_round="bf16")
    want = oracle.swiglu_expert_backward(a, w1, w3, w2, dy, gu_round="bf16", dgu_round="bf16")
    np.testing.assert_allclose(got["da"], want["da"], rtol=1e-12, atol=1e-15)
    q = oracle.fp8_swiglu_expert_backward_dx(a, w1, w3, w2, dy, dgu_round="bf16")
    assert np.all(oracle.round_bf16(q["dg"]) == q["dg"]) and np.all(oracle.round_bf16(q["du"]) == q["du"])


@pytest.mark.parametrize("R", [1, 100, 300])
def test_weight_gradient_without_quantisation_is_exact(R):
    rng = np.random.default_rng(R)
    dy, h = rng.normal(size=(R, 256)), rng.normal(size=(R, 128))
    np.testing.assert_allclose(oracle.fp8_weight_grad(dy, h, quant=False), dy.T @ h, rtol=1e-13)


@pytest.mark.parametrize("R", [100, 300])
def test_weight_gradient_error_and_tiles(R):
    """Tiles run along the rows (R = 300: two full tiles and one of 44): the
    dequantised operands reproduce the product exactly in float64, the error
    against the exact product stays within the formats' precision, and
    scaling either operand by a power of two scales the result exactly."""
    rng = np.random.default_rng(R + 1)
    dy, h = rng.normal(size=(R, 256)) * 1e-3, rng.normal(size=(R, 128))
    got = oracle.fp8_weight_grad(dy, h)
    qd, sd = oracle.quant_cols_1x128(dy, "e5m2")
    qh, sh = oracle.quant_cols_1x128(h, "e4m3")
    assert sd.shape == ((R + 127) // 128, 256) and qd.shape == dy.shape
    vd = oracle.e5m2_decode(qd) * np.repeat(sd.astype(np.float64), 128, axis=0)[:R]
    vh = oracle.e4m3_decode(qh) * np.repeat(sh.astype(np.float64), 128, axis=0)[:R]
    np.testing.assert_allclose(got, vd.T @ vh, rtol=1e-12, atol=1e-15)
    exact = dy.T @ h
    assert 1e-3 <= np.linalg.norm(got - exact) / np.linalg.norm(exact) <= 0.15
    np.testing.assert_array_equal(oracle.fp8_weight_grad(dy * 2.0 ** 12, h), got * 2.0 ** 12)
    np.testing.assert_array_equal(oracle.fp8_weight_grad(dy, h * 2.0 ** -7), got * 2.0 ** -7)


def test_column_tiles_are_independent_of_other_columns():
    """Each (column, 128-row tile) has its own scale: changing one column
    changes no other column's codes or scales."""
    rng = np.random.default_rng(9)
    m = rng.normal(size=(200, 6))
    q0, s0 = oracle.quant_cols_1x128(m)
    m2 = m.copy()
    m2[:, 3] *= 1000.0
    q1, s1 = oracle.quant_cols_1x128(m2)
    keep = [0, 1, 2, 4, 5]
    np.testing.assert_array_equal(q0[:, keep], q1[:, keep])
    np.testing.assert_array_equal(s0[:, keep], s1[:, keep])
