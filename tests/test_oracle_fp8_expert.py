"""Pins for oracle.fp8_swiglu_expert, the E4M3 forward of one SwiGLU expert.

The function composes pinned parts (the E4M3 codec, the 1x128 row and
128x128 block quantisers, the block-scaled GEMM).  These pins fix the
composition itself against things it cannot agree with by accident:
  * with the quantisation off it is the exact expert ``swiglu_expert``
    (pinned by the dense brute-force MoE and by torch's SiLU);
  * with operands that quantise losslessly (every tile's max-abs is
    448 * 2^k and every value sits on the E4M3 grid times 2^k) and
    W2 = (7/8) I, the output is the dequantised hidden activation itself,
    so its values must lie on the E4M3 grid of each row's 128-wide tiles
    along f, with the scale fixed by the tile's max-abs ([P1] §4.1: 1x128
    activation tiles, online max-abs);
  * with random operands it stays within E4M3 precision of the exact
    expert, and no closer than quantisation allows;
  * every row is computed independently (each activation scale belongs to
    one row);
  * it equals the SwiGLU of the dequantised operands, with h replaced by its
    dequantised 1x128 quantisation along f."""
import numpy as np
import pytest

import oracle

E4M3_GRID = oracle.e4m3_all_values()[:0x7F]          # 0 .. 448, the non-negative codes


def _lossless(rng, rows, cols, tile_rows, tile_cols, exp2):
    """A matrix whose tiles quantise without error: values on the E4M3 grid
    (codes 0x20..0x7D, random signs), each tile's first element +-448, all
    times 2^exp2."""
    codes = rng.integers(0x20, 0x7E, size=(rows, cols))
    v = E4M3_GRID[codes] * rng.choice([-1.0, 1.0], size=(rows, cols))
    for i in range(0, rows, tile_rows):
        for j in range(0, cols, tile_cols):
            v[i, j] = 448.0 * rng.choice([-1.0, 1.0])
    return v * 2.0 ** exp2


def _random_case(seed, M=8, d=384, f=256):
    rng = np.random.default_rng(seed)
    a = oracle.round_bf16(rng.normal(size=(M, d)))
    w1 = oracle.round_bf16(rng.normal(size=(f, d)) / np.sqrt(d))
    w3 = oracle.round_bf16(rng.normal(size=(f, d)) / np.sqrt(d))
    w2 = rng.normal(size=(d, f)) / np.sqrt(f)
    # W2's 128x128 blocks at different magnitudes, so that a scale applied to
    # the wrong block shows
    mag = np.array([[1.0, 16.0], [1.0 / 16, 1.0], [4.0, 0.25]])
    w2 = oracle.round_bf16(w2 * np.kron(mag, np.ones((128, 128))))
    return a, w1, w3, w2


@pytest.mark.parametrize("seed", [0, 1])
def test_without_quantisation_it_is_the_exact_expert(seed):
    a, w1, w3, w2 = _random_case(seed)
    got = oracle.fp8_swiglu_expert(a, w1, w3, w2, quant=False)
    want = oracle.swiglu_expert(a, w1, w3, w2)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def test_lossless_operands_leave_the_1x128_quantisation_of_h_along_f():
    """a per 1x128 along d and W1, W3 per 128x128 block quantise exactly, and
    W2 = (7/8) I does too (block max 7/8 gives scale 2^-9, code 448), so the
    output is 7/8 of the dequantised h.  Each row's 128-wide tile of it must
    be E4M3 codes times that tile's scale float32(amax / 448)."""
    rng = np.random.default_rng(10)
    M, d = 6, 256
    f = d
    a = _lossless(rng, M, d, 1, 128, -8)
    w1 = _lossless(rng, f, d, 128, 128, -13)
    w3 = _lossless(rng, f, d, 128, 128, -13)
    w2 = 0.875 * np.eye(d)
    h = oracle.swiglu_expert(a, w1, w3, np.eye(d))             # the exact hidden activation
    y = oracle.fp8_swiglu_expert(a, w1, w3, w2) / 0.875
    h32 = h.astype(np.float32)
    assert np.any(y != h), "h was not quantised"
    for r in range(M):
        for j in range(f // 128):
            cols = slice(128 * j, 128 * (j + 1))
            amax = np.float32(np.abs(h32[r, cols]).max())
            s = float(np.float32(amax / np.float32(448.0)))
            q = y[r, cols] / s
            # on the E4M3 grid of this row's tile
            assert np.all(np.isin(np.abs(q), E4M3_GRID)), (r, j)
            # the tile's largest element lands on (or next to) the top code
            assert np.abs(q).max() >= 416.0
            # within half a step of h (3 mantissa bits, plus the subnormal floor)
            err = np.abs(y[r, cols] - h[r, cols])
            assert np.all(err <= np.abs(h[r, cols]) * 2.0 ** -4 * 1.0001 + s * 2.0 ** -10)


@pytest.mark.parametrize("seed", [2, 3])
def test_error_stays_within_e4m3_precision(seed):
    """Four E4M3 quantisations in a chain (a, W1 and W3, h, W2; 3 mantissa
    bits each, so at most 2^-4 relative per element, about 2% RMS): the
    output lands within 10% of the exact expert in norm, but is not exact."""
    a, w1, w3, w2 = _random_case(seed)
    got = oracle.fp8_swiglu_expert(a, w1, w3, w2)
    exact = oracle.swiglu_expert(a, w1, w3, w2)
    rel = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    assert 1e-3 <= rel <= 0.1, rel
    # row by row too: no row may be far off
    rel_rows = np.linalg.norm(got - exact, axis=1) / np.linalg.norm(exact, axis=1)
    assert np.all(rel_rows <= 0.15), rel_rows


def test_rows_are_independent():
    a, w1, w3, w2 = _random_case(4, M=5)
    whole = oracle.fp8_swiglu_expert(a, w1, w3, w2)
    for r in range(5):
        one = oracle.fp8_swiglu_expert(a[r:r + 1], w1, w3, w2)
        np.testing.assert_array_equal(one[0], whole[r])


def test_equals_swiglu_of_the_dequantised_operands():
    """Written out from the pinned quantisers and codec with dense float64
    matmuls (no per-slice sums): a, W1, W3, W2 dequantised, h formed from
    them, then h replaced by the dequantised 1x128 quantisation of each of
    its rows along f."""
    a, w1, w3, w2 = _random_case(5)

    def deq_rows(m):
        q, s = oracle.quant_rows_1x128(np.asarray(m, np.float32))
        return oracle.e4m3_decode(q) * np.repeat(s.astype(np.float64), 128, axis=1)

    def deq_blocks(w):
        q, s = oracle.quant_blocks_128(np.asarray(w, np.float32))
        return oracle.e4m3_decode(q) * np.kron(s.astype(np.float64), np.ones((128, 128)))

    A, W1, W3, W2 = deq_rows(a), deq_blocks(w1), deq_blocks(w3), deq_blocks(w2)
    g, u = A @ W1.T, A @ W3.T
    h = g / (1.0 + np.exp(-g)) * u
    want = deq_rows(h.astype(np.float32)) @ W2.T
    np.testing.assert_allclose(oracle.fp8_swiglu_expert(a, w1, w3, w2), want,
                               rtol=1e-10, atol=1e-12 * np.abs(want).max())
