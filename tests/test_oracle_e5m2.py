"""Pins for the oracle's E5M2 codec and gradient quantiser (oracle.e5m2_*,
oracle.quant_rows_1x128_e5m2): the OCP E5M2 definition written out
independently, every one of the 256 codes, torch's float8_e5m2 conversion
on in-range values, and the error bound of 1x128 scaling."""
import numpy as np
import pytest
import torch

import oracle


def _definition(code):
    """E5M2 value of one code from the format definition, field by field."""
    s, e, m = code >> 7, (code >> 2) & 31, code & 3
    if e == 31:
        return (-1) ** s * (float("inf") if m == 0 else float("nan"))
    if e == 0:
        return (-1) ** s * (m / 4) * 2.0 ** -14
    return (-1) ** s * (1 + m / 4) * 2.0 ** (e - 15)


def test_exhaustive_code_table():
    vals = oracle.e5m2_all_values()
    for c in range(256):
        want = _definition(c)
        if np.isnan(want):
            assert np.isnan(vals[c])
        else:
            assert vals[c] == want, c
    fin = np.isfinite(vals)
    assert fin.sum() == 256 - 8                       # 2 infinities, 6 NaNs
    assert vals[fin].max() == 57344.0 and vals[0x01] == 2.0 ** -16 and vals[0x04] == 2.0 ** -14
    # every finite code round-trips (signed zero included)
    codes = np.arange(256, dtype=np.uint8)[fin]
    np.testing.assert_array_equal(oracle.e5m2_encode(vals[fin]), codes)


def test_midpoints_round_to_even_and_saturate():
    vals = oracle.e5m2_all_values()[:124]             # 0 .. 57344 increasing
    mids = (vals[:-1] + vals[1:]) / 2
    got = oracle.e5m2_encode(mids)
    lo = np.arange(123)
    want = np.where(lo % 2 == 0, lo, lo + 1)          # the code with an even mantissa
    np.testing.assert_array_equal(got, want.astype(np.uint8))
    # just off a midpoint goes to the nearer code
    np.testing.assert_array_equal(oracle.e5m2_encode(np.nextafter(mids, 0)), lo.astype(np.uint8))
    np.testing.assert_array_equal(oracle.e5m2_encode(np.nextafter(mids, np.inf)),
                                  (lo + 1).astype(np.uint8))
    big = np.array([57344.0, 61439.0, 61440.0, 1e9, np.inf, -np.inf])
    np.testing.assert_array_equal(oracle.e5m2_encode(big),
                                  np.array([0x7B] * 5 + [0xFB], dtype=np.uint8))
    assert oracle.e5m2_encode(np.nan) == 0x7F


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.normal(size=20000) * 10.0 ** rng.uniform(-6, 4, size=20000),
                        oracle.e5m2_all_values()[:124]]).astype(np.float32)
    v = v[np.abs(v) <= 57344.0]
    ours = oracle.e5m2_decode(oracle.e5m2_encode(v))
    theirs = torch.from_numpy(v).to(torch.float8_e5m2).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, theirs)


def test_e5m2_differs_from_e4m3_where_the_formats_differ():
    """Wider range, coarser steps: 1.125 is exact in E4M3 and a tie in E5M2;
    1000 overflows E4M3 (saturates at 448) but not E5M2."""
    assert oracle.e4m3_decode(oracle.e4m3_encode(1.125)) == 1.125
    assert oracle.e5m2_decode(oracle.e5m2_encode(1.125)) == 1.0
    assert oracle.e4m3_decode(oracle.e4m3_encode(1000.0)) == 448.0
    assert oracle.e5m2_decode(oracle.e5m2_encode(1000.0)) == 1024.0


@pytest.mark.parametrize("scale_exp", [-20, 0, 12])
def test_gradient_quantisation_error_bound(scale_exp):
    """Each 1x128 tile: scale = amax/57344, the tile's max-abs element maps to
    the top code, and every dequantised element is within half a step of its
    value: |q s - g| <= 2^-3 |g| for normal codes, <= 2^-17 s below them."""
    rng = np.random.default_rng(scale_exp + 100)
    g = (rng.normal(size=(6, 256)) * 2.0 ** scale_exp).astype(np.float32)
    g[2, :128] = 0.0                                  # an all-zero tile
    codes, scales = oracle.quant_rows_1x128_e5m2(g)
    assert codes.shape == g.shape and scales.shape == (6, 2)
    assert scales[2, 0] == 1.0 and np.all(codes[2, :128] == 0)
    deq = oracle.e5m2_decode(codes) * np.repeat(scales.astype(np.float64), 128, axis=1)
    g64 = g.astype(np.float64)
    s64 = np.repeat(scales.astype(np.float64), 128, axis=1)
    bound = np.maximum(2.0 ** -3 * np.abs(g64), 2.0 ** -17 * s64) * (1 + 1e-6)
    assert np.all(np.abs(deq - g64) <= bound)
    for r in range(6):
        for t in range(2):
            tile = g64[r, 128 * t:128 * (t + 1)]
            if np.abs(tile).max() == 0:
                continue
            assert scales[r, t] == np.float32(np.float32(np.abs(tile).max()) / np.float32(57344))
            top = codes[r, 128 * t + int(np.argmax(np.abs(tile)))]
            assert abs(oracle.e5m2_decode(top)) == 57344.0


def test_mixed_format_block_gemm_equals_the_dequantised_product():
    """An E5M2 gradient operand (1x128 scales) against E4M3 weights (128x128
    blocks): the block-scaled product equals the plain matmul of the two
    dequantised matrices, and naming the wrong format changes it."""
    rng = np.random.default_rng(21)
    dy = rng.normal(size=(5, 256)) * 1e-3
    w = rng.normal(size=(256, 256)) / 16
    qa, sa = oracle.quant_rows_1x128_e5m2(dy)
    qb, sb = oracle.quant_blocks_128(w)
    got = oracle.fp8_gemm_ref(qa, sa, qb, sb, a_format="e5m2", b_format="e4m3")
    a = oracle.e5m2_decode(qa) * np.repeat(sa.astype(np.float64), 128, axis=1)
    b = oracle.e4m3_decode(qb) * np.kron(sb.astype(np.float64), np.ones((128, 128)))
    np.testing.assert_allclose(got, a @ b.T, rtol=1e-12, atol=1e-18)
    assert not np.allclose(oracle.fp8_gemm_ref(qa, sa, qb, sb), got)
    # and it stays within the E5M2/E4M3 rounding of the exact product
    assert np.linalg.norm(got - dy @ w.T) <= 0.15 * np.linalg.norm(dy @ w.T)
