"""Pins for the oracle's E4M3 codec and block quantisation (CPU)."""
import numpy as np
import pytest
import torch

import oracle


def test_exhaustive_code_table():
    v = oracle.e4m3_all_values()
    assert v[0x00] == 0.0 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x08] == 2.0 ** -6 and v[0x38] == 1.0 and v[0x7E] == 448.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.isnan(v).sum() == 2
    np.testing.assert_array_equal(v[0x80:0xFF], -v[0x00:0x7F])
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)
    # every finite code round-trips
    fin = np.isfinite(v)
    np.testing.assert_array_equal(oracle.e4m3_encode(v[fin]), np.arange(256)[fin])
    # the library routine agrees on every finite value
    t = torch.from_numpy(v[fin]).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(t, v[fin])


def test_midpoints_round_to_even_and_saturate():
    pos = oracle.e4m3_all_values()[:0x7F]
    mids = 0.5 * (pos[:-1] + pos[1:])
    codes = oracle.e4m3_encode(mids)
    lo = np.arange(0x7E)
    want = np.where(lo % 2 == 0, lo, lo + 1)              # even mantissa wins
    np.testing.assert_array_equal(codes, want)
    assert oracle.e4m3_encode(np.array([449.0, 1e9, -1e30]))[0] == 0x7E
    assert oracle.e4m3_encode(np.array([-1e30]))[0] == 0xFE
    assert oracle.e4m3_encode(np.array([np.nan]))[0] == 0x7F
    assert not np.isnan(oracle.e4m3_decode(oracle.e4m3_encode(np.array([1e30, -1e30])))).any()


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * 10.0 ** rng.uniform(-3, 2.5, 200000)).astype(np.float32)
    x = x[np.abs(x) < 448]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(x), want)


def test_quant_rows_scale_and_error_bound():
    rng = np.random.default_rng(1)
    a = rng.standard_normal((5, 384)).astype(np.float32)
    a[2, 128:256] = 0.0
    codes, sc = oracle.quant_rows_1x128(a)
    assert sc.shape == (5, 3) and sc.dtype == np.float32
    assert sc[2, 1] == 1.0 and np.all(codes[2, 128:256] == 0)
    deq = oracle.e4m3_decode(codes) * np.repeat(sc.astype(np.float64), 128, axis=1)
    for m in range(5):
        for kb in range(3):
            tile = a[m, kb * 128:(kb + 1) * 128].astype(np.float64)
            amax = np.abs(tile).max()
            if amax == 0:
                continue
            assert sc[m, kb] == np.float32(np.float32(amax) / np.float32(448))
            # the max-abs element lands on (or next to) the top code
            assert np.abs(oracle.e4m3_decode(codes[m, kb * 128:(kb + 1) * 128])).max() >= 416
            err = np.abs(deq[m, kb * 128:(kb + 1) * 128] - tile)
            # relative half-ulp bound of a 3-bit mantissa, plus the subnormal floor
            assert np.all(err <= np.abs(tile) * 2.0 ** -4 * 1.0001 + sc[m, kb] * 2.0 ** -10 + 1e-30)


def test_block_quant_layout():
    rng = np.random.default_rng(2)
    w = rng.standard_normal((256, 384)).astype(np.float32)
    w[128:, 256:] *= 100.0
    codes, sc = oracle.quant_blocks_128(w)
    assert sc.shape == (2, 3)
    for i in range(2):
        for j in range(3):
            blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            # one 128x128 block is quantised as a single tile with its own scale
            amax = np.float32(np.abs(blk).max())
            assert sc[i, j] == amax / np.float32(448)
            inv = np.float32(448) / amax
            np.testing.assert_array_equal(codes[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128],
                                          oracle.e4m3_encode((blk * inv).astype(np.float32)))


def test_fp8_gemm_equals_dequantised_matmul():
    rng = np.random.default_rng(3)
    a = rng.standard_normal((7, 256)).astype(np.float32)
    w = rng.standard_normal((256, 256)).astype(np.float32)
    qa, sa = oracle.quant_rows_1x128(a)
    qb, sb = oracle.quant_blocks_128(w)
    A = oracle.e4m3_decode(qa) * np.repeat(sa.astype(np.float64), 128, axis=1)
    B = oracle.e4m3_decode(qb) * np.kron(sb.astype(np.float64), np.ones((128, 128)))
    np.testing.assert_allclose(oracle.fp8_gemm_ref(qa, sa, qb, sb), A @ B.T, rtol=1e-12, atol=1e-12)
    # and it stays close to the unquantised product (E4M3 relative error ~2^-4 per factor)
    rel = np.linalg.norm(A @ B.T - a.astype(np.float64) @ w.T.astype(np.float64)) / np.linalg.norm(a @ w.T)
    assert rel < 0.05
