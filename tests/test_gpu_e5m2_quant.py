"""1x128 E5M2 quantisation of gradient rows (moe_quantize_rows_e5m2) against
oracle.quant_rows_1x128_e5m2: codes and scales bit-exact.

Both sides take the same fp32 steps (amax, scale = amax/57344 and inverse
57344/amax by IEEE division, v * inverse, round to nearest even with
saturation), so every integer code and every scale must agree.  The rows mix
magnitudes from 1e-8 to 1e4 and include an all-zero tile."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols", [(1, 128), (300, 256), (2048, 7168)])
def test_e5m2_gradient_quantisation_is_bit_exact(rows, cols):
    import torch
    import sparse_moe_layer_limited_b200 as M
    rng = np.random.default_rng(rows + cols)
    g = rng.normal(size=(rows, cols)) * 10.0 ** rng.uniform(-8, 4, size=(rows, 1))
    g[0, :128] = 0.0
    g = oracle.round_bf16(g).astype(np.float32)          # the stored bf16 values
    sc_ld = (rows + 3) // 4 * 4
    gd = torch.from_numpy(g).to(torch.bfloat16).cuda()
    codes = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    scales = torch.full((cols // 128, sc_ld), -1.0, dtype=torch.float32, device="cuda")
    M.moe_quantize_rows_e5m2(gd, codes, scales)
    torch.cuda.synchronize()
    want_codes, want_scales = oracle.quant_rows_1x128_e5m2(g)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_codes)
    got_scales = scales.cpu().numpy()
    np.testing.assert_array_equal(got_scales[:, :rows].T, want_scales)
    assert np.all(got_scales[:, rows:] == -1.0)           # the padding is not written
