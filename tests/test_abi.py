"""The C ABI without a GPU: the library loads, exports every declared
symbol, and rejects bad shapes and pointers before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def L():
    from sparse_moe_layer_limited_b200 import build
    if not os.path.exists(build.LIB_PATH):
        build.build()
    from sparse_moe_layer_limited_b200 import _lib
    return _lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_bias_update",
              "moe_workspace_size", "moe_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    raw = ctypes.CDLL(L.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), name
    assert set(declared_functions()) <= set(L._SIGS), "binding misses a declared entry point"


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5, 7):
        assert isinstance(L.status_string(code), str) and L.status_string(code)


def test_shape_checks(L):
    from synth import CONFIGS
    from tests.support import moe_shape
    for cfg in CONFIGS.values():
        s = moe_shape(cfg)
        assert L.check_shape(s) == L.OK, cfg.name
        assert L.workspace_size(s) > 0
    ok = L.shape(128, 64, 16, 4, 1, 1, 32, L.DTYPE_FP32)
    assert L.check_shape(ok) == L.OK
    bad = [
        (L.shape(0, 64, 16, 4, 1, 1, 32, 0), L.ERR_ARG),        # T = 0
        (L.shape(128, 64, 16, 4, 3, 1, 32, 0), L.ERR_UNSUPPORTED),  # G does not divide N
        (L.shape(128, 64, 16, 4, 4, 5, 32, 0), L.ERR_UNSUPPORTED),  # topG > G
        (L.shape(128, 64, 16, 17, 1, 1, 32, 0), L.ERR_UNSUPPORTED),  # K > N
        (L.shape(128, 64, 16, 5, 4, 1, 32, 0), L.ERR_UNSUPPORTED),  # K > topG * N/G
        (L.shape(128, 64, 512, 4, 1, 1, 32, 0), L.ERR_UNSUPPORTED),  # N > 256
        (L.shape(128, 100, 16, 4, 1, 1, 32, 0), L.ERR_UNSUPPORTED),  # d % 32
        (L.shape(128, 128, 16, 4, 1, 1, 256, 1), L.ERR_UNSUPPORTED),  # bf16 needs d % 256
        (L.shape(128, 256, 16, 4, 1, 1, 200, 1), L.ERR_UNSUPPORTED),  # bf16 needs f % 128
        (L.shape(128, 256, 16, 4, 1, 1, 256, 9), L.ERR_UNSUPPORTED),  # dtype
    ]
    for s, want in bad:
        assert L.check_shape(s) == want, s
        assert L.workspace_size(s) == 0


def test_null_pointers_rejected_before_any_launch(L):
    s = L.shape(128, 64, 16, 4, 1, 1, 32, L.DTYPE_FP32)
    f = L.lib()
    p = ctypes.byref(s)
    assert f.moe_route(p, None, None, None, None, None, None, None, None) == L.ERR_ARG
    assert f.moe_dispatch(p, *([None] * 10)) == L.ERR_ARG
    assert f.moe_expert_ffn(p, *([None] * 12)) == L.ERR_ARG
    assert f.moe_combine(p, *([None] * 6)) == L.ERR_ARG
    assert f.moe_bias_update(p, None, None, ctypes.c_float(0.001), None) == L.ERR_ARG
    assert f.moe_route(None, *([None] * 8)) == L.ERR_ARG
    # misaligned (not 16-byte aligned) pointers are rejected too
    mis = ctypes.c_void_p(0x1001)
    assert f.moe_combine(p, mis, mis, mis, mis, mis, None) == L.ERR_ARG


def test_workspace_layout_grows_with_shape(L):
    a = L.workspace_size(L.shape(1024, 256, 8, 2, 2, 1, 256, L.DTYPE_BF16))
    b = L.workspace_size(L.shape(2048, 256, 8, 2, 2, 1, 256, L.DTYPE_BF16))
    assert 0 < a < b
    assert a % 256 == 0


def test_backward_entry_points_reject_bad_arguments_before_any_launch(L):
    f = L.lib()
    fp32 = ctypes.byref(L.shape(128, 64, 16, 4, 1, 1, 32, L.DTYPE_FP32))
    bf16 = ctypes.byref(L.shape(128, 256, 16, 4, 1, 1, 256, L.DTYPE_BF16))
    bf16_f128 = ctypes.byref(L.shape(128, 256, 16, 4, 1, 1, 128, L.DTYPE_BF16))
    mis = ctypes.c_void_p(0x1001)
    ok = ctypes.c_void_p(0x1000)   # aligned, never dereferenced: the checks fail first
    # layer backward steps: every pointer is required (dx_route may be NULL)
    for s in (fp32, bf16):
        assert f.moe_combine_backward(s, *([None] * 7)) == L.ERR_ARG
        assert f.moe_route_backward(s, *([None] * 11)) == L.ERR_ARG
        assert f.moe_dispatch_backward(s, *([None] * 6)) == L.ERR_ARG
        assert f.moe_combine_backward(s, ok, ok, ok, ok, ok, mis, None) == L.ERR_ARG
        assert f.moe_route_backward(s, *([ok] * 9), mis, ok, None) == L.ERR_ARG
        # a misaligned optional dx_route is still rejected
        assert f.moe_dispatch_backward(s, ok, ok, ok, mis, ok, None) == L.ERR_ARG
        assert f.moe_dispatch_backward(s, ok, None, ok, None, ok, None) == L.ERR_ARG
    assert f.moe_combine_backward(None, *([ok] * 6), None) == L.ERR_ARG
    # expert backward and weight transposes: BF16 only; weight gradients need f % 256
    assert f.moe_transpose_weights(fp32, ok, ok, ok, ok, None) == L.ERR_UNSUPPORTED
    assert f.moe_expert_ffn_backward_dx(fp32, *([ok] * 11), None) == L.ERR_UNSUPPORTED
    assert f.moe_expert_ffn_backward_dw(fp32, *([ok] * 8), None) == L.ERR_UNSUPPORTED
    assert f.moe_expert_ffn_backward_dw(bf16_f128, *([ok] * 8), None) == L.ERR_UNSUPPORTED
    assert f.moe_expert_ffn_backward_dx(bf16, *([None] * 11), None) == L.ERR_ARG
    assert f.moe_expert_ffn_backward_dw(bf16, *([None] * 8), None) == L.ERR_ARG
    assert f.moe_backward_workspace_size(fp32) == 0
    assert f.moe_backward_workspace_size(bf16) > 0


def test_e5m2_quantiser_rejects_bad_sizes_before_any_launch(L):
    f = L.lib()
    ok = ctypes.c_void_p(0x1000)
    mis = ctypes.c_void_p(0x1008)
    assert f.moe_quantize_rows_e5m2(ok, 0, 128, ok, ok, 1, None) == L.ERR_ARG      # no rows
    assert f.moe_quantize_rows_e5m2(ok, 4, 200, ok, ok, 4, None) == L.ERR_ARG      # cols % 128
    assert f.moe_quantize_rows_e5m2(ok, 4, 128, ok, ok, 3, None) == L.ERR_ARG      # sc_ld < rows
    assert f.moe_quantize_rows_e5m2(None, 4, 128, ok, ok, 4, None) == L.ERR_ARG
    assert f.moe_quantize_rows_e5m2(ok, 4, 128, mis, ok, 4, None) == L.ERR_ARG


def test_fp8_backward_entry_points_reject_bad_arguments_before_any_launch(L):
    f = L.lib()
    ok = ctypes.c_void_p(0x1000)
    e4m3 = ctypes.byref(L.shape(128, 256, 16, 4, 1, 1, 256, L.DTYPE_E4M3))
    e4m3_f128 = ctypes.byref(L.shape(128, 256, 16, 4, 1, 1, 128, L.DTYPE_E4M3))
    bf16 = ctypes.byref(L.shape(128, 256, 16, 4, 1, 1, 256, L.DTYPE_BF16))
    fp32 = ctypes.byref(L.shape(128, 64, 16, 4, 1, 1, 32, L.DTYPE_FP32))
    assert f.moe_expert_ffn_backward_dx_fp8(bf16, *([ok] * 15), None) == L.ERR_UNSUPPORTED
    assert f.moe_expert_ffn_backward_dx_fp8(e4m3_f128, *([ok] * 15), None) == L.ERR_UNSUPPORTED
    assert f.moe_expert_ffn_backward_dx_fp8(e4m3, *([None] * 15), None) == L.ERR_ARG
    assert f.moe_quantize_weights_transposed(bf16, *([ok] * 6), None) == L.ERR_UNSUPPORTED
    assert f.moe_quantize_weights_transposed(e4m3, *([None] * 6), None) == L.ERR_ARG
    assert f.moe_transpose_weights(fp32, ok, ok, ok, ok, None) == L.ERR_UNSUPPORTED
    assert f.moe_transpose_weights(e4m3, None, ok, ok, ok, None) == L.ERR_ARG
    assert f.moe_backward_workspace_size(e4m3) > 0


def test_fp8_weight_gradient_entry_point_rejects_bad_arguments(L):
    f = L.lib()
    ok = ctypes.c_void_p(0x1000)
    e4m3 = ctypes.byref(L.shape(128, 256, 16, 4, 1, 1, 256, L.DTYPE_E4M3))
    bf16 = ctypes.byref(L.shape(128, 256, 16, 4, 1, 1, 256, L.DTYPE_BF16))
    assert f.moe_expert_ffn_backward_dw_fp8(bf16, *([ok] * 8), None) == L.ERR_UNSUPPORTED
    assert f.moe_expert_ffn_backward_dw_fp8(e4m3, *([None] * 8), None) == L.ERR_ARG


def test_gather_rows_rejects_bad_arguments_before_any_launch(L):
    f = L.lib().moe_gather_rows
    fake = ctypes.c_void_p(1 << 20)                        # never dereferenced
    odd = ctypes.c_void_p((1 << 20) + 8)                   # not 16-byte aligned
    assert f(fake, 10, fake, 4, 24, fake, None) == L.ERR_ARG      # row bytes not a multiple of 16
    assert f(fake, 10, fake, -1, 32, fake, None) == L.ERR_ARG     # negative count
    assert f(None, 10, fake, 4, 32, fake, None) == L.ERR_ARG
    assert f(fake, 10, None, 4, 32, fake, None) == L.ERR_ARG
    assert f(odd, 10, fake, 4, 32, fake, None) == L.ERR_ARG
    assert f(fake, 10, fake, 0, 32, fake, None) == L.OK          # nothing to do


def test_gemm_clock_reader_rejects_null(L):
    import ctypes as C
    c = (C.c_uint64 * 4)()
    assert L.lib().moe_read_gemm_clock(None, None, c, 0) == L.ERR_ARG
    assert L.lib().moe_read_gemm_clock(C.c_void_p(1 << 20), None, None, 0) == L.ERR_ARG
