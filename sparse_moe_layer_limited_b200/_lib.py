"""ctypes binding of libmoe_b200.so: argument marshalling only.

Each function takes torch tensors (device memory from PyTorch), checks their
dtype/shape/placement, and calls the C entry point of the same name; every
step of the computation runs in the library's CUDA kernels.  A missing
library is an error: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB_PATH

DTYPE_FP32, DTYPE_BF16, DTYPE_E4M3 = 0, 1, 2
OK, ERR_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE = 0, -1, -2, -3, -4, -5

_c_p = ctypes.c_void_p


class MoEShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("N", ctypes.c_int32),
                ("K", ctypes.c_int32), ("G", ctypes.c_int32), ("topG", ctypes.c_int32),
                ("f", ctypes.c_int32), ("dtype", ctypes.c_int32)]

    def __repr__(self):
        return "MoEShape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        detail = lib().moe_last_error().decode() if status == ERR_CUDA else ""
        super().__init__(f"{fn} failed: {status} ({status_string(status)})"
                         + (f": {detail}" if detail else ""))
        self.status = status


_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_check_shape": (ctypes.c_int, [ctypes.POINTER(MoEShape)]),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(MoEShape)]),
    "moe_workspace_init": (ctypes.c_int, [_c_p, _c_p]),
    "moe_read_device_status": (ctypes.c_int, [_c_p, _c_p, ctypes.POINTER(ctypes.c_uint32),
                                              ctypes.c_int]),
    "moe_read_gemm_clock": (ctypes.c_int, [_c_p, _c_p, ctypes.POINTER(ctypes.c_uint64),
                                           ctypes.c_int]),
    "moe_route": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 8),
    "moe_route_softmax": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 8),
    "moe_dispatch": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 10),
    "moe_expert_ffn": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 12),
    "moe_expert_ffn_gathered": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 9),
    "moe_expert_ffn_combine": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 13),
    "moe_combine": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 6),
    "moe_combine_backward": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 7),
    "moe_route_backward": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 11),
    "moe_dispatch_backward": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 6),
    "moe_quantize_rows_e5m2": (ctypes.c_int, [_c_p, ctypes.c_int64, ctypes.c_int, _c_p, _c_p,
                                              ctypes.c_int64, _c_p]),
    "moe_quantize_weights_transposed": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 7),
    "moe_expert_ffn_backward_dx_fp8": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 16),
    "moe_expert_ffn_backward_dw_fp8": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 9),
    "moe_backward_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(MoEShape)]),
    "moe_transpose_weights": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 5),
    "moe_expert_ffn_backward_dx": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 12),
    "moe_expert_ffn_backward_dw": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 9),
    "moe_dispatch_noalloc": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 9),
    "moe_bias_update": (ctypes.c_int, [ctypes.POINTER(MoEShape), _c_p, _c_p, ctypes.c_float,
                                       _c_p]),
    "moe_gather_rows": (ctypes.c_int, [_c_p, ctypes.c_int64, _c_p, ctypes.c_int64, ctypes.c_int,
                                       _c_p, _c_p]),
    "moe_pack_w13": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 4),
    "moe_quantize_weights": (ctypes.c_int, [ctypes.POINTER(MoEShape)] + [_c_p] * 7),
    "moe_forward": (ctypes.c_int, [ctypes.POINTER(MoEShape), _c_p, _c_p, _c_p, ctypes.c_float]
                    + [_c_p] * 17),
}

_lib = None


def lib():
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def shape(T, d, N, K, G, topG, f, dtype) -> MoEShape:
    return MoEShape(T, d, N, K, G, topG, f, dtype)


def check_shape(s: MoEShape) -> int:
    return lib().moe_check_shape(ctypes.byref(s))


def workspace_size(s: MoEShape) -> int:
    return lib().moe_workspace_size(ctypes.byref(s))


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _call(name, *args):
    rc = getattr(lib(), name)(*args)
    if rc != OK:
        raise MoEError(name, rc)


def _expect(t, dtype, numel, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name}: expected {numel} elements, got {t.numel()}")


def x_torch_dtype(s: MoEShape):
    return torch.float32 if s.dtype == DTYPE_FP32 else torch.bfloat16


def w_torch_dtype(s: MoEShape):
    return {DTYPE_FP32: torch.float32, DTYPE_BF16: torch.bfloat16,
            DTYPE_E4M3: torch.float8_e4m3fn}[s.dtype]


def moe_workspace_init(ws, stream=None):
    _call("moe_workspace_init", _ptr(ws), _stream(stream))


def moe_read_gemm_clock(ws, stream=None, clear=False) -> dict:
    """Average SM clock (MHz) of the bf16 and FP8 expert GEMM launches since
    the last clear, from the kernels' own cycle and nanosecond counters
    (None where no launch was recorded)."""
    c = (ctypes.c_uint64 * 4)()
    _call("moe_read_gemm_clock", _ptr(ws), _stream(stream), c, int(clear))
    mhz = lambda cyc, ns: (1e3 * cyc / ns) if ns else None  # noqa: E731
    return {"bf16_mhz": mhz(c[0], c[1]), "fp8_mhz": mhz(c[2], c[3]), "bf16_ns": c[1],
            "fp8_ns": c[3]}


def moe_read_device_status(ws, stream=None, clear=False) -> int:
    v = ctypes.c_uint32(0)
    rc = lib().moe_read_device_status(_ptr(ws), _stream(stream), ctypes.byref(v), int(clear))
    if rc not in (OK, ERR_DEVICE):
        raise MoEError("moe_read_device_status", rc)
    return int(v.value)


def moe_route(s, x, router_w, bias, topk_idx, topk_gate, counts, ws, stream=None):
    _expect(x, x_torch_dtype(s), s.T * s.d, "x")
    _expect(router_w, torch.float32, s.N * s.d, "router_w")
    _expect(bias, torch.float32, s.N, "bias")
    _expect(topk_idx, torch.int32, s.T * s.K, "topk_idx")
    _expect(topk_gate, torch.float32, s.T * s.K, "topk_gate")
    _expect(counts, torch.int32, s.N, "counts")
    _call("moe_route", ctypes.byref(s), _ptr(x), _ptr(router_w), _ptr(bias), _ptr(topk_idx),
          _ptr(topk_gate), _ptr(counts), _ptr(ws), _stream(stream))


def moe_route_softmax(s, x, router_w, topk_idx, topk_gate, counts, prob_sum, ws,
                      stream=None):
    _expect(topk_idx, torch.int32, s.T * s.K, "topk_idx")
    _expect(topk_gate, torch.float32, s.T * s.K, "topk_gate")
    _expect(counts, torch.int32, s.N, "counts")
    if prob_sum is not None:
        _expect(prob_sum, torch.float32, s.N, "prob_sum")
    _call("moe_route_softmax", ctypes.byref(s), _ptr(x), _ptr(router_w), _ptr(topk_idx),
          _ptr(topk_gate), _ptr(counts), _ptr(prob_sum), _ptr(ws), _stream(stream))


def moe_dispatch(s, x, topk_idx, counts, offsets, perm_tok, slot, x_perm, x_perm_scales, ws,
                 stream=None):
    _expect(offsets, torch.int32, s.N + 1, "offsets")
    _expect(perm_tok, torch.int32, s.T * s.K, "perm_tok")
    _expect(slot, torch.int32, s.T * s.K, "slot")
    if x_perm is not None:  # None: rows not copied (BF16/FP32, moe_expert_ffn_gathered)
        _expect(x_perm, w_torch_dtype(s) if s.dtype == DTYPE_E4M3 else x_torch_dtype(s),
                s.T * s.K * s.d, "x_perm")
    _call("moe_dispatch", ctypes.byref(s), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
          _ptr(perm_tok), _ptr(slot), _ptr(x_perm), _ptr(x_perm_scales), _ptr(ws),
          _stream(stream))


def moe_dispatch_noalloc(s, x, topk_idx, counts, offsets, perm_tok, slot, x_perm,
                         x_perm_scales=None, stream=None):
    """moe_dispatch without a workspace (fixed static device scratch)."""
    _expect(offsets, torch.int32, s.N + 1, "offsets")
    _expect(perm_tok, torch.int32, s.T * s.K, "perm_tok")
    _expect(slot, torch.int32, s.T * s.K, "slot")
    _call("moe_dispatch_noalloc", ctypes.byref(s), _ptr(x), _ptr(topk_idx), _ptr(counts),
          _ptr(offsets), _ptr(perm_tok), _ptr(slot), _ptr(x_perm), _ptr(x_perm_scales),
          _stream(stream))


def moe_expert_ffn(s, x_perm, x_perm_scales, offsets, x, w13, w2, w13_scales, w2_scales,
                   y_perm, y_shared, ws, stream=None):
    _expect(w13, w_torch_dtype(s), (s.N + 1) * 2 * s.f * s.d, "w13")
    _expect(w2, w_torch_dtype(s), (s.N + 1) * s.d * s.f, "w2")
    _expect(y_perm, x_torch_dtype(s), s.T * s.K * s.d, "y_perm")
    _expect(y_shared, x_torch_dtype(s), s.T * s.d, "y_shared")
    _call("moe_expert_ffn", ctypes.byref(s), _ptr(x_perm), _ptr(x_perm_scales), _ptr(offsets),
          _ptr(x), _ptr(w13), _ptr(w2), _ptr(w13_scales), _ptr(w2_scales), _ptr(y_perm),
          _ptr(y_shared), _ptr(ws), _stream(stream))


def moe_expert_ffn_gathered(s, x, perm_tok, offsets, w13, w2, y_perm, y_shared, ws,
                            stream=None):
    _expect(w13, w_torch_dtype(s), (s.N + 1) * 2 * s.f * s.d, "w13")
    _expect(w2, w_torch_dtype(s), (s.N + 1) * s.d * s.f, "w2")
    _expect(y_perm, x_torch_dtype(s), s.T * s.K * s.d, "y_perm")
    _expect(y_shared, x_torch_dtype(s), s.T * s.d, "y_shared")
    _call("moe_expert_ffn_gathered", ctypes.byref(s), _ptr(x), _ptr(perm_tok), _ptr(offsets),
          _ptr(w13), _ptr(w2), _ptr(y_perm), _ptr(y_shared), _ptr(ws), _stream(stream))


def moe_expert_ffn_combine(s, x_perm, offsets, perm_tok, slot, topk_gate, x, w13, w2, y_perm,
                           y_shared, y, ws, stream=None):
    _expect(w13, w_torch_dtype(s), (s.N + 1) * 2 * s.f * s.d, "w13")
    _expect(w2, w_torch_dtype(s), (s.N + 1) * s.d * s.f, "w2")
    _expect(y_perm, x_torch_dtype(s), s.T * s.K * s.d, "y_perm")
    _expect(y_shared, x_torch_dtype(s), s.T * s.d, "y_shared")
    _expect(y, x_torch_dtype(s), s.T * s.d, "y")
    _expect(slot, torch.int32, s.T * s.K, "slot")
    _expect(topk_gate, torch.float32, s.T * s.K, "topk_gate")
    _call("moe_expert_ffn_combine", ctypes.byref(s), _ptr(x_perm), _ptr(offsets), _ptr(perm_tok),
          _ptr(slot), _ptr(topk_gate), _ptr(x), _ptr(w13), _ptr(w2), _ptr(y_perm),
          _ptr(y_shared), _ptr(y), _ptr(ws), _stream(stream))


def backward_workspace_size(s) -> int:
    return lib().moe_backward_workspace_size(ctypes.byref(s))


def moe_transpose_weights(s, w13, w2, w13t, w2t, stream=None):
    _expect(w13t, x_torch_dtype(s), (s.N + 1) * 2 * s.f * s.d, "w13t")   # bf16 weights
    _expect(w2t, x_torch_dtype(s), (s.N + 1) * s.d * s.f, "w2t")
    _call("moe_transpose_weights", ctypes.byref(s), _ptr(w13), _ptr(w2), _ptr(w13t), _ptr(w2t),
          _stream(stream))


def moe_expert_ffn_backward_dx(s, x_perm, offsets, x, w13, w13t, w2t, dy_perm, dy_shared,
                               dx_perm, dx_shared, ws_bwd, stream=None):
    _expect(dx_perm, x_torch_dtype(s), s.T * s.K * s.d, "dx_perm")
    _expect(dx_shared, x_torch_dtype(s), s.T * s.d, "dx_shared")
    _call("moe_expert_ffn_backward_dx", ctypes.byref(s), _ptr(x_perm), _ptr(offsets), _ptr(x),
          _ptr(w13), _ptr(w13t), _ptr(w2t), _ptr(dy_perm), _ptr(dy_shared), _ptr(dx_perm),
          _ptr(dx_shared), _ptr(ws_bwd), _stream(stream))


def moe_quantize_weights_transposed(s, w13t, w2t, w13t_q, w13t_scales, w2t_q, w2t_scales,
                                    stream=None):
    _expect(w13t_q, torch.float8_e4m3fn, (s.N + 1) * s.d * 2 * s.f, "w13t_q")
    _expect(w2t_q, torch.float8_e4m3fn, (s.N + 1) * s.f * s.d, "w2t_q")
    _expect(w13t_scales, torch.float32, (s.N + 1) * (s.d // 128) * (2 * s.f // 128),
            "w13t_scales")
    _expect(w2t_scales, torch.float32, (s.N + 1) * (s.f // 128) * (s.d // 128), "w2t_scales")
    _call("moe_quantize_weights_transposed", ctypes.byref(s), _ptr(w13t), _ptr(w2t),
          _ptr(w13t_q), _ptr(w13t_scales), _ptr(w2t_q), _ptr(w2t_scales), _stream(stream))


def moe_expert_ffn_backward_dx_fp8(s, x_perm, x_perm_scales, offsets, x, w13, w13_scales, w13t,
                                   w13t_scales, w2t, w2t_scales, dy_perm, dy_shared, dx_perm,
                                   dx_shared, ws_bwd, stream=None):
    _expect(dx_perm, torch.bfloat16, s.T * s.K * s.d, "dx_perm")
    _expect(dx_shared, torch.bfloat16, s.T * s.d, "dx_shared")
    _call("moe_expert_ffn_backward_dx_fp8", ctypes.byref(s), _ptr(x_perm), _ptr(x_perm_scales),
          _ptr(offsets), _ptr(x), _ptr(w13), _ptr(w13_scales), _ptr(w13t), _ptr(w13t_scales),
          _ptr(w2t), _ptr(w2t_scales), _ptr(dy_perm), _ptr(dy_shared), _ptr(dx_perm),
          _ptr(dx_shared), _ptr(ws_bwd), _stream(stream))


def moe_expert_ffn_backward_dw_fp8(s, perm_tok, offsets, x, dy_perm, dy_shared, dw13, dw2,
                                   ws_bwd, stream=None):
    _expect(dw13, torch.bfloat16, (s.N + 1) * 2 * s.f * s.d, "dw13")
    _expect(dw2, torch.bfloat16, (s.N + 1) * s.d * s.f, "dw2")
    _call("moe_expert_ffn_backward_dw_fp8", ctypes.byref(s), _ptr(perm_tok), _ptr(offsets),
          _ptr(x), _ptr(dy_perm), _ptr(dy_shared), _ptr(dw13), _ptr(dw2), _ptr(ws_bwd),
          _stream(stream))


def moe_expert_ffn_backward_dw(s, x_perm, offsets, x, dy_perm, dy_shared, dw13, dw2, ws_bwd,
                               stream=None):
    _expect(dw13, w_torch_dtype(s), (s.N + 1) * 2 * s.f * s.d, "dw13")
    _expect(dw2, w_torch_dtype(s), (s.N + 1) * s.d * s.f, "dw2")
    _call("moe_expert_ffn_backward_dw", ctypes.byref(s), _ptr(x_perm), _ptr(offsets), _ptr(x),
          _ptr(dy_perm), _ptr(dy_shared), _ptr(dw13), _ptr(dw2), _ptr(ws_bwd), _stream(stream))


def moe_combine(s, y_perm, y_shared, slot, topk_gate, y, stream=None):
    _expect(y, x_torch_dtype(s), s.T * s.d, "y")
    _call("moe_combine", ctypes.byref(s), _ptr(y_perm), _ptr(y_shared), _ptr(slot),
          _ptr(topk_gate), _ptr(y), _stream(stream))


def moe_combine_backward(s, dy, y_perm, slot, topk_gate, dy_perm, dgate, stream=None):
    _expect(dy_perm, x_torch_dtype(s), s.T * s.K * s.d, "dy_perm")
    _expect(dgate, torch.float32, s.T * s.K, "dgate")
    _call("moe_combine_backward", ctypes.byref(s), _ptr(dy), _ptr(y_perm), _ptr(slot),
          _ptr(topk_gate), _ptr(dy_perm), _ptr(dgate), _stream(stream))


def moe_route_backward(s, x, router_w, topk_idx, dgate, offsets, perm_tok, slot, dlogit,
                       dx_route, drouter, stream=None):
    _expect(dlogit, torch.float32, s.T * s.K, "dlogit")
    _expect(dx_route, torch.float32, s.T * s.d, "dx_route")
    _expect(drouter, torch.float32, s.N * s.d, "drouter")
    _call("moe_route_backward", ctypes.byref(s), _ptr(x), _ptr(router_w), _ptr(topk_idx),
          _ptr(dgate), _ptr(offsets), _ptr(perm_tok), _ptr(slot), _ptr(dlogit), _ptr(dx_route),
          _ptr(drouter), _stream(stream))


def moe_dispatch_backward(s, dx_perm, dx_shared, slot, dx_route, dx, stream=None):
    _expect(dx, x_torch_dtype(s), s.T * s.d, "dx")
    _call("moe_dispatch_backward", ctypes.byref(s), _ptr(dx_perm), _ptr(dx_shared), _ptr(slot),
          _ptr(dx_route), _ptr(dx), _stream(stream))


def moe_quantize_rows_e5m2(g, codes, scales, stream=None):
    """g [rows, cols] bf16 -> codes [rows, cols] uint8 (E5M2 bits) and scales
    [cols/128, sc_ld] fp32 (sc_ld = scales.shape[1] >= rows)."""
    rows, cols = g.shape
    _expect(g, torch.bfloat16, rows * cols, "g")
    _expect(codes, torch.uint8, rows * cols, "codes")
    if scales.dtype != torch.float32 or scales.dim() != 2 or scales.shape[0] != cols // 128:
        raise ValueError("scales: expected float32 [cols/128, sc_ld]")
    _call("moe_quantize_rows_e5m2", _ptr(g), ctypes.c_int64(rows), ctypes.c_int(cols),
          _ptr(codes), _ptr(scales), ctypes.c_int64(scales.shape[1]), _stream(stream))


def moe_bias_update(s, counts, bias, gamma, stream=None):
    _expect(counts, torch.int32, s.N, "counts")
    _expect(bias, torch.float32, s.N, "bias")
    _call("moe_bias_update", ctypes.byref(s), _ptr(counts), _ptr(bias), ctypes.c_float(gamma),
          _stream(stream))


def moe_gather_rows(src, idx, dst, stream=None):
    """dst[i] = src[idx[i]] (whole rows); src and dst 2-D with equal row bytes."""
    if src.dim() != 2 or dst.dim() != 2 or src.dtype != dst.dtype or src.shape[1] != dst.shape[1]:
        raise ValueError("src and dst: 2-D tensors of one dtype and row length")
    _expect(idx, torch.int32, dst.shape[0], "idx")
    row_bytes = src.shape[1] * src.element_size()
    _call("moe_gather_rows", _ptr(src), ctypes.c_int64(src.shape[0]), _ptr(idx),
          ctypes.c_int64(dst.shape[0]), ctypes.c_int(row_bytes), _ptr(dst), _stream(stream))


def moe_pack_w13(s, w1, w3, w13, stream=None):
    _call("moe_pack_w13", ctypes.byref(s), _ptr(w1), _ptr(w3), _ptr(w13), _stream(stream))


def moe_quantize_weights(s, w13_bf16, w2_bf16, w13_q, w13_scales, w2_q, w2_scales, stream=None):
    _call("moe_quantize_weights", ctypes.byref(s), _ptr(w13_bf16), _ptr(w2_bf16), _ptr(w13_q),
          _ptr(w13_scales), _ptr(w2_q), _ptr(w2_scales), _stream(stream))


def moe_forward(s, x, router_w, bias, gamma, w13, w2, w13_scales, w2_scales, topk_idx,
                topk_gate, counts, offsets, perm_tok, slot, x_perm, x_perm_scales, y_perm,
                y_shared, y, ws, stream=None):
    _call("moe_forward", ctypes.byref(s), _ptr(x), _ptr(router_w), _ptr(bias),
          ctypes.c_float(gamma), _ptr(w13), _ptr(w2), _ptr(w13_scales), _ptr(w2_scales),
          _ptr(topk_idx), _ptr(topk_gate), _ptr(counts), _ptr(offsets), _ptr(perm_tok),
          _ptr(slot), _ptr(x_perm), _ptr(x_perm_scales), _ptr(y_perm), _ptr(y_shared), _ptr(y),
          _ptr(ws), _stream(stream))
