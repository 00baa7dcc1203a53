"""MoELayer: owns the device buffers of one layer shape and runs the forward
through the C-ABI calls (route -> dispatch -> experts -> combine -> bias update)
and, in BF16 mode, the layer backward."""
from __future__ import annotations

import torch

from . import _lib as L


class MoELayer:
    """DeepSeekMoE layer on one GPU.

    router_w [N, d] fp32, bias [N] fp32 (updated in place by forward), w13
    [N+1, 2f, d] packed (see moe_pack_w13), w2 [N+1, d, f]; for E4M3 the
    quantised weights and their 128x128-block scales.  All tensors must be on
    the same CUDA device.  Intermediate buffers are allocated once here.

    gather (BF16 only): GEMM1 reads each routed row straight from x through
    perm_tok (moe_expert_ffn_gathered) instead of a permuted copy; dispatch
    then writes no x_perm.

    fused_combine (BF16 only, not with gather): the combine runs inside
    GEMM2's epilogue (moe_expert_ffn_combine) instead of as its own kernel;
    the output is bit-identical."""

    def __init__(self, shape: L.MoEShape, router_w, bias, w13, w2, w13_scales=None,
                 w2_scales=None, gamma: float = 0.001, gather: bool = False,
                 fused_combine: bool = False):
        rc = L.check_shape(shape)
        if rc != L.OK:
            raise L.MoEError("moe_check_shape", rc)
        self.shape = s = shape
        self.router_w, self.bias, self.w13, self.w2 = router_w, bias, w13, w2
        self.w13_scales, self.w2_scales = w13_scales, w2_scales
        self.gamma = float(gamma)
        self.gather = bool(gather) and s.dtype == L.DTYPE_BF16
        self.fused_combine = (bool(fused_combine) and s.dtype == L.DTYPE_BF16
                              and not self.gather)
        dev = router_w.device
        i32 = dict(dtype=torch.int32, device=dev)
        xdt = L.x_torch_dtype(s)
        self.topk_idx = torch.empty(s.T, s.K, **i32)
        self.topk_gate = torch.empty(s.T, s.K, dtype=torch.float32, device=dev)
        self.counts = torch.empty(s.N, **i32)
        self.offsets = torch.empty(s.N + 1, **i32)
        self.perm_tok = torch.empty(s.T * s.K, **i32)
        self.slot = torch.empty(s.T, s.K, **i32)
        pdt = torch.float8_e4m3fn if s.dtype == L.DTYPE_E4M3 else xdt
        self.x_perm = (None if self.gather
                       else torch.empty(s.T * s.K, s.d, dtype=pdt, device=dev))
        self.x_perm_scales = (torch.empty(s.d // 128, (s.T * s.K + 3) // 4 * 4, dtype=torch.float32,
                                          device=dev)
                              if s.dtype == L.DTYPE_E4M3 else None)
        self.y_perm = torch.empty(s.T * s.K, s.d, dtype=xdt, device=dev)
        self.y_shared = torch.empty(s.T, s.d, dtype=xdt, device=dev)
        self.y = torch.empty(s.T, s.d, dtype=xdt, device=dev)
        self.ws = torch.zeros(L.workspace_size(s), dtype=torch.uint8, device=dev)

    def route(self, x, stream=None):
        s = self.shape
        L.moe_route(s, x, self.router_w, self.bias, self.topk_idx, self.topk_gate, self.counts,
                    self.ws, stream)

    def forward(self, x, update_bias: bool = True, stream=None):
        """y = shared(x) + sum_k gate_k expert_k(x); then (optionally) the bias
        update from this batch's counts.  Returns self.y (overwritten next call)."""
        s = self.shape
        L.moe_route(s, x, self.router_w, self.bias, self.topk_idx, self.topk_gate, self.counts,
                    self.ws, stream)
        L.moe_dispatch(s, x, self.topk_idx, self.counts, self.offsets, self.perm_tok, self.slot,
                       self.x_perm, self.x_perm_scales, self.ws, stream)
        self.experts_and_combine(x, stream)
        if update_bias:
            L.moe_bias_update(s, self.counts, self.bias, self.gamma, stream)
        return self.y

    def experts_and_combine(self, x, stream=None):
        """The expert GEMMs and the COMBINE step (one fused launch pair when
        fused_combine is set); writes self.y."""
        s = self.shape
        if self.fused_combine:
            L.moe_expert_ffn_combine(s, self.x_perm, self.offsets, self.perm_tok, self.slot,
                                     self.topk_gate, x, self.w13, self.w2, self.y_perm,
                                     self.y_shared, self.y, self.ws, stream)
        else:
            self.experts(x, stream)
            L.moe_combine(s, self.y_perm, self.y_shared, self.slot, self.topk_gate, self.y,
                          stream)

    def experts(self, x, stream=None):
        """The expert GEMMs on the dispatched rows (gathered from x or read from x_perm)."""
        s = self.shape
        if self.gather:
            L.moe_expert_ffn_gathered(s, x, self.perm_tok, self.offsets, self.w13, self.w2,
                                      self.y_perm, self.y_shared, self.ws, stream)
        else:
            L.moe_expert_ffn(s, self.x_perm, self.x_perm_scales, self.offsets, x, self.w13,
                             self.w2, self.w13_scales, self.w2_scales, self.y_perm,
                             self.y_shared, self.ws, stream)

    def backward(self, x, dy, w13t, w2t, weight_grads: bool = True, stream=None):
        """Gradients of the last forward (its routing held fixed) given
        dy = dL/dy [T, d], BF16 mode without gather, in the backward order
        COMBINE -> MLP_B -> MLP_W -> DISPATCH:
          moe_combine_backward -> moe_expert_ffn_backward_dx (-> _dw)
          -> moe_route_backward -> moe_dispatch_backward.
        w13t, w2t: the transposed weights (moe_transpose_weights).  Returns
        dict(dx [T, d] bf16, drouter [N, d] fp32, dgate [T, K] fp32, and with
        weight_grads dw13, dw2 laid out like w13, w2).  The bias gets no
        gradient (it only selects experts)."""
        s = self.shape
        if s.dtype != L.DTYPE_BF16 or self.gather:
            raise ValueError("the layer backward runs in BF16 mode on the x_perm path")
        dev, xdt = x.device, L.x_torch_dtype(s)
        if getattr(self, "_bwd", None) is None:
            self._bwd = dict(
                ws=torch.zeros(L.backward_workspace_size(s), dtype=torch.uint8, device=dev),
                dy_perm=torch.empty(s.T * s.K, s.d, dtype=xdt, device=dev),
                dgate=torch.empty(s.T, s.K, dtype=torch.float32, device=dev),
                dx_perm=torch.empty(s.T * s.K, s.d, dtype=xdt, device=dev),
                dx_shared=torch.empty(s.T, s.d, dtype=xdt, device=dev),
                dlogit=torch.empty(s.T, s.K, dtype=torch.float32, device=dev),
                dx_route=torch.empty(s.T, s.d, dtype=torch.float32, device=dev))
        B = self._bwd
        dx = torch.empty(s.T, s.d, dtype=xdt, device=dev)
        drouter = torch.empty(s.N, s.d, dtype=torch.float32, device=dev)
        L.moe_combine_backward(s, dy, self.y_perm, self.slot, self.topk_gate, B["dy_perm"],
                               B["dgate"], stream)
        L.moe_expert_ffn_backward_dx(s, self.x_perm, self.offsets, x, self.w13, w13t, w2t,
                                     B["dy_perm"], dy, B["dx_perm"], B["dx_shared"], B["ws"],
                                     stream)
        out = dict(dx=dx, drouter=drouter, dgate=B["dgate"])
        if weight_grads:
            out["dw13"] = torch.empty_like(self.w13)
            out["dw2"] = torch.empty_like(self.w2)
            L.moe_expert_ffn_backward_dw(s, self.x_perm, self.offsets, x, B["dy_perm"], dy,
                                         out["dw13"], out["dw2"], B["ws"], stream)
        L.moe_route_backward(s, x, self.router_w, self.topk_idx, B["dgate"], self.offsets,
                             self.perm_tok, self.slot, B["dlogit"], B["dx_route"], drouter,
                             stream)
        L.moe_dispatch_backward(s, B["dx_perm"], B["dx_shared"], self.slot, B["dx_route"], dx,
                                stream)
        return out

    def capture(self, x, update_bias: bool = True):
        """Record one forward (route, dispatch, experts, combine and, with
        update_bias, the bias update) on the buffer x into a CUDA graph, so
        that replay() reruns the whole step with one launch from the host.
        One eager forward runs first (it also moves the bias once) so that
        every launch-time set-up happens outside the capture.  The graph keeps
        x's address: copy each new batch into x before replay().  Returns the
        graph."""
        side = torch.cuda.Stream(x.device)
        side.wait_stream(torch.cuda.current_stream(x.device))
        with torch.cuda.stream(side):
            self.forward(x, update_bias)
        torch.cuda.current_stream(x.device).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.forward(x, update_bias)
        self._graph = graph
        return graph

    def replay(self):
        """Rerun the captured step; returns self.y."""
        self._graph.replay()
        return self.y

    def backward_status(self, clear: bool = False) -> int:
        """Status word of the backward workspace (0 = no device-side problem)."""
        B = getattr(self, "_bwd", None)
        return 0 if B is None else L.moe_read_device_status(B["ws"], None, clear)

    def device_status(self, clear: bool = False) -> int:
        return L.moe_read_device_status(self.ws, None, clear)
