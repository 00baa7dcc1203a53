"""DeepSeekMoE layer forward for one NVIDIA B200 (sm_100a).

The compute runs in ``libmoe_b200.so`` (hand-written CUDA, C ABI declared in
``include/moe_b200.h``); this package only marshals arguments.  The library is
loaded on first use, and any call fails loudly when it has not been built.
"""
from ._lib import (  # noqa: F401
    backward_workspace_size, moe_expert_ffn_backward_dw, moe_expert_ffn_backward_dx,
    moe_transpose_weights, moe_combine_backward, moe_route_backward, moe_dispatch_backward,
    moe_quantize_rows_e5m2, moe_quantize_weights_transposed, moe_expert_ffn_backward_dx_fp8,
    moe_expert_ffn_backward_dw_fp8,
    DTYPE_BF16, DTYPE_E4M3, DTYPE_FP32, MoEError, MoEShape, check_shape, lib, moe_bias_update,
    moe_combine, moe_dispatch, moe_dispatch_noalloc, moe_expert_ffn, moe_expert_ffn_gathered,
    moe_gather_rows, moe_expert_ffn_combine,
    moe_forward, moe_pack_w13, moe_quantize_weights,
    moe_read_device_status, moe_read_gemm_clock, moe_route, moe_route_softmax, moe_workspace_init, shape,
    status_string,
    workspace_size, x_torch_dtype, w_torch_dtype,
)
from .layer import MoELayer  # noqa: F401
