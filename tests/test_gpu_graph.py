"""The layer step captured in a CUDA graph and replayed.

A graph replay launches the same kernels with the same arguments as the
eager forward, so outputs and the bias after every step must be bit-identical
to an eager layer run step for step on the same batches (bf16 with and
without the fused combine, and E4M3)."""
import numpy as np
import pytest

from synth import CONFIGS, gen
from tests import support as S

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,fused", [("bf16", False), ("bf16", True), ("e4m3", False)])
def test_graph_replay_matches_eager(dtype, fused):
    import torch
    import sparse_moe_layer_limited_b200 as M
    base = CONFIGS[1] if dtype == "bf16" else CONFIGS[3]
    cfg = base.with_(T=600, d=512, N=16, K=4, G=4, topG=2, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    W = S.device_weights(cfg)
    s = S.moe_shape(cfg)

    def make():
        return M.MoELayer(s, torch.from_numpy(R).cuda(),
                          torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                          W.get("w13_scales"), W.get("w2_scales"), gamma=cfg.gamma,
                          fused_combine=fused)
    eager, graphed = make(), make()
    batches = [S.to_dev_x(S.tie_free_x(cfg, R, b, batch=i)[0], cfg) for i in range(4)]
    x_buf = batches[0].clone()
    graphed.capture(x_buf)                 # its eager warm-up is step 0 on batch 0
    y0 = eager.forward(batches[0]).clone()
    torch.cuda.synchronize()
    assert torch.equal(graphed.y, y0) and torch.equal(graphed.bias, eager.bias)
    for i in range(1, 4):
        x_buf.copy_(batches[i])
        y_g = graphed.replay().clone()
        y_e = eager.forward(batches[i]).clone()
        torch.cuda.synchronize()
        assert torch.equal(y_g, y_e), i
        assert torch.equal(graphed.bias, eager.bias), i
    assert graphed.device_status() == 0 and eager.device_status() == 0
