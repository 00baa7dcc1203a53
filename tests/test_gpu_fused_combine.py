"""The COMBINE step fused into GEMM2's epilogue (moe_expert_ffn_combine).

Each token's K+1-th arrival forms its output with the standalone combine's
operations in the same order, so y must be bit-identical to moe_expert_ffn
followed by moe_combine: on small layers with ragged experts, idle experts
and a single token, and on the full V3 layer; y_perm and y_shared too.  The
standalone path is itself checked against the oracle by the parity tests;
here the fused layer is also checked against the oracle directly on one
small case."""
import numpy as np
import pytest

import oracle
from synth import BY_NAME, CONFIGS, gen
from tests import support as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import sparse_moe_layer_limited_b200 as M
    return M


def _pair(M, cfg, W, R, b):
    import torch
    s = S.moe_shape(cfg)
    Rd = torch.from_numpy(R).cuda()
    mk = lambda fused: M.MoELayer(s, Rd, torch.from_numpy(np.asarray(b, np.float32)).cuda(),  # noqa
                                  W["w13"], W["w2"], gamma=cfg.gamma, fused_combine=fused)
    return mk(False), mk(True)


@pytest.mark.parametrize("T,N,K,G,topG", [(1000, 16, 4, 4, 2), (129, 8, 2, 2, 1), (1, 16, 4, 4, 2),
                                          (300, 32, 8, 8, 4)])
def test_fused_combine_bitexact_small(M, T, N, K, G, topG):
    import torch
    cfg = CONFIGS[1].with_(T=T, d=512, N=N, K=K, G=G, topG=topG, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    ref, fused = _pair(M, cfg, W, R, b)
    xd = S.to_dev_x(x, cfg)
    for step in range(2):                  # the second call reuses the arrival counters
        y0 = ref.forward(xd).clone()
        y1 = fused.forward(xd).clone()
        torch.cuda.synchronize()
        assert torch.equal(y1, y0), step
        assert torch.equal(fused.y_perm, ref.y_perm) and torch.equal(fused.y_shared, ref.y_shared)
        assert torch.equal(fused.bias, ref.bias)
    assert fused.device_status() == 0
    if T == 1000:
        want = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K,
                                  h_round="bf16")["y"]
        fresh = _pair(M, cfg, W, R, b)[1]
        got = fresh.forward(xd, update_bias=False).float().cpu().numpy()
        assert S.rel_fro(got, want) <= 1e-2


def test_fused_combine_bitexact_v3(M):
    import torch
    from synth import device as sdev
    cfg = BY_NAME["v3_bf16"]
    s = S.moe_shape(cfg)
    dev = torch.device("cuda")
    w1 = sdev.expert_weights_bf16(cfg, 0, "w1", dev)
    w3 = sdev.expert_weights_bf16(cfg, 0, "w3", dev)
    w13 = torch.empty(cfg.N + 1, 2 * cfg.f, cfg.d, dtype=torch.bfloat16, device=dev)
    M.moe_pack_w13(s, w1, w3, w13)
    del w1, w3
    w2 = sdev.expert_weights_bf16(cfg, 0, "w2", dev)
    R = gen.make_router(cfg)
    b = gen.make_bias(cfg)
    ref, fused = _pair(M, cfg, dict(w13=w13, w2=w2), R, b)
    x = sdev.x_bf16(cfg, 0, device=dev)
    for step in range(3):
        y0 = ref.forward(x).clone()
        y1 = fused.forward(x).clone()
        torch.cuda.synchronize()
        assert torch.equal(y1, y0), step
    assert fused.device_status() == 0 and ref.device_status() == 0
