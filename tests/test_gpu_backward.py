"""Expert backward, input gradients (moe_expert_ffn_backward_dx) against the
oracle's SwiGLU backward, and the weight transposes it uses."""
import numpy as np
import pytest

import oracle
from synth import CONFIGS, gen
from tests import support as S

pytestmark = pytest.mark.gpu
TOL_BF16 = 1e-2


@pytest.fixture(scope="module")
def M():
    import sparse_moe_layer_limited_b200 as M
    return M


def _grads(cfg, seed):
    """Seeded output gradients dy_perm [T*K, d] and dy_shared [T, d] (bf16 values)."""
    dyp = gen.make_x(cfg.with_(T=cfg.T * cfg.K), seed=seed)
    dys = gen.make_x(cfg, seed=seed + 1)
    return dyp, dys


@pytest.mark.parametrize("T", [600, 129, 1])
def test_backward_dx_matches_oracle(M, T):
    import torch
    cfg = CONFIGS[1].with_(T=T, d=256, N=8, K=2, G=2, topG=1, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    s = S.moe_shape(cfg)
    layer = M.MoELayer(s, torch.from_numpy(R).cuda(),
                       torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                       gamma=cfg.gamma)
    xd = S.to_dev_x(x, cfg)
    layer.forward(xd, update_bias=False)
    w13t = torch.empty(cfg.N + 1, cfg.d, 2 * cfg.f, dtype=torch.bfloat16, device="cuda")
    w2t = torch.empty(cfg.N + 1, cfg.f, cfg.d, dtype=torch.bfloat16, device="cuda")
    M.moe_transpose_weights(s, W["w13"], W["w2"], w13t, w2t)
    torch.cuda.synchronize()
    assert torch.equal(w13t, W["w13"].transpose(1, 2))
    assert torch.equal(w2t, W["w2"].transpose(1, 2))

    dyp, dys = _grads(cfg, 31)
    dyp_d, dys_d = S.to_dev_x(dyp, cfg), S.to_dev_x(dys, cfg)
    dxp = torch.empty_like(layer.x_perm)
    dxs = torch.empty_like(xd)
    ws = torch.zeros(M.backward_workspace_size(s), dtype=torch.uint8, device="cuda")
    M.moe_expert_ffn_backward_dx(s, layer.x_perm, layer.offsets, xd, W["w13"], w13t, w2t,
                                 dyp_d, dys_d, dxp, dxs, ws)
    assert M.moe_read_device_status(ws) == 0

    get = S.host_weights(cfg)
    offs = layer.offsets.cpu().numpy()
    perm = layer.perm_tok.cpu().numpy()
    dxp_h = dxp.float().cpu().numpy()
    for e in range(cfg.N):
        a, z = offs[e], offs[e + 1]
        if z == a:
            continue
        want = oracle.swiglu_expert_backward(x[perm[a:z]], *get(e), dyp[a:z], gu_round="bf16",
                                             dgu_round="bf16")["da"]
        assert S.rel_fro(dxp_h[a:z], want) <= TOL_BF16, e
    want = oracle.swiglu_expert_backward(x, *get(cfg.N), dys, gu_round="bf16",
                                         dgu_round="bf16")["da"]
    assert S.rel_fro(dxs.float().cpu().numpy(), want) <= TOL_BF16


def test_v3_backward_dx_sampled(M):
    """The full V3 layer shape: input gradients of three routed experts (every
    row) and of 192 shared-expert rows against the oracle (rows are
    independent in the backward, so the oracle takes only the sampled ones)."""
    import torch
    cfg = CONFIGS[2]
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    s = S.moe_shape(cfg)
    layer = M.MoELayer(s, torch.from_numpy(R).cuda(),
                       torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                       gamma=cfg.gamma)
    xd = S.to_dev_x(x, cfg)
    layer.forward(xd, update_bias=False)
    w13t = torch.empty(cfg.N + 1, cfg.d, 2 * cfg.f, dtype=torch.bfloat16, device="cuda")
    w2t = torch.empty(cfg.N + 1, cfg.f, cfg.d, dtype=torch.bfloat16, device="cuda")
    M.moe_transpose_weights(s, W["w13"], W["w2"], w13t, w2t)
    dyp, dys = _grads(cfg, 41)
    dxp = torch.empty_like(layer.x_perm)
    dxs = torch.empty_like(xd)
    ws = torch.zeros(M.backward_workspace_size(s), dtype=torch.uint8, device="cuda")
    M.moe_expert_ffn_backward_dx(s, layer.x_perm, layer.offsets, xd, W["w13"], w13t, w2t,
                                 S.to_dev_x(dyp, cfg), S.to_dev_x(dys, cfg), dxp, dxs, ws)
    assert M.moe_read_device_status(ws) == 0
    get = S.streaming_weights(cfg)
    offs = layer.offsets.cpu().numpy()
    perm = layer.perm_tok.cpu().numpy()
    for e in (0, 101, 255):
        a, z = offs[e], offs[e + 1]
        want = oracle.swiglu_expert_backward(x[perm[a:z]], *get(e), dyp[a:z], gu_round="bf16",
                                             dgu_round="bf16")["da"]
        assert S.rel_fro(dxp[a:z].float().cpu().numpy(), want) <= TOL_BF16, e
    rows = np.random.default_rng(3).choice(cfg.T, 192, replace=False)
    want = oracle.swiglu_expert_backward(x[rows], *get(cfg.N), dys[rows], gu_round="bf16",
                                         dgu_round="bf16")["da"]
    assert S.rel_fro(dxs.float().cpu().numpy()[rows], want) <= TOL_BF16


def _unpack_w13(dw13, f):
    """Packed [2f, d] (per 128-row block j: W1 rows then W3 rows) -> (dW1, dW3)."""
    blocks = dw13.reshape(f // 128, 2, 128, -1)
    return blocks[:, 0].reshape(f, -1), blocks[:, 1].reshape(f, -1)


@pytest.mark.parametrize("T,bias_shift", [(600, 0.0), (129, 0.0), (300, 0.5)])
def test_backward_dw_matches_oracle(M, T, bias_shift):
    """Weight gradients of every routed expert and of the shared expert
    against the oracle; with the bias shifted onto two groups, most experts
    get no rows and their gradients must be zero."""
    import torch
    cfg = CONFIGS[1].with_(T=T, d=256, N=16, K=2, G=4, topG=2, f=256)
    R = gen.make_router(cfg)
    b = gen.make_bias(cfg).copy()
    b[:8] += bias_shift
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    s = S.moe_shape(cfg)
    layer = M.MoELayer(s, torch.from_numpy(R).cuda(),
                       torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                       gamma=cfg.gamma)
    xd = S.to_dev_x(x, cfg)
    layer.forward(xd, update_bias=False)
    w13t = torch.empty(cfg.N + 1, cfg.d, 2 * cfg.f, dtype=torch.bfloat16, device="cuda")
    w2t = torch.empty(cfg.N + 1, cfg.f, cfg.d, dtype=torch.bfloat16, device="cuda")
    M.moe_transpose_weights(s, W["w13"], W["w2"], w13t, w2t)
    dyp, dys = _grads(cfg, 51)
    dyp_d, dys_d = S.to_dev_x(dyp, cfg), S.to_dev_x(dys, cfg)
    dxp, dxs = torch.empty_like(layer.x_perm), torch.empty_like(xd)
    ws = torch.zeros(M.backward_workspace_size(s), dtype=torch.uint8, device="cuda")
    M.moe_expert_ffn_backward_dx(s, layer.x_perm, layer.offsets, xd, W["w13"], w13t, w2t,
                                 dyp_d, dys_d, dxp, dxs, ws)
    dw13 = torch.full_like(W["w13"], float("nan"))
    dw2 = torch.full_like(W["w2"], float("nan"))
    M.moe_expert_ffn_backward_dw(s, layer.x_perm, layer.offsets, xd, dyp_d, dys_d, dw13, dw2, ws)
    assert M.moe_read_device_status(ws) == 0
    get = S.host_weights(cfg)
    offs = layer.offsets.cpu().numpy()
    perm = layer.perm_tok.cpu().numpy()
    g13 = dw13.float().cpu().numpy()
    g2 = dw2.float().cpu().numpy()
    empty = 0
    for e in range(cfg.N + 1):
        if e < cfg.N:
            a, z = offs[e], offs[e + 1]
            rows_x, rows_dy = x[perm[a:z]], dyp[a:z]
        else:
            rows_x, rows_dy = x, dys
        d1, d3 = _unpack_w13(g13[e], cfg.f)
        if rows_x.shape[0] == 0:
            empty += 1
            assert np.all(d1 == 0) and np.all(d3 == 0) and np.all(g2[e] == 0), e
            continue
        r = oracle.swiglu_expert_backward(rows_x, *get(e), rows_dy, gu_round="bf16",
                                          dgu_round="bf16")
        assert S.rel_fro(d1, r["dw1"]) <= TOL_BF16, ("dw1", e)
        assert S.rel_fro(d3, r["dw3"]) <= TOL_BF16, ("dw3", e)
        assert S.rel_fro(g2[e], r["dw2"]) <= TOL_BF16, ("dw2", e)
    assert (empty > 0) == (bias_shift > 0)
