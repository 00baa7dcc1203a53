"""FP8 input gradients of the experts (moe_expert_ffn_backward_dx_fp8) and
the transposed E4M3 weights they use (moe_quantize_weights_transposed)
against the oracle's FP8 expert backward, with the GPU's rounding points
(g, u and dg, du stored bf16).  Differences left are fp32 against float64
accumulation, so the bound is the bf16 one."""
import numpy as np
import pytest

import oracle
from synth import CONFIGS, gen
from tests import support as S

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module")
def M():
    import sparse_moe_layer_limited_b200 as M
    return M


@pytest.mark.parametrize("T", [300, 1])
def test_fp8_backward_dx_matches_oracle(M, T):
    import torch
    cfg = CONFIGS[3].with_(T=T, d=256, N=16, K=4, G=4, topG=2, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)                          # E4M3 codes and 128x128 scales
    Wb = S.device_weights(cfg.with_(dtype="bf16"))     # the same weights in bf16
    s = S.moe_shape(cfg)
    layer = M.MoELayer(s, torch.from_numpy(R).cuda(),
                       torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                       W["w13_scales"], W["w2_scales"], gamma=cfg.gamma)
    xd = S.to_dev_x(x, cfg)
    layer.forward(xd, update_bias=False)
    E, d, f = cfg.N + 1, cfg.d, cfg.f
    w13t = torch.empty(E, d, 2 * f, dtype=torch.bfloat16, device="cuda")
    w2t = torch.empty(E, f, d, dtype=torch.bfloat16, device="cuda")
    M.moe_transpose_weights(s, Wb["w13"], Wb["w2"], w13t, w2t)
    w13tq = torch.empty(E, d, 2 * f, dtype=torch.float8_e4m3fn, device="cuda")
    w2tq = torch.empty(E, f, d, dtype=torch.float8_e4m3fn, device="cuda")
    w13ts = torch.empty(E, d // 128, 2 * f // 128, dtype=torch.float32, device="cuda")
    w2ts = torch.empty(E, f // 128, d // 128, dtype=torch.float32, device="cuda")
    M.moe_quantize_weights_transposed(s, w13t, w2t, w13tq, w13ts, w2tq, w2ts)
    torch.cuda.synchronize()
    # the transposed blocks are the forward's blocks transposed
    assert torch.equal(w13tq.view(torch.uint8), W["w13"].view(torch.uint8).transpose(1, 2))
    assert torch.equal(w2tq.view(torch.uint8), W["w2"].view(torch.uint8).transpose(1, 2))
    assert torch.equal(w13ts, W["w13_scales"].transpose(1, 2))
    assert torch.equal(w2ts, W["w2_scales"].transpose(1, 2))

    dyp = gen.make_x(cfg.with_(T=cfg.T * cfg.K, dtype="bf16"), seed=51)
    dys = gen.make_x(cfg.with_(dtype="bf16"), seed=52)
    dxp = torch.empty(cfg.T * cfg.K, d, dtype=torch.bfloat16, device="cuda")
    dxs = torch.empty(cfg.T, d, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(M.backward_workspace_size(s), dtype=torch.uint8, device="cuda")
    M.moe_expert_ffn_backward_dx_fp8(s, layer.x_perm, layer.x_perm_scales, layer.offsets, xd,
                                     W["w13"], W["w13_scales"], w13tq, w13ts, w2tq, w2ts,
                                     S.to_dev_x(dyp, cfg), S.to_dev_x(dys, cfg), dxp, dxs, ws)
    assert M.moe_read_device_status(ws) == 0

    get = S.host_weights(cfg)
    offs = layer.offsets.cpu().numpy()
    perm = layer.perm_tok.cpu().numpy()
    got = dxp.float().cpu().numpy()
    for e in range(cfg.N):
        a, z = offs[e], offs[e + 1]
        if z == a:
            continue
        want = oracle.fp8_swiglu_expert_backward_dx(x[perm[a:z]], *get(e), dyp[a:z],
                                                    dgu_round="bf16")["da"]
        assert S.rel_fro(got[a:z], want) <= TOL, e
    want = oracle.fp8_swiglu_expert_backward_dx(x, *get(cfg.N), dys, dgu_round="bf16")["da"]
    assert S.rel_fro(dxs.float().cpu().numpy(), want) <= TOL


def _packed(dg, du):
    """[dg du] in the packed W13 column order: per 128 features, the gate
    block then the up block."""
    R, f = dg.shape
    out = np.empty((R, 2 * f))
    for j in range(f // 128):
        out[:, 256 * j:256 * j + 128] = dg[:, 128 * j:128 * (j + 1)]
        out[:, 256 * j + 128:256 * (j + 1)] = du[:, 128 * j:128 * (j + 1)]
    return out


def test_fp8_backward_dw_matches_oracle(M):
    """moe_expert_ffn_backward_dw_fp8 after the _dx_fp8 call: dW2 and the
    packed dW13 of every expert against oracle.fp8_weight_grad on the
    oracle's own g, u, dg, du (bf16 where the GPU stores them); idle
    experts get zeros."""
    import torch
    cfg = CONFIGS[3].with_(T=300, d=256, N=16, K=4, G=4, topG=2, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    Wb = S.device_weights(cfg.with_(dtype="bf16"))
    s = S.moe_shape(cfg)
    layer = M.MoELayer(s, torch.from_numpy(R).cuda(),
                       torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                       W["w13_scales"], W["w2_scales"], gamma=cfg.gamma)
    xd = S.to_dev_x(x, cfg)
    layer.forward(xd, update_bias=False)
    E, d, f = cfg.N + 1, cfg.d, cfg.f
    w13t = torch.empty(E, d, 2 * f, dtype=torch.bfloat16, device="cuda")
    w2t = torch.empty(E, f, d, dtype=torch.bfloat16, device="cuda")
    M.moe_transpose_weights(s, Wb["w13"], Wb["w2"], w13t, w2t)
    w13tq = torch.empty(E, d, 2 * f, dtype=torch.float8_e4m3fn, device="cuda")
    w2tq = torch.empty(E, f, d, dtype=torch.float8_e4m3fn, device="cuda")
    w13ts = torch.empty(E, d // 128, 2 * f // 128, dtype=torch.float32, device="cuda")
    w2ts = torch.empty(E, f // 128, d // 128, dtype=torch.float32, device="cuda")
    M.moe_quantize_weights_transposed(s, w13t, w2t, w13tq, w13ts, w2tq, w2ts)
    dyp = gen.make_x(cfg.with_(T=cfg.T * cfg.K, dtype="bf16"), seed=53)
    dys = gen.make_x(cfg.with_(dtype="bf16"), seed=54)
    dyp_d, dys_d = S.to_dev_x(dyp, cfg), S.to_dev_x(dys, cfg)
    dxp = torch.empty(cfg.T * cfg.K, d, dtype=torch.bfloat16, device="cuda")
    dxs = torch.empty(cfg.T, d, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(M.backward_workspace_size(s), dtype=torch.uint8, device="cuda")
    M.moe_expert_ffn_backward_dx_fp8(s, layer.x_perm, layer.x_perm_scales, layer.offsets, xd,
                                     W["w13"], W["w13_scales"], w13tq, w13ts, w2tq, w2ts,
                                     dyp_d, dys_d, dxp, dxs, ws)
    dw13 = torch.empty(E, 2 * f, d, dtype=torch.bfloat16, device="cuda")
    dw2 = torch.empty(E, d, f, dtype=torch.bfloat16, device="cuda")
    M.moe_expert_ffn_backward_dw_fp8(s, layer.perm_tok, layer.offsets, xd, dyp_d, dys_d, dw13,
                                     dw2, ws)
    torch.cuda.synchronize()
    assert M.moe_read_device_status(ws) == 0

    get = S.host_weights(cfg)
    offs = layer.offsets.cpu().numpy()
    perm = layer.perm_tok.cpu().numpy()
    g13, g2 = dw13.float().cpu().numpy(), dw2.float().cpu().numpy()
    for e in range(E):
        if e < cfg.N:
            a_, z = offs[e], offs[e + 1]
            rows, dy_e = x[perm[a_:z]], dyp[a_:z]
        else:
            rows, dy_e = x, dys
        if rows.shape[0] == 0:
            assert np.all(g13[e] == 0) and np.all(g2[e] == 0), e
            continue
        bw = oracle.fp8_swiglu_expert_backward_dx(rows, *get(e), dy_e, dgu_round="bf16")
        h = oracle.round_bf16(oracle.silu(bw["g"]) * bw["u"])
        assert S.rel_fro(g2[e], oracle.fp8_weight_grad(dy_e, h)) <= 2 * TOL, ("dw2", e)
        want13 = oracle.fp8_weight_grad(_packed(bw["dg"], bw["du"]), rows)
        assert S.rel_fro(g13[e], want13) <= 2 * TOL, ("dw13", e)
