"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Routing indices, counts, offsets, the permutation and slots must match bit
for bit; gates within 1e-6; layer outputs within rel-Frobenius 1e-5 (fp32
layer) and 1e-2 (bf16 layer, oracle on bf16-rounded operands with the hidden
activation rounded to bf16).
"""
import numpy as np
import pytest

import oracle
from synth import CONFIGS, gen
from tests import support as S

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-5, "bf16": 1e-2, "e4m3": 2e-2}


@pytest.fixture(scope="module")
def M():
    import sparse_moe_layer_limited_b200 as M
    return M


def _torch():
    import torch
    return torch


def _run_route(M, cfg, x, R, b, T=None):
    torch = _torch()
    s = S.moe_shape(cfg, T)
    xd = S.to_dev_x(x, cfg)
    Rd = torch.from_numpy(R).cuda()
    bd = torch.from_numpy(np.asarray(b, np.float32)).cuda()
    idx = torch.empty(s.T, s.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(s.T, s.K, dtype=torch.float32, device="cuda")
    counts = torch.empty(s.N, dtype=torch.int32, device="cuda")
    ws = torch.zeros(M.workspace_size(s), dtype=torch.uint8, device="cuda")
    M.moe_route(s, xd, Rd, bd, idx, gate, counts, ws)
    assert M.moe_read_device_status(ws) == 0
    return idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy()


def _check_route(cfg, r, idx, gate, counts):
    np.testing.assert_array_equal(idx, r["idx"])
    np.testing.assert_array_equal(counts, r["counts"])
    np.testing.assert_allclose(gate, r["gate"], rtol=0, atol=1e-6)


def test_device_generator_matches_host():
    torch = _torch()
    from synth import device as sdev
    cfg = CONFIGS[1]
    w = sdev.expert_weights_bf16(cfg, 0, "w2")
    for e in (0, 17, cfg.N):
        host = gen.make_expert_weight(cfg, 0, "w2", e)
        dev = w[e].float().cpu().numpy()
        np.testing.assert_array_equal(dev, host)


@pytest.mark.parametrize("cfg_id", [0, 1])
def test_route_bitexact(M, cfg_id):
    cfg = CONFIGS[cfg_id]
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    _check_route(cfg, r, *_run_route(M, cfg, x, R, b))


def test_route_ragged_and_hot_expert(M):
    """T not a multiple of the 32-token tile; a +10 bias forces one expert."""
    cfg = CONFIGS[1].with_(T=1000)
    R = gen.make_router(cfg)
    b = gen.make_bias(cfg).copy()
    b[13] = 10.0
    x, _ = S.tie_free_x(cfg, R, b)
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    assert r["counts"][13] == cfg.T
    _check_route(cfg, r, *_run_route(M, cfg, x, R, b))


def _layer(M, cfg, x, R, b, W):
    torch = _torch()
    s = S.moe_shape(cfg)
    layer = M.MoELayer(s, torch.from_numpy(R).cuda(),
                       torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                       W["w13_scales"], W["w2_scales"], gamma=cfg.gamma)
    xd = S.to_dev_x(x, cfg)
    return layer, xd


def _check_dispatch(layer, r, xd=None):
    """offsets, perm_tok and slot equal the oracle's; with the device input
    xd, every dispatched row (bf16 or fp32) is its token's row bit for bit."""
    import torch
    d = oracle.dispatch(r["idx"], layer.shape.N)
    np.testing.assert_array_equal(layer.offsets.cpu().numpy(), d["offsets"])
    np.testing.assert_array_equal(layer.perm_tok.cpu().numpy(), d["perm_tok"])
    np.testing.assert_array_equal(layer.slot.cpu().numpy(), d["slot"])
    if xd is not None and layer.x_perm is not None and layer.x_perm.dtype == xd.dtype:
        pt = torch.from_numpy(d["perm_tok"].astype(np.int64)).to(xd.device)
        assert torch.equal(layer.x_perm[:len(pt)], xd[pt])
    return d


def test_tiny_fp32_layer_full(M):
    """The tiny fp32 layer end to end, every output element."""
    cfg = CONFIGS[0]
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    layer, xd = _layer(M, cfg, x, R, b, W)
    y = layer.forward(xd).cpu().numpy()
    ref = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K)
    r = ref["route"]
    _check_route(cfg, r, layer.topk_idx.cpu().numpy(), layer.topk_gate.cpu().numpy(),
                 layer.counts.cpu().numpy())
    _check_dispatch(layer, r, xd)
    err = S.rel_fro(y, ref["y"])
    assert err <= TOL["fp32"], err
    nb = oracle.bias_update(b, r["counts"], cfg.T, cfg.K, cfg.gamma)
    np.testing.assert_array_equal(layer.bias.cpu().numpy(), nb)
    assert layer.device_status() == 0


def _small_bf16(T=1000):
    # several m-tiles per expert with a ragged tail, 2 n-tiles in GEMM1
    return CONFIGS[1].with_(T=T, d=256, N=8, K=2, G=2, topG=1, f=256)


@pytest.mark.parametrize("T", [1000, 129, 1])
def test_small_bf16_layer_full(M, T):
    cfg = _small_bf16(T)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    layer, xd = _layer(M, cfg, x, R, b, W)
    y = layer.forward(xd).float().cpu().numpy()
    ref = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K,
                             h_round="bf16")
    r = ref["route"]
    _check_route(cfg, r, layer.topk_idx.cpu().numpy(), layer.topk_gate.cpu().numpy(),
                 layer.counts.cpu().numpy())
    d = _check_dispatch(layer, r, xd)
    # per-expert rows of the grouped GEMM output
    get = S.host_weights(cfg)
    yp = layer.y_perm.float().cpu().numpy()
    for e in range(cfg.N):
        a, z = d["offsets"][e], d["offsets"][e + 1]
        if z == a:
            continue
        want = oracle.swiglu_expert(x[d["perm_tok"][a:z]], *get(e), h_round="bf16")
        assert S.rel_fro(yp[a:z], want) <= TOL["bf16"], e
    ysh = layer.y_shared.float().cpu().numpy()
    assert S.rel_fro(ysh, oracle.swiglu_expert(x, *get(cfg.N), h_round="bf16")) <= TOL["bf16"]
    err = S.rel_fro(y, ref["y"])
    assert err <= TOL["bf16"], err
    assert layer.device_status() == 0


@pytest.mark.parametrize("T", [1000, 129, 1])
def test_gathered_expert_rows_bitexact(M, T):
    """moe_expert_ffn_gathered (GEMM1 gathers x rows through perm_tok, dispatch
    copies nothing) gives bit-identical expert outputs to the x_perm path, and
    the gathered layer matches the oracle."""
    torch = _torch()
    cfg = _small_bf16(T)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    layer, xd = _layer(M, cfg, x, R, b, W)
    layer.forward(xd, update_bias=False)
    s = layer.shape
    perm_tok, slot = torch.empty_like(layer.perm_tok), torch.empty_like(layer.slot)
    offsets = torch.empty_like(layer.offsets)
    yp, ysh = torch.empty_like(layer.y_perm), torch.empty_like(layer.y_shared)
    M.moe_dispatch(s, xd, layer.topk_idx, layer.counts, offsets, perm_tok, slot, None, None,
                   layer.ws)
    M.moe_expert_ffn_gathered(s, xd, perm_tok, offsets, layer.w13, layer.w2, yp, ysh, layer.ws)
    torch.cuda.synchronize()
    assert torch.equal(perm_tok, layer.perm_tok) and torch.equal(slot, layer.slot)
    assert torch.equal(yp, layer.y_perm)
    assert torch.equal(ysh, layer.y_shared)
    # the layer built to gather end to end, against the oracle
    lg = M.MoELayer(s, layer.router_w, torch.from_numpy(np.asarray(b, np.float32)).cuda(),
                    W["w13"], W["w2"], gamma=cfg.gamma, gather=True)
    assert lg.gather and lg.x_perm is None
    y = lg.forward(xd).float().cpu().numpy()
    ref = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K,
                             h_round="bf16")
    assert S.rel_fro(y, ref["y"]) <= TOL["bf16"]
    assert lg.device_status() == 0 and layer.device_status() == 0


def test_mid_bf16_layer_full(M):
    """The mid-size bf16 layer: full routing/dispatch and the output of every
    token."""
    torch = _torch()
    cfg = CONFIGS[1]
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    layer, xd = _layer(M, cfg, x, R, b, W)
    y = layer.forward(xd).float().cpu().numpy()
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    _check_route(cfg, r, layer.topk_idx.cpu().numpy(), layer.topk_gate.cpu().numpy(),
                 layer.counts.cpu().numpy())
    d = _check_dispatch(layer, r, xd)
    ref = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K,
                             h_round="bf16")
    err = S.rel_fro(y, ref["y"])
    assert err <= TOL["bf16"], err
    # every token on its own too: no row may hide behind the others
    row_err = np.linalg.norm(y - ref["y"], axis=1) / np.linalg.norm(ref["y"], axis=1)
    assert row_err.max() <= 3 * TOL["bf16"], row_err.max()
    assert layer.device_status() == 0
    del torch


# ---------------------------------------------------------------------------
# FP8-E4M3 layer
# ---------------------------------------------------------------------------

def _small_fp8(T=1000):
    return CONFIGS[3].with_(T=T, d=256, N=8, K=2, G=2, topG=1, f=256)


def test_fp8_weight_quantisation_bitexact(M):
    """Per-128x128-block E4M3 codes and fp32 scales of the packed W1/W3 and W2
    equal the oracle's quantisation of the same bf16 weights."""
    cfg = CONFIGS[3].with_(N=16)
    W = S.device_weights(cfg)
    q13 = W["w13"].view(__import__("torch").uint8).cpu().numpy()
    s13 = W["w13_scales"].cpu().numpy()
    q2 = W["w2"].view(__import__("torch").uint8).cpu().numpy()
    s2 = W["w2_scales"].cpu().numpy()
    get = S.host_weights(cfg)
    for e in (0, cfg.N):
        w1, w3, w2 = get(e)
        c1, sc1 = oracle.quant_blocks_128(w1)
        c3, sc3 = oracle.quant_blocks_128(w3)
        c2, sc2 = oracle.quant_blocks_128(w2)
        for j in range(cfg.f // 128):          # packed: W1 block j, then W3 block j
            np.testing.assert_array_equal(q13[e, 256 * j:256 * j + 128], c1[128 * j:128 * j + 128])
            np.testing.assert_array_equal(q13[e, 256 * j + 128:256 * j + 256],
                                          c3[128 * j:128 * j + 128])
            np.testing.assert_array_equal(s13[e, 2 * j], sc1[j])
            np.testing.assert_array_equal(s13[e, 2 * j + 1], sc3[j])
        np.testing.assert_array_equal(q2[e], c2)
        np.testing.assert_array_equal(s2[e], sc2)


@pytest.mark.parametrize("T", [1000, 1])
def test_small_fp8_layer_full(M, T):
    torch = _torch()
    cfg = _small_fp8(T)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    layer, xd = _layer(M, cfg, x, R, b, W)
    y = layer.forward(xd).float().cpu().numpy()
    ref = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K,
                             expert_fn=oracle.fp8_swiglu_expert)
    r = ref["route"]
    _check_route(cfg, r, layer.topk_idx.cpu().numpy(), layer.topk_gate.cpu().numpy(),
                 layer.counts.cpu().numpy())
    d = _check_dispatch(layer, r, xd)
    # dispatched rows are quantised per 1x128 tile exactly as the oracle does
    codes, scales = oracle.quant_rows_1x128(x[d["perm_tok"]])
    np.testing.assert_array_equal(layer.x_perm.view(torch.uint8).cpu().numpy(), codes)
    # scales are stored block-major, [d/128, T*K rounded up to 4]
    got = layer.x_perm_scales.cpu().numpy()
    assert got.shape == (cfg.d // 128, (cfg.T * cfg.K + 3) // 4 * 4)
    np.testing.assert_array_equal(got[:, :cfg.T * cfg.K], scales.T)
    get = S.host_weights(cfg)
    yp = layer.y_perm.float().cpu().numpy()
    for e in range(cfg.N):
        a, z = d["offsets"][e], d["offsets"][e + 1]
        if z == a:
            continue
        want = oracle.fp8_swiglu_expert(x[d["perm_tok"][a:z]], *get(e))
        assert S.rel_fro(yp[a:z], want) <= TOL["e4m3"], e
    err = S.rel_fro(y, ref["y"])
    assert err <= TOL["e4m3"], err
    assert layer.device_status() == 0


# ---------------------------------------------------------------------------
# degenerate and maximum-size routing / layer cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,G,topG", [
    (8, 8, 1, 1),       # K = N: every expert on every token
    (16, 4, 16, 4),     # one expert per group: group score = that expert's biased score
    (256, 32, 8, 4),    # the largest K and N the kernels take
    (64, 1, 8, 1),      # K = 1, a single group kept
])
def test_route_degenerate_and_max(M, N, K, G, topG):
    cfg = CONFIGS[1].with_(T=777, d=256, N=N, K=K, G=G, topG=topG, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    _check_route(cfg, r, *_run_route(M, cfg, x, R, b))


@pytest.mark.parametrize("N,K,T", [(64, 6, 1000), (256, 8, 777), (256, 13, 500), (16, 16, 97)])
def test_softmax_route_baseline(M, N, K, T):
    """moe_route_softmax against the oracle's softmax top-K: indices and
    counts bit-exact, gates within fp32 rounding, per-expert probability sums
    and the balance statistic within fp32 summation error."""
    torch = _torch()
    cfg = CONFIGS[1].with_(T=T, d=256, N=N, K=K, G=1, topG=1, f=256)
    R = gen.make_router(cfg)
    x, _ = S.tie_free_x(cfg, R, None,
                        margins=lambda xr: oracle.route_softmax_margins(xr, R, cfg.K))
    ref = oracle.route_softmax(x, R, cfg.K)
    s = S.moe_shape(cfg)
    idx = torch.empty(s.T, s.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(s.T, s.K, dtype=torch.float32, device="cuda")
    counts = torch.empty(s.N, dtype=torch.int32, device="cuda")
    psum = torch.empty(s.N, dtype=torch.float32, device="cuda")
    ws = torch.zeros(M.workspace_size(s), dtype=torch.uint8, device="cuda")
    M.moe_route_softmax(s, S.to_dev_x(x, cfg), torch.from_numpy(R).cuda(), idx, gate, counts,
                        psum, ws)
    assert M.moe_read_device_status(ws) == 0
    _check_route(cfg, ref, idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy())
    ps = psum.cpu().numpy()
    np.testing.assert_allclose(ps, ref["prob_sum"], rtol=1e-5, atol=1e-6 * T)
    assert abs(ps.sum() - T) <= 1e-4 * T
    got = oracle.balance_loss(counts.cpu().numpy(), ps, T, K)
    assert got == pytest.approx(oracle.balance_loss(ref["counts"], ref["prob_sum"], T, K),
                                rel=1e-5)


def test_layer_k13_same_node_budget(M):
    """K = 13 experts per token within the same 4 of 8 groups, the larger
    expert count the pages give for the same communication budget."""
    cfg = CONFIGS[1].with_(T=600, d=256, N=256, K=13, G=8, topG=4, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    layer, xd = _layer(M, cfg, x, R, b, W)
    y = layer.forward(xd).float().cpu().numpy()
    ref = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K,
                             h_round="bf16")
    _check_route(cfg, ref["route"], layer.topk_idx.cpu().numpy(),
                 layer.topk_gate.cpu().numpy(), layer.counts.cpu().numpy())
    _check_dispatch(layer, ref["route"], xd)
    assert S.rel_fro(y, ref["y"]) <= TOL["bf16"]
    assert layer.device_status() == 0


def test_layer_all_experts_every_token(M):
    """K = N: each expert's group holds every token (several m-tiles each)."""
    cfg = CONFIGS[1].with_(T=300, d=256, N=4, K=4, G=1, topG=1, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    layer, xd = _layer(M, cfg, x, R, b, W)
    y = layer.forward(xd).float().cpu().numpy()
    ref = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K,
                             h_round="bf16")
    assert np.all(layer.counts.cpu().numpy() == cfg.T)
    _check_dispatch(layer, ref["route"], xd)
    assert S.rel_fro(y, ref["y"]) <= TOL["bf16"]
    assert layer.device_status() == 0


def test_layer_with_idle_experts(M):
    """Biases push all tokens into two groups, so most experts get no rows."""
    cfg = CONFIGS[1].with_(T=500, d=256, N=32, K=2, G=8, topG=2, f=256)
    R = gen.make_router(cfg)
    b = gen.make_bias(cfg).copy()
    b[:8] += 0.5                                    # groups 0 and 1 win every token
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    layer, xd = _layer(M, cfg, x, R, b, W)
    y = layer.forward(xd).float().cpu().numpy()
    ref = oracle.moe_forward(x, R, b, S.host_weights(cfg), cfg.G, cfg.topG, cfg.K,
                             h_round="bf16")
    counts = layer.counts.cpu().numpy()
    assert counts[8:].sum() == 0 and counts.sum() == cfg.T * cfg.K
    _check_dispatch(layer, ref["route"], xd)
    assert S.rel_fro(y, ref["y"]) <= TOL["bf16"]
    assert layer.device_status() == 0
