"""Backward of COMBINE, of the gates and of DISPATCH (moe_combine_backward,
moe_route_backward, moe_dispatch_backward) against the oracle, step by step
on seeded inputs; then the whole layer backward (MoELayer.backward) against
oracle.moe_backward.

Routing and dispatch come from each side's own forward on the same tie-free
input (the slots are checked to be identical first); every other input of a
step is seeded and given to both sides as the same stored values."""
import numpy as np
import pytest

import oracle
from synth import CONFIGS, gen
from tests import support as S

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32": CONFIGS[0],
    "small_bf16": CONFIGS[1].with_(T=300, d=256, N=16, K=4, G=4, topG=2, f=256),
    # more than eight selected experts: the gate kernel's wide instantiation
    "k13_bf16": CONFIGS[1].with_(T=200, d=256, N=64, K=13, G=8, topG=4, f=256),
}


@pytest.fixture(scope="module")
def M():
    import sparse_moe_layer_limited_b200 as M
    return M


def _layer(M, cfg):
    import torch
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    s = S.moe_shape(cfg)
    layer = M.MoELayer(s, torch.from_numpy(R).cuda(),
                       torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                       gamma=cfg.gamma)
    xd = S.to_dev_x(x, cfg)
    layer.forward(xd, update_bias=False)
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    dsp = oracle.dispatch(r["idx"], cfg.N)
    torch.cuda.synchronize()
    assert np.array_equal(layer.slot.cpu().numpy(), dsp["slot"])
    assert np.array_equal(layer.topk_idx.cpu().numpy(), r["idx"])
    return dict(x=x, xd=xd, R=R, b=b, W=W, s=s, layer=layer, r=r, dsp=dsp)


def _rounding(cfg):
    return 2.0 ** -8 if cfg.dtype != "fp32" else 2.0 ** -23


@pytest.mark.parametrize("name", sorted(CASES))
def test_combine_backward_matches_oracle(M, name):
    import torch
    cfg = CASES[name]
    c = _layer(M, cfg)
    dy = gen.make_x(cfg, seed=41)
    yp = gen.make_x(cfg.with_(T=cfg.T * cfg.K), seed=42)
    dyd, ypd = S.to_dev_x(dy, cfg), S.to_dev_x(yp, cfg)
    dyp = torch.empty_like(ypd)
    dg = torch.empty(cfg.T, cfg.K, dtype=torch.float32, device="cuda")
    M.moe_combine_backward(c["s"], dyd, ypd, c["layer"].slot, c["layer"].topk_gate, dyp, dg)
    want = oracle.combine_backward(dy, yp, c["dsp"]["slot"], c["r"]["gate"])
    got = dyp.float().cpu().numpy()
    # one rounding of gate * dy; the fp32 gate is within 1e-6 of the oracle's
    assert np.all(np.abs(got - want["dy_perm"]) <= (_rounding(cfg) + 2e-6)
                  * np.abs(want["dy_perm"]) + 1e-30)
    # dy . y_perm: exact products, fp32 sum of d terms
    absd = np.abs(dy)[:, None, :] * np.abs(yp[c["dsp"]["slot"]])
    err = np.abs(dg.cpu().numpy() - want["dgate"])
    assert np.all(err <= 1e-5 * absd.sum(axis=2) + 1e-30)


@pytest.mark.parametrize("name", sorted(CASES))
def test_route_backward_matches_oracle(M, name):
    import torch
    cfg = CASES[name]
    c = _layer(M, cfg)
    dgate = np.random.default_rng(43).normal(size=(cfg.T, cfg.K)).astype(np.float32)
    dl = torch.empty(cfg.T, cfg.K, dtype=torch.float32, device="cuda")
    dxr = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    dR = torch.empty(cfg.N, cfg.d, dtype=torch.float32, device="cuda")
    L = c["layer"]
    M.moe_route_backward(c["s"], c["xd"], L.router_w, L.topk_idx, torch.from_numpy(dgate).cuda(),
                         L.offsets, L.perm_tok, L.slot, dl, dxr, dR)
    want = oracle.route_backward(c["x"], c["R"], c["r"]["idx"], dgate)
    assert S.rel_fro(dl.cpu().numpy(), want["dz"]) <= 1e-4
    assert S.rel_fro(dxr.cpu().numpy(), want["dx"]) <= 1e-4
    got_R = dR.cpu().numpy()
    assert S.rel_fro(got_R, want["drouter"]) <= 1e-4
    idle = np.bincount(c["r"]["idx"].ravel(), minlength=cfg.N) == 0
    assert np.all(got_R[idle] == 0.0)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("with_route", [True, False])
def test_dispatch_backward_matches_oracle(M, name, with_route):
    import torch
    cfg = CASES[name]
    c = _layer(M, cfg)
    dxp = gen.make_x(cfg.with_(T=cfg.T * cfg.K), seed=44)
    dxs = gen.make_x(cfg, seed=45)
    dxr = (np.random.default_rng(46).normal(size=(cfg.T, cfg.d)).astype(np.float32)
           if with_route else None)
    dt = torch.float32 if cfg.dtype == "fp32" else torch.bfloat16
    dx = torch.empty(cfg.T, cfg.d, dtype=dt, device="cuda")
    M.moe_dispatch_backward(c["s"], S.to_dev_x(dxp, cfg), S.to_dev_x(dxs, cfg), c["layer"].slot,
                            None if dxr is None else torch.from_numpy(dxr).cuda(), dx)
    slot = c["dsp"]["slot"]
    want = oracle.dispatch_backward(dxp, dxs, slot, dxr)
    absw = oracle.dispatch_backward(np.abs(dxp), np.abs(dxs), slot,
                                    None if dxr is None else np.abs(dxr))
    err = np.abs(dx.float().cpu().numpy() - want)
    assert np.all(err <= _rounding(cfg) * np.abs(want) + 1e-6 * absw + 1e-30)


def test_layer_backward_matches_oracle(M):
    """MoELayer.backward (14 launches: combine, expert input and weight
    gradients, gate and router, dispatch) against the oracle's layer backward
    on the same stored inputs.  The GPU rounds g, u, h, dg, du, y_perm and
    dy_perm to bf16 where they are stored; the oracle keeps float64, so the
    bound is a few bf16 roundings."""
    import torch
    cfg = CASES["small_bf16"]
    c = _layer(M, cfg)
    L = c["layer"]
    dy = gen.make_x(cfg, seed=47)
    w13t = torch.empty(cfg.N + 1, cfg.d, 2 * cfg.f, dtype=torch.bfloat16, device="cuda")
    w2t = torch.empty(cfg.N + 1, cfg.f, cfg.d, dtype=torch.bfloat16, device="cuda")
    M.moe_transpose_weights(c["s"], L.w13, L.w2, w13t, w2t)
    g = L.backward(c["xd"], S.to_dev_x(dy, cfg), w13t, w2t)
    torch.cuda.synchronize()
    assert L.backward_status() == 0
    want = oracle.moe_backward(c["x"], c["R"], c["b"], S.host_weights(cfg), cfg.G, cfg.topG,
                               cfg.K, dy, h_round="bf16")
    assert S.rel_fro(g["dgate"].cpu().numpy(), want["dgate"]) <= 2e-2
    assert S.rel_fro(g["dx"].float().cpu().numpy(), want["dx"]) <= 2e-2
    assert S.rel_fro(g["drouter"].cpu().numpy(), want["drouter"]) <= 3e-2
    dw2 = g["dw2"].float().cpu().numpy()
    for e in range(cfg.N + 1):
        assert S.rel_fro(dw2[e], want["dw"][e][2]) <= 2e-2, e
