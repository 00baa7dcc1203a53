"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (the MoELayer / C-ABI calls on one stream).

* V3 bf16 layer: routing for all 8192 tokens over 10 passes with the bias
  update between passes (indices, counts and bias bit-exact every pass), then
  the rows of every expert's ragged last m-tile and the whole output of 64
  tokens against the oracle.
* V3 FP8 layer (T=16384): routing bit-exact, dispatched E4M3 codes and scales
  bit-exact on sampled rows, then the same tail-row and 64-token checks
  against the oracle's E4M3 emulation.
* Decode workload (256 tokens, Zipf expert popularity): 200 route + bias
  update steps bit-exact, with a full forward every 20 steps checked on all
  tokens at two of them.
"""
import numpy as np
import pytest

import oracle
from synth import CONFIGS, gen
from tests import support as S

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def M():
    import sparse_moe_layer_limited_b200 as M
    return M


def _check_tails_and_tokens(layer, x, r, d, cfg, y, kind, tol, n_tokens=64):
    """Expert rows against the oracle, run per expert in a process pool:
    * for every routed expert, the rows of its last (ragged) m-tile: the
      GPU's y_perm rows within `tol` (rel-Frobenius) of the oracle expert;
    * for 64 sampled tokens (the last dispatched token of every 16th expert,
      the last token, and a low-fan-out rest), their K routed rows and their
      shared-expert row, combined with the oracle's gates into y: within
      `tol` of the GPU's y."""
    import torch
    offs, perm, slot, idx = d["offsets"], d["perm_tok"], d["slot"], r["idx"]
    must = [int(perm[offs[e + 1] - 1]) for e in range(0, cfg.N, 16) if offs[e + 1] > offs[e]]
    tokens, _ = S.greedy_token_sample(idx, n_tokens, must=must + [cfg.T - 1])
    rows = {e: S.tail_tile_rows(offs, e) for e in range(cfg.N)}
    for t in tokens:
        for k in range(cfg.K):
            e = int(idx[t, k])
            rows[e] = np.union1d(rows[e], [int(slot[t, k])])
    jobs = {e: x[perm[rw]].astype(np.float32) for e, rw in rows.items() if len(rw)}
    jobs[cfg.N] = x[tokens].astype(np.float32)          # shared expert on the sampled tokens
    want = S.expert_outputs_parallel(cfg, jobs, kind)
    every = np.concatenate([rw for rw in rows.values() if len(rw)])
    got_rows = layer.y_perm[torch.from_numpy(every).cuda()].float().cpu().numpy()
    where = {}
    pos = 0
    for e, rw in rows.items():
        if len(rw):
            where[e] = (rw, got_rows[pos:pos + len(rw)])
            pos += len(rw)
    for e, (rw, got) in where.items():
        tail = S.tail_tile_rows(offs, e)
        sel = np.isin(rw, tail)
        assert S.rel_fro(got[sel], want[e][sel]) <= tol, ("expert tail rows", e)
    # the sampled tokens' outputs from the oracle's expert rows and gates
    routed = {}
    for e, (rw, _) in where.items():
        for j, row in enumerate(rw):
            routed[(int(perm[row]), e)] = want[e][j]
    ref = oracle.combine(want[cfg.N], routed, idx, r["gate"], tokens)
    err = S.rel_fro(y.float().cpu().numpy()[tokens], ref)
    assert err <= tol, err


def _layer(M, cfg, R, b, W):
    import torch
    return M.MoELayer(S.moe_shape(cfg), torch.from_numpy(R).cuda(),
                      torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"],
                      W["w13_scales"], W["w2_scales"], gamma=cfg.gamma)


def test_v3_bf16_passes_and_sampled_outputs(M):
    import torch
    cfg = CONFIGS[2]
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    W = S.device_weights(cfg)
    layer = _layer(M, cfg, R, b, W)
    x = gen.make_x(cfg)
    redrawn = []
    for p in range(cfg.passes):
        x, n = S.tie_free_x(cfg, R, b, batch=0, x=x)
        redrawn.append(n)
        xd = S.to_dev_x(x, cfg)
        y = layer.forward(xd)                      # route, dispatch, experts, combine, bias
        r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
        np.testing.assert_array_equal(layer.topk_idx.cpu().numpy(), r["idx"])
        np.testing.assert_array_equal(layer.counts.cpu().numpy(), r["counts"])
        np.testing.assert_allclose(layer.topk_gate.cpu().numpy(), r["gate"], rtol=0, atol=1e-6)
        b_next = oracle.bias_update(b, r["counts"], cfg.T, cfg.K, cfg.gamma)
        np.testing.assert_array_equal(layer.bias.cpu().numpy(), b_next)
        if p == cfg.passes - 1:
            d = oracle.dispatch(r["idx"], cfg.N)
            np.testing.assert_array_equal(layer.offsets.cpu().numpy(), d["offsets"])
            np.testing.assert_array_equal(layer.perm_tok.cpu().numpy(), d["perm_tok"])
            np.testing.assert_array_equal(layer.slot.cpu().numpy(), d["slot"])
            # every dispatched row is its token's row, bit for bit (65,536 rows)
            pt = torch.from_numpy(d["perm_tok"].astype(np.int64)).to(xd.device)
            assert torch.equal(layer.x_perm[:len(pt)], xd[pt])
            # every expert's ragged last m-tile, and the whole output of 64 tokens
            _check_tails_and_tokens(layer, x, r, d, cfg, y, "bf16", 1e-2)
        b = b_next
    assert layer.device_status() == 0
    print("near-tie rows re-drawn per pass:", redrawn)
    del torch


def test_v3_bf16_gathered_rows_bitexact(M):
    """At the full V3 size the gathered expert GEMMs (no x_perm) reproduce the
    x_perm path's expert outputs bit for bit."""
    import torch
    cfg = CONFIGS[2]
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    W = S.device_weights(cfg)
    layer = _layer(M, cfg, R, b, W)
    x, _ = S.tie_free_x(cfg, R, b)
    xd = S.to_dev_x(x, cfg)
    layer.forward(xd, update_bias=False)
    s = layer.shape
    yp, ysh = torch.empty_like(layer.y_perm), torch.empty_like(layer.y_shared)
    M.moe_expert_ffn_gathered(s, xd, layer.perm_tok, layer.offsets, layer.w13, layer.w2, yp, ysh,
                              layer.ws)
    torch.cuda.synchronize()
    assert torch.equal(yp, layer.y_perm)
    assert torch.equal(ysh, layer.y_shared)
    assert layer.device_status() == 0


def test_decode_zipf_200_steps(M):
    import torch
    cfg = CONFIGS[4]
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    W = S.device_weights(cfg)
    layer = _layer(M, cfg, R, b, W)
    loads = []
    checked = 0
    for step in range(cfg.steps):
        x, _ = S.tie_free_x(cfg, R, b, batch=step)
        xd = S.to_dev_x(x, cfg)
        forward = step % cfg.forward_every == 0
        if forward:
            y = layer.forward(xd, update_bias=False)
        else:
            layer.route(xd)
        r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
        np.testing.assert_array_equal(layer.topk_idx.cpu().numpy(), r["idx"])
        np.testing.assert_array_equal(layer.counts.cpu().numpy(), r["counts"])
        if forward and step in (0, 100):
            ref = oracle.moe_forward(x, R, b, S.streaming_weights(cfg), cfg.G, cfg.topG, cfg.K,
                                     h_round="bf16")
            err = S.rel_fro(y.float().cpu().numpy(), ref["y"])
            assert err <= 1e-2, (step, err)
            checked += 1
        M.moe_bias_update(layer.shape, layer.counts, layer.bias, cfg.gamma)
        b = oracle.bias_update(b, r["counts"], cfg.T, cfg.K, cfg.gamma)
        np.testing.assert_array_equal(layer.bias.cpu().numpy(), b)
        loads.append(r["counts"].max() / r["counts"].mean())
    assert checked == 2
    assert layer.device_status() == 0
    # max/mean load is reported, not asserted: at gamma = 1e-3 the bias moves at
    # most 0.2 in score units over 200 steps
    print("max/mean load: first", loads[0], "last", loads[-1])
    del torch


def test_v3_fp8_routing_and_sampled_outputs(M):
    """The V3 layer with E4M3 expert GEMMs at T=16384: routing bit-exact for all
    tokens, dispatched-row quantisation bit-exact on sampled rows, outputs of
    sampled tokens within rel-Frobenius 2e-2 of the oracle's FP8 emulation."""
    import torch
    cfg = CONFIGS[3]
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    W = S.device_weights(cfg)
    layer = _layer(M, cfg, R, b, W)
    x, _ = S.tie_free_x(cfg, R, b)
    y = layer.forward(S.to_dev_x(x, cfg))
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    np.testing.assert_array_equal(layer.topk_idx.cpu().numpy(), r["idx"])
    np.testing.assert_array_equal(layer.counts.cpu().numpy(), r["counts"])
    d = oracle.dispatch(r["idx"], cfg.N)
    np.testing.assert_array_equal(layer.perm_tok.cpu().numpy(), d["perm_tok"])
    rows = np.random.default_rng(1).choice(cfg.T * cfg.K, 512, replace=False)
    codes, scales = oracle.quant_rows_1x128(x[d["perm_tok"][rows]])
    np.testing.assert_array_equal(layer.x_perm.view(torch.uint8)[rows].cpu().numpy(), codes)
    # scales are block-major [d/128, T*K rounded up to 4]; index on the host
    np.testing.assert_array_equal(layer.x_perm_scales.cpu().numpy()[:, rows].T, scales)
    # every expert's ragged last m-tile, and the whole output of 64 tokens
    _check_tails_and_tokens(layer, x, r, d, cfg, y, "fp8", 2e-2)
    assert layer.device_status() == 0
