"""The workspace-free dispatch entry point (moe_dispatch_noalloc).

Some callers cannot allocate device memory at the moment they call the
layer (for example while a framework forbids new allocations, or when a host
application passes only its own input and output buffers), so they cannot
supply the workspace moe_dispatch needs.  moe_dispatch_noalloc keeps that
scratch in a fixed static device array instead.  These tests call it
through the C ABI and require the same results as moe_dispatch on two calls
in a row with different shapes (the shared array keeps the previous call's
contents), and check that shapes beyond the array are refused up front.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import oracle
from synth import CONFIGS, gen
from tests import support as S


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import sparse_moe_layer_limited_b200 as M
    f = M.lib()
    fake = ctypes.c_void_p(1 << 20)                                # never dereferenced
    for T in (20000, 16385):       # at N = 256 the array holds the tables of T <= 16384
        big = M.shape(T, 256, 256, 8, 8, 4, 256, M.DTYPE_BF16)
        rc = f.moe_dispatch_noalloc(ctypes.byref(big), fake, fake, fake, fake, fake, fake, fake,
                                    None, None)
        assert rc == M._lib.ERR_WORKSPACE, T
    ok = M.shape(1000, 256, 8, 2, 2, 1, 256, M.DTYPE_BF16)
    assert f.moe_dispatch_noalloc(ctypes.byref(ok), None, fake, fake, fake, fake, fake, fake,
                                  None, None) == M._lib.ERR_ARG


def _inputs(cfg):
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    r = oracle.route(x, R, b, cfg.G, cfg.topG, cfg.K)
    return x, r


def _dispatch_both(M, cfg, x, r, slots_only=False, statuses=None):
    """moe_dispatch (with a workspace) and moe_dispatch_noalloc on the same
    inputs, outputs pre-filled with -7; with `statuses` a list, the
    workspace call's device status word is appended to it."""
    import torch
    s = S.moe_shape(cfg)
    xd = S.to_dev_x(x, cfg)
    idx = torch.from_numpy(r["idx"].astype(np.int32)).cuda()
    counts = torch.from_numpy(r["counts"].astype(np.int32)).cuda()
    outs = []
    for which in ("ws", "noalloc"):
        off = torch.full((s.N + 1,), -7, dtype=torch.int32, device="cuda")
        perm = torch.full((s.T * s.K,), -7, dtype=torch.int32, device="cuda")
        slot = torch.full((s.T, s.K), -7, dtype=torch.int32, device="cuda")
        xp = torch.zeros(s.T * s.K, s.d, dtype=xd.dtype, device="cuda")
        xp_arg = None if slots_only else xp
        if which == "ws":
            ws = torch.zeros(M.workspace_size(s), dtype=torch.uint8, device="cuda")
            M.moe_dispatch(s, xd, idx, counts, off, perm, slot, xp_arg, None, ws)
            if statuses is not None:
                statuses.append(M.moe_read_device_status(ws))
        else:
            rc = M.lib().moe_dispatch_noalloc(
                ctypes.byref(s), ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
                ctypes.c_void_p(counts.data_ptr()), ctypes.c_void_p(off.data_ptr()),
                ctypes.c_void_p(perm.data_ptr()), ctypes.c_void_p(slot.data_ptr()),
                None if slots_only else ctypes.c_void_p(xp.data_ptr()), None,
                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
            assert rc == 0, M.status_string(rc)
        torch.cuda.synchronize()
        outs.append((off.cpu().numpy(), perm.cpu().numpy(), slot.cpu().numpy(),
                     xp.float().cpu().numpy()))
    return outs


@pytest.mark.gpu
def test_noalloc_matches_workspace_dispatch_twice():
    import sparse_moe_layer_limited_b200 as M
    cases = [CONFIGS[1], CONFIGS[1].with_(T=1000, d=256, N=8, K=2, G=2, topG=1, f=256)]
    for cfg in cases:                      # two calls in a row, different shapes
        x, r = _inputs(cfg)
        (o1, p1, s1, x1), (o2, p2, s2, x2) = _dispatch_both(M, cfg, x, r)
        # integer outputs bit-exact; the gathered rows are copies, so exact too
        np.testing.assert_array_equal(o2, o1)
        np.testing.assert_array_equal(p2, p1)
        np.testing.assert_array_equal(s2, s1)
        np.testing.assert_array_equal(x2, x1)
        d = oracle.dispatch(r["idx"], cfg.N)
        np.testing.assert_array_equal(o2, d["offsets"])
        np.testing.assert_array_equal(p2, d["perm_tok"])


@pytest.mark.gpu
def test_noalloc_at_its_largest_shape_and_slots_only():
    """T = 16384 at N = 256 is the largest shape the array holds (1 MiB of
    tables); and with x_perm NULL only offsets, perm_tok and slot are written,
    as with moe_dispatch."""
    import sparse_moe_layer_limited_b200 as M
    big = CONFIGS[1].with_(T=16384, d=256, N=256, K=8, G=8, topG=4, f=256)
    small = CONFIGS[1].with_(T=300, d=256, N=16, K=4, G=4, topG=2, f=256)
    for cfg, slots_only in ((big, False), (small, True)):
        x, r = _inputs(cfg)
        (o1, p1, s1, x1), (o2, p2, s2, x2) = _dispatch_both(M, cfg, x, r, slots_only)
        np.testing.assert_array_equal(o2, o1)
        np.testing.assert_array_equal(p2, p1)
        np.testing.assert_array_equal(s2, s1)
        np.testing.assert_array_equal(x2, x1)
        d = oracle.dispatch(r["idx"], cfg.N)
        np.testing.assert_array_equal(o2, d["offsets"])
        np.testing.assert_array_equal(p2, d["perm_tok"])
        np.testing.assert_array_equal(s2, d["slot"])
        if slots_only:
            assert not x2.any()            # the rows were not copied


MOE_DEV_BAD_INDEX = 4  # the device status bit for an expert index outside [0, N)


@pytest.mark.gpu
def test_noalloc_bad_expert_index_stays_in_bounds():
    """One (token, k) pair names expert N, outside [0, N).  moe_dispatch
    reports it in its workspace status; moe_dispatch_noalloc, whose status
    word cannot be read back, must still write only in bounds: both leave
    that pair's slot untouched (-7) and place no row for it, and every other
    pair's slot and row, perm_tok and the offsets agree between the two."""
    import sparse_moe_layer_limited_b200 as M
    cfg = CONFIGS[1].with_(T=1000, d=256, N=8, K=2, G=2, topG=1, f=256)
    x, r = _inputs(cfg)
    idx = r["idx"].astype(np.int32).copy()
    counts = r["counts"].astype(np.int64).copy()
    t_bad, k_bad = 3, 1
    counts[idx[t_bad, k_bad]] -= 1         # counts describe the valid pairs only
    idx[t_bad, k_bad] = cfg.N
    statuses = []
    (o1, p1, s1, x1), (o2, p2, s2, x2) = _dispatch_both(M, cfg, x, dict(r, idx=idx, counts=counts),
                                                        statuses=statuses)
    assert statuses[0] & MOE_DEV_BAD_INDEX
    TK1 = cfg.T * cfg.K - 1                # rows placed: every pair but the bad one
    np.testing.assert_array_equal(o2, o1)
    assert o1[cfg.N] == TK1
    np.testing.assert_array_equal(p2[:TK1], p1[:TK1])
    assert p1[TK1] == -7 and p2[TK1] == -7  # the row past the placed ones is not written
    np.testing.assert_array_equal(s2, s1)
    assert s1[t_bad, k_bad] == -7 and s2[t_bad, k_bad] == -7
    np.testing.assert_array_equal(x2[:TK1], x1[:TK1])
    np.testing.assert_array_equal(x1[:TK1], x[p1[:TK1]].astype(np.float32))
