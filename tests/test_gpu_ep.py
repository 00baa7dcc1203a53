"""Expert parallelism on the GPU: the row gather kernel, and the whole
expert-parallel forward on one rank.

With one rank (NCCL, world size 1) every collective is a copy to itself and
the regroup is the identity, so ExpertParallelMoE over the library's kernels
must reproduce MoELayer's output and bias bit for bit; this runs every
kernel and every collective call of the expert-parallel path.  The exchange
between two ranks is covered on CPU (tests/test_ep_cpu.py)."""
import socket

import numpy as np
import pytest

from synth import CONFIGS, gen
from tests import support as S

pytestmark = pytest.mark.gpu


def test_gather_rows_matches_numpy():
    import torch
    import sparse_moe_layer_limited_b200 as M
    g = torch.Generator(device="cuda").manual_seed(3)
    for dtype, d in ((torch.bfloat16, 256), (torch.float32, 72), (torch.uint8, 7168)):
        src = torch.randint(0, 255, (1000, d), generator=g, device="cuda").to(dtype)
        idx = torch.randint(0, 1000, (1537,), generator=g, device="cuda", dtype=torch.int32)
        idx[5], idx[9] = -1, 1000                       # out of range: zero rows
        dst = torch.full((1537, d), 7, dtype=dtype, device="cuda")
        M.moe_gather_rows(src, idx, dst)
        torch.cuda.synchronize()
        i = idx.cpu().numpy()
        want = np.zeros((1537, d), dtype=np.float64)
        okr = (i >= 0) & (i < 1000)
        want[okr] = src.cpu().double().numpy()[i[okr]]
        np.testing.assert_array_equal(dst.cpu().double().numpy(), want)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_parallel_single_rank_equals_layer():
    import torch
    import torch.distributed as dist
    import sparse_moe_layer_limited_b200 as M
    from sparse_moe_layer_limited_b200 import ep
    cfg = CONFIGS[1].with_(T=300, d=256, N=16, K=4, G=4, topG=2, f=256)
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    x, _ = S.tie_free_x(cfg, R, b)
    W = S.device_weights(cfg)
    s = S.moe_shape(cfg)
    Rd = torch.from_numpy(R).cuda()
    layer = M.MoELayer(s, Rd, torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"],
                       W["w2"], gamma=cfg.gamma)
    xd = S.to_dev_x(x, cfg)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        ops = ep.LibraryOps(s, ep.local_shape(s, 1), Rd,
                            torch.from_numpy(np.asarray(b, np.float32)).cuda(), W["w13"], W["w2"])
        epl = ep.ExpertParallelMoE(ops, cfg.N, gamma=cfg.gamma)
        for step in range(3):                          # the bias moves between steps
            y_ep = epl.forward(xd).clone()
            y_ref = layer.forward(xd).clone()
            torch.cuda.synchronize()
            assert torch.equal(y_ep, y_ref), step
            assert torch.equal(ops.bias, layer.bias), step
        assert layer.device_status() == 0
        assert M.moe_read_device_status(ops.ws) == 0
        assert M.moe_read_device_status(ops.ws_loc) == 0
    finally:
        dist.destroy_process_group()
