"""Expert parallelism on the GPU: the row gather kernel, and the whole
expert-parallel forward on one rank.

With one rank (NCCL, world size 1) every collective is a copy to itself and
the regroup is the identity, so ExpertParallelMoE over the library's kernels
must reproduce MoELayer's output and bias bit for bit; this runs every
kernel and every collective call of the expert-parallel path.

With two ranks, two processes share the GPU and exchange through gloo: the
collectives run on the host, so no kernel of one rank ever waits on the
other's.  Each rank holds half of the routed experts; every row an expert
receives is computed by the same kernel as in the single-GPU layer, so each
rank's output must equal MoELayer's on that rank's batch bit for bit, the
regroup sends every row to exactly one rank, and both ranks end with the
bias the oracle's update gives for the two batches' summed counts.  The
exchange between ranks is also covered on CPU against the oracle
(tests/test_ep_cpu.py)."""
import os
import socket
import sys

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


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _two_rank_worker(rank, world, port, dtype, q, replicas=0):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import sparse_moe_layer_limited_b200 as M
    from sparse_moe_layer_limited_b200 import ep
    from synth import CONFIGS, gen
    from tests import support as S
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        cfg = CONFIGS[1].with_(T=300, d=256, N=16, K=4, G=4, topG=2, f=256, dtype=dtype)
        R, b = gen.make_router(cfg), gen.make_bias(cfg)
        if replicas:  # three hot experts, so that the placement makes replicas
            b = np.asarray(b, np.float32).copy()
            b[[1, 2, 9]] += np.float32(0.3)
        x, _ = S.tie_free_x(cfg, R, b, batch=rank)          # each rank its own batch
        W = S.device_weights(cfg)
        s = S.moe_shape(cfg)
        Rd = torch.from_numpy(R).cuda()
        bd = torch.from_numpy(np.asarray(b, np.float32)).cuda()
        lo, hi = ep.expert_range(cfg.N, world, rank)
        keep = list(range(lo, hi)) + [cfg.N]                # this rank's experts + shared
        w13 = W["w13"][keep].contiguous()
        w2 = W["w2"][keep].contiguous()
        ops = ep.LibraryOps(s, ep.local_shape(s, world, replicas), Rd, bd.clone(), w13, w2,
                            replicas=replicas)
        epl = ep.ExpertParallelMoE(ops, cfg.N, gamma=cfg.gamma, redundant=replicas,
                                   replan_every=1 if replicas else 0)
        layer = M.MoELayer(s, Rd, bd.clone(), W["w13"], W["w2"], gamma=cfg.gamma)
        xd = S.to_dev_x(x, cfg)
        out = dict(equal=[], recv=[], counts=None, bias=None, hosted=None)
        for step in range(2):                 # step 1 routes with the updated bias
            layer.bias.copy_(ops.bias)
            y_ep = epl.forward(xd).clone()
            y_ref = layer.forward(xd, update_bias=False).clone()
            torch.cuda.synchronize()
            out["equal"].append(bool(torch.equal(y_ep, y_ref)))
            out["recv"].append(sum(epl.last_plan["recv_splits"]))
            if step == 0:
                out["counts"] = layer.counts.cpu().numpy().astype(np.int64)
                out["bias"] = ops.bias.cpu().numpy()
                out["hosted"] = epl.hosted
        out["status"] = [int(layer.device_status()), int(M.moe_read_device_status(ops.ws)),
                         int(M.moe_read_device_status(ops.ws_loc))]
        q.put((rank, out))
    except Exception as e:  # report instead of leaving the parent's queue read to time out
        q.put((rank, dict(error=repr(e))))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype,replicas", [("bf16", 0), ("fp32", 0), ("bf16", 2)])
def test_expert_parallel_two_ranks_one_gpu(dtype, replicas):
    """replicas=2: after the first step the three hot experts (and one more)
    get copies on the other rank, so the second step splits their rows
    between two GPUs' worth of slots and moves their weights first."""
    import oracle
    import torch.multiprocessing as mp
    from sparse_moe_layer_limited_b200 import ep
    from synth import CONFIGS
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_two_rank_worker, args=(r, 2, port, dtype, q, replicas))
             for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = dict(q.get(timeout=600) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=120)
    for r in (0, 1):
        assert "error" not in res[r], res[r]
        assert res[r]["equal"] == [True, True], res[r]["equal"]
        assert res[r]["status"] == [0, 0, 0]
    for p in procs:
        assert p.exitcode == 0
    cfg = CONFIGS[1].with_(T=300, d=256, N=16, K=4, G=4, topG=2, f=256, dtype=dtype)
    for step in (0, 1):                               # every routed row went to one rank
        assert res[0]["recv"][step] + res[1]["recv"][step] == 2 * cfg.T * cfg.K
    b0 = gen.make_bias(cfg)
    if replicas:
        b0 = np.asarray(b0, np.float32).copy()
        b0[[1, 2, 9]] += np.float32(0.3)
        placed = res[0]["hosted"]
        assert placed == res[1]["hosted"]
        assert placed == ep.place_redundant(res[0]["counts"] + res[1]["counts"], cfg.N, 2, replicas)
        assert all(e >= 0 for h in placed for e in h[cfg.N // 2:])
    want_b = oracle.bias_update(b0, res[0]["counts"] + res[1]["counts"], 2 * cfg.T, cfg.K,
                                cfg.gamma)
    np.testing.assert_array_equal(res[0]["bias"], want_b)
    np.testing.assert_array_equal(res[1]["bias"], want_b)
