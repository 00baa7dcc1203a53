"""Expert parallelism inside one node, on CPU with the gloo backend.

The exchange (``ExpertParallelMoE.forward``: the all-to-all of the counts,
the all-to-all of the dispatched rows, the regroup by local expert, the
reverse all-to-all, the all-reduce of the counts before the bias update)
runs for real between two ranks; each rank's own steps (route, dispatch, the
expert FFN on the rows it holds, combine, bias update) are done here with
the float64 oracle.  Each rank's output must equal the oracle's whole-layer
forward of that rank's batch, and both ranks must end with the bias the
oracle's update gives for the two batches' summed counts.  The planning
tables are also checked on their own.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg():
    from synth import CONFIGS
    return CONFIGS[0].with_(T=48, d=64, N=16, K=4, G=4, topG=2, f=32)


class OracleOps:
    """A rank's own steps in float64 with the oracle (test infrastructure);
    same interface as sparse_moe_layer_limited_b200.ep.LibraryOps."""

    def __init__(self, cfg, router, bias, get, lo, hi, cap):
        self.cfg, self.R, self.b, self.get, self.lo, self.hi = cfg, router, bias.copy(), get, lo, hi
        self.recv = torch.zeros(cap, cfg.d, dtype=torch.float64)
        self.y_perm = torch.zeros(cfg.T * cfg.K, cfg.d, dtype=torch.float64)
        self.capacity = cap

    def route_dispatch(self, x):
        import oracle
        c = self.cfg
        self.x = np.asarray(x, np.float64)
        self.r = oracle.route(self.x, self.R, self.b, c.G, c.topG, c.K)
        self.d = oracle.dispatch(self.r["idx"], c.N)
        x_perm = torch.from_numpy(self.x[self.d["perm_tok"]])
        return torch.from_numpy(self.r["counts"].astype(np.int32)), x_perm

    def set_plan(self, plan):
        self.plan = plan
        return len(plan["gather"])

    def experts(self, R, x):
        import oracle
        p = self.plan
        x_loc = self.recv[:R].numpy()[p["gather"]]
        y_loc = np.zeros_like(x_loc)
        offs = p["offsets"]
        for e in range(self.hi - self.lo):
            a, z = offs[e], offs[e + 1]
            if z > a:
                y_loc[a:z] = oracle.swiglu_expert(x_loc[a:z], *self.get(self.lo + e))
        self.y_shared = oracle.swiglu_expert(self.x, *self.get(self.cfg.N))
        out = torch.zeros_like(self.recv)
        out[:R] = torch.from_numpy(y_loc[p["scatter"]])
        return out

    def combine(self):
        y = self.y_shared.copy()
        yp = self.y_perm.numpy()
        for t in range(self.cfg.T):
            for k in range(self.cfg.K):
                y[t] += self.r["gate"][t, k] * yp[self.d["slot"][t, k]]
        return y

    def bias_update(self, counts_all, T_all, gamma):
        import oracle
        self.b = oracle.bias_update(self.b, counts_all.numpy(), T_all, self.cfg.K, gamma)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_moe_layer_limited_b200 import ep
    from synth import gen
    from tests import support as S
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = _cfg()
        R, b = gen.make_router(cfg), gen.make_bias(cfg)
        get = S.host_weights(cfg)
        x, _ = S.tie_free_x(cfg, R, b, batch=rank)            # each rank its own batch
        lo, hi = ep.expert_range(cfg.N, world, rank)
        ops = OracleOps(cfg, R, b, get, lo, hi, cap=cfg.T * min(32, cfg.N // world))
        layer = ep.ExpertParallelMoE(ops, cfg.N, gamma=cfg.gamma)
        y = layer.forward(x)
        want = oracle.moe_forward(x, R, b, get, cfg.G, cfg.topG, cfg.K)
        err = float(np.max(np.abs(y - want["y"])) / np.max(np.abs(want["y"])))
        q.put((rank, dict(err=err, counts=want["route"]["counts"], bias=ops.b,
                          recv=layer.last_plan["recv_splits"])))
    except Exception as e:  # report instead of hanging the other rank's queue read
        q.put((rank, dict(error=repr(e))))
        raise
    finally:
        dist.destroy_process_group()


def test_two_ranks_match_the_oracle_forward_and_bias():
    import oracle
    from synth import gen
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    for r in (0, 1):
        assert "error" not in res[r], res[r]
        assert res[r]["err"] <= 1e-12, res[r]["err"]
    for p in procs:
        assert p.exitcode == 0
    cfg = _cfg()
    b0 = gen.make_bias(cfg)
    counts = res[0]["counts"] + res[1]["counts"]
    want_b = oracle.bias_update(b0, counts, 2 * cfg.T, cfg.K, cfg.gamma)
    np.testing.assert_array_equal(res[0]["bias"], want_b)
    np.testing.assert_array_equal(res[1]["bias"], want_b)
    # every routed row went to exactly one rank
    assert sum(res[0]["recv"]) + sum(res[1]["recv"]) == 2 * cfg.T * cfg.K


@pytest.mark.parametrize("W,E,seed", [(2, 8, 0), (4, 3, 1), (8, 32, 2), (1, 5, 3)])
def test_regroup_plan_tables(W, E, seed):
    from sparse_moe_layer_limited_b200 import ep
    rng = np.random.default_rng(seed)
    cnt = rng.integers(0, 9, size=(W, E))
    cnt[0, 0] = 0                                      # an empty (src, expert) block
    p = ep.regroup_plan(cnt)
    R = int(cnt.sum())
    assert p["recv_splits"] == [int(v) for v in cnt.sum(axis=1)]
    np.testing.assert_array_equal(np.diff(p["offsets"]), cnt.sum(axis=0))
    assert sorted(p["gather"].tolist()) == list(range(R))
    np.testing.assert_array_equal(p["gather"][p["scatter"]], np.arange(R))
    # label every received row with (src, expert, rank within the block) and
    # check the expert-major order: experts ascending, then sources, then rank
    labels = []
    for s in range(W):
        for e in range(E):
            labels += [(e, s, i) for i in range(cnt[s, e])]
    regrouped = [labels[j] for j in p["gather"]]
    assert regrouped == sorted(labels)


def test_send_splits_and_expert_ranges():
    from sparse_moe_layer_limited_b200 import ep
    counts = np.arange(16)
    assert ep.send_splits(counts, 4) == [6, 22, 38, 54]
    assert [ep.expert_range(256, 8, r) for r in (0, 7)] == [(0, 32), (224, 256)]
    with pytest.raises(ValueError):
        ep.expert_range(10, 4, 0)
