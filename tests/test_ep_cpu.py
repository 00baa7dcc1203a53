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

With redundant experts, a first forward on a batch with hot experts is
followed by a re-placement from the node-wide counts and the real weight
exchange into the ranks' replica slots (float64 tensors here); the second
forward, whose rows for the replicated experts are split between copies,
must again equal the oracle's forward, and the replica slots must hold the
weights of their experts.
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
    same interface as sparse_moe_layer_limited_b200.ep.LibraryOps.  The
    rank's expert slots (primaries, then `replicas` replica slots, then the
    shared expert) hold W1/W3 in w13 [S + 1, 2, f, d] and W2 in w2 [S + 1,
    d, f]; replica slots start at zero and are filled by the exchange."""

    def __init__(self, cfg, router, bias, get, lo, hi, cap, replicas=0):
        self.cfg, self.R, self.b, self.get, self.lo, self.hi = cfg, router, bias.copy(), get, lo, hi
        self.recv = torch.zeros(cap, cfg.d, dtype=torch.float64)
        self.y_perm = torch.zeros(cfg.T * cfg.K, cfg.d, dtype=torch.float64)
        self.y_send = torch.zeros(cfg.T * cfg.K, cfg.d, dtype=torch.float64)
        self.capacity = cap
        S = (hi - lo) + replicas
        self.S = S
        self.w13 = torch.zeros(S + 1, 2, cfg.f, cfg.d, dtype=torch.float64)
        self.w2 = torch.zeros(S + 1, cfg.d, cfg.f, dtype=torch.float64)
        for i, e in enumerate(list(range(lo, hi)) + [None] * replicas + [cfg.N]):
            if e is not None:
                w1, w3, w2 = get(e)
                self.w13[i, 0] = torch.from_numpy(w1)
                self.w13[i, 1] = torch.from_numpy(w3)
                self.w2[i] = torch.from_numpy(w2)

    def gather_send(self, order):
        self.order = np.asarray(order)
        return torch.from_numpy(self.x_perm_np[self.order])

    def unsend(self, n):
        out = np.zeros_like(self.y_send.numpy()[:n])
        out[self.order] = self.y_send.numpy()[:n]
        self.y_perm[:n] = torch.from_numpy(out)

    def route_dispatch(self, x):
        import oracle
        c = self.cfg
        self.x = np.asarray(x, np.float64)
        self.r = oracle.route(self.x, self.R, self.b, c.G, c.topG, c.K)
        self.d = oracle.dispatch(self.r["idx"], c.N)
        self.x_perm_np = self.x[self.d["perm_tok"]]
        x_perm = torch.from_numpy(self.x_perm_np)
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
        for i in range(len(offs) - 1):
            a, z = offs[i], offs[i + 1]
            if z > a:  # slot i's weights as this rank holds them
                y_loc[a:z] = oracle.swiglu_expert(x_loc[a:z], self.w13[i, 0].numpy(),
                                                  self.w13[i, 1].numpy(), self.w2[i].numpy())
        S = self.S
        self.y_shared = oracle.swiglu_expert(self.x, self.w13[S, 0].numpy(), self.w13[S, 1].numpy(),
                                             self.w2[S].numpy())
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


def _skewed_bias(cfg):
    """The configuration's bias with three experts made hot (a Zipf-like
    skew of the routed load), so that the placement has replicas to make."""
    from synth import gen
    b = gen.make_bias(cfg).astype(np.float32).copy()
    b[[1, 2, 9]] += np.float32(0.3)
    return b


def _redundant_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_moe_layer_limited_b200 import ep
    from synth import gen
    from tests import support as S
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = _cfg()
        R, b = gen.make_router(cfg), _skewed_bias(cfg)
        get = S.host_weights(cfg)
        x, _ = S.tie_free_x(cfg, R, b, batch=rank)
        lo, hi = ep.expert_range(cfg.N, world, rank)
        r = 2
        cap = cfg.T * min(32, cfg.N // world + r)
        ops = OracleOps(cfg, R, b, get, lo, hi, cap, replicas=r)
        layer = ep.ExpertParallelMoE(ops, cfg.N, gamma=cfg.gamma, redundant=r, replan_every=1)
        y0 = layer.forward(x)                 # no replicas yet; then re-placed from its counts
        want0 = oracle.moe_forward(x, R, b, get, cfg.G, cfg.topG, cfg.K)
        b1 = ops.b.copy()
        x2, _ = S.tie_free_x(cfg, R, b1, batch=10 + rank)
        y1 = layer.forward(x2, update_bias=False)
        want1 = oracle.moe_forward(x2, R, b1, get, cfg.G, cfg.topG, cfg.K)
        err = max(float(np.max(np.abs(y0 - want0["y"])) / np.max(np.abs(want0["y"]))),
                  float(np.max(np.abs(y1 - want1["y"])) / np.max(np.abs(want1["y"]))))
        # the replica slots hold their experts' weights
        wok = True
        for i, e in enumerate(layer.hosted[rank]):
            if e >= 0:
                w1, w3, w2 = get(e)
                wok &= bool(np.array_equal(ops.w13[i, 0].numpy(), w1) and
                            np.array_equal(ops.w13[i, 1].numpy(), w3) and
                            np.array_equal(ops.w2[i].numpy(), w2))
        q.put((rank, dict(err=err, hosted=layer.hosted, wok=wok, counts0=want0["route"]["counts"],
                          recv=sum(layer.last_plan["recv_splits"]))))
    except Exception as e:  # report instead of hanging the other rank's queue read
        q.put((rank, dict(error=repr(e))))
        raise
    finally:
        dist.destroy_process_group()


def test_two_ranks_with_redundant_experts_match_the_oracle():
    from sparse_moe_layer_limited_b200 import ep
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_redundant_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    for r in (0, 1):
        assert "error" not in res[r], res[r]
        assert res[r]["err"] <= 1e-12, res[r]["err"]
        assert res[r]["wok"]
    for p in procs:
        assert p.exitcode == 0
    cfg = _cfg()
    hosted = res[0]["hosted"]
    assert hosted == res[1]["hosted"]
    # the placement is the one the summed first-step counts give, and it has replicas
    load = res[0]["counts0"] + res[1]["counts0"]
    assert hosted == ep.place_redundant(load, cfg.N, 2, 2)
    assert sum(1 for q_ in hosted for e in q_[cfg.N // 2:] if e >= 0) == 4
    # every routed row of the second step went to exactly one copy
    assert res[0]["recv"] + res[1]["recv"] == 2 * cfg.T * cfg.K


def test_place_redundant_properties():
    from sparse_moe_layer_limited_b200 import ep
    N, W, r = 32, 4, 2
    rng = np.random.default_rng(5)
    load = rng.integers(10, 40, size=N).astype(np.int64)
    load[[3, 17]] = [900, 400]                    # two hot experts
    hosted = ep.place_redundant(load, N, W, r)
    assert hosted == ep.place_redundant(load.copy(), N, W, r)          # deterministic
    per = N // W
    for q_ in range(W):
        assert hosted[q_][:per] == list(range(q_ * per, (q_ + 1) * per))
        reps = [e for e in hosted[q_][per:] if e >= 0]
        assert len(hosted[q_]) == per + r
        assert len(set(reps)) == len(reps) and not set(reps) & set(hosted[q_][:per])
    copies = {e: sum(e in h for h in hosted) for e in range(N)}
    assert copies[3] == W                          # the hottest expert is on every rank
    assert copies[17] >= 2
    # every replicated expert carries at least the load of any unreplicated one
    rep = [e for e in range(N) if copies[e] > 1]
    assert all(load[e] >= max(load[f] for f in range(N) if copies[f] == 1) for e in rep)
    assert sum(copies.values()) == N + W * r       # every slot is used
    assert ep.place_redundant(load, N, W, 0) == ep.primary_placement(N, W)


@pytest.mark.parametrize("sender", [0, 1, 2])
def test_send_tables_cover_every_row_once(sender):
    from sparse_moe_layer_limited_b200 import ep
    N, W, r = 12, 3, 2
    rng = np.random.default_rng(sender)
    counts = rng.integers(0, 9, size=N)
    load = rng.integers(0, 50, size=N)
    hosted = ep.place_redundant(load, N, W, r)
    st = ep.send_tables(counts, hosted, sender, N // W)
    order = st["order"]
    assert sorted(order.tolist()) == list(range(int(counts.sum())))
    assert st["sends"] == [int(v) for v in st["sendcnt"].sum(axis=1)]
    off = np.concatenate([[0], np.cumsum(counts)])
    pos = 0
    for q_ in range(W):
        for i, e in enumerate(hosted[q_]):
            m = int(st["sendcnt"][q_, i])
            if e < 0:
                assert m == 0
                continue
            rows = order[pos:pos + m]
            pos += m
            # a contiguous chunk of expert e's rows
            assert np.all(np.diff(rows) == 1) or m <= 1
            assert np.all((rows >= off[e]) & (rows < off[e + 1]))
    for e in range(N):
        chunks = [int(st["sendcnt"][q_, i]) for q_ in range(W) for i, f in enumerate(hosted[q_])
                  if f == e]
        assert sum(chunks) == counts[e]
        assert max(chunks) - min(chunks) <= 1
