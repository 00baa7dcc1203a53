"""Expert parallelism inside one node: the routed experts split over GPUs.

The mhpq.cn article "DeepSeek-V3 高效训练关键技术分析" describes the
experts spread over devices (§2.1, 64-way expert parallelism) and tokens
reaching the experts of other devices by all-to-all, with each token limited
to a few nodes (§3.1).  Here W ranks of one node (one process per GPU) share
the layer:

* rank r holds the routed experts [r*N/W, (r+1)*N/W) (contiguous, so when W
  divides the group count G a rank holds whole groups), plus replicas of the
  router, the bias and the shared expert; every rank routes its own batch of
  T tokens;
* forward, on every rank: route and dispatch (local kernels); an all-to-all
  of the per-expert counts, giving each rank the count matrix cnt[src, e] of
  the rows it will receive; an all-to-all of the dispatched rows (dispatch
  orders rows by expert, so the rows for one destination are one contiguous
  range); a regroup of the received rows by local expert (moe_gather_rows);
  the grouped expert FFN, with the shared expert on the rank's own tokens;
  the inverse regroup; the reverse all-to-all, which returns every row to
  its place in the sender's dispatch order; the local combine;
* bias update: an all-reduce of the counts, after which every rank applies
  the same +-gamma with the threshold of the whole node's batch (W*T*K/N),
  so the replicated biases stay identical.

Inside one NVSwitch node every peer is reached at the same bandwidth, so the
group limit constrains nothing here; it stays part of the routing rule.

The exchange uses torch.distributed collectives (NCCL between GPUs; with
gloo, device tensors are staged through host memory).  The
per-rank computation is behind a small operations interface: the library's
CUDA kernels (``LibraryOps``) on the product path.  The host-side planning
(send splits, the regroup tables) is plain integer work in NumPy.

Local expert capacity: the grouped FFN runs with a local shape of T tokens
and K_cap = min(32, N/W) rows per token, i.e. at most T*K_cap received rows
(4x the average T*K at V3 sizes on 8 GPUs, and at least 4x with two ranks);
a batch that sends more rows to one rank raises an error rather than
dropping tokens.  BF16 and FP32 layers; the E4M3 mode is not expert-parallel
here.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L


# ---- host-side planning (integer bookkeeping, no arithmetic of the method) -------------

def expert_range(N: int, W: int, r: int):
    """Routed experts [lo, hi) of rank r."""
    if N % W:
        raise ValueError(f"N={N} routed experts do not split over {W} ranks")
    n = N // W
    return r * n, (r + 1) * n


def send_splits(counts: np.ndarray, W: int) -> list:
    """Rows this rank sends to each rank: the counts of that rank's experts."""
    c = np.asarray(counts, dtype=np.int64).reshape(W, -1)
    return [int(v) for v in c.sum(axis=1)]


def regroup_plan(cnt: np.ndarray) -> dict:
    """From the received count matrix cnt[src, e] (rows that rank `src`
    sends for local expert e; rows arrive ordered by src, then by expert,
    then in the sender's token order), the tables of the local expert pass:
      recv_splits [W]       rows from each source
      offsets [E + 1]       expert-major row offsets (expert e: src 0's rows,
                            then src 1's, ...)
      gather [R]            expert-major row i <- received row gather[i]
      scatter [R]           received row j <- expert-major row scatter[j]."""
    cnt = np.asarray(cnt, dtype=np.int64)
    W, E = cnt.shape
    recv_splits = cnt.sum(axis=1)
    src_base = np.concatenate([[0], np.cumsum(recv_splits)[:-1]])
    # first received row of (src, e)
    in_src = np.concatenate([np.zeros((W, 1), np.int64), np.cumsum(cnt, axis=1)[:, :-1]], axis=1)
    first_recv = src_base[:, None] + in_src
    per_expert = cnt.sum(axis=0)
    offsets = np.concatenate([[0], np.cumsum(per_expert)]).astype(np.int64)
    R = int(offsets[-1])
    gather = np.empty(R, dtype=np.int64)
    pos = 0
    for e in range(E):
        for s in range(W):
            n = int(cnt[s, e])
            gather[pos:pos + n] = first_recv[s, e] + np.arange(n)
            pos += n
    scatter = np.empty(R, dtype=np.int64)
    scatter[gather] = np.arange(R)
    return dict(recv_splits=[int(v) for v in recv_splits], offsets=offsets.astype(np.int32),
                gather=gather.astype(np.int32), scatter=scatter.astype(np.int32))


# ---- the per-rank operations on the product path ----------------------------------------

class LibraryOps:
    """The per-rank steps through the C-ABI library (CUDA kernels only).

    shape: the layer shape with this rank's T; local_shape: (T, d, N/W,
    K_cap, 1, 1, f) for the grouped FFN over this rank's experts.  w13, w2:
    this rank's routed experts then the shared expert ([N/W + 1, 2f, d],
    [N/W + 1, d, f], packed as for MoELayer)."""

    def __init__(self, shape, local_shape, router_w, bias, w13, w2):
        s, sl = shape, local_shape
        for sh in (s, sl):
            rc = L.check_shape(sh)
            if rc != L.OK:
                raise L.MoEError("moe_check_shape", rc)
        if s.dtype == L.DTYPE_E4M3:
            raise ValueError("the expert-parallel layer runs in BF16 or FP32 mode")
        self.shape, self.local_shape = s, sl
        self.router_w, self.bias, self.w13, self.w2 = router_w, bias, w13, w2
        dev = router_w.device
        xdt = L.x_torch_dtype(s)
        i32 = dict(dtype=torch.int32, device=dev)
        cap = sl.T * sl.K
        self.capacity = cap
        self.idx = torch.empty(s.T, s.K, **i32)
        self.gate = torch.empty(s.T, s.K, dtype=torch.float32, device=dev)
        self.counts = torch.empty(s.N, **i32)
        self.offsets = torch.empty(s.N + 1, **i32)
        self.perm_tok = torch.empty(s.T * s.K, **i32)
        self.slot = torch.empty(s.T, s.K, **i32)
        self.x_perm = torch.empty(s.T * s.K, s.d, dtype=xdt, device=dev)
        self.y_perm = torch.empty(s.T * s.K, s.d, dtype=xdt, device=dev)
        self.recv = torch.empty(cap, s.d, dtype=xdt, device=dev)
        self.x_loc = torch.empty(cap, s.d, dtype=xdt, device=dev)
        self.y_loc = torch.empty(cap, s.d, dtype=xdt, device=dev)
        self.y_back = torch.empty(cap, s.d, dtype=xdt, device=dev)
        self.y_shared = torch.empty(s.T, s.d, dtype=xdt, device=dev)
        self.y = torch.empty(s.T, s.d, dtype=xdt, device=dev)
        self.offsets_loc = torch.empty(sl.N + 1, **i32)
        self.gather_idx = torch.empty(cap, **i32)
        self.scatter_idx = torch.empty(cap, **i32)
        self.ws = torch.zeros(L.workspace_size(s), dtype=torch.uint8, device=dev)
        self.ws_loc = torch.zeros(L.workspace_size(sl), dtype=torch.uint8, device=dev)

    def route_dispatch(self, x):
        s = self.shape
        L.moe_route(s, x, self.router_w, self.bias, self.idx, self.gate, self.counts, self.ws)
        L.moe_dispatch(s, x, self.idx, self.counts, self.offsets, self.perm_tok, self.slot,
                       self.x_perm, None, self.ws)
        return self.counts, self.x_perm

    def set_plan(self, plan):
        R = len(plan["gather"])
        if R > self.capacity:
            raise RuntimeError(f"rank receives {R} rows, above its capacity {self.capacity}")
        self.offsets_loc.copy_(torch.from_numpy(plan["offsets"]))
        self.gather_idx[:R].copy_(torch.from_numpy(plan["gather"]))
        self.scatter_idx[:R].copy_(torch.from_numpy(plan["scatter"]))
        return R

    def experts(self, R, x):
        """Regroup the R received rows by expert, run the grouped FFN (the
        shared expert on this rank's x), regroup the outputs back."""
        L.moe_gather_rows(self.recv[:R], self.gather_idx[:R], self.x_loc[:R])
        L.moe_expert_ffn(self.local_shape, self.x_loc, None, self.offsets_loc, x, self.w13,
                         self.w2, None, None, self.y_loc, self.y_shared, self.ws_loc)
        L.moe_gather_rows(self.y_loc[:R], self.scatter_idx[:R], self.y_back[:R])
        return self.y_back

    def combine(self):
        L.moe_combine(self.shape, self.y_perm, self.y_shared, self.slot, self.gate, self.y)
        return self.y

    def bias_update(self, counts_all, T_all, gamma):
        s = self.shape
        node = L.shape(T_all, s.d, s.N, s.K, s.G, s.topG, s.f, s.dtype)
        L.moe_bias_update(node, counts_all, self.bias, gamma)


def local_shape(shape, W: int):
    """The grouped-FFN shape of one rank: T tokens, N/W experts, K_cap =
    min(32, N/W) rows per token of capacity, one group."""
    n = shape.N // W
    k = min(32, n)
    return L.shape(shape.T, shape.d, n, k, 1, 1, shape.f, shape.dtype)


def _all_to_all(dist, group, out, inp, out_splits=None, in_splits=None):
    """all_to_all_single; with a backend that exchanges host memory only
    (gloo), device tensors go through host copies."""
    if inp.is_cuda and dist.get_backend(group) == "gloo":
        o = torch.empty(out.shape, dtype=out.dtype)
        dist.all_to_all_single(o, inp.cpu(), output_split_sizes=out_splits,
                               input_split_sizes=in_splits, group=group)
        out.copy_(o)
        return
    dist.all_to_all_single(out, inp, output_split_sizes=out_splits, input_split_sizes=in_splits,
                           group=group)


def _all_reduce(dist, group, t):
    if t.is_cuda and dist.get_backend(group) == "gloo":
        h = t.cpu()
        dist.all_reduce(h, group=group)
        t.copy_(h)
        return
    dist.all_reduce(t, group=group)


class ExpertParallelMoE:
    """One rank of the expert-parallel layer.  `ops` carries the per-rank
    steps (the library's kernels by default: ``LibraryOps``); `group` is the
    torch.distributed process group (the default group when None)."""

    def __init__(self, ops, N: int, gamma: float = 0.001, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.N = N
        self.lo, self.hi = expert_range(N, self.W, self.rank)
        self.ops = ops
        self.gamma = float(gamma)
        self.last_plan = None

    def forward(self, x, update_bias: bool = True):
        dist, ops, W = self.dist, self.ops, self.W
        counts, x_perm = ops.route_dispatch(x)
        # per-expert counts: rank r's counts of rank q's experts go to q
        cnt = torch.empty_like(counts)
        _all_to_all(dist, self.group, cnt, counts)
        cnt_h = cnt.cpu().numpy().reshape(W, -1)
        sends = send_splits(counts.cpu().numpy(), W)
        plan = regroup_plan(cnt_h)
        self.last_plan = plan
        R = ops.set_plan(plan)
        n_send = sum(sends)
        _all_to_all(dist, self.group, ops.recv[:R], x_perm[:n_send], plan["recv_splits"], sends)
        y_back = ops.experts(R, x)
        _all_to_all(dist, self.group, ops.y_perm[:n_send], y_back[:R], sends, plan["recv_splits"])
        y = ops.combine()
        if update_bias:
            counts_all = counts.clone()
            _all_reduce(dist, self.group, counts_all)
            ops.bias_update(counts_all, x.shape[0] * W, self.gamma)
        return y
