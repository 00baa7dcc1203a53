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

Redundant experts: the inference deployment in the DeepSeek-V3
walk-through (kaiyunto.com), deployment section (decoding stage), and the
"解读 DeepSeek-V3" notes (gkm0120.cn), Q10, place extra copies of high-load
experts on other GPUs and adjust the placement as the load moves.
Here every rank keeps r replica slots beside its N/W primary experts.
`place_redundant` fills the W*r slots greedily from the node-wide counts:
the expert with the highest load per copy receives another copy on the
least-loaded rank that has a free slot and does not hold it yet.  Every
sender splits its rows for an expert with c copies into c contiguous,
balanced chunks, one per copy (which copy takes a remainder row rotates with
the sender).  The rows are sent in destination order (a row gather), the
outputs come back the same way and are put back by the inverse gather, so
the local FFN and the combine are unchanged.  When the placement changes,
`exchange_replica_weights` moves each replicated expert's weights from its
primary rank to its new hosts.  The pages do not say how replicas share an
expert's rows; the chunk split is this library's reading.

Local expert capacity: the grouped FFN runs with a local shape of T tokens
and K_cap = min(32, N/W + r) rows per token, i.e. at most T*K_cap received
rows (4x the average T*K at V3 sizes on 8 GPUs, and at least 4x with two
ranks); a batch that sends more rows to one rank raises an error rather than
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


def primary_placement(N: int, W: int):
    """hosted[q]: rank q's primary experts (contiguous), no replica slots."""
    return [list(range(*expert_range(N, W, q))) for q in range(W)]


def place_redundant(load, N: int, W: int, r: int):
    """hosted[q] = rank q's N/W primary experts, then its r replica slots
    (expert ids, -1 for an empty slot), from the node-wide per-expert row
    counts `load`.  Greedy and deterministic: while slots are free, the
    expert with the largest load per copy (ties: smaller id) gets one more
    copy, on the eligible rank (a free slot, no copy of it yet) with the
    smallest load (ties: smaller rank); an expert no rank can take is skipped."""
    load = np.asarray(load, dtype=np.float64).reshape(N)
    hosted = primary_placement(N, W)
    copies = {e: [q] for q in range(W) for e in hosted[q]}
    per = N // W
    rank_load = np.array([load[q * per:(q + 1) * per].sum() for q in range(W)])
    free = [r] * W
    slots = [[] for _ in range(W)]
    skipped = set()
    while sum(free) > 0:
        cand = [(-(load[e] / len(copies[e])), e) for e in range(N)
                if e not in skipped and load[e] > 0]
        if not cand:
            break
        _, e = min(cand)
        elig = [q for q in range(W) if free[q] > 0 and q not in copies[e]]
        if not elig:
            skipped.add(e)
            continue
        c = len(copies[e])
        # the copies of e share its load evenly: move load/c - load/(c+1) from
        # each of the c current holders' sums to the new one
        share_old, share_new = load[e] / c, load[e] / (c + 1)
        q = min(elig, key=lambda q: (rank_load[q], q))
        for h in copies[e]:
            rank_load[h] -= share_old - share_new
        rank_load[q] += share_new
        copies[e].append(q)
        slots[q].append(e)
        free[q] -= 1
    return [hosted[q] + slots[q] + [-1] * (r - len(slots[q])) for q in range(W)]


def send_tables(counts, hosted, sender: int, n_primary: int):
    """For one sender with per-expert row counts `counts` (its dispatch order:
    rows of expert e at offsets [off[e], off[e+1])): the rows it sends, in
    destination order.
      sendcnt [W, S]  rows for slot i of rank q (S = slots per rank)
      sends   [W]     rows to each rank
      order   [sum]   x_perm row of each sent row
    Expert e with c copies (primary first): chunk j of its rows goes to copy
    j; chunk sizes differ by at most one, and the first n mod c chunks after
    rotating by the sender's rank take the extra rows."""
    counts = np.asarray(counts, dtype=np.int64)
    W, S = len(hosted), len(hosted[0])
    off = np.concatenate([[0], np.cumsum(counts)])
    copies = {}
    for q in range(W):
        for i, e in enumerate(hosted[q]):
            if e >= 0:
                copies.setdefault(e, []).append((q, i))
    for e in copies:
        copies[e].sort(key=lambda qi: (qi[1] >= n_primary, qi[0]))
    sendcnt = np.zeros((W, S), dtype=np.int64)
    start = {}
    for e, lst in copies.items():
        n, c = int(counts[e]), len(lst)
        base, extra = divmod(n, c)
        pos = int(off[e])
        for j, (q, i) in enumerate(lst):
            m = base + (1 if (j - sender) % c < extra else 0)
            sendcnt[q, i] = m
            start[(q, i)] = pos
            pos += m
    parts = [np.arange(start[(q, i)], start[(q, i)] + sendcnt[q, i], dtype=np.int64)
             for q in range(W) for i in range(S) if sendcnt[q, i]]
    order = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
    return dict(sendcnt=sendcnt, sends=[int(v) for v in sendcnt.sum(axis=1)], order=order)


def exchange_replica_weights(dist, group, w13, w2, hosted, old_hosted, n_primary: int):
    """Fill this rank's replica slots that changed between `old_hosted` and
    `hosted` with the weights of their experts, sent by the experts' primary
    ranks.  w13 [S + 1, 2f, d], w2 [S + 1, d, f]: slots 0..n_primary-1 hold
    the primaries, n_primary..S-1 the replicas, S the shared expert.  One
    all_to_all of whole expert blocks (zero-length for pairs with nothing to
    move); every rank calls it with the same tables."""
    W = len(hosted)
    rank = dist.get_rank(group)
    need = [[] for _ in range(W)]     # need[q]: (slot on q, expert) that q fetches
    for q in range(W):
        for i in range(n_primary, len(hosted[q])):
            e = hosted[q][i]
            if e >= 0 and (old_hosted is None or old_hosted[q][i] != e):
                need[q].append((i, e))
    blk13, blk2 = w13[0].numel(), w2[0].numel()
    per_block = blk13 + blk2
    # this rank sends, to each q, the primaries of its own that q needs, in q's slot order
    send_parts, send_sizes = [], []
    for q in range(W):
        mine = [(i, e) for i, e in need[q] if e // n_primary == rank]
        for _, e in mine:
            j = e - rank * n_primary
            send_parts += [w13[j].view(-1), w2[j].view(-1)]
        send_sizes.append(len(mine) * per_block)
    recv_list = [(i, e) for i, e in need[rank]]
    recv_sizes = [sum(1 for _, e in recv_list if e // n_primary == p) * per_block
                  for p in range(W)]
    # every rank takes part in the collective, also with nothing to move
    send = (torch.cat(send_parts) if send_parts
            else torch.empty(0, dtype=w13.dtype, device=w13.device))
    recv = torch.empty(sum(recv_sizes), dtype=w13.dtype, device=w13.device)
    _all_to_all(dist, group, recv, send, recv_sizes, send_sizes)
    pos = 0
    for p in range(W):
        for i, e in recv_list:
            if e // n_primary != p:
                continue
            w13[i].view(-1).copy_(recv[pos:pos + blk13])     # view: the slot itself
            w2[i].view(-1).copy_(recv[pos + blk13:pos + per_block])
            pos += per_block


# ---- the per-rank operations on the product path ----------------------------------------

class LibraryOps:
    """The per-rank steps through the C-ABI library (CUDA kernels only).

    shape: the layer shape with this rank's T; local_shape: (T, d, N/W + r,
    K_cap, 1, 1, f) for the grouped FFN over this rank's slots.  w13, w2:
    this rank's primary experts then the shared expert ([N/W + 1, 2f, d],
    [N/W + 1, d, f], packed as for MoELayer); with r replica slots the
    weights are copied once into [N/W + r + 1, ...] buffers whose slots
    N/W .. N/W + r - 1 take the replicas (`exchange_replica_weights`)."""

    def __init__(self, shape, local_shape, router_w, bias, w13, w2, replicas: int = 0):
        s, sl = shape, local_shape
        for sh in (s, sl):
            rc = L.check_shape(sh)
            if rc != L.OK:
                raise L.MoEError("moe_check_shape", rc)
        if s.dtype == L.DTYPE_E4M3:
            raise ValueError("the expert-parallel layer runs in BF16 or FP32 mode")
        self.shape, self.local_shape = s, sl
        self.router_w, self.bias = router_w, bias
        self.replicas = int(replicas)
        if self.replicas:
            n = w13.shape[0] - 1
            if sl.N != n + self.replicas:
                raise ValueError("local shape: N/W + r slots expected")
            self.w13 = torch.zeros((sl.N + 1,) + tuple(w13.shape[1:]), dtype=w13.dtype,
                                   device=w13.device)
            self.w2 = torch.zeros((sl.N + 1,) + tuple(w2.shape[1:]), dtype=w2.dtype,
                                  device=w2.device)
            self.w13[:n].copy_(w13[:n])
            self.w13[sl.N].copy_(w13[n])
            self.w2[:n].copy_(w2[:n])
            self.w2[sl.N].copy_(w2[n])
        else:
            self.w13, self.w2 = w13, w2
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
        if self.replicas:  # rows in destination order and back
            self.send_idx = torch.empty(s.T * s.K, **i32)
            self.unsend_idx = torch.empty(s.T * s.K, **i32)
            self.x_send = torch.empty(s.T * s.K, s.d, dtype=xdt, device=dev)
            self.y_send = torch.empty(s.T * s.K, s.d, dtype=xdt, device=dev)
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

    def gather_send(self, order):
        """x_perm rows in the given order (destination-major) for the send."""
        n = len(order)
        self.send_idx[:n].copy_(torch.from_numpy(order.astype(np.int32)))
        inv = np.empty(n, dtype=np.int32)
        inv[order] = np.arange(n, dtype=np.int32)
        self.unsend_idx[:n].copy_(torch.from_numpy(inv))
        L.moe_gather_rows(self.x_perm[:n], self.send_idx[:n], self.x_send[:n])
        return self.x_send

    def unsend(self, n):
        """y_perm rows from the rows returned in send order."""
        L.moe_gather_rows(self.y_send[:n], self.unsend_idx[:n], self.y_perm[:n])

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


def local_shape(shape, W: int, replicas: int = 0):
    """The grouped-FFN shape of one rank: T tokens, N/W + r expert slots,
    K_cap = min(32, N/W + r) rows per token of capacity, one group."""
    n = shape.N // W + replicas
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
    torch.distributed process group (the default group when None).

    redundant = r replica slots per rank (``ops`` built with the same r);
    replan_every = k > 0 re-places the replicas from the node-wide counts
    after every k-th forward (0: only by an explicit ``replan``)."""

    def __init__(self, ops, N: int, gamma: float = 0.001, group=None, redundant: int = 0,
                 replan_every: int = 0):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.N = N
        self.lo, self.hi = expert_range(N, self.W, self.rank)
        self.n_primary = N // self.W
        self.ops = ops
        self.gamma = float(gamma)
        self.r = int(redundant)
        self.replan_every = int(replan_every)
        self.steps = 0
        self.hosted = [h + [-1] * self.r for h in primary_placement(N, self.W)]
        self.last_plan = None

    def replan(self, load):
        """Place the replicas for the node-wide per-expert loads `load` and
        move the weights of the newly placed ones (a collective: every rank
        calls it with the same loads)."""
        new = place_redundant(load, self.N, self.W, self.r)
        exchange_replica_weights(self.dist, self.group, self.ops.w13, self.ops.w2, new,
                                 self.hosted, self.n_primary)
        self.hosted = new

    def forward(self, x, update_bias: bool = True):
        dist, ops, W = self.dist, self.ops, self.W
        counts, x_perm = ops.route_dispatch(x)
        if self.r == 0:
            # per-expert counts: rank r's counts of rank q's experts go to q
            cnt = torch.empty_like(counts)
            _all_to_all(dist, self.group, cnt, counts)
            cnt_h = cnt.cpu().numpy().reshape(W, -1)
            sends = send_splits(counts.cpu().numpy(), W)
            send_rows = x_perm
            y_dst = ops.y_perm
        else:
            st = send_tables(counts.cpu().numpy(), self.hosted, self.rank, self.n_primary)
            S = len(self.hosted[0])
            sendcnt = torch.from_numpy(st["sendcnt"].astype(np.int32).reshape(-1)).to(counts.device)
            cnt = torch.empty_like(sendcnt)
            _all_to_all(dist, self.group, cnt, sendcnt)
            cnt_h = cnt.cpu().numpy().reshape(W, S)
            sends = st["sends"]
            send_rows = ops.gather_send(st["order"])
            y_dst = ops.y_send
        plan = regroup_plan(cnt_h)
        self.last_plan = plan
        R = ops.set_plan(plan)
        n_send = sum(sends)
        _all_to_all(dist, self.group, ops.recv[:R], send_rows[:n_send], plan["recv_splits"], sends)
        y_back = ops.experts(R, x)
        _all_to_all(dist, self.group, y_dst[:n_send], y_back[:R], sends, plan["recv_splits"])
        if self.r:
            ops.unsend(n_send)
        y = ops.combine()
        self.steps += 1
        replan = self.r > 0 and self.replan_every > 0 and self.steps % self.replan_every == 0
        if update_bias or replan:
            counts_all = counts.clone()
            _all_reduce(dist, self.group, counts_all)
            if update_bias:
                ops.bias_update(counts_all, x.shape[0] * W, self.gamma)
            if replan:
                self.replan(counts_all.cpu().numpy())
        return y
