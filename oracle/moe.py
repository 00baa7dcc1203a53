"""Float64 oracle of the DeepSeekMoE layer forward (test infrastructure only).

Each function is the plain definition of one step, written for a reader to
check against the pages by eye; see the package docstring for the [P*] page
keys.  All arithmetic is float64 unless a step names another precision.
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------------------
# rounding helpers (storage precision of operands the method stores)
# ---------------------------------------------------------------------------

def round_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits,
    ties to even), returned as float64.  Written as an exact power-of-two
    rescale plus numpy's half-to-even ``rint`` (finite, in-range inputs)."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                      # v = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                 # bf16 subnormal spacing is 2**-133
    step_exp = e - 8                        # 8 significant bits
    return np.ldexp(np.rint(np.ldexp(v, -step_exp)), step_exp)


def silu(u):
    """SiLU(u) = u * sigmoid(u) = u / (1 + exp(-u))."""
    u = np.asarray(u, dtype=np.float64)
    return u / (1.0 + np.exp(-u))


# ---------------------------------------------------------------------------
# routing: affinity, bias, group limit, top-K, gates, counts
# ---------------------------------------------------------------------------

def affinity(x, router) -> np.ndarray:
    """s[t, i] = sigmoid(x_t . e_i) in float64 from the stored operands.

    [P4] DeepSeekMoE paragraph: V3 computes the token-to-expert affinity with
    a sigmoid (not a softmax)."""
    z = np.asarray(x, dtype=np.float64) @ np.asarray(router, dtype=np.float64).T
    return 1.0 / (1.0 + np.exp(-z))


def biased_scores(s, bias) -> np.ndarray:
    """s'[t, i] = s[t, i] + b_i, the score used only to choose experts.

    [P2] Q3 and [P1] §1.2: a per-expert bias is added to the affinity score
    to steer routing; it never enters the gate value."""
    return np.asarray(s, dtype=np.float64) + np.asarray(bias, dtype=np.float64)[None, :]


def group_scores(sb, G: int) -> np.ndarray:
    """Score of each of G contiguous expert groups (expert i in group
    i // (N/G)): the sum of the two largest biased scores in the group (the
    whole group when it holds one expert).

    [P1] §3.1 limits each token to at most 4 nodes; with experts laid out
    contiguously over nodes a group is a node.  The top-2-sum group score is
    the reading this library takes (the pages give no formula)."""
    T, N = sb.shape
    gs = N // G
    out = np.empty((T, G), dtype=np.float64)
    for g in range(G):
        block = np.sort(sb[:, g * gs:(g + 1) * gs], axis=1)    # ascending
        out[:, g] = block[:, -min(2, gs):].sum(axis=1)
    return out


def kept_groups(gscore, topG: int) -> np.ndarray:
    """Indices of the topG highest-scoring groups per token (lower index wins
    an exact tie), [T, topG]."""
    order = np.argsort(-gscore, axis=1, kind="stable")
    return order[:, :topG]


def route(x, router, bias, G: int, topG: int, K: int) -> dict:
    """Group-limited top-K routing with the bias-for-selection-only rule.

    Steps (per token):
      1. s = sigmoid(x . e_i)                             [P4]
      2. s' = s + b                                       [P2] Q3, [P1] §1.2
      3. keep the topG groups by group score (top-2 sum)  [P1] §3.1
      4. idx = the K largest s' among experts of kept groups ([P5] §二(一)4
         top-K by affinity); reported in ascending expert id
      5. gate_k = s[idx_k] / sum_j s[idx_j] with the *un-biased* s
         ([P4]: normalise over the selected affinities; [P2] Q3: the bias
         does not affect the gate)
      6. counts_i = number of tokens that selected expert i
    Returns dict(idx [T,K] int64, gate [T,K] f64, counts [N] int64, s, sb)."""
    s = affinity(x, router)
    sb = biased_scores(s, bias)
    T, N = sb.shape
    allowed = np.zeros((T, N), dtype=bool)
    gs = N // G
    for t, groups in enumerate(kept_groups(group_scores(sb, G), topG)):
        for g in groups:
            allowed[t, g * gs:(g + 1) * gs] = True
    masked = np.where(allowed, sb, -np.inf)
    top = np.argsort(-masked, axis=1, kind="stable")[:, :K]
    idx = np.sort(top, axis=1)
    sel = np.take_along_axis(s, idx, axis=1)
    gate = sel / sel.sum(axis=1, keepdims=True)
    counts = np.bincount(idx.ravel(), minlength=N).astype(np.int64)
    return dict(idx=idx.astype(np.int64), gate=gate, counts=counts, s=s, sb=sb)


def route_margins(x, router, bias, G: int, topG: int, K: int) -> np.ndarray:
    """Per token, the smaller of two gaps that decide the discrete routing:
    (K-th minus (K+1)-th biased score among experts of the kept groups) and
    (topG-th minus (topG+1)-th group score).  +inf where a gap does not exist
    (K = number of allowed experts, or topG = G)."""
    s = affinity(x, router)
    sb = biased_scores(s, bias)
    T, N = sb.shape
    gsc = group_scores(sb, G)
    gsorted = -np.sort(-gsc, axis=1)
    gmargin = (gsorted[:, topG - 1] - gsorted[:, topG]) if topG < G else np.full(T, np.inf)
    gs = N // G
    emargin = np.full(T, np.inf)
    for t, groups in enumerate(kept_groups(gsc, topG)):
        vals = np.sort(np.concatenate([sb[t, g * gs:(g + 1) * gs] for g in groups]))[::-1]
        if K < vals.size:
            emargin[t] = vals[K - 1] - vals[K]
    return np.minimum(gmargin, emargin)


# ---------------------------------------------------------------------------
# the conventional softmax gate (the baseline the method replaces)
# ---------------------------------------------------------------------------

def route_softmax(x, router, K: int) -> dict:
    """Softmax top-K routing, the conventional gate that the bias method
    replaces, kept as a baseline.

    [P4] (gating paragraph): a conventional gating network is a softmax on
    top of a classifier, balanced by an auxiliary penalty term; [P2] Q3:
    conventional MoE models add an auxiliary loss for balance.  The pages give
    no formula; the plainest reading, per token:
      1. z_i = x . e_i,  p = softmax(z) over all N experts
      2. idx = the K largest p (no groups, no bias), ascending expert id
      3. gate_k = p[idx_k] / sum_j p[idx_j]  (the softmax over the selected)
      4. counts_i as in route(); prob_sum_i = sum_t p[t, i]
    Returns dict(idx, gate, counts, p, prob_sum)."""
    z = np.asarray(x, dtype=np.float64) @ np.asarray(router, dtype=np.float64).T
    e = np.exp(z - z.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    T, N = p.shape
    top = np.argsort(-z, axis=1, kind="stable")[:, :K]
    idx = np.sort(top, axis=1)
    sel = np.take_along_axis(p, idx, axis=1)
    gate = sel / sel.sum(axis=1, keepdims=True)
    counts = np.bincount(idx.ravel(), minlength=N).astype(np.int64)
    return dict(idx=idx.astype(np.int64), gate=gate, counts=counts, p=p,
                prob_sum=p.sum(axis=0))


def route_softmax_margins(x, router, K: int) -> np.ndarray:
    """Per token, the K-th minus the (K+1)-th largest logit z (+inf when
    K = N): the gap that decides the softmax top-K."""
    z = np.asarray(x, dtype=np.float64) @ np.asarray(router, dtype=np.float64).T
    zs = -np.sort(-z, axis=1)
    if K >= z.shape[1]:
        return np.full(z.shape[0], np.inf)
    return zs[:, K - 1] - zs[:, K]


def balance_loss(counts, prob_sum, T: int, K: int) -> float:
    """The conventional auxiliary balance statistic of a routing batch:
    L = N * sum_i f_i * P_i with f_i = counts_i / (K T), the share of the
    T*K selections that went to expert i, and P_i = prob_sum_i / T, the mean
    softmax probability of expert i.  L = 1 when both are uniform and grows
    as routing concentrates.  [P4]: the penalty discourages over-confident
    gate outputs; [P1] §1.2: per-sequence load concentration is what it
    measures when the batch is one sequence.  The product form is the reading
    this library takes (the pages give no formula)."""
    counts = np.asarray(counts, dtype=np.float64)
    prob_sum = np.asarray(prob_sum, dtype=np.float64)
    N = counts.size
    f = counts / (K * T)
    P = prob_sum / T
    return float(N * np.sum(f * P))


# ---------------------------------------------------------------------------
# dispatch, experts, combine
# ---------------------------------------------------------------------------

def dispatch(idx, N: int) -> dict:
    """Group the (token, expert) pairs by expert for the expert GEMMs
    ([P1] §2.2: DISPATCH precedes MLP).

    Row order: experts ascending, and within one expert tokens ascending.
    offsets[i] = first row of expert i (exclusive prefix sum of the counts),
    perm_tok[r] = token of row r, slot[t, k] = row holding (t, idx[t, k])."""
    idx = np.asarray(idx)
    T, K = idx.shape
    counts = np.bincount(idx.ravel(), minlength=N)
    offsets = np.zeros(N + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm_tok = np.empty(T * K, dtype=np.int64)
    slot = np.empty((T, K), dtype=np.int64)
    fill = offsets[:-1].copy()
    for t in range(T):                      # tokens in ascending order
        for k in range(K):
            e = idx[t, k]
            perm_tok[fill[e]] = t
            slot[t, k] = fill[e]
            fill[e] += 1
    return dict(offsets=offsets, perm_tok=perm_tok, slot=slot, counts=counts)


def swiglu_expert(a, w1, w3, w2, h_round: str = "none") -> np.ndarray:
    """One expert FFN on the rows ``a`` [M, d]:
    y = (silu(a W1^T) * (a W3^T)) W2^T, with W1, W3 [f, d] and W2 [d, f].

    The expert is an FFN ([P1] §1.1, [P5]); its SwiGLU form is this library's
    reading.  ``h_round='bf16'`` rounds the hidden activation to bf16 before
    the W2 contraction (it is stored as a bf16 GEMM operand)."""
    a = np.asarray(a, dtype=np.float64)
    h = silu(a @ np.asarray(w1, np.float64).T) * (a @ np.asarray(w3, np.float64).T)
    if h_round == "bf16":
        h = round_bf16(h)
    return h @ np.asarray(w2, np.float64).T


def swiglu_expert_backward(a, w1, w3, w2, dy, gu_round: str = "none",
                           dgu_round: str = "none") -> dict:
    """Gradients of one expert FFN y = (silu(a W1^T) * (a W3^T)) W2^T given
    dy = dL/dy [M, d].

    [P1] §2.2: the backward pass runs COMBINE -> MLP_B (input gradients) ->
    MLP_W (weight gradients) -> DISPATCH.  With g = a W1^T and u = a W3^T
    (the gate and up products) and h = silu(g) * u, the chain rule gives
        dh  = dy W2
        dg  = dh * u * silu'(g),  silu'(g) = sigma(g) (1 + g (1 - sigma(g)))
        du  = dh * silu(g)
        da  = dg W1 + du W3
        dW2 = dy^T h,  dW1 = dg^T a,  dW3 = du^T a
    ``gu_round='bf16'``: g and u are the bf16 values a recompute stores;
    ``dgu_round='bf16'``: dg and du are rounded to bf16 (a GEMM operand)
    before the da and dW contractions.  Returns dict(da, dw1, dw3, dw2, dg,
    du, dh)."""
    a = np.asarray(a, dtype=np.float64)
    w1, w3, w2 = (np.asarray(w, np.float64) for w in (w1, w3, w2))
    dy = np.asarray(dy, dtype=np.float64)
    g, u = a @ w1.T, a @ w3.T
    if gu_round == "bf16":
        g, u = round_bf16(g), round_bf16(u)
    sig = 1.0 / (1.0 + np.exp(-g))
    h = g * sig * u
    dh = dy @ w2
    dg = dh * u * sig * (1.0 + g * (1.0 - sig))
    du = dh * g * sig
    if dgu_round == "bf16":
        dg, du = round_bf16(dg), round_bf16(du)
    return dict(da=dg @ w1 + du @ w3, dw1=dg.T @ a, dw3=du.T @ a, dw2=dy.T @ h, dg=dg, du=du,
                dh=dh)


def expert_outputs(x, idx, get_weights, N: int, tokens=None, h_round: str = "none",
                   expert_fn=None) -> dict:
    """Per-expert outputs for the selected tokens.

    Returns {'shared': y_sh [len(tokens), d], 'routed': {(t, e): y [d]}} where
    y_sh = E_N(x_t) is the always-on shared expert ([P1] §1.1: the shared
    expert processes every token) and routed entries are E_e(x_t) for each
    selected expert e of each token t.  ``get_weights(e)`` -> (W1, W3, W2);
    ``expert_fn(a, w1, w3, w2)`` overrides the expert math (FP8 emulation)."""
    x = np.asarray(x, dtype=np.float64)
    tokens = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    fn = expert_fn or (lambda a, w1, w3, w2: swiglu_expert(a, w1, w3, w2, h_round))
    routed = {}
    users = {}
    for t in tokens:
        for e in idx[t]:
            users.setdefault(int(e), []).append(int(t))
    for e in sorted(users):
        w1, w3, w2 = get_weights(e)
        ts = users[e]
        y = fn(x[ts], w1, w3, w2)
        for j, t in enumerate(ts):
            routed[(t, e)] = y[j]
    w1, w3, w2 = get_weights(N)
    shared = fn(x[tokens], w1, w3, w2)
    return dict(shared=shared, routed=routed, tokens=tokens)


def combine(shared, routed, idx, gate, tokens) -> np.ndarray:
    """y_t = y_shared_t + sum_k gate[t,k] * E_{idx[t,k]}(x_t), float64
    ([P1] §2.2 COMBINE; [P4] gate-weighted sum of the routed outputs)."""
    out = np.array(shared, dtype=np.float64, copy=True)
    for j, t in enumerate(tokens):
        for k in range(idx.shape[1]):
            out[j] += gate[t, k] * routed[(int(t), int(idx[t, k]))]
    return out


# ---------------------------------------------------------------------------
# auxiliary-loss-free bias update
# ---------------------------------------------------------------------------

def bias_update(bias, counts, T: int, K: int, gamma: float) -> np.ndarray:
    """b_i <- b_i - gamma if expert i is overloaded, b_i + gamma if it is
    under-loaded, unchanged if its load is exactly the mean T*K/N.  Computed
    in float32 (the stored precision of b), one rounding per step.

    [P4] DeepSeekMoE paragraph (decrease by gamma when overloaded, increase by
    gamma when under-loaded; gamma is the bias update speed); [P1] §1.2 (the
    bias is not a gradient update and is adjusted at every step)."""
    b = np.asarray(bias, dtype=np.float32)
    c = np.asarray(counts, dtype=np.int64)
    N = b.size
    g = np.float32(gamma)
    out = b.copy()
    for i in range(N):
        if c[i] * N > T * K:          # c_i > T*K/N, compared exactly
            out[i] = np.float32(b[i] - g)
        elif c[i] * N < T * K:
            out[i] = np.float32(b[i] + g)
    return out


# ---------------------------------------------------------------------------
# backward of COMBINE, of the gates and of DISPATCH
# ---------------------------------------------------------------------------

def combine_backward(dy, y_perm, slot, gate) -> dict:
    """Backward of y_t = y_shared_t + sum_k gate[t,k] * y_perm[slot[t,k]].

    [P1] §2.2 runs the backward pass COMBINE -> MLP_B -> MLP_W -> DISPATCH;
    this is its first step.  For each (t, k):
        dy_perm[slot[t,k]] = gate[t,k] * dy_t      (the routed expert's output gradient)
        dgate[t,k]         = dy_t . y_perm[slot[t,k]]
    and the shared expert's output gradient is dy itself.  float64.
    Returns dict(dy_perm [T*K, d], dgate [T, K])."""
    dy = np.asarray(dy, dtype=np.float64)
    y_perm = np.asarray(y_perm, dtype=np.float64)
    slot = np.asarray(slot)
    gate = np.asarray(gate, dtype=np.float64)
    T, K = slot.shape
    dy_perm = np.zeros((T * K, dy.shape[1]), dtype=np.float64)
    dgate = np.empty((T, K), dtype=np.float64)
    for t in range(T):
        for k in range(K):
            r = slot[t, k]
            dy_perm[r] = gate[t, k] * dy[t]
            dgate[t, k] = float(np.dot(dy[t], y_perm[r]))
    return dict(dy_perm=dy_perm, dgate=dgate)


def route_backward(x, router, idx, dgate) -> dict:
    """Gradient of the gates with respect to the router logits, the layer
    input and the router weights, the selection held fixed (the bias enters
    only the selection, [P2] Q3, so it receives no gradient).

    With z = x e_i (the logits), s = sigmoid(z) ([P4]: sigmoid affinity) and,
    over the K selected experts, gate_k = s_k / S with S = sum_j s_j ([P4]:
    normalisation over the selected affinities):
        ds_k = (dgate_k - sum_j gate_j dgate_j) / S
        dz_k = ds_k * s_k (1 - s_k)
        dx_t += sum_k dz_k e_{idx_k},    de_i += sum over (t, k) with idx = i of dz_k x_t
    Returns dict(dz [T, K], dx [T, d], drouter [N, d], s [T, K], gate [T, K])."""
    x = np.asarray(x, dtype=np.float64)
    R = np.asarray(router, dtype=np.float64)
    idx = np.asarray(idx)
    dgate = np.asarray(dgate, dtype=np.float64)
    T, K = idx.shape
    z = np.einsum("td,tkd->tk", x, R[idx])
    s = 1.0 / (1.0 + np.exp(-z))
    S = s.sum(axis=1, keepdims=True)
    gate = s / S
    ds = (dgate - (gate * dgate).sum(axis=1, keepdims=True)) / S
    dz = ds * s * (1.0 - s)
    dx = np.einsum("tk,tkd->td", dz, R[idx])
    drouter = np.zeros_like(R)
    for t in range(T):
        for k in range(K):
            drouter[idx[t, k]] += dz[t, k] * x[t]
    return dict(dz=dz, dx=dx, drouter=drouter, s=s, gate=gate)


def dispatch_backward(dx_perm, dx_shared, slot, dx_route=None) -> np.ndarray:
    """Last step of the backward order ([P1] §2.2): every copy of token t
    that DISPATCH made sends its input gradient back,
        dx_t = dx_shared_t + sum_k dx_perm[slot[t,k]] (+ dx_route_t),
    where dx_shared is the shared expert's input gradient and dx_route the
    gradient through the router logits.  float64, [T, d]."""
    dx = np.array(dx_shared, dtype=np.float64, copy=True)
    dx_perm = np.asarray(dx_perm, dtype=np.float64)
    slot = np.asarray(slot)
    T, K = slot.shape
    for t in range(T):
        for k in range(K):
            dx[t] += dx_perm[slot[t, k]]
    if dx_route is not None:
        dx += np.asarray(dx_route, dtype=np.float64)
    return dx


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------

def moe_forward(x, router, bias, get_weights, G: int, topG: int, K: int,
                tokens=None, h_round: str = "none", expert_fn=None) -> dict:
    """Routing for every token, then the layer output for ``tokens`` (all by
    default): y = E_shared(x) + sum_k gate_k * E_{idx_k}(x), float64.
    Forward order DISPATCH -> MLP -> COMBINE as in [P1] §2.2."""
    N = np.asarray(router).shape[0]
    r = route(x, router, bias, G, topG, K)
    d = dispatch(r["idx"], N)
    ex = expert_outputs(x, r["idx"], get_weights, N, tokens, h_round, expert_fn)
    y = combine(ex["shared"], ex["routed"], r["idx"], r["gate"], ex["tokens"])
    return dict(route=r, dispatch=d, y=y, tokens=ex["tokens"], shared=ex["shared"],
                routed=ex["routed"])


def moe_backward(x, router, bias, get_weights, G: int, topG: int, K: int, dy,
                 h_round: str = "none") -> dict:
    """The layer backward for every token, in the order of [P1] §2.2:
    COMBINE backward, MLP_B and MLP_W of every expert (routed and shared),
    then DISPATCH backward with the router path added.  The routing is the
    forward's and held fixed.  float64.
    Returns dict(dx [T, d], drouter [N, d], dw {e: (dW1, dW3, dW2)}, dgate,
    dz, route, dispatch)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    N = np.asarray(router).shape[0]
    T, d = x.shape
    r = route(x, router, bias, G, topG, K)
    dsp = dispatch(r["idx"], N)
    offs, perm_tok, slot = dsp["offsets"], dsp["perm_tok"], dsp["slot"]
    y_perm = np.zeros((T * K, d), dtype=np.float64)
    for e in range(N):
        rows = np.arange(offs[e], offs[e + 1])
        if rows.size:
            w1, w3, w2 = get_weights(e)
            y_perm[rows] = swiglu_expert(x[perm_tok[rows]], w1, w3, w2, h_round)
    cb = combine_backward(dy, y_perm, slot, r["gate"])
    dx_perm = np.zeros((T * K, d), dtype=np.float64)
    dw = {}
    for e in range(N):
        rows = np.arange(offs[e], offs[e + 1])
        w1, w3, w2 = get_weights(e)
        if rows.size:
            b = swiglu_expert_backward(x[perm_tok[rows]], w1, w3, w2, cb["dy_perm"][rows])
            dx_perm[rows] = b["da"]
            dw[e] = (b["dw1"], b["dw3"], b["dw2"])
        else:
            dw[e] = tuple(np.zeros_like(np.asarray(w, np.float64)) for w in (w1, w3, w2))
    w1, w3, w2 = get_weights(N)
    bs = swiglu_expert_backward(x, w1, w3, w2, dy)
    dw[N] = (bs["dw1"], bs["dw3"], bs["dw2"])
    rb = route_backward(x, router, r["idx"], cb["dgate"])
    dx = dispatch_backward(dx_perm, bs["da"], slot, rb["dx"])
    return dict(dx=dx, drouter=rb["drouter"], dw=dw, dgate=cb["dgate"], dz=rb["dz"],
                route=r, dispatch=dsp)
