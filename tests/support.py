"""Test helpers: seeded inputs for both sides, near-tie rejection, metrics.

Inputs come from ``synth`` (the shared generator).  The near-tie rule uses
the oracle's margins: a token whose K-th/(K+1)-th biased-score gap or whose
topG-th/(topG+1)-th group-score gap is below 1e-4 has its x row re-drawn from
its own sub-stream, so fp32 (GPU) and fp64 (oracle) reach the same discrete
routing.  Expected values are always the oracle's; nothing here reads a GPU
result into the oracle.
"""
from __future__ import annotations

import numpy as np

import oracle
from synth import gen
from synth.configs import MoEConfig

NEAR_TIE = 1e-4


def tie_free_x(cfg: MoEConfig, router, bias, seed: int = 0, batch: int = 0, x=None,
               max_attempts: int = 64, margins=None):
    """x [T, d] (float32 array of stored values) with no near-tie token under
    (router, bias), or under `margins` (x rows -> per-row decision gaps) when
    given.  Returns (x, number of rows re-drawn)."""
    x = gen.make_x(cfg, seed, batch) if x is None else x.copy()
    rows = np.arange(cfg.T)
    redrawn = 0
    if margins is None:
        def margins(xr):
            return oracle.route_margins(xr, router, bias, cfg.G, cfg.topG, cfg.K)
    for attempt in range(max_attempts):
        m = margins(x[rows])
        bad = rows[m < NEAR_TIE]
        if bad.size == 0:
            return x, redrawn
        for t in bad:
            x[t] = gen.redraw_x_row(cfg, seed, batch, int(t), attempt)
        redrawn += bad.size
        rows = bad
    raise RuntimeError("could not remove near-ties")


def host_weights(cfg: MoEConfig, seed: int = 0):
    """Oracle-side accessor e -> (W1, W3, W2) as float64 arrays (cached)."""
    cache = {}

    def get(e):
        if e not in cache:
            cache[e] = tuple(gen.make_expert_weight(cfg, seed, w, e).astype(np.float64)
                             for w in ("w1", "w3", "w2"))
        return cache[e]
    return get


def streaming_weights(cfg: MoEConfig, seed: int = 0):
    """Oracle-side accessor e -> (W1, W3, W2) float64 that regenerates each
    expert into the same three buffers (the oracle uses one expert at a time),
    for full-size layers whose weights do not fit in host memory at once."""
    bufs = {w: np.empty(gen.weight_shape(cfg, w), np.float64) for w in ("w1", "w3", "w2")}

    def get(e):
        return tuple(gen.make_expert_weight(cfg, seed, w, e, out=bufs[w])
                     for w in ("w1", "w3", "w2"))
    return get


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def h_round_for(cfg: MoEConfig) -> str:
    return "none" if cfg.dtype == "fp32" else "bf16"


def greedy_token_sample(idx: np.ndarray, n: int, seed: int = 0, must=()):
    """Pick ~n tokens whose selected experts overlap as much as possible (so
    the oracle needs few experts' weights); always includes ``must``."""
    rng = np.random.default_rng(seed)
    chosen = list(dict.fromkeys(int(t) for t in must))
    experts = set()
    for t in chosen:
        experts.update(idx[t].tolist())
    cand = rng.permutation(idx.shape[0])[:4096]
    while len(chosen) < n:
        best, best_new = None, None
        for t in cand[:512]:
            if t in chosen:
                continue
            new = len(set(idx[t].tolist()) - experts)
            if best_new is None or new < best_new:
                best, best_new = int(t), new
        chosen.append(best)
        experts.update(idx[best].tolist())
        cand = rng.permutation(cand)
    return np.array(chosen), sorted(experts)


# ---------------------------------------------------------------------------
# GPU-side construction (imports torch and the package lazily)
# ---------------------------------------------------------------------------

def moe_shape(cfg: MoEConfig, T: int | None = None):
    import sparse_moe_layer_limited_b200 as M
    dt = {"fp32": M.DTYPE_FP32, "bf16": M.DTYPE_BF16, "e4m3": M.DTYPE_E4M3}[cfg.dtype]
    return M.shape(T or cfg.T, cfg.d, cfg.N, cfg.K, cfg.G, cfg.topG, cfg.f, dt)


def to_dev_x(x, cfg: MoEConfig):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return (t if cfg.dtype == "fp32" else t.to(torch.bfloat16)).cuda()


def device_weights(cfg: MoEConfig, seed: int = 0):
    """Packed w13 [N+1, 2f, d] and w2 [N+1, d, f] on the GPU for the layer's
    arithmetic dtype (bf16 weights are generated on the device, fp32 on the
    host), plus the E4M3 codes and scales when cfg.dtype == 'e4m3'."""
    import torch
    import sparse_moe_layer_limited_b200 as M
    from synth import device as sdev
    s = moe_shape(cfg)
    if cfg.dtype == "fp32":
        w1 = torch.from_numpy(np.stack([gen.make_expert_weight(cfg, seed, "w1", e)
                                        for e in range(cfg.N + 1)])).cuda()
        w3 = torch.from_numpy(np.stack([gen.make_expert_weight(cfg, seed, "w3", e)
                                        for e in range(cfg.N + 1)])).cuda()
        w2 = torch.from_numpy(np.stack([gen.make_expert_weight(cfg, seed, "w2", e)
                                        for e in range(cfg.N + 1)])).cuda()
    else:
        w1 = sdev.expert_weights_bf16(cfg, seed, "w1")
        w3 = sdev.expert_weights_bf16(cfg, seed, "w3")
        w2 = sdev.expert_weights_bf16(cfg, seed, "w2")
    w13 = torch.empty(cfg.N + 1, 2 * cfg.f, cfg.d, dtype=w1.dtype, device=w1.device)
    M.moe_pack_w13(s, w1, w3, w13)
    del w1, w3
    out = dict(w13=w13, w2=w2, w13_scales=None, w2_scales=None)
    if cfg.dtype == "e4m3":
        w13q = torch.empty_like(w13, dtype=torch.float8_e4m3fn)
        w2q = torch.empty_like(w2, dtype=torch.float8_e4m3fn)
        s13 = torch.empty(cfg.N + 1, 2 * cfg.f // 128, cfg.d // 128, dtype=torch.float32,
                          device=w13.device)
        s2 = torch.empty(cfg.N + 1, cfg.d // 128, cfg.f // 128, dtype=torch.float32,
                         device=w13.device)
        M.moe_quantize_weights(s, w13, w2, w13q, s13, w2q, s2)
        out = dict(w13=w13q, w2=w2q, w13_scales=s13, w2_scales=s2)
    torch.cuda.synchronize()
    return out


# ---------------------------------------------------------------------------
# Per-expert oracle jobs in parallel (full-size layers)
# ---------------------------------------------------------------------------

def _expert_job(args):
    """Worker: one expert's oracle outputs on its rows (weights regenerated
    from the seeded generator inside the worker)."""
    cfg, seed, e, rows, kind = args
    w = tuple(gen.make_expert_weight(cfg, seed, n, e).astype(np.float64)
              for n in ("w1", "w3", "w2"))
    if kind == "fp8":
        return e, oracle.fp8_swiglu_expert(rows, *w)
    return e, oracle.swiglu_expert(rows, *w, h_round="bf16")


def expert_outputs_parallel(cfg: MoEConfig, jobs: dict, kind: str, seed: int = 0,
                            workers: int | None = None, timeout: float = 1800.0) -> dict:
    """{expert: rows [n, d]} -> {expert: oracle outputs [n, d]}, one process
    per expert job in a pool started with 'spawn' (no CUDA state is inherited);
    kind 'fp8' runs the E4M3 expert emulation, 'bf16' the expert with h
    rounded to bf16."""
    import multiprocessing as mp
    import os
    n = workers or max(1, min(16, len(os.sched_getaffinity(0))))
    items = [(cfg, seed, int(e), np.asarray(r, np.float64), kind) for e, r in jobs.items()]
    with mp.get_context("spawn").Pool(n) as pool:
        # bounded: a pool whose workers cannot start would otherwise wait forever
        return dict(pool.map_async(_expert_job, items, chunksize=1).get(timeout=timeout))


def tail_tile_rows(offsets: np.ndarray, e: int, tile: int = 128) -> np.ndarray:
    """Rows (expert-major) of expert e's last m-tile: the ragged tail the
    expert GEMMs handle with a partly filled (or M=64) tile."""
    a, z = int(offsets[e]), int(offsets[e + 1])
    if z == a:
        return np.zeros(0, dtype=np.int64)
    full = (z - a - 1) // tile * tile
    return np.arange(a + full, z)
