"""Throughput of the DeepSeekMoE layer forward on B200 GPUs.

A step is one whole forward of the layer over one batch (route -> dispatch
-> experts -> combine) plus the bias update, on synthetic seeded inputs of the
DeepSeek-V3 shape (T=8192 tokens, d=7168, 256 routed + 1 shared experts,
K=8, 8 groups / top-4, f=2048, bf16).  `value` is tokens/s over all ranks
with inputs resident in HBM; `e2e` adds the host->device copy of x and the
device->host copy of y to every step.  Each rank is an independent replica
(the layer needs no exchange on one GPU), so scaling is weak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth import BY_NAME, gen  # noqa: E402

METRIC = "MoE-layer tokens/s at 1 B200 (bf16, FP8) and % of tensor/HBM roofline"
L2_BYTES = 126 * 1024 * 1024


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", default="v3_bf16")
    p.add_argument("--cpu-sample", type=int, default=2, help="tokens per oracle sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the FP8 and decode workloads reported beside the headline")
    p.add_argument("--gather", choices=["on", "off"], default="off",
                   help="bf16: GEMM1 gathers routed rows from x through perm_tok (on) or "
                        "reads the permuted copy written by dispatch (off)")
    p.add_argument("--fused-combine", choices=["on", "off"], default="off",
                   help="bf16: the combine runs inside GEMM2's epilogue (on) or as its own "
                        "kernel (off); the output is bit-identical")
    p.add_argument("--only", choices=["backward", "backward_fp8"], default=None,
                   help="run one of the line's measurements alone and print its object "
                        "(backward: the bf16 expert backward on --config's shapes; "
                        "backward_fp8: the FP8 expert backward on the V3 FP8 shapes)")
    p.add_argument("--T", type=int, default=None, help="override tokens (profiling runs)")
    p.add_argument("--N", type=int, default=None, help="override routed experts (profiling)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"],
                    bf16_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    sustained_mhz=p.get("clocks_under_load", {}).get("sm_mhz_median"),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, sustained_mhz=1300.0,
                source="fallback")


def workload_name(cfg):
    return (f"{cfg.name}: T={cfg.T} d={cfg.d} N={cfg.N}+1 K={cfg.K} groups={cfg.G}/top{cfg.topG} "
            f"f={cfg.f} {cfg.dtype}")


def flops_per_forward(cfg):
    """Algorithmic FLOPs: router 2*T*d*N, experts 6*d*f per (token, expert)
    for the K routed experts and the shared one."""
    return 2.0 * cfg.T * cfg.d * cfg.N + 6.0 * cfg.d * cfg.f * cfg.T * (cfg.K + 1)


def ffn_flops(cfg):
    return 6.0 * cfg.d * cfg.f * cfg.T * (cfg.K + 1)


def bytes_per_forward(cfg, counts):
    """Algorithmic HBM bytes: weights of the experts that received rows plus
    the shared expert, x in, y out, the fp32 router (bf16 elements)."""
    used = int(np.count_nonzero(counts)) + 1
    wb = used * 3 * cfg.d * cfg.f * 2
    return wb + 2 * cfg.T * cfg.d * 2 + cfg.N * cfg.d * 4


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.5)  # let nvidia-smi start sampling before the timed region
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for name, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


def cpu_oracle_baseline(cfg, n_tokens, seed=0, batch=1000):
    """The float64 oracle as it stands on this host's cores: routing plus the
    expert and combine work of `n_tokens` tokens of a fresh batch.  Weight
    generation (into reused buffers) is excluded from the time.
    Returns (tokens/s, cores, note)."""
    import oracle
    R, b = gen.make_router(cfg), gen.make_bias(cfg)
    cores = len(os.sched_getaffinity(0))
    x = gen.make_x(cfg, seed, batch=batch)[:max(n_tokens, 1)]
    bufs = {w: np.empty(gen.weight_shape(cfg, w), np.float64) for w in ("w1", "w3", "w2")}
    gen_time = [0.0]

    def get(e):
        t0 = time.perf_counter()
        out = tuple(gen.make_expert_weight(cfg, seed, w, e, out=bufs[w])
                    for w in ("w1", "w3", "w2"))
        gen_time[0] += time.perf_counter() - t0
        return out

    t0 = time.perf_counter()
    oracle.moe_forward(x, R, b, get, cfg.G, cfg.topG, cfg.K,
                       h_round="none" if cfg.dtype == "fp32" else "bf16")
    dt = time.perf_counter() - t0 - gen_time[0]
    note = (f"{x.shape[0]} token(s) of the {cfg.name} workload per sample (full routing, the "
            f"K+1 expert FFNs and the combine; weight generation excluded), numpy float64 "
            f"on {cores} cores")
    return x.shape[0] / dt, cores, note


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        import torch
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
        pg = dist
    return world, rank, local, pg


def pair_gemm():
    """True when the bf16 expert GEMMs run on CTA pairs (MOE_BF16_GEMM=pair)."""
    return os.environ.get("MOE_BF16_GEMM") == "pair"


def reduce_max(values, pg, device):
    """Element-wise max of a list of floats over all ranks (identity on one rank)."""
    if pg is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return t.tolist()


def run_reference(args, cfg):
    world, rank, local, pg = dist_setup(args)
    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    times = []
    n = max(1, args.cpu_sample)
    for w in range(args.warmup):
        cpu_oracle_baseline(cfg, 1, batch=2000 + w)
    cores = len(os.sched_getaffinity(0))
    note = ""
    for k in range(args.steps):
        v, cores, note = cpu_oracle_baseline(cfg, n, batch=3000 + k)
        times.append(n / v)
    value = n * len(times) / sum(times)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(cfg), "sample_tokens_per_step": n},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": note},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def main():
    global GATHER, FUSED_COMBINE
    args = parse()
    GATHER = args.gather == "on"
    FUSED_COMBINE = args.fused_combine == "on"
    cfg = BY_NAME[args.config]
    if args.T:
        cfg = cfg.with_(T=args.T)
    if args.N:
        cfg = cfg.with_(N=args.N)
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.only == "backward":
        import torch
        out = run_backward(cfg, torch.device("cuda"), calls=max(1, args.steps),
                           warmup=args.warmup)
        print(json.dumps({"backward_dx": out}), flush=True)
        return out
    if args.only == "backward_fp8":
        import torch
        c8 = BY_NAME["v3_fp8"]
        if args.T:
            c8 = c8.with_(T=args.T)
        if args.N:
            c8 = c8.with_(N=args.N)
        out = run_backward_fp8(c8, torch.device("cuda"), calls=max(1, args.steps),
                               warmup=args.warmup)
        print(json.dumps({"backward_fp8": out}), flush=True)
        return out

    import torch

    world, rank, local, pg = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    main_res = run_layer(cfg, dev, args.steps, max(3, args.warmup), pg, local, e2e=True)
    extra = {}
    if not args.no_extra and not (args.T or args.N):
        # the FP8 layer, the decode workload and the mid-size bf16 layer,
        # reported beside the bf16 headline
        extra["fp8"] = run_layer(BY_NAME["v3_fp8"], dev, max(5, args.steps // 5), 3, pg, local)
        extra["mid"] = run_layer(BY_NAME["mid_bf16"], dev, max(20, args.steps), 3, pg, local)
        extra["decode"] = run_layer(BY_NAME["decode_zipf"], dev, max(20, args.steps), 3, pg,
                                    local)
    bwd = layer_bwd = bwd_fp8 = None
    if not args.no_extra and cfg.dtype == "bf16" and world == 1:
        bwd = run_backward(cfg, dev)
        layer_bwd = run_layer_backward(cfg, dev)
        bwd_fp8 = run_backward_fp8(BY_NAME["v3_fp8"], dev)

    if rank == 0:
        P = peaks()
        r = main_res
        ms_step = r["total_ms"] / args.steps
        value = world * cfg.T * args.steps / (r["total_ms"] / 1e3)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; random-init weights of the DeepSeek-V3 MoE layer shape)",
            "config": {"workload": workload_name(cfg), "global_batch": world * cfg.T,
                       "l2": "inputs larger than L2: the expert weights "
                             f"({(cfg.N + 1) * 3 * cfg.d * cfg.f * 2 / 1e9:.1f} GB) stream "
                             "through it every step",
                       "parallelism": f"replicas x{world}",
                       "combine": ("fused into GEMM2's epilogue" if FUSED_COMBINE
                                   else "own kernel")},
            "roofline": r["roofline"],
            "layer_roofline": r["layer_roofline"],
            "phases_ms": r["phases_ms"],
            "e2e": {"value": world * cfg.T * args.steps / (r["e2e_ms"] / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": cfg.T * cfg.d * 2,
                    "d2h_bytes_per_step": cfg.T * cfg.d * 2},
            "gpu_launches": r["launches_per_step"] * args.steps,
            "clocks": r["clocks"],
            "device_status": r["status"],
            "load_max_over_mean": r["load_max_over_mean"],
        }
        if r.get("softmax_route"):
            line["softmax_route"] = r["softmax_route"]
        if r.get("graph"):
            line["graph_replay"] = r["graph"]
        for k, v in extra.items():
            line[k] = {"workload": workload_name(v["cfg"]),
                       "value": world * v["cfg"].T * v["steps"] / (v["total_ms"] / 1e3),
                       "unit": "tokens/s", "ms_per_step": v["total_ms"] / v["steps"],
                       "steps": v["steps"], "roofline": v["roofline"],
                       "layer_roofline": v["layer_roofline"], "phases_ms": v["phases_ms"],
                       "clocks": v["clocks"], "device_status": v["status"],
                       "load_max_over_mean": v["load_max_over_mean"]}
        if bwd is not None:
            line["backward_dx"] = bwd
        if layer_bwd is not None:
            line["layer_backward"] = layer_bwd
        if bwd_fp8 is not None:
            line["backward_fp8"] = bwd_fp8
        if world == 1 and not args.no_cpu_baseline:
            v, cores, note = cpu_oracle_baseline(cfg, args.cpu_sample)
            line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores,
                                    "kind": "oracle", "sample": note}
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_e2e(M, s, layer, x, w13, w2, s13, s2, cfg, steps, stream):
    """End to end through the C-ABI calls with host buffers: every step copies
    its x from pinned host memory to the GPU and its y back.  The copies run on
    two copy streams (PCIe is full duplex) so step k+1's upload and step k-1's
    download overlap step k's compute; x and y are double-buffered on the
    device.  Returns ms from the first upload to the last download."""
    import torch
    dev = x.device
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_host = [x.cpu().pin_memory() for _ in range(2)]
    y_host = [torch.empty(cfg.T, cfg.d, dtype=layer.y.dtype).pin_memory() for _ in range(2)]
    xs = [torch.empty_like(x) for _ in range(2)]
    ys = [torch.empty_like(layer.y) for _ in range(2)]
    ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731

    def run(n):
        x_ready = [ev() for _ in range(2)]
        done = [None, None]
        y_out = [None, None]
        for k in range(n):
            b = k & 1
            # upload step k's input once step k-2 (same buffer) has finished with it
            if done[b] is not None:
                h2d.wait_event(done[b])
            with torch.cuda.stream(h2d):
                xs[b].copy_(x_host[b], non_blocking=True)
            x_ready[b].record(h2d)
            stream.wait_event(x_ready[b])
            if y_out[b] is not None:  # ys[b] is being read back for step k-2
                stream.wait_event(y_out[b])
            xb = xs[b]
            M.moe_route(s, xb, layer.router_w, layer.bias, layer.topk_idx, layer.topk_gate,
                        layer.counts, layer.ws, stream)
            M.moe_dispatch(s, xb, layer.topk_idx, layer.counts, layer.offsets, layer.perm_tok,
                           layer.slot, layer.x_perm, layer.x_perm_scales, layer.ws, stream)
            if layer.fused_combine:
                M.moe_expert_ffn_combine(s, layer.x_perm, layer.offsets, layer.perm_tok,
                                         layer.slot, layer.topk_gate, xb, layer.w13, layer.w2,
                                         layer.y_perm, layer.y_shared, ys[b], layer.ws, stream)
            else:
                layer.experts(xb, stream)
                M.moe_combine(s, layer.y_perm, layer.y_shared, layer.slot, layer.topk_gate,
                              ys[b], stream)
            M.moe_bias_update(s, layer.counts, layer.bias, cfg.gamma, stream)
            done[b] = ev()
            done[b].record(stream)
            d2h.wait_event(done[b])
            with torch.cuda.stream(d2h):
                y_host[b].copy_(ys[b], non_blocking=True)
            y_out[b] = ev()
            y_out[b].record(d2h)

    run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d)          # before the first upload
    stream.wait_stream(h2d)
    d2h.wait_stream(h2d)
    run(steps)
    h2d.wait_stream(d2h)
    h2d.wait_stream(stream)
    e1.record(h2d)          # after the last download
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


GATHER = False  # set from --gather in main()
FUSED_COMBINE = False  # set from --fused-combine in main()


def run_backward(cfg, dev, calls=10, warmup=3):
    """The expert backward, input gradients (moe_expert_ffn_backward_dx), on the
    layer's routing of one synthetic batch: GEMM1 recomputed, dY W2^T with the
    SwiGLU-backward epilogue, dGU W13 -- 10*d*f FLOP per dispatched or shared
    row.  dY is seeded synthetic N(0, 1) bf16.  CUDA events over `calls` calls
    after `warmup`."""
    import torch
    import sparse_moe_layer_limited_b200 as M
    from synth import device as sdev
    s = M.shape(cfg.T, cfg.d, cfg.N, cfg.K, cfg.G, cfg.topG, cfg.f, M.DTYPE_BF16)
    w1 = sdev.expert_weights_bf16(cfg, 0, "w1", dev)
    w3 = sdev.expert_weights_bf16(cfg, 0, "w3", dev)
    w13 = torch.empty(cfg.N + 1, 2 * cfg.f, cfg.d, dtype=torch.bfloat16, device=dev)
    M.moe_pack_w13(s, w1, w3, w13)
    del w1, w3
    w2 = sdev.expert_weights_bf16(cfg, 0, "w2", dev)
    w13t = torch.empty(cfg.N + 1, cfg.d, 2 * cfg.f, dtype=torch.bfloat16, device=dev)
    w2t = torch.empty(cfg.N + 1, cfg.f, cfg.d, dtype=torch.bfloat16, device=dev)
    M.moe_transpose_weights(s, w13, w2, w13t, w2t)
    router = torch.from_numpy(gen.make_router(cfg)).to(dev)
    bias = torch.from_numpy(gen.make_bias(cfg)).to(dev)
    layer = M.MoELayer(s, router, bias, w13, w2, gamma=cfg.gamma)
    x = sdev.x_bf16(cfg, 0, device=dev)
    layer.forward(x, update_bias=False)
    g = torch.Generator(device=dev).manual_seed(7)
    dyp = torch.randn(cfg.T * cfg.K, cfg.d, generator=g, device=dev).to(torch.bfloat16)
    dys = torch.randn(cfg.T, cfg.d, generator=g, device=dev).to(torch.bfloat16)
    dxp, dxs = torch.empty_like(dyp), torch.empty_like(dys)
    ws = torch.zeros(M.backward_workspace_size(s), dtype=torch.uint8, device=dev)

    dw13, dw2 = torch.empty_like(w13), torch.empty_like(w2)

    def call_dx():
        M.moe_expert_ffn_backward_dx(s, layer.x_perm, layer.offsets, x, w13, w13t, w2t, dyp, dys,
                                     dxp, dxs, ws)

    def call_dw():
        M.moe_expert_ffn_backward_dw(s, layer.x_perm, layer.offsets, x, dyp, dys, dw13, dw2, ws)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(calls):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / calls

    ms = timed(call_dx)
    call_dx()                # the weight pass reads what the input pass leaves in ws
    ms_dw = timed(call_dw)
    ms_wt = timed(lambda: M.moe_transpose_weights(s, w13, w2, w13t, w2t))
    wt_bytes = 2.0 * 2 * (cfg.N + 1) * 3 * cfg.d * cfg.f  # read + write, bf16
    status = M.moe_read_device_status(ws)
    rows = cfg.T * cfg.K + cfg.T
    fl = 10.0 * cfg.d * cfg.f * rows
    fl_dw = 6.0 * cfg.d * cfg.f * rows
    P = peaks()
    pk, pk_sus = P["bf16"], P["bf16_sustained"]
    achieved = fl / (ms / 1e3) / 1e12
    achieved_dw = fl_dw / (ms_dw / 1e3) / 1e12
    return {"workload": workload_name(cfg), "ms": ms, "tokens_per_s": cfg.T / (ms / 1e3),
            "roofline": {"bound": "tensor", "achieved": achieved, "unit": "TFLOP/s",
                         "peak": pk, "frac": achieved / pk, "peak_source": P["source"] +
                         " bf16 burst", "frac_of_sustained": achieved / pk_sus,
                         "flops_per_call": fl},
            "gpu_launches_per_call": 3, "device_status": status,
            "weight_gradients": {"ms": ms_dw, "achieved": achieved_dw, "unit": "TFLOP/s",
                                 "frac": achieved_dw / pk,
                                 "frac_of_sustained": achieved_dw / pk_sus,
                                 "flops_per_call": fl_dw,
                                 "gpu_launches_per_call": 7,
                                 "kernel": ("one CTA" if os.environ.get("MOE_WGRAD") == "single"
                                            else "CTA pair"),
                                 "note": "dW2 and dW13 of every expert (6 d f FLOP per row), "
                                         "including the transposes into per-expert blocks"},
            "weight_transpose": {"ms": ms_wt, "bytes": wt_bytes,
                                 "achieved_gbs": wt_bytes / (ms_wt / 1e3) / 1e9,
                                 "frac_of_hbm": wt_bytes / (ms_wt / 1e3) / 1e9 / P["hbm"],
                                 "note": "moe_transpose_weights (W13^T, W2^T of every expert), "
                                         "once per weight update, outside the timed steps"},
            "note": "expert FFN input gradients: GEMM1 recomputed, dh with the SwiGLU-backward "
                    "epilogue, dx (3 launches); weight gradients beside them"}


def run_backward_fp8(cfg, dev, calls=5, warmup=2):
    """The FP8 expert backward on the layer's routing of one synthetic batch
    (E4M3 weights and activations, E5M2 gradients): input gradients
    (moe_expert_ffn_backward_dx_fp8: GEMM1 recomputed, dY quantised, dY W2^T
    with the SwiGLU-backward epilogue, dGU quantised, dGU W13; 10*d*f FLOP per
    dispatched or shared row) and weight gradients
    (moe_expert_ffn_backward_dw_fp8: layout, four quantisations, dW2 and
    dW13; 6*d*f FLOP per row).  dY is seeded N(0, 1) bf16.  CUDA events over
    `calls` calls after `warmup`; peak = the measured bf16 burst rate x 2."""
    import torch
    import sparse_moe_layer_limited_b200 as M
    from synth import device as sdev
    s = M.shape(cfg.T, cfg.d, cfg.N, cfg.K, cfg.G, cfg.topG, cfg.f, M.DTYPE_E4M3)
    E, d, f = cfg.N + 1, cfg.d, cfg.f
    w1 = sdev.expert_weights_bf16(cfg, 0, "w1", dev)
    w3 = sdev.expert_weights_bf16(cfg, 0, "w3", dev)
    w13 = torch.empty(E, 2 * f, d, dtype=torch.bfloat16, device=dev)
    M.moe_pack_w13(s, w1, w3, w13)
    del w1, w3
    w2 = sdev.expert_weights_bf16(cfg, 0, "w2", dev)
    q = lambda *shape: torch.empty(*shape, dtype=torch.float8_e4m3fn, device=dev)  # noqa: E731
    f32 = lambda *shape: torch.empty(*shape, dtype=torch.float32, device=dev)  # noqa: E731
    w13q, w2q = q(E, 2 * f, d), q(E, d, f)
    s13, s2 = f32(E, 2 * f // 128, d // 128), f32(E, d // 128, f // 128)
    M.moe_quantize_weights(s, w13, w2, w13q, s13, w2q, s2)
    w13t = torch.empty(E, d, 2 * f, dtype=torch.bfloat16, device=dev)
    w2t = torch.empty(E, f, d, dtype=torch.bfloat16, device=dev)
    M.moe_transpose_weights(s, w13, w2, w13t, w2t)
    del w13, w2
    w13tq, w2tq = q(E, d, 2 * f), q(E, f, d)
    s13t, s2t = f32(E, d // 128, 2 * f // 128), f32(E, f // 128, d // 128)
    M.moe_quantize_weights_transposed(s, w13t, w2t, w13tq, s13t, w2tq, s2t)
    torch.cuda.synchronize()
    del w13t, w2t
    router = torch.from_numpy(gen.make_router(cfg)).to(dev)
    bias = torch.from_numpy(gen.make_bias(cfg)).to(dev)
    layer = M.MoELayer(s, router, bias, w13q, w2q, s13, s2, gamma=cfg.gamma)
    x = sdev.x_bf16(cfg, 0, device=dev)
    layer.forward(x, update_bias=False)
    g = torch.Generator(device=dev).manual_seed(7)
    dyp = torch.randn(cfg.T * cfg.K, d, generator=g, device=dev).to(torch.bfloat16)
    dys = torch.randn(cfg.T, d, generator=g, device=dev).to(torch.bfloat16)
    dxp, dxs = torch.empty_like(dyp), torch.empty_like(dys)
    ws = torch.zeros(M.backward_workspace_size(s), dtype=torch.uint8, device=dev)
    dw13 = torch.empty(E, 2 * f, d, dtype=torch.bfloat16, device=dev)
    dw2 = torch.empty(E, d, f, dtype=torch.bfloat16, device=dev)

    def call_dx():
        M.moe_expert_ffn_backward_dx_fp8(s, layer.x_perm, layer.x_perm_scales, layer.offsets, x,
                                         w13q, s13, w13tq, s13t, w2tq, s2t, dyp, dys, dxp, dxs,
                                         ws)

    def call_dw():
        M.moe_expert_ffn_backward_dw_fp8(s, layer.perm_tok, layer.offsets, x, dyp, dys, dw13,
                                         dw2, ws)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(calls):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / calls

    ms = timed(call_dx)
    call_dx()                # the weight pass reads what the input pass leaves in ws
    ms_dw = timed(call_dw)
    status = M.moe_read_device_status(ws)
    rows = cfg.T * cfg.K + cfg.T
    fl, fl_dw = 10.0 * d * f * rows, 6.0 * d * f * rows
    P = peaks()
    pk = 2.0 * P["bf16"]
    a, a_dw = fl / (ms / 1e3) / 1e12, fl_dw / (ms_dw / 1e3) / 1e12
    return {"workload": workload_name(cfg), "ms": ms, "tokens_per_s": cfg.T / (ms / 1e3),
            "roofline": {"bound": "tensor", "achieved": a, "unit": "TFLOP/s", "peak": pk,
                         "frac": a / pk, "peak_source": P["source"] + " bf16 burst x nominal "
                         "fp8/bf16 ratio 2", "flops_per_call": fl},
            "gpu_launches_per_call": 7, "device_status": status,
            "weight_gradients": {"ms": ms_dw, "achieved": a_dw, "unit": "TFLOP/s",
                                 "frac": a_dw / pk, "flops_per_call": fl_dw,
                                 "gpu_launches_per_call": 11,
                                 "note": "dW2 and dW13 of every expert (6 d f FLOP per row), "
                                         "including the layout pass and the four 1x128 "
                                         "quantisations"},
            "note": "E4M3 operands, E5M2 gradients: input gradients (GEMM1 recomputed, dY "
                    "quantised, dh with the SwiGLU-backward epilogue, dGU quantised, dx)"}


def run_layer_backward(cfg, dev, calls=10, warmup=3):
    """The backward steps around the experts on the layer's routing of one
    synthetic batch (BF16): moe_combine_backward, moe_route_backward,
    moe_dispatch_backward, each against the HBM roofline of its algorithmic
    bytes, and the whole MoELayer.backward (14 launches).  dy is seeded
    N(0, 1) bf16.  CUDA events over `calls` calls after `warmup`."""
    import torch
    import sparse_moe_layer_limited_b200 as M
    from synth import device as sdev
    s = M.shape(cfg.T, cfg.d, cfg.N, cfg.K, cfg.G, cfg.topG, cfg.f, M.DTYPE_BF16)
    w1 = sdev.expert_weights_bf16(cfg, 0, "w1", dev)
    w3 = sdev.expert_weights_bf16(cfg, 0, "w3", dev)
    w13 = torch.empty(cfg.N + 1, 2 * cfg.f, cfg.d, dtype=torch.bfloat16, device=dev)
    M.moe_pack_w13(s, w1, w3, w13)
    del w1, w3
    w2 = sdev.expert_weights_bf16(cfg, 0, "w2", dev)
    w13t = torch.empty(cfg.N + 1, cfg.d, 2 * cfg.f, dtype=torch.bfloat16, device=dev)
    w2t = torch.empty(cfg.N + 1, cfg.f, cfg.d, dtype=torch.bfloat16, device=dev)
    M.moe_transpose_weights(s, w13, w2, w13t, w2t)
    router = torch.from_numpy(gen.make_router(cfg)).to(dev)
    bias = torch.from_numpy(gen.make_bias(cfg)).to(dev)
    layer = M.MoELayer(s, router, bias, w13, w2, gamma=cfg.gamma)
    x = sdev.x_bf16(cfg, 0, device=dev)
    layer.forward(x, update_bias=False)
    g = torch.Generator(device=dev).manual_seed(11)
    T, K, d, N = cfg.T, cfg.K, cfg.d, cfg.N
    dy = torch.randn(T, d, generator=g, device=dev).to(torch.bfloat16)
    dyp = torch.empty(T * K, d, dtype=torch.bfloat16, device=dev)
    dgate = torch.empty(T, K, dtype=torch.float32, device=dev)
    dl = torch.empty(T, K, dtype=torch.float32, device=dev)
    dxr = torch.empty(T, d, dtype=torch.float32, device=dev)
    dR = torch.empty(N, d, dtype=torch.float32, device=dev)
    dxp = torch.randn(T * K, d, generator=g, device=dev).to(torch.bfloat16)
    dx = torch.empty(T, d, dtype=torch.bfloat16, device=dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(calls):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / calls

    P = peaks()
    steps = {
        "combine_backward": (
            lambda: M.moe_combine_backward(s, dy, layer.y_perm, layer.slot, layer.topk_gate, dyp,
                                           dgate),
            2.0 * (T * d + 2 * T * K * d), "dy + y_perm read, dy_perm written (bf16)"),
        "route_backward": (
            lambda: M.moe_route_backward(s, x, router, layer.topk_idx, dgate, layer.offsets,
                                         layer.perm_tok, layer.slot, dl, dxr, dR),
            2.0 * T * d + 4.0 * (N * d + T * d + N * d),
            "x and the router read once, dx_route and drouter written (fp32)"),
        "dispatch_backward": (
            lambda: M.moe_dispatch_backward(s, dxp, dy, layer.slot, dxr, dx),
            2.0 * (T * K * d + 2 * T * d) + 4.0 * T * d,
            "dx_perm, dx_shared, dx_route read, dx written"),
    }
    out = {"workload": workload_name(cfg)}
    for name, (fn, nbytes, what) in steps.items():
        ms = timed(fn)
        out[name] = {"ms": ms, "bytes": nbytes, "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
                     "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / P["hbm"], "bytes_note": what}
    ms_all = timed(lambda: layer.backward(x, dy, w13t, w2t))
    out["layer_backward"] = {"ms": ms_all, "tokens_per_s": T / (ms_all / 1e3),
                             "gpu_launches_per_call": 14,
                             "note": "combine, expert input and weight gradients, gate and "
                                     "router, dispatch"}
    out["device_status"] = layer.backward_status()
    return out


def graph_step_timing(layer, x, steps, warmup=3):
    """The same layer step (route -> bias update) captured in one CUDA graph
    and replayed `steps` times after `warmup` replays, CUDA events around the
    replays: the step without host launch overhead."""
    import torch
    layer.capture(x)
    for _ in range(warmup):
        layer.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        layer.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return {"ms_per_step": ms, "value": x.shape[0] / (ms / 1e3), "unit": "tokens/s",
            "note": "one CUDA graph per step (route, dispatch, experts, combine, bias update), "
                    "replayed back to back"}


def softmax_route_baseline(M, s, x, router, layer, cfg, stream, reps=20):
    """The conventional softmax top-K router (moe_route_softmax) on the same
    input, for contrast with the method's routing: time per call (CUDA events,
    after 3 warm-up calls) and the balance statistic N * sum f_i P_i of its
    selections (1 = uniform)."""
    import torch
    dev = x.device
    idx = torch.empty(s.T, s.K, dtype=torch.int32, device=dev)
    gate = torch.empty(s.T, s.K, dtype=torch.float32, device=dev)
    cnt = torch.empty(s.N, dtype=torch.int32, device=dev)
    psum = torch.empty(s.N, dtype=torch.float32, device=dev)
    for _ in range(3):
        M.moe_route_softmax(s, x, router, idx, gate, cnt, psum, layer.ws, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        M.moe_route_softmax(s, x, router, idx, gate, cnt, psum, layer.ws, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    c = cnt.cpu().numpy().astype(np.float64)
    P = psum.cpu().numpy().astype(np.float64) / s.T
    f = c / (s.K * s.T)
    return {"ms": e0.elapsed_time(e1) / reps, "balance": float(s.N * np.sum(f * P)),
            "load_max_over_mean": float(c.max() / c.mean()),
            "note": "softmax top-K over all experts, no bias or group limit (the baseline "
                    "the method replaces); balance = N * sum_i f_i * P_i"}


_READ_GBS = {}


def hbm_read_stream_gbs(dev, gib=4, reps=10):
    """Read-only HBM bandwidth over a `gib` GiB bf16 buffer (larger than L2):
    the better of a float32 sum over it and a matrix-vector product that
    streams it as a [rows, 8192] matrix, each best of `reps` CUDA-event
    timings; bytes read / time."""
    import torch
    if dev in _READ_GBS:
        return _READ_GBS[dev]
    n = gib * (1 << 30) // 2
    buf = torch.ones(n, dtype=torch.bfloat16, device=dev)
    mat = buf.view(-1, 8192)
    vec = torch.ones(8192, dtype=torch.bfloat16, device=dev)

    def best(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        out = 1e30
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            out = min(out, e0.elapsed_time(e1))
        return out

    ms = min(best(lambda: buf.sum(dtype=torch.float32)), best(lambda: torch.mv(mat, vec)))
    del buf, mat, vec
    torch.cuda.empty_cache()
    _READ_GBS[dev] = 2.0 * n / (ms / 1e3) / 1e9
    return _READ_GBS[dev]


def run_layer(cfg, dev, steps, warmup, pg, local, e2e=False):
    """Build one layer of `cfg` on `dev` (weights generated on the device), run
    `warmup` untimed steps and `steps` timed steps, each a full forward plus
    the bias update, with CUDA events around every entry point."""
    import torch
    import sparse_moe_layer_limited_b200 as M
    from synth import device as sdev

    dt = {"fp32": M.DTYPE_FP32, "bf16": M.DTYPE_BF16, "e4m3": M.DTYPE_E4M3}[cfg.dtype]
    s = M.shape(cfg.T, cfg.d, cfg.N, cfg.K, cfg.G, cfg.topG, cfg.f, dt)
    w1 = sdev.expert_weights_bf16(cfg, 0, "w1", dev)
    w3 = sdev.expert_weights_bf16(cfg, 0, "w3", dev)
    w13 = torch.empty(cfg.N + 1, 2 * cfg.f, cfg.d, dtype=torch.bfloat16, device=dev)
    M.moe_pack_w13(s, w1, w3, w13)
    del w1, w3
    w2 = sdev.expert_weights_bf16(cfg, 0, "w2", dev)
    s13 = s2 = None
    if cfg.dtype == "e4m3":
        w13q = torch.empty(w13.shape, dtype=torch.float8_e4m3fn, device=dev)
        w2q = torch.empty(w2.shape, dtype=torch.float8_e4m3fn, device=dev)
        s13 = torch.empty(cfg.N + 1, 2 * cfg.f // 128, cfg.d // 128, dtype=torch.float32,
                          device=dev)
        s2 = torch.empty(cfg.N + 1, cfg.d // 128, cfg.f // 128, dtype=torch.float32, device=dev)
        M.moe_quantize_weights(s, w13, w2, w13q, s13, w2q, s2)
        torch.cuda.synchronize()
        del w13, w2
        w13, w2 = w13q, w2q
    router = torch.from_numpy(gen.make_router(cfg)).to(dev)
    bias = torch.from_numpy(gen.make_bias(cfg)).to(dev)
    if cfg.zipf_s is None:
        x = sdev.x_bf16(cfg, 0, 0, dev)
    else:
        x = torch.from_numpy(gen.make_x(cfg)).to(torch.bfloat16).to(dev)
    layer = M.MoELayer(s, router, bias, w13, w2, s13, s2, gamma=cfg.gamma, gather=GATHER,
                       fused_combine=FUSED_COMBINE)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)
    phases = ["route", "dispatch", "experts", "combine", "bias"]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        M.moe_route(s, x, router, layer.bias, layer.topk_idx, layer.topk_gate, layer.counts,
                    layer.ws, stream)
        if ev is not None:
            ev[1].record(stream)
        M.moe_dispatch(s, x, layer.topk_idx, layer.counts, layer.offsets, layer.perm_tok,
                       layer.slot, layer.x_perm, layer.x_perm_scales, layer.ws, stream)
        if ev is not None:
            ev[2].record(stream)
        if layer.fused_combine:   # experts and combine in one pair of launches
            layer.experts_and_combine(x, stream)
        else:
            layer.experts(x, stream)
        if ev is not None:
            ev[3].record(stream)
        if not layer.fused_combine:
            M.moe_combine(s, layer.y_perm, layer.y_shared, layer.slot, layer.topk_gate, layer.y,
                          stream)
        if ev is not None:
            ev[4].record(stream)
        M.moe_bias_update(s, layer.counts, layer.bias, cfg.gamma, stream)
        if ev is not None:
            ev[5].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    if pg is not None:
        pg.barrier()
    M.moe_read_gemm_clock(layer.ws, clear=True)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for k in range(steps):
            step(evs[k])
        torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    # the SM clock the expert GEMMs themselves ran at (their first CTA's
    # cycle and nanosecond counters over the timed steps)
    gclk = M.moe_read_gemm_clock(layer.ws)
    per_phase = {p: [evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(steps)]
                 for i, p in enumerate(phases)}
    total_ms = evs[0][0].elapsed_time(evs[-1][5])
    counts = layer.counts.cpu().numpy()
    status = layer.device_status()

    e2e_ms = None
    baseline = None
    graph = None
    if e2e:
        e2e_ms = run_e2e(M, s, layer, x, w13, w2, s13, s2, cfg, steps, stream)
        if cfg.dtype != "fp32":  # the softmax router takes bf16 activations
            baseline = softmax_route_baseline(M, s, x, router, layer, cfg, stream)
        graph = graph_step_timing(layer, x, steps)

    total_ms, e2e_ms = reduce_max([total_ms, e2e_ms or 0.0], pg, dev)

    P = peaks()
    fp8 = cfg.dtype == "e4m3"
    # Denominator: the measured burst bf16 GEMM rate (cuBLAS 8192^3, best of
    # 10), x2 for E4M3 (the nominal dense fp8/bf16 ratio, 4.5 / 2.25 PFLOP/s).
    # The measured sustained rate (a seconds-long loop under the power cap)
    # and the fraction against it are reported beside it for context.
    ratio = 2.0 if fp8 else 1.0
    peak = P["bf16"] * ratio
    peak_sus = P["bf16_sustained"] * ratio
    peak_src = P["source"] + (" bf16 burst x nominal fp8/bf16 ratio 2" if fp8
                              else " bf16 burst")
    ffn_ms = statistics.mean(per_phase["experts"])
    wbytes = 1 if fp8 else 2
    fl = flops_per_forward(cfg)
    used = int(np.count_nonzero(counts)) + 1
    by = used * 3 * cfg.d * cfg.f * wbytes + 2 * cfg.T * cfg.d * 2 + cfg.N * cfg.d * 4
    roof_ms = max(fl / (peak * 1e12), by / (P["hbm"] * 1e9)) * 1e3
    ms_step = total_ms / steps
    kmhz = gclk["fp8_mhz"] if fp8 else gclk["bf16_mhz"]
    if cfg.zipf_s is None:
        achieved = ffn_flops(cfg) / (ffn_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": "moe_expert_ffn (grouped GEMM1+SwiGLU, GEMM2)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": peak_src, "peak_sustained": peak_sus,
                "frac_of_sustained": achieved / peak_sus, "traffic": None,
                "kernel_sm_mhz": kmhz}
        if kmhz and P.get("sustained_mhz"):
            # the measured cuBLAS rate per MHz (its sustained run and that run's
            # median clock) at the clock these kernels ran at
            at_clk = peak_sus * kmhz / P["sustained_mhz"]
            roof["peak_at_kernel_clock"] = at_clk
            roof["frac_at_kernel_clock"] = achieved / at_clk
        if cfg.name == "v3_bf16" and cfg.T == 8192 and cfg.N == 256 and not pair_gemm():
            # DRAM bytes of one moe_expert_ffn call (GEMM1 + GEMM2), from the ncu
            # capture of the same kernels on the T=1024 / 32+1-expert case
            # (3.28 GB), scaled by the expert weights (x 257/33) and the
            # activation rows (x 8)
            roof["traffic"] = 25.6e9
            roof["traffic_note"] = ("bytes per call, ncu capture of a smaller case scaled to "
                                    "the full layer; algorithmic 25.35e9")
        if cfg.name == "v3_fp8" and cfg.T == 16384 and cfg.N == 256:
            # DRAM bytes of one moe_expert_ffn call (both FP8 GEMMs): the ncu
            # capture on the T=1024 / 32+1-expert case measured 1.719 GB against
            # 1.693 GB algorithmic; the same ratio applied to the full layer's
            # 15.15 GB algorithmic
            roof["traffic"] = 15.38e9
            roof["traffic_note"] = ("bytes per call, ncu capture of a smaller case scaled to "
                                    "the full layer; algorithmic 15.15e9")
    else:
        # decode: the experts stream the weights of the experts that received rows
        wb = used * 3 * cfg.d * cfg.f * wbytes
        achieved = wb / (ffn_ms / 1e3) / 1e9
        # the experts only read weights: the denominator is the better of the
        # measured read+write copy and a read-only stream measured here
        rd = hbm_read_stream_gbs(dev)
        pk = max(P["hbm"], rd)
        roof = {"bound": "hbm", "kernel": "moe_expert_ffn (weights of the experts hit)",
                "achieved": achieved, "peak": pk, "unit": "GB/s", "frac": achieved / pk,
                "peak_source": ("read-only stream measured in this run" if rd >= P["hbm"]
                                else P["source"] + " copy"),
                "peak_copy": P["hbm"], "peak_read_stream": rd, "nominal_gbs": 7700.0,
                "frac_of_nominal": achieved / 7700.0,
                "traffic": None, "experts_hit": used - 1, "kernel_sm_mhz": kmhz}
        if cfg.name == "decode_zipf" and cfg.d == 7168 and cfg.f == 2048:
            # DRAM bytes of the two expert GEMM launches, from an ncu capture
            # of the same workload (1-pass dram__bytes metrics): 14.66 GB read +
            # written for 166 experts hit, 1.0023x their weight bytes; the
            # same ratio applied to this run's experts
            roof["traffic"] = wb * 1.0023
            roof["traffic_note"] = ("bytes per experts phase (GEMM1 + GEMM2), ncu capture of "
                                    "this workload scaled by the experts hit")
    return {"cfg": cfg, "steps": steps, "total_ms": total_ms, "e2e_ms": e2e_ms,
            "softmax_route": baseline, "graph": graph,
            "phases_ms": {p: statistics.mean(v) for p, v in per_phase.items()},
            "roofline": roof,
            "layer_roofline": {"ms": roof_ms, "frac": roof_ms / ms_step, "flops": fl, "bytes": by},
            "clocks": clk.summary(), "status": status,
            "load_max_over_mean": float(counts.max() / counts.mean()),
            # route 3 (split, score GEMM, select), dispatch 3, experts 2 (+1 quantiser
            # for FP8), combine 1, bias 1
            "launches_per_step": (10 if not fp8 else 11) - (1 if layer.fused_combine else 0),
            "fused_combine": bool(layer.fused_combine)}


if __name__ == "__main__":
    main()
