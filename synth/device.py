"""Device-side fill of the synthetic tensors (same values as ``synth.gen``).

Only the large bf16 tensors (expert weights, big activations) are generated on
the GPU; everything is keyed exactly as in ``synth.gen`` so the host can
regenerate any expert's weights for the oracle.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import gen
from .configs import MoEConfig

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(verbose: bool = False) -> str:
    import subprocess
    cmd = ["nvcc", "-shared", "-Xcompiler", "-fPIC", "-O3",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-o", LIB_PATH, os.path.join(_HERE, "csrc", "gen.cu")]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run __graft_entry__.build()")
        _lib = ctypes.CDLL(LIB_PATH)
        _lib.synth_fill_table_u16.restype = ctypes.c_int
        _lib.synth_fill_table_u16.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                              ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    return _lib


def fill_bf16(out, keys, per_stream: int, sigma: float):
    """Fill torch bf16 tensor ``out`` (len(keys) * per_stream elements) with the
    N(0, sigma^2) streams ``keys``."""
    import torch
    dev = out.device
    table = torch.from_numpy(gen.f32_to_bf16_bits(gen.normal_table(float(sigma), "bf16"))
                             .view(np.int16)).to(dev)
    keys_t = torch.from_numpy(np.array(keys, dtype=np.uint64).view(np.int64)).to(dev)
    assert out.dtype == torch.bfloat16 and out.is_contiguous()
    assert out.numel() == len(keys) * per_stream
    rc = lib().synth_fill_table_u16(out.data_ptr(), keys_t.data_ptr(), len(keys), per_stream,
                                    table.data_ptr(), torch.cuda.current_stream(dev).cuda_stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_table_u16 failed: {rc}")
    return out


def expert_weights_bf16(cfg: MoEConfig, seed: int, which: str, device="cuda"):
    """All N+1 experts' W1/W3 ([N+1, f, d]) or W2 ([N+1, d, f]) as bf16 on the GPU."""
    import torch
    shape = gen.weight_shape(cfg, which)
    out = torch.empty((cfg.N + 1,) + shape, dtype=torch.bfloat16, device=device)
    keys = [gen.weight_key(cfg, seed, which, e) for e in range(cfg.N + 1)]
    return fill_bf16(out, keys, shape[0] * shape[1], gen.weight_sigma(cfg, which))


def x_bf16(cfg: MoEConfig, seed: int = 0, batch: int = 0, device="cuda"):
    """The layer input x [T, d] as bf16 on the GPU (plain N(0,1) workloads)."""
    import torch
    assert cfg.zipf_s is None and gen.x_dtype(cfg) == "bf16"
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=device)
    return fill_bf16(out, [gen.stream_key(seed, cfg.cfg_id, gen.T_X, batch)], cfg.T * cfg.d, 1.0)
