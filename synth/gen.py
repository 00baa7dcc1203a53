"""Seeded synthetic inputs for the MoE-layer workloads.

This module is shared by the float64 oracle (tests) and the CUDA path (tests,
bench).  It holds no arithmetic of the MoE method: only counter-based random
streams, the distributions named for each workload, and rounding to the
storage dtype.

Random stream
-------------
Every tensor (and, for expert weights, every expert) has its own 64-bit key,
folded from (seed, config id, tensor id, sub-ids) with the SplitMix64 finaliser
(Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014).  Element i of a stream is ``u_i = mix64(key + (i+1)*GOLDEN)``.

Normal draws use the top 16 bits of ``u_i`` to index a table of the 65536
mid-point quantiles of N(0,1) (``Phi^-1((j+0.5)/65536)``, float64), times
sigma, rounded to float32 and then (bf16 tensors) to bfloat16 with
round-to-nearest-even.  Because a draw is an integer hash plus a table look-up,
the device generator (``synth/csrc/gen.cu``) reproduces it bit for bit.

Uniform draws use the top 53 bits: ``lo + (hi-lo) * (u >> 11) * 2**-53`` in
float64, rounded to float32.
"""
from __future__ import annotations

import math
import os
from functools import lru_cache
from statistics import NormalDist

import numpy as np

from .configs import MoEConfig

GOLDEN = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1

# tensor ids for key folding
T_X, T_ROUTER, T_BIAS, T_W1, T_W3, T_W2, T_ZIPF_U, T_ZIPF_PERM, T_XREDRAW = range(1, 10)


def _mix64_int(z: int) -> int:
    z &= M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def stream_key(seed: int, *fields: int) -> int:
    """Fold (seed, fields...) into one 64-bit stream key."""
    k = _mix64_int((seed + 1) * GOLDEN)
    for v in fields:
        k = _mix64_int(k + ((int(v) + 1) * GOLDEN))
    return k


_CHUNK = 1 << 20


def _mix64_inplace(z: np.ndarray, t: np.ndarray) -> None:
    """SplitMix64 finaliser applied in place to ``z`` (``t`` is scratch)."""
    np.right_shift(z, np.uint64(30), out=t)
    np.bitwise_xor(z, t, out=z)
    np.multiply(z, np.uint64(0xBF58476D1CE4E5B9), out=z)
    np.right_shift(z, np.uint64(27), out=t)
    np.bitwise_xor(z, t, out=z)
    np.multiply(z, np.uint64(0x94D049BB133111EB), out=z)
    np.right_shift(z, np.uint64(31), out=t)
    np.bitwise_xor(z, t, out=z)


def _stream_chunks(key: int, n: int, start: int = 0):
    """Yield (offset, uint64 chunk) covering stream elements start..start+n-1.
    The chunk buffer is reused between yields."""
    z = np.empty(min(n, _CHUNK), dtype=np.uint64)
    t = np.empty_like(z)
    base = np.arange(1, z.size + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for off in range(0, n, _CHUNK):
            m = min(_CHUNK, n - off)
            zz, tt = z[:m], t[:m]
            # z = key + (start + off + j + 1) * GOLDEN  (mod 2^64)
            np.add(base[:m], np.uint64(start + off), out=zz)
            np.multiply(zz, np.uint64(GOLDEN), out=zz)
            np.add(zz, np.uint64(key), out=zz)
            _mix64_inplace(zz, tt)
            yield off, zz


def raw_u64(key: int, n: int, start: int = 0) -> np.ndarray:
    """Elements start..start+n-1 of the stream ``key`` as uint64."""
    out = np.empty(n, dtype=np.uint64)
    for off, z in _stream_chunks(key, n, start):
        out[off:off + z.size] = z
    return out


_HOST_LIB = None
_HOST_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsynth_host.so")


def build_host(verbose: bool = False) -> str:
    """Compile the C twin of the table draw (same values, many times faster)."""
    import subprocess
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc", "host_gen.c")
    cmd = ["gcc", "-O3", "-fopenmp", "-shared", "-fPIC", "-o", _HOST_LIB_PATH, src]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return _HOST_LIB_PATH


def _host_lib():
    global _HOST_LIB
    if _HOST_LIB is None and os.path.exists(_HOST_LIB_PATH):
        import ctypes
        lib = ctypes.CDLL(_HOST_LIB_PATH)
        for name in ("synth_host_fill_f32", "synth_host_fill_f64"):
            fn = getattr(lib, name)
            fn.restype = None
            fn.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                           ctypes.c_void_p]
        _HOST_LIB = lib
    return _HOST_LIB


def _table_draw_numpy(key: int, n: int, table: np.ndarray, start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=table.dtype)
    for off, z in _stream_chunks(key, n, start):
        np.take(table, (z >> np.uint64(48)).astype(np.int64), out=out[off:off + z.size])
    return out


def _table_draw(key: int, n: int, table: np.ndarray, start: int = 0) -> np.ndarray:
    lib = _host_lib()
    if lib is None or table.dtype not in (np.float32, np.float64):
        return _table_draw_numpy(key, n, table, start)
    table = np.ascontiguousarray(table)
    out = np.empty(n, dtype=table.dtype)
    fn = lib.synth_host_fill_f32 if table.dtype == np.float32 else lib.synth_host_fill_f64
    fn(out.ctypes.data, key, start, n, table.ctypes.data)
    return out


@lru_cache(maxsize=None)
def normal_quantiles() -> np.ndarray:
    """The 65536 mid-point quantiles of N(0,1), float64."""
    nd = NormalDist()
    return np.array([nd.inv_cdf((j + 0.5) / 65536.0) for j in range(65536)], dtype=np.float64)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rnd = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + rnd) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_storage(v64: np.ndarray, dtype: str) -> np.ndarray:
    """float64 draw -> float32 array holding the stored (fp32 or bf16) value."""
    f = np.asarray(v64, dtype=np.float64).astype(np.float32)
    if dtype == "fp32":
        return f
    return bf16_bits_to_f32(f32_to_bf16_bits(f))


@lru_cache(maxsize=64)
def normal_table(sigma: float, dtype: str) -> np.ndarray:
    """The 65536 stored values sigma*q_j for one distribution, as float32."""
    return round_storage(normal_quantiles() * sigma, dtype)


def normal(key: int, shape, sigma: float, dtype: str, start: int = 0) -> np.ndarray:
    """N(0, sigma^2) draws (table-quantised) rounded to ``dtype``; float32 array."""
    n = int(np.prod(shape))
    return _table_draw(key, n, normal_table(float(sigma), dtype), start).reshape(shape)


def normal64(key: int, shape, start: int = 0) -> np.ndarray:
    """Unrounded float64 N(0,1) table draws (used to build composite inputs)."""
    n = int(np.prod(shape))
    return _table_draw(key, n, normal_quantiles(), start).reshape(shape)


def uniform(key: int, shape, lo: float, hi: float) -> np.ndarray:
    n = int(np.prod(shape))
    u = raw_u64(key, n)
    unit = (u >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return (lo + (hi - lo) * unit).astype(np.float32).reshape(shape)


# ---------------------------------------------------------------------------
# Per-workload tensors
# ---------------------------------------------------------------------------

MU = 4.0  # length of the common direction added to x in the Zipf workload


def _zipf_pick_probabilities(N: int, K: int, s: float) -> np.ndarray:
    """Per-token pick probability by popularity rank: min(1, lam * r^-s),
    with lam chosen so the probabilities sum to K (water-filling by bisection)."""
    r = np.arange(1, N + 1, dtype=np.float64)
    w = r ** (-s)
    lo, hi = 0.0, float(K) / w[-1] + 1.0
    for _ in range(200):
        lam = 0.5 * (lo + hi)
        if np.minimum(1.0, lam * w).sum() > K:
            hi = lam
        else:
            lo = lam
    return np.minimum(1.0, 0.5 * (lo + hi) * w)


def zipf_shift(cfg: MoEConfig, seed: int):
    """Closed-form logit shifts delta_i that give expert popularity close to
    Zipf(s): with x = z + MU*u and e_i = e0_i + (delta_i/MU)*u, the logit of
    expert i is about N(delta_i, 1 + delta_i^2/MU^2); delta_i is set so that
    P(logit_i > 0) equals the water-filled Zipf pick probability of its rank.
    Returns (delta[N], rank_of_expert[N], u[d])."""
    assert cfg.zipf_s is not None
    pi = _zipf_pick_probabilities(cfg.N, cfg.K, cfg.zipf_s)
    nd = NormalDist()
    q = np.array([nd.inv_cdf(min(max(p, 1e-6), 1 - 1e-6)) for p in pi])
    q = np.clip(q, -3.0, 3.0)
    delta_by_rank = q / np.sqrt(1.0 - q * q / (MU * MU))
    # seeded assignment of popularity ranks to experts
    h = raw_u64(stream_key(seed, cfg.cfg_id, T_ZIPF_PERM), cfg.N)
    order = np.argsort(h, kind="stable")          # order[r] = expert with rank r
    rank = np.empty(cfg.N, dtype=np.int64)
    rank[order] = np.arange(cfg.N)
    delta = delta_by_rank[rank]
    g = normal64(stream_key(seed, cfg.cfg_id, T_ZIPF_U), (cfg.d,))
    u = g / math.sqrt(float(np.dot(g, g)))
    return delta, rank, u


def make_router(cfg: MoEConfig, seed: int = 0) -> np.ndarray:
    """Router vectors e_i, [N, d] float32 (e_i ~ N(0, 1/d))."""
    key = stream_key(seed, cfg.cfg_id, T_ROUTER)
    if cfg.zipf_s is None:
        return normal(key, (cfg.N, cfg.d), 1.0 / math.sqrt(cfg.d), "fp32")
    e0 = normal64(key, (cfg.N, cfg.d)) / math.sqrt(cfg.d)
    delta, _, u = zipf_shift(cfg, seed)
    return (e0 + (delta / MU)[:, None] * u[None, :]).astype(np.float32)


def make_bias(cfg: MoEConfig, seed: int = 0) -> np.ndarray:
    """Initial per-expert routing bias b ~ U(-0.01, 0.01), float32 [N]."""
    return uniform(stream_key(seed, cfg.cfg_id, T_BIAS), (cfg.N,), -0.01, 0.01)


def x_dtype(cfg: MoEConfig) -> str:
    """Storage dtype of the layer input: fp32 for the fp32 layer, else bf16."""
    return "fp32" if cfg.dtype == "fp32" else "bf16"


def _x_from_key(cfg: MoEConfig, seed: int, key: int, rows: int) -> np.ndarray:
    if cfg.zipf_s is None:
        return normal(key, (rows, cfg.d), 1.0, x_dtype(cfg))
    _, _, u = zipf_shift(cfg, seed)
    z = normal64(key, (rows, cfg.d))
    return round_storage(z + MU * u[None, :], x_dtype(cfg))


def make_x(cfg: MoEConfig, seed: int = 0, batch: int = 0) -> np.ndarray:
    """Layer input x [T, d] (float32 array holding fp32 or bf16 values).
    ``batch`` selects a fresh batch (decode steps); 0 is the default batch."""
    return _x_from_key(cfg, seed, stream_key(seed, cfg.cfg_id, T_X, batch), cfg.T)


def redraw_x_row(cfg: MoEConfig, seed: int, batch: int, token: int, attempt: int) -> np.ndarray:
    """A replacement row for token ``token`` (near-tie rejection), [d]."""
    key = stream_key(seed, cfg.cfg_id, T_XREDRAW, batch, token, attempt)
    return _x_from_key(cfg, seed, key, 1)[0]


def weight_key(cfg: MoEConfig, seed: int, which: str, expert: int) -> int:
    tid = {"w1": T_W1, "w3": T_W3, "w2": T_W2}[which]
    return stream_key(seed, cfg.cfg_id, tid, expert)


def weight_shape(cfg: MoEConfig, which: str):
    return (cfg.f, cfg.d) if which in ("w1", "w3") else (cfg.d, cfg.f)


def weight_sigma(cfg: MoEConfig, which: str) -> float:
    fan_in = cfg.d if which in ("w1", "w3") else cfg.f
    return 1.0 / math.sqrt(fan_in)


def weight_dtype(cfg: MoEConfig) -> str:
    """Weights are drawn in bf16 for the bf16 and FP8 layers (FP8 quantises
    from them), fp32 for the fp32 layer."""
    return "fp32" if cfg.dtype == "fp32" else "bf16"


def make_expert_weight(cfg: MoEConfig, seed: int, which: str, expert: int,
                       out: np.ndarray | None = None) -> np.ndarray:
    """W1[e], W3[e] ([f, d]) or W2[e] ([d, f]) of expert e (e == N is the
    shared expert); entries ~ N(0, 1/fan_in), as a float32 array of stored
    values, or written into ``out`` (float32 or float64, right shape)."""
    key = weight_key(cfg, seed, which, expert)
    shape = weight_shape(cfg, which)
    table = normal_table(weight_sigma(cfg, which), weight_dtype(cfg))
    if out is None:
        return normal(key, shape, weight_sigma(cfg, which), weight_dtype(cfg))
    assert out.shape == shape and out.flags.c_contiguous
    lib = _host_lib()
    flat = out.reshape(-1)
    if lib is not None and out.dtype in (np.float32, np.float64):
        t = np.ascontiguousarray(table, dtype=out.dtype)
        fn = lib.synth_host_fill_f32 if out.dtype == np.float32 else lib.synth_host_fill_f64
        fn(flat.ctypes.data, key, 0, flat.size, t.ctypes.data)
    else:
        flat[:] = _table_draw_numpy(key, flat.size, table)
    return out
