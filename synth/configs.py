"""The five synthetic MoE-layer workloads (shapes, dtypes, schedule).

Pure data: no arithmetic of the MoE method lives here.  Both the float64
oracle (tests only) and the CUDA path read these shapes.

Notation follows the DeepSeek-V3 pages: T tokens, d model width, N routed
experts plus one always-on shared expert, K routed experts per token, G expert
groups ("nodes"), topG groups a token may reach, f the expert inner width.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class MoEConfig:
    name: str
    cfg_id: int
    T: int
    d: int
    N: int
    K: int
    G: int
    topG: int
    f: int
    dtype: str          # "fp32" | "bf16" | "e4m3" (expert GEMM operands)
    passes: int = 1     # forward passes, bias update applied between them
    gamma: float = 0.001
    zipf_s: float | None = None
    steps: int = 1      # route + bias-update steps (decode workload)
    forward_every: int = 1

    @property
    def rows(self) -> int:
        """Routed rows after dispatch: one per (token, selected expert)."""
        return self.T * self.K

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


# Tiny fp32 layer: the oracle runs it in well under a second; no group limit.
TINY = MoEConfig("tiny_fp32", 0, T=128, d=64, N=16, K=4, G=1, topG=1, f=32, dtype="fp32")
# Mid-size bf16 layer with group-limited routing (8 groups, top-4).
MID = MoEConfig("mid_bf16", 1, T=4096, d=2048, N=64, K=6, G=8, topG=4, f=1408, dtype="bf16")
# DeepSeek-V3-shaped layer (256 routed + 1 shared, K=8, 8 groups / top-4), bf16,
# 10 forward passes with the bias update between them.
V3_BF16 = MoEConfig("v3_bf16", 2, T=8192, d=7168, N=256, K=8, G=8, topG=4, f=2048,
                    dtype="bf16", passes=10, gamma=0.001)
# The same layer with FP8-E4M3 expert GEMMs (1x128 activation tiles, 128x128
# weight blocks, fp32 scales); the router stays fp32.
V3_FP8 = MoEConfig("v3_fp8", 3, T=16384, d=7168, N=256, K=8, G=8, topG=4, f=2048,
                   dtype="e4m3", passes=1, gamma=0.001)
# Decode-like: 256 tokens, V3 shape, Zipf(1.2) expert popularity, 200
# route + bias-update steps with one full forward every 20 steps.
DECODE = MoEConfig("decode_zipf", 4, T=256, d=7168, N=256, K=8, G=8, topG=4, f=2048,
                   dtype="bf16", gamma=0.001, zipf_s=1.2, steps=200, forward_every=20)

CONFIGS = {c.cfg_id: c for c in (TINY, MID, V3_BF16, V3_FP8, DECODE)}
BY_NAME = {c.name: c for c in CONFIGS.values()}
