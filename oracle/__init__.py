"""Float64 CPU oracle of the DeepSeekMoE layer forward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import or run anything in this package.  It shares no code with the
CUDA path (``sparse_moe_layer_limited_b200``); the one thing both sides share
is the seeded input generator ``synth`` (which holds no arithmetic of the
method).

Sources (the pages that define the method), cited in docstrings as:

* [P1] "DeepSeek-V3 高效训练关键技术分析" (mhpq.cn/news/1102932):
  §1.1 DeepSeekMoE 架构 (1 shared + 256 routed experts, 8 active),
  §1.2 无辅助损失负载均衡 (per-expert bias, adjusted every step from the load),
  §2.2 forward order ATTN -> DISPATCH -> MLP -> COMBINE,
  §3.1 限制路由范围 (a token reaches at most 4 nodes),
  §4.1 精细量化策略 / 在线量化 (1x128 activation and 128x128 weight scaling,
  scale from the online max-abs).
* [P2] "解读 DeepSeek-V3" reading notes (gkm0120.cn/p/38322), Q3
  (bias added to the affinity for routing only; never in the gate value).
* [P4] DeepSeek-V3 technical-report walk-through (kaiyunto.com/.../3873),
  DeepSeekMoE paragraphs: sigmoid affinity, gate = normalisation over the
  selected affinities, bias decreased by gamma when the expert is overloaded
  and increased by gamma when under-loaded.
* [P5] "DeepSeek-V3核心技术解析：MoE、MLA、MTP与FP8训练详解" (wenxiaobai),
  §二(一)4 top-K selection by affinity; shared expert always participates.

Readings where the pages are silent (all also listed in the design notes):
group score = sum of the two largest biased scores in a group; 8 contiguous
groups with the top 4 kept; SwiGLU experts without biases; no routed scaling
factor; lower index wins exact ties; an expert exactly at the T*K/N load keeps
its bias; FP8 scale = amax/448 in fp32 (amax = 0 gives scale 1, codes 0).

Parity status: every function here is pinned by the tests in
``tests/test_oracle_*.py`` (brute force, closed forms, invariants, special
cases, the exhaustive E4M3 table, a hand-worked routing fixture).
"""
from .moe import (  # noqa: F401
    affinity, biased_scores, group_scores, kept_groups, route, route_margins,
    route_softmax, route_softmax_margins, balance_loss,
    dispatch, swiglu_expert, swiglu_expert_backward, expert_outputs, combine, bias_update,
    moe_forward, combine_backward, route_backward, dispatch_backward, moe_backward,
    round_bf16, silu,
)
from .fp8 import (  # noqa: F401
    e4m3_decode, e4m3_encode, e4m3_all_values, quant_rows_1x128, quant_blocks_128,
    e5m2_decode, e5m2_encode, e5m2_all_values, quant_rows_1x128_e5m2,
    fp8_gemm_ref, fp8_swiglu_expert, fp8_swiglu_expert_backward_dx, quant_cols_1x128,
    fp8_weight_grad,
)
