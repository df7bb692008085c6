"""Named layer shapes and their synthetic-input recipes.

A ``LayerConfig`` carries the layer's shape (what the C ABI's ``moe_config``
holds) and the recipe that ``inputs.make_inputs`` follows to draw seeded
router logits, activations and expert weights for it.

The shapes follow the family the MegaFlux paper evaluates ("MegaFlux:
Skew-Resilient MoE Megakernels via Pipelined Expert Replication", §4.1
"Platform and configurations": SwiGLU experts, top-8 routing, a per-GPU
budget of spare replicas, 128-row token blocks) scaled to one GPU whose
expert-parallel ranks are virtual.
"""
from __future__ import annotations

import dataclasses

BF16 = 0
FP32 = 1
GATE_SOFTMAX_TOPK = 0
GATE_SIGMOID_TOPK = 1
PLAN_EXACT = 0    # exactly S*K entries per rank (greedy refill from the biggest donor)
PLAN_BLOCKS = 1   # block-granular four-candidate search, pruning and refinement


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int          # tokens
    d: int          # hidden size
    E: int          # routed experts
    K: int          # experts per token (top-k)
    F: int          # expert FFN width (SwiGLU intermediate size)
    R: int          # virtual expert-parallel ranks
    tile: int       # token-block rows (beta)
    budget: int     # replicas a rank may host
    dtype: int = BF16
    gating: int = GATE_SOFTMAX_TOPK
    plan_mode: int = PLAN_EXACT
    # input recipe
    logits: str = "xwr"      # "xwr": x @ Wr + bias; "normal": N(0,1) + bias
    zipf_s: float = 0.0      # bias_e = -s * ln(rank_e) over a seeded expert permutation
    hot_bias: float = 0.0    # >0: one seeded hot expert gets this bias
    hot_frac: float = 1.0    # fraction of tokens that carry the hot bias
    w_std: float = 0.02      # std of router and expert weights

    def replace(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == BF16 else 4

    @property
    def S(self) -> int:
        return self.T // self.R

    @property
    def N(self) -> int:
        return self.T * self.K


TINY = LayerConfig("tiny", T=256, d=128, E=8, K=2, F=256, R=4, tile=16, budget=1,
                   dtype=FP32, zipf_s=1.0)
OLMOE = LayerConfig("olmoe", T=8192, d=2048, E=64, K=8, F=1024, R=8, tile=128, budget=2,
                    zipf_s=0.8)
QWEN3 = LayerConfig("qwen3", T=16384, d=2048, E=128, K=8, F=768, R=8, tile=128, budget=2,
                    zipf_s=1.0)
EXTREME = LayerConfig("extreme", T=32768, d=4096, E=64, K=4, F=1536, R=8, tile=128, budget=1,
                      hot_bias=30.0)
DSV3 = LayerConfig("dsv3", T=8192, d=7168, E=256, K=8, F=2048, R=32, tile=128, budget=4,
                   gating=GATE_SIGMOID_TOPK, logits="normal", zipf_s=1.2)

# A reduced DeepSeek-V3-like shape for profiler captures of the GEMM: the
# full shape's d and F with about 256 rows per expert and 2.8 GB of weights.
DSV3_SMALL = DSV3.replace(name="dsv3_small", T=1024, E=32, R=4, budget=4)

NAMED = {c.name: c for c in (TINY, OLMOE, QWEN3, EXTREME, DSV3, DSV3_SMALL)}

# The Qwen3-shaped skew sweep.
QWEN3_SWEEP = tuple(QWEN3.replace(name=f"qwen3_s{s}", zipf_s=s) for s in (0.0, 0.5, 1.0, 1.5))


def describe(c: LayerConfig) -> dict:
    return {"workload": c.name, "T": c.T, "d": c.d, "E": c.E, "top_k": c.K, "F": c.F,
            "R": c.R, "tile": c.tile, "budget": c.budget,
            "dtype": "bf16" if c.dtype == BF16 else "fp32",
            "gating": "softmax_topk" if c.gating == GATE_SOFTMAX_TOPK else "sigmoid_topk",
            "planner": "exact_SK" if c.plan_mode == PLAN_EXACT else "blocks",
            "router": c.logits, "zipf_s": c.zipf_s, "hot_bias": c.hot_bias,
            "hot_frac": c.hot_frac}
