"""The MoE layer shapes exercised by tests and the benchmark (pure data)."""
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                 # tokens
    H: int                 # hidden size
    E: int                 # routed experts
    I: int                 # routed expert intermediate size
    I_s: int               # merged shared-expert intermediate size (0 = none)
    k: int                 # experts per token
    n_group: int
    topk_group: int
    scoring: str           # "softmax" | "sigmoid"
    norm_topk_prob: bool
    scale: float           # routed_scaling_factor
    dtype: str             # "bf16" | "e4m3" (expert weights / activations)
    has_bias: bool         # selection-only bias b ~ U(-0.05, 0.05)
    skew_experts: int = 0  # experts whose gate rows get +0.5*xbar (skewed load)
    bias_steps: int = 0    # aux-loss-free bias update steps between forwards
    gamma: float = 0.001   # bias update speed
    seed: int = 0

    @property
    def rows(self) -> int:
        return self.T * self.k

    def flops(self) -> float:
        """Algorithmic FLOPs of one forward: gate + routed SwiGLU + shared."""
        gate = 2.0 * self.T * self.H * self.E
        routed = 2.0 * self.T * self.k * 3 * self.H * self.I
        shared = 2.0 * self.T * 3 * self.H * self.I_s
        return gate + routed + shared


CONFIGS = {
    # Tiny layer: softmax, greedy top-4, no renorm, scale 1.0.
    "tiny": MoEConfig("tiny", T=64, H=256, E=16, I=128, I_s=128, k=4,
                      n_group=1, topk_group=1, scoring="softmax",
                      norm_topk_prob=False, scale=1.0, dtype="bf16",
                      has_bias=False, seed=1001),
    # DeepSeek-V2-Lite MoE layer (2 shared experts merged into I_s = 2816).
    "v2lite": MoEConfig("v2lite", T=4096, H=2048, E=64, I=1408, I_s=2816, k=6,
                        n_group=1, topk_group=1, scoring="softmax",
                        norm_topk_prob=False, scale=1.0, dtype="bf16",
                        has_bias=False, seed=1002),
    # DeepSeek-V3 MoE layer, prefill-shaped.
    "v3": MoEConfig("v3", T=8192, H=7168, E=256, I=2048, I_s=2048, k=8,
                    n_group=8, topk_group=4, scoring="sigmoid",
                    norm_topk_prob=True, scale=2.5, dtype="bf16",
                    has_bias=True, seed=1003),
    # DeepSeek-V3 MoE layer, FP8 E4M3 decode-shaped.
    "v3_fp8_decode": MoEConfig("v3_fp8_decode", T=256, H=7168, E=256, I=2048,
                               I_s=2048, k=8, n_group=8, topk_group=4,
                               scoring="sigmoid", norm_topk_prob=True,
                               scale=2.5, dtype="e4m3", has_bias=True,
                               seed=1004),
    # Skewed-load V3 layer with 10 aux-loss-free bias steps.
    "v3_skewed": MoEConfig("v3_skewed", T=32768, H=7168, E=256, I=2048,
                           I_s=2048, k=8, n_group=8, topk_group=4,
                           scoring="sigmoid", norm_topk_prob=True, scale=2.5,
                           dtype="bf16", has_bias=True, skew_experts=16,
                           bias_steps=10, gamma=0.001, seed=1005),
    # V3 shapes and V3's tokens per expert (T*k/E = 256) on 32 experts: the
    # small case the profiler captures (2.8 GB of weights, larger than L2).
    "v3_e32": MoEConfig("v3_e32", T=1024, H=7168, E=32, I=2048, I_s=2048, k=8,
                        n_group=8, topk_group=4, scoring="sigmoid",
                        norm_topk_prob=True, scale=2.5, dtype="bf16",
                        has_bias=True, seed=1006),
}


def get_config(name: str, **overrides) -> MoEConfig:
    cfg = CONFIGS[name]
    return replace(cfg, **overrides) if overrides else cfg


def tiny_grouped_config(**overrides) -> MoEConfig:
    """Tiny layer with V3-style grouped sigmoid routing (4 groups, keep 2)."""
    base = replace(CONFIGS["tiny"], name="tiny_grouped", n_group=4,
                   topk_group=2, scoring="sigmoid", norm_topk_prob=True,
                   scale=2.5, has_bias=True, seed=1011)
    return replace(base, **overrides) if overrides else base
