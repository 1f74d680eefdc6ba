"""Workload shapes of the sparse MoE FFN forward (GLM-4.5 / GLM-5 style).

Each configuration names the sizes of one layer call: N tokens of hidden size D,
E routed experts in n_group contiguous groups of which topk_group are kept, k
experts per token, expert width d_moe, one shared expert of width d_sh, and the
routed scaling factor alpha.  Model shapes follow the pages: GLM-4.5 has 160
routed experts of width 1536 and alpha 2.5, GLM-4.5-Air 128 of width 1408 and
alpha 1.0 ("GLM-4.5 MoE Forward", Overview; "GLM-4.5 Group Router", How it
works); GLM-5 has D 6144, 256 experts of width 2048, a bf16 router matrix and an
fp32 bias ("GLM-5 Mixture of experts", Parameters and In numbers).
"""

from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    N: int
    D: int
    E: int
    n_group: int
    topk_group: int
    k: int
    d_moe: int
    d_sh: int
    alpha: float
    norm_topk_prob: bool
    dtype: torch.dtype  # x, experts, shared expert and y
    wg_dtype: torch.dtype  # router matrix W_g
    beta: float  # correction bias b ~ U(-beta, beta)
    skew: bool = False  # Zipf-like expert popularity via router-row offsets
    description: str = ""

    def with_(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    # Algorithmic work of one layer call (routed k experts + shared + router).
    def flops(self) -> float:
        return self.N * (2.0 * self.k * 3 * self.D * self.d_moe
                         + 2.0 * 3 * self.D * self.d_sh + 2.0 * self.D * self.E)

    def weight_bytes(self, hit_experts: int) -> float:
        es = torch.tensor([], dtype=self.dtype).element_size()
        ws = torch.tensor([], dtype=self.wg_dtype).element_size()
        return ((hit_experts * 3.0 * self.D * self.d_moe + 3.0 * self.D * self.d_sh) * es
                + self.E * self.D * ws + self.E * 4.0 + 2.0 * self.N * self.D * es)


F32, BF16 = torch.float32, torch.bfloat16

CONFIGS = {
    "tiny_fp32": MoEConfig(
        "tiny_fp32", N=64, D=256, E=16, n_group=4, topk_group=2, k=4, d_moe=128, d_sh=128,
        alpha=2.5, norm_topk_prob=True, dtype=F32, wg_dtype=F32, beta=0.1,
        description="tiny general group-routed path, fp32 throughout"),
    "air_decode": MoEConfig(
        "air_decode", N=32, D=4096, E=128, n_group=1, topk_group=1, k=8, d_moe=1408, d_sh=1408,
        alpha=1.0, norm_topk_prob=True, dtype=BF16, wg_dtype=F32, beta=0.05,
        description="GLM-4.5-Air-shaped decode, 32 tokens, bf16 experts, fp32 router"),
    "glm45_prefill": MoEConfig(
        "glm45_prefill", N=8192, D=5120, E=160, n_group=1, topk_group=1, k=8, d_moe=1536,
        d_sh=1536, alpha=2.5, norm_topk_prob=True, dtype=BF16, wg_dtype=F32, beta=0.05,
        description="GLM-4.5-shaped prefill, 8192 tokens, bf16 experts, fp32 router"),
    "glm5_prefill": MoEConfig(
        "glm5_prefill", N=4096, D=6144, E=256, n_group=1, topk_group=1, k=8, d_moe=2048,
        d_sh=2048, alpha=2.5, norm_topk_prob=True, dtype=BF16, wg_dtype=BF16, beta=0.05,
        description="GLM-5-shaped block, 4096-token prefill, bf16 experts and router matrix"),
    "glm5_decode": MoEConfig(
        "glm5_decode", N=64, D=6144, E=256, n_group=1, topk_group=1, k=8, d_moe=2048,
        d_sh=2048, alpha=2.5, norm_topk_prob=True, dtype=BF16, wg_dtype=BF16, beta=0.05,
        description="GLM-5-shaped block, 64-token decode, bf16 experts and router matrix"),
    "skew_grouped": MoEConfig(
        "skew_grouped", N=16384, D=6144, E=256, n_group=8, topk_group=4, k=8, d_moe=2048,
        d_sh=2048, alpha=2.5, norm_topk_prob=True, dtype=BF16, wg_dtype=BF16, beta=0.1,
        skew=True,
        description="group-restricted routing (8 groups of 32, keep 4) with Zipf-skewed "
                    "expert load, 16384 tokens, bf16"),
}

# The bench's headline workload: the largest single-GPU configuration (the layer's
# tokens/s metric names prefill and decode but no configuration), the skewed
# group-routed 16384-token prefill.  The other performance configurations are
# measured in the same run and reported beside it.
DEFAULT_WORKLOAD = "skew_grouped"
PERF_WORKLOADS = ("skew_grouped", "glm45_prefill", "glm5_prefill", "glm5_decode", "air_decode")
