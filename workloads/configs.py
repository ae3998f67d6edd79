"""The five named workloads.

Shapes follow the pages' running example: Qwen2.5-7B has 28 layers and 512
K/V values per token per layer ("PagedAttention, Visualized", Part 2), which is
4 KV heads x 128 dims; the pool holds blocks of 16 tokens ("PagedAttention",
section "PagedAttention in one picture").  One workload is one layer's decode
step.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    num_seqs: int
    num_heads: int          # query heads (Hq)
    num_kv_heads: int       # KV heads (Hkv); GQA group G = Hq / Hkv
    head_dim: int           # D
    dtype: str              # "f32" | "f16" | "bf16"
    num_blocks: int         # physical blocks in the pool (NB)
    ctx_kind: str           # how context lengths are drawn, see gen.py
    ctx_args: tuple = ()
    placement: str = "permuted"  # "permuted" | "identity" | "churned" | "shared_prefix"
    block_size: int = 16
    partition_size: int = 0      # 0 = library's choice
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / float(self.head_dim) ** 0.5

    @property
    def elt_bytes(self) -> int:
        return {"f32": 4, "f16": 2, "bf16": 2}[self.dtype]


CONFIGS = {
    "tiny": WorkloadConfig(
        name="tiny", num_seqs=4, num_heads=4, num_kv_heads=2, head_dim=64,
        dtype="f32", num_blocks=32, ctx_kind="fixed", ctx_args=(1, 15, 16, 37),
        placement="permuted",
        description="4 seqs, ctx {1,15,16,37}, 4/2 heads, D=64, fp32, 32-block pool"),
    "qwen_layer": WorkloadConfig(
        name="qwen_layer", num_seqs=32, num_heads=28, num_kv_heads=4, head_dim=128,
        dtype="f16", num_blocks=4096, ctx_kind="uniform", ctx_args=(128, 2048),
        placement="permuted",
        description="Qwen2.5-7B-shaped layer: B=32, ctx U[128,2048], 28/4 heads, D=128, fp16"),
    "long32k": WorkloadConfig(
        name="long32k", num_seqs=8, num_heads=28, num_kv_heads=4, head_dim=128,
        dtype="bf16", num_blocks=16384, ctx_kind="fixed", ctx_args=(32768,) * 8,
        placement="permuted", partition_size=512,
        description="B=8, ctx 32768 each, 28/4 heads, D=128, bf16, shuffled 16384-block pool"),
    "churned256": WorkloadConfig(
        name="churned256", num_seqs=256, num_heads=28, num_kv_heads=4, head_dim=128,
        dtype="f16", num_blocks=80000, ctx_kind="lognormal", ctx_args=(300.0, 1.0, 8, 4096),
        placement="churned",
        description="B=256, ctx lognormal(median 300, sigma 1) clipped to [8,4096], 28/4 heads, "
                    "D=128, fp16, 80000-block pool fragmented by allocate/free churn"),
    "shared_prefix": WorkloadConfig(
        name="shared_prefix", num_seqs=1024, num_heads=28, num_kv_heads=4, head_dim=128,
        dtype="bf16", num_blocks=40000, ctx_kind="shared_prefix", ctx_args=(512, 16, 1024, 64),
        placement="shared_prefix",
        description="1024 seqs sharing a 512-token prefix (32 blocks), suffix U[16,1024], "
                    "28/4 heads, D=128, bf16; 64 forks copy-on-write their partial last block"),
}


def get_config(name: str, **overrides) -> WorkloadConfig:
    cfg = CONFIGS[name]
    return replace(cfg, **overrides) if overrides else cfg
