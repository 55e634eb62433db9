"""Model shapes and workloads of the masked block-diffusion denoiser.

Shapes follow the pages: a 256-position canvas ("Diffusion LLMs are not a good
fit for distributed inference", canvas paragraph; "Diffusion LLMs: what changes
...", section 4.2 "Block decoding"), a mixture-of-experts backbone with about
3.8B active of 26B parameters (same page, section 4.2; "DiffusionGemma: 4x
Faster ...", "Memory Optimization"), up to 48 denoising steps and about 12 on
average (section 4.2 "Few steps"), a 4096-token prompt with 1024 output tokens at
batch 1 (section 4.2 "Speed"), and concurrency up to about 32 users (section 3).
Layer counts and widths are the ones the workload list fixes; the pages do not
give them.
"""

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int          # 0 = dense SwiGLU FFN
    top_k: int              # experts per token (1 for dense)
    ffn_dim: int            # expert (or dense) FFN width
    vocab: int
    canvas: int             # positions per canvas
    weight_dtype: str = "bf16"   # "bf16" or "f32"
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    weight_seed: int = 1000

    @property
    def mask_id(self) -> int:
        # [MASK] is the last vocabulary entry; prompts never contain it.
        return self.vocab - 1

    @property
    def dense(self) -> bool:
        return self.n_experts == 0

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def with_layers(self, n_layers: int, name: Optional[str] = None) -> "ModelConfig":
        return replace(self, n_layers=n_layers, name=name or f"{self.name}-{n_layers}L")


@dataclass(frozen=True)
class Workload:
    name: str
    model: ModelConfig
    prefix: int                  # prompt length P per request
    batch: int                   # independent requests
    n_canvases: int              # canvases generated per request (appended after each)
    policy: str                  # "topk" or "threshold"
    k: int = 0                   # top-k commits per step
    tau: float = 0.9             # threshold for "threshold"
    floor: bool = True           # step-budget floor for "threshold"
    max_steps: int = 48          # step budget S_max per canvas
    prompt_seed: int = 2000      # request r of workload w uses prompt_seed + r
    batches: Tuple[int, ...] = field(default_factory=tuple)  # sweep values (config 5)


TINY_DENSE = ModelConfig(
    name="tiny-dense", n_layers=2, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64,
    n_experts=0, top_k=1, ffn_dim=1024, vocab=1024, canvas=32, weight_dtype="f32",
    weight_seed=1001)

SMALL_MOE = ModelConfig(
    name="small-moe", n_layers=8, d_model=1024, n_heads=16, n_kv_heads=4, head_dim=64,
    n_experts=32, top_k=4, ffn_dim=512, vocab=32768, canvas=256, weight_dtype="bf16",
    weight_seed=1002)

MOE_26B = ModelConfig(
    name="moe-26b-a4b", n_layers=30, d_model=2816, n_heads=16, n_kv_heads=8, head_dim=176,
    n_experts=128, top_k=8, ffn_dim=704, vocab=65536, canvas=256, weight_dtype="bf16",
    weight_seed=1003)

CONFIGS = {c.name: c for c in (TINY_DENSE, SMALL_MOE, MOE_26B)}

WORKLOADS = {
    # 1: tiny dense denoiser, prefix 64, canvas 32, top-4 x 8 steps
    "c1-tiny-dense": Workload("c1-tiny-dense", TINY_DENSE, prefix=64, batch=1, n_canvases=1,
                              policy="topk", k=4, max_steps=8, prompt_seed=2100),
    # 2: small MoE, prefix 1024, canvas 256, top-16 x 16 steps
    "c2-small-moe": Workload("c2-small-moe", SMALL_MOE, prefix=1024, batch=1, n_canvases=1,
                             policy="topk", k=16, max_steps=16, prompt_seed=2200),
    # 3: 26B MoE, prefix 4096, canvas 256, threshold 0.9 + floor, at most 48 steps
    "c3-moe26b-canvas": Workload("c3-moe26b-canvas", MOE_26B, prefix=4096, batch=1,
                                 n_canvases=1, policy="threshold", tau=0.9, floor=True,
                                 max_steps=48, prompt_seed=2300),
    # 4: same model, 4 canvases of 256 (1024 output tokens), 12 steps each, append after each
    "c4-moe26b-1024out": Workload("c4-moe26b-1024out", MOE_26B, prefix=4096, batch=1,
                                  n_canvases=4, policy="threshold", tau=0.9, floor=True,
                                  max_steps=12, prompt_seed=2400),
    # 5: same model, concurrency sweep, 12 fixed steps (threshold never fires)
    "c5-moe26b-batch": Workload("c5-moe26b-batch", MOE_26B, prefix=4096, batch=1,
                                n_canvases=1, policy="threshold", tau=float("inf"),
                                floor=True, max_steps=12, prompt_seed=2500,
                                batches=(1, 4, 8, 16, 32, 64)),
}


def get_config(name: str) -> ModelConfig:
    return CONFIGS[name]


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]
