"""CPU oracle for the masked block-diffusion denoising step (TEST INFRASTRUCTURE).

Plain, slow numpy code that states what one denoising pass computes, used to check
the CUDA path. Only the test suite, the smoke check and the benchmark's CPU-baseline
leg may import it; the library itself never does and shares no code with it.

Parity status of each function is listed in ``oracle/model.py``'s header.
"""

from .model import (
    Policy,
    OracleModel,
    bf16,
    rmsnorm,
    rope_cos_sin,
    apply_rope,
    attention,
    router_topk,
    swiglu_expert,
    moe_ffn,
    lm_head_conf,
    commit_count,
    commit_select,
    edit_select,
    sequence_forward,
)

__all__ = [
    "Policy", "OracleModel", "bf16", "rmsnorm", "rope_cos_sin", "apply_rope", "attention",
    "router_topk", "swiglu_expert", "moe_ffn", "lm_head_conf", "commit_count",
    "commit_select", "edit_select", "sequence_forward",
]
