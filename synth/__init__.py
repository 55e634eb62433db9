"""Seeded synthetic inputs for the masked block-diffusion denoising step.

This package is shared by the CPU oracle and by the CUDA path. It holds only
input generation (model shapes, random-init weights, prompt tokens) and none of
the method's arithmetic. Every value is produced by integer operations on a
counter-based generator, so the numpy generator here and the device generator in
``synth/csrc/synth_fill.cu`` give bit-identical tensors.
"""

from .configs import ModelConfig, Workload, CONFIGS, WORKLOADS, get_config, get_workload
from .gen import (
    splitmix64,
    tensor_specs,
    blob_layout,
    gen_tensor,
    gen_weights,
    gen_blob,
    blob_from_weights,
    prompt_tokens,
    normal_f32,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
    uniform_f32,
)

__all__ = [
    "ModelConfig", "Workload", "CONFIGS", "WORKLOADS", "get_config", "get_workload",
    "splitmix64", "tensor_specs", "blob_layout", "gen_tensor", "gen_weights", "gen_blob", "blob_from_weights",
    "prompt_tokens", "normal_f32", "f32_to_bf16_bits", "bf16_bits_to_f32", "uniform_f32",
]
