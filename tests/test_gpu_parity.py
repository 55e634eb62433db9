"""Model-level parity of the CUDA path with the oracle, step by step (GPU).

Workloads: the tiny dense denoiser and the small MoE denoiser at their full sizes,
and the 26B model's layer shapes (E = 128, top-8, F = 704, head_dim 176, V = 65536)
with two layers. Every oracle step is replayed on the GPU from the oracle's canvas.
"""

import numpy as np
import pytest

from oracle import Policy
from parity_util import build_pair, check_generate_invariants, compare_trace
from synth import WORKLOADS

pytestmark = pytest.mark.gpu


def run_workload(name, n_layers=None, prefix=None, s_max=None, append_check=True):
    w = WORKLOADS[name]
    cfg = w.model if n_layers is None else w.model.with_layers(n_layers)
    P = w.prefix if prefix is None else prefix
    S = w.max_steps if s_max is None else s_max
    C = cfg.canvas
    max_ctx = P + 3 * C
    orc, den, prompt = build_pair(cfg, P, w.prompt_seed, max_ctx)
    pol = Policy(w.policy, k=w.k, tau=w.tau, floor=w.floor)
    canvas, steps, trace = orc.generate_block(0, pol, S, trace=True)
    stats = compare_trace(cfg, trace, den, pol, S)
    # the full loop on the GPU completes the canvas within the budget
    gpu_canvas, gpu_steps = check_generate_invariants(cfg, den, pol, S, expect_steps=steps)
    if append_check:
        # append the oracle's canvas on both sides, then compare the next canvas's first step
        import torch
        orc.append(0, canvas)
        den.append_kv(1, torch.from_numpy(canvas.astype(np.int32)[None]).cuda())
        assert den.prefix_len(0) == P + C
        _, _, trace2 = orc.generate_block(0, pol, S, trace=True)
        compare_trace(cfg, trace2[:2], den, pol, S)
    den.close()
    return stats, steps, gpu_steps, float(np.mean(gpu_canvas == canvas))


def test_parity_tiny_dense():
    stats, steps, gsteps, agree = run_workload("c1-tiny-dense")
    assert steps == 8 and gsteps == 8
    assert stats["arg_pinned"] > 0.9 * stats["arg_total"]


def test_parity_small_moe():
    stats, steps, gsteps, agree = run_workload("c2-small-moe")
    assert steps == 16 and gsteps == 16
    assert stats["route_pinned"] > 0.9 * stats["route_total"]
    assert stats["arg_pinned"] > 0.9 * stats["arg_total"]


def test_parity_moe26b_shapes_two_layers():
    # full-width layers of the 26B model; threshold 0.9 + floor, 12-step budget
    stats, steps, gsteps, agree = run_workload("c4-moe26b-1024out", n_layers=2, prefix=1024)
    assert steps == 12 and gsteps == 12
    assert stats["route_pinned"] > 0.9 * stats["route_total"]
