"""Parity of the kernel variants the engine can select, against the oracle (GPU).

test_gpu_parity.py covers the default selections. Here each alternative is switched on
through the environment variable the engine reads when a handle is created, and the
same step-by-step comparison with the oracle runs on a two-layer model:

- DLLM_MOE_PAIR=0: one weight tile per grouped down work item instead of two;
- DLLM_NO_GRAPH=1: every pass launched eagerly instead of replaying its CUDA graph.

A GQA group of 3 (6 query heads over 2 KV heads) does not divide the 128-row query tile
of the tensor-core attention, so that model runs both its prefill and its canvas passes
on the mma.sync attention kernel; its 16 experts (not a multiple of 32) run the SIMT
router instead of the tensor-core router GEMM.
"""

from dataclasses import replace

import pytest

from oracle import Policy
from parity_util import build_pair, check_generate_invariants, compare_trace
from synth import WORKLOADS

pytestmark = pytest.mark.gpu


def _run(cfg, prefix, policy, s_max, prompt_seed):
    orc, den, _ = build_pair(cfg, prefix, prompt_seed, prefix + 2 * cfg.canvas)
    try:
        _, steps, trace = orc.generate_block(0, policy, s_max, trace=True)
        stats = compare_trace(cfg, trace, den, policy, s_max)
        check_generate_invariants(cfg, den, policy, s_max, expect_steps=steps)
    finally:
        den.close()
    return stats, steps


VARIANTS = {
    "down-one-tile-per-item": {"DLLM_MOE_PAIR": "0"},
    "no-graph": {"DLLM_NO_GRAPH": "1"},
}


@pytest.mark.parametrize("name", list(VARIANTS))
def test_variant_small_moe(name, monkeypatch):
    for k, v in VARIANTS[name].items():
        monkeypatch.setenv(k, v)
    w = WORKLOADS["c2-small-moe"]
    cfg = w.model.with_layers(2)
    stats, steps = _run(cfg, 512, Policy("topk", k=32), 8, w.prompt_seed + 7)
    assert steps == 8
    assert stats["route_pinned"] > 0.9 * stats["route_total"]
    assert stats["arg_pinned"] > 0.9 * stats["arg_total"]


def test_gqa_group_of_three_on_mma_sync_attention():
    base = WORKLOADS["c2-small-moe"].model
    cfg = replace(base, name="gqa3-moe", n_layers=2, d_model=512, n_heads=6, n_kv_heads=2, head_dim=64,
                  n_experts=16, top_k=4, ffn_dim=256, vocab=8192, canvas=64, weight_seed=1010)
    stats, steps = _run(cfg, 300, Policy("threshold", tau=0.9, floor=True), 8, 2700)
    assert steps <= 8
    assert stats["route_pinned"] > 0.9 * stats["route_total"]
    assert stats["arg_pinned"] > 0.9 * stats["arg_total"]


_FAULT_SCRIPT = """
import sys
sys.path.insert(0, {root!r})
from masked_block_diffusion_b200 import binding
from synth import WORKLOADS, blob_from_weights, gen_weights
cfg = WORKLOADS["c1-tiny-dense"].model
blob = blob_from_weights(cfg, gen_weights(cfg))
c = binding.make_config(cfg, max_ctx=256, max_batch=1)
try:
    h = binding.dllm_create(c, blob.ctypes.data, blob.nbytes, False, 0)
    print("CODE", 0)
    binding.dllm_destroy(h)
except binding.DllmError as e:
    print("CODE", e.code)
"""


def test_allocation_failure_is_reported_cleanly():
    """The n-th device allocation fails on the host (DLLM_FAULT_ALLOC_AT): dllm_create
    returns DLLM_E_OOM with no handle, after releasing what it had allocated."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for n in (1, 5, 20):
        env = dict(os.environ, DLLM_FAULT_ALLOC_AT=str(n))
        out = subprocess.run([sys.executable, "-c", _FAULT_SCRIPT.format(root=root)], env=env,
                             capture_output=True, text=True, timeout=300)
        assert out.returncode == 0, out.stderr[-2000:]
        line = [x for x in out.stdout.splitlines() if x.startswith("CODE")][-1]
        assert line == "CODE -2", line
