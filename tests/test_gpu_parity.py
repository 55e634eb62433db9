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


def test_parity_batched_requests_small_moe():
    """Two requests with different prompts (and prefix lengths) in one batched pass: each
    request's conf / argmax / commits equal the oracle run on that request alone."""
    import torch
    from masked_block_diffusion_b200 import Denoiser, make_policy
    from oracle import OracleModel
    from parity_util import MARGIN, REL
    from synth import blob_from_weights, gen_weights, prompt_tokens

    w = WORKLOADS["c2-small-moe"]
    cfg = w.model.with_layers(2)
    C = cfg.canvas
    W = gen_weights(cfg)
    orc = OracleModel(cfg, W)
    den = Denoiser(cfg, blob_from_weights(cfg, W), max_ctx=1024 + 2 * C, max_batch=2)
    prompts = [prompt_tokens(cfg.vocab, 2600, 512), prompt_tokens(cfg.vocab, 2601, 700)]
    den.set_debug(True)
    recs = []
    for r, p in enumerate(prompts):
        rec = {}
        orc.prefill(r, p, rec)
        den.force_routing(np.stack(rec["topk_idx"]))
        den.prefill(r, p)
    # one batched pass on both requests' step-2 canvases of a top-16 schedule
    pol = Policy("topk", k=16)
    canv, masks, refs = [], [], []
    for r in range(2):
        _, _, tr = orc.generate_block(r, pol, 16, trace=True)
        e = tr[2]
        canv.append(e["canvas"])
        masks.append(e["mask"])
        refs.append(e)
    force = np.concatenate([np.stack(e["rec"]["topk_idx"]) for e in refs], axis=1)
    den.force_routing(force)
    cv = torch.from_numpy(np.stack(canv).astype(np.int32)).cuda()
    mk = torch.from_numpy(np.stack(masks).astype(np.uint8)).cuda()
    conf, arg, rem = den.denoise_step(cv, mk, make_policy("topk", 16), 2, 16)
    conf, arg, rem = conf.cpu().numpy(), arg.cpu().numpy(), rem.cpu().numpy()
    new_mask = mk.cpu().numpy().astype(bool)
    for r in range(2):
        e = refs[r]
        assert np.all(np.abs(conf[r] / e["conf"] - 1.0) <= REL)
        sel = e["rec"]["logit_margin"] > MARGIN
        assert np.array_equal(arg[r][sel], e["argmax"][sel])
        assert rem[r] == int(e["mask"].sum()) - 16
        gpu_commit = e["mask"] & ~new_mask[r]
        assert int(gpu_commit.sum()) == 16
    den.force_routing(None)
    den.set_debug(False)
    # a batched generate_block completes both canvases within the budget
    code, out, steps = den.generate_block(2, 16, make_policy("topk", 16))
    assert code == 0 and steps == [16, 16]
    o = out.cpu().numpy()
    assert np.all((o >= 0) & (o <= cfg.vocab - 2))
    den.close()


def test_parity_moe26b_shapes_two_layers():
    # full-width layers of the 26B model; threshold 0.9 + floor, 12-step budget
    stats, steps, gsteps, agree = run_workload("c4-moe26b-1024out", n_layers=2, prefix=1024)
    assert steps == 12 and gsteps == 12
    assert stats["route_pinned"] > 0.9 * stats["route_total"]
