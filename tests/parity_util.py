"""Step-by-step parity of the CUDA path against the oracle (used by the GPU tests).

Each denoising step of the oracle's trace is replayed on the GPU from the oracle's
own (canvas, mask), so a near-tie decided differently at one step cannot compound.
Tolerances (fixed for this path): routing sets, argmax tokens and commit sets equal
wherever the oracle's margin at the decision exceeds 1e-3 (router logit units, LM
logit units, log-confidence units); conf within 2e-2 relative; final hidden state
within 2e-2 of the row's largest magnitude.
"""

from __future__ import annotations

import functools
import math
import os

import numpy as np
import torch

from masked_block_diffusion_b200 import Denoiser, make_policy
from oracle import OracleModel, Policy
from synth import blob_from_weights, gen_weights, prompt_tokens

MARGIN = 1e-3
REL = 2e-2


@functools.lru_cache(maxsize=1)
def cached_weights(cfg):
    """The seeded weights of cfg, generated once for the tests that share a model."""
    return gen_weights(cfg, threads=os.cpu_count() or 8)


def build_pair(cfg, prefix: int, prompt_seed: int, max_ctx: int, max_batch: int = 1, expert_fp8: bool = False):
    W = cached_weights(cfg)
    blob = blob_from_weights(cfg, W)
    orc = OracleModel(cfg, W, f64_matrices=cfg.d_model >= 2048, expert_fp8=expert_fp8)
    den = Denoiser(cfg, blob, max_ctx=max_ctx, max_batch=max_batch, expert_fp8=expert_fp8)
    del blob
    prompt = prompt_tokens(cfg.vocab, prompt_seed, prefix)
    rec = {}
    orc.prefill(0, prompt, rec)
    if not cfg.dense:
        # the prefix K/V feed every later pass: prefill on the oracle's experts too, so
        # that a near-tie routed differently in the prompt cannot move the canvas passes
        den.set_debug(True)
        den.force_routing(np.stack(rec["topk_idx"]))
    den.prefill(0, prompt)
    if not cfg.dense:
        den.force_routing(None)
        den.set_debug(False)
    return orc, den, prompt


def commit_margin(conf: np.ndarray, mask: np.ndarray, n: int, policy: Policy) -> float:
    """log-confidence gap at the commit boundary (and at tau for the threshold policy)."""
    masked = np.nonzero(mask)[0]
    c = np.asarray(conf, np.float64)[masked]
    order = np.lexsort((masked, -c))
    cs = c[order]
    m = math.inf
    if 0 < n < cs.size:
        m = math.log(cs[n - 1]) - math.log(cs[n])
    if policy.kind == "threshold" and math.isfinite(policy.tau):
        m = min(m, float(np.min(np.abs(np.log(cs) - math.log(policy.tau)))))
    return m


def compare_trace(cfg, orc_trace, den: Denoiser, policy: Policy, s_max: int, stats=None, margin: float = MARGIN):
    """Replays every oracle step on the GPU and checks the decisions and values.

    Decisions whose oracle margin exceeds `margin` must agree. With a margin above 1e-3,
    decisions with margins between 1e-3 and `margin` that differ are counted in
    stats["near_flips"] instead (the caller bounds them).
    """
    C = cfg.canvas
    stats = stats if stats is not None else {"route_pinned": 0, "route_total": 0, "arg_pinned": 0,
                                             "arg_total": 0, "commit_pinned": 0, "steps": 0, "edits": 0,
                                             "edit_pinned": 0, "near_flips": 0, "near_total": 0}
    stats.setdefault("near_flips", 0)
    stats.setdefault("near_total", 0)
    pol = make_policy(policy.kind, policy.k, policy.tau, policy.floor, policy.t2t, policy.edit_tau)
    den.set_debug(True)
    for e in orc_trace:
        rec = e["rec"]
        canvas = torch.from_numpy(e["canvas"].astype(np.int32)[None]).cuda()
        mask = torch.from_numpy(e["mask"].astype(np.uint8)[None]).cuda()
        old_mask = e["mask"].copy()
        if not cfg.dense:
            # each layer runs on the oracle's experts, so a near-tie flip in one layer
            # cannot move the inputs of the next; every layer's own choice is still checked
            den.force_routing(np.stack(rec["topk_idx"]))
        conf, arg, rem = den.denoise_step(canvas, mask, pol, e["step"], s_max)
        conf = conf.cpu().numpy()[0]
        arg = arg.cpu().numpy()[0]
        new_mask = mask.cpu().numpy()[0].astype(bool)
        new_canvas = canvas.cpu().numpy()[0]

        # hidden state after the last layer
        x_gpu = den.debug_read(0, 0, (C, cfg.d_model), np.float32).astype(np.float64)
        x_ref = rec["final_x"]
        row_err = np.abs(x_gpu - x_ref).max(axis=1) / np.abs(x_ref).max(axis=1)
        assert row_err.max() <= REL, f"step {e['step']}: hidden rel err {row_err.max():.3g}"

        # routing, layer by layer
        if not cfg.dense:
            k = cfg.top_k
            for l in range(cfg.n_layers):
                lg = rec["router_logits"][l]
                srt = -np.sort(-lg, axis=1)
                rmargin = srt[:, k - 1] - srt[:, k]
                sel = rmargin > margin
                near = (rmargin > MARGIN) & ~sel
                gi = den.debug_read(2, l, (C, k), np.int32)
                ri = rec["topk_idx"][l]
                same = np.array([set(gi[t]) == set(ri[t]) for t in range(C)])
                bad = np.nonzero(sel & ~same)[0]
                if bad.size:
                    gl = den.debug_read(1, l, (C, cfg.n_experts), np.float32)
                    xl = den.debug_read(5, l - 1, (C, cfg.d_model), np.float32) if l > 0 else None
                    lines = []
                    for t in bad[:4]:
                        order = np.argsort(-lg[t], kind="stable")[:k + 1]
                        lines.append(f"token {t}: margin {margin[t]:.3e}; oracle logits {lg[t][order]} "
                                     f"gpu logits {gl[t][order]} (experts {order}); gpu picked {sorted(gi[t])}")
                        if xl is not None:
                            xr = rec["x"][l - 1][t]
                            lines.append(f"  input row rel err {np.abs(xl[t] - xr).max() / np.abs(xr).max():.3e}")
                    raise AssertionError(f"step {e['step']} layer {l}: routing differs at tokens {bad[:8]}\n"
                                         + "\n".join(lines))
                stats["route_pinned"] += int(sel.sum())
                stats["route_total"] += C
                stats["near_flips"] += int((near & ~same).sum())
                stats["near_total"] += int(near.sum())
                gl = den.debug_read(1, l, (C, cfg.n_experts), np.float32)
                assert np.abs(gl - lg).max() <= REL * np.abs(lg).max()

        # LM head: conf and argmax
        assert np.all(np.abs(conf / e["conf"] - 1.0) <= REL), f"step {e['step']}: conf"
        lm_sel = rec["logit_margin"] > margin
        lm_near = (rec["logit_margin"] > MARGIN) & ~lm_sel
        bad = np.nonzero(lm_sel & (arg != e["argmax"]))[0]
        assert bad.size == 0, (f"step {e['step']}: argmax differs at {bad[:8]} (margins "
                               f"{rec['logit_margin'][bad[:8]]}, conf rel err {(conf / e['conf'] - 1)[bad[:8]]})")
        stats["near_flips"] += int((lm_near & (arg != e["argmax"])).sum())
        stats["near_total"] += int(lm_near.sum())
        stats["arg_pinned"] += int(lm_sel.sum())
        stats["arg_total"] += C

        # commit
        gpu_commit = old_mask & ~new_mask
        n = int(e["commit"].sum())
        assert int(gpu_commit.sum()) == n, f"step {e['step']}: commit count {gpu_commit.sum()} vs {n}"
        assert int(rem.cpu().numpy()[0]) == int(old_mask.sum()) - n
        cm = commit_margin(e["conf"], old_mask, n, policy)
        if cm > margin:
            assert np.array_equal(gpu_commit, e["commit"]), f"step {e['step']}: commit set differs"
            stats["commit_pinned"] += 1
        elif cm > MARGIN:
            stats["near_flips"] += int(not np.array_equal(gpu_commit, e["commit"]))
            stats["near_total"] += 1
        # newly committed positions hold the pass's argmax
        assert np.array_equal(new_canvas[gpu_commit], arg[gpu_commit])
        # earlier commits: untouched (M2T); with T2T, re-written exactly where the oracle
        # edits, wherever that decision is pinned (argmax margin, and the log-confidence
        # margin to edit_tau, above 1e-3), and only ever to the pass's argmax
        committed = ~old_mask
        gpu_edit = committed & (new_canvas != e["canvas"])
        if policy.t2t:
            pinned = committed & lm_sel & (np.abs(np.log(e["conf"].astype(np.float64))
                                                  - math.log(policy.edit_tau)) > margin)
            bad = np.nonzero(pinned & (gpu_edit != e["edit"]))[0]
            assert bad.size == 0, f"step {e['step']}: edit set differs at {bad[:8]}"
            assert np.array_equal(new_canvas[gpu_edit], arg[gpu_edit])
            stats["edits"] += int(gpu_edit.sum())
            stats["edit_pinned"] += int((pinned & e["edit"]).sum())
        else:
            assert not gpu_edit.any(), f"step {e['step']}: a committed token changed"
        assert not np.any(new_mask & ~old_mask)
        stats["steps"] += 1
    if not cfg.dense:
        den.force_routing(None)
    den.set_debug(False)
    return stats


def check_generate_invariants(cfg, den: Denoiser, policy: Policy, s_max: int, expect_steps=None):
    pol = make_policy(policy.kind, policy.k, policy.tau, policy.floor, policy.t2t, policy.edit_tau)
    code, canvas, steps = den.generate_block(1, s_max, pol)
    assert code == 0, code
    c = canvas.cpu().numpy()[0]
    assert np.all((c >= 0) & (c <= cfg.vocab - 2)), "a [MASK] or out-of-range token survived"
    assert steps[0] <= s_max
    if expect_steps is not None:
        assert steps[0] == expect_steps
    return c, steps[0]
