"""Planted mistakes: every pin of the oracle must notice a plausible error in it.

Each case below replaces one oracle function with a copy that carries a single
plausible mistake (a dropped term, a wrong sign or index, a transposed operand, a wrong
tie rule), then runs the pins that guard that function. The case passes only if at
least one of those pins fails on the mutant. A pin that cannot tell a mutant from the
real function pins nothing, and this file says so by failing.
"""

import math

import numpy as np
import pytest

import oracle
import oracle.model as om
import test_oracle_pins as pins


# ---------------------------------------------------------------- mutants

def rmsnorm_sum(x, g, eps):            # sum of squares instead of their mean
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * np.asarray(g, np.float64)


def rmsnorm_eps_outside(x, g, eps):    # eps added after the square root
    x = np.asarray(x, np.float64)
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * np.asarray(g, np.float64)


def rmsnorm_no_gain(x, g, eps):        # gains dropped
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def bf16_truncate(x):                  # truncation instead of round-to-nearest-even
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)


def bf16_half_up(x):                   # ties away from zero instead of to even
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + np.uint64(0x8000)) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def attention_no_scale(q, k, v, allowed=None):
    return om.__dict__["_orig_attention"](q * math.sqrt(q.shape[2]), k, v, allowed)


def attention_gqa_modulo(q, k, v, allowed=None):   # head h reads KV head h % Hkv
    Tq, H, hd = q.shape
    Hkv = k.shape[1]
    out = np.zeros((Tq, H, v.shape[2]))
    for h in range(H):
        s = q[:, h] @ k[:, h % Hkv].T / math.sqrt(hd)
        if allowed is not None:
            s = np.where(allowed, s, -np.inf)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        out[:, h] = (e / e.sum(axis=1, keepdims=True)) @ v[:, h % Hkv]
    return out


def attention_ignores_mask(q, k, v, allowed=None):
    return om.__dict__["_orig_attention"](q, k, v, None)


def attention_softmax_over_queries(q, k, v, allowed=None):   # normalised over the wrong axis
    Tq, H, hd = q.shape
    Hkv = k.shape[1]
    out = np.zeros((Tq, H, v.shape[2]))
    for h in range(H):
        g = h * Hkv // H
        s = q[:, h] @ k[:, g].T / math.sqrt(hd)
        if allowed is not None:
            s = np.where(allowed, s, -np.inf)
        e = np.exp(s - s.max(axis=0, keepdims=True))
        out[:, h] = (e / e.sum(axis=0, keepdims=True)) @ v[:, g]
    return out


def rope_sign_swapped(x, cos, sin):
    half = x.shape[-1] // 2
    a, b = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([a * c + b * s, b * c - a * s], axis=-1)


def rope_adjacent_pairs(x, cos, sin):  # pairs (2i, 2i+1) instead of (i, i + hd/2)
    a, b = x[..., 0::2], x[..., 1::2]
    c, s = cos[:, None, :], sin[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = b * c + a * s
    return out


def rope_freq_wrong(positions, head_dim, theta):   # theta^(-i/hd) instead of theta^(-2i/hd)
    half = head_dim // 2
    inv = theta ** (-1.0 * np.arange(half, dtype=np.float64) / head_dim)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def router_ties_high(y, wr, k):        # ties resolved toward the higher expert
    logits = om.f32(np.asarray(y, np.float64) @ np.asarray(wr, np.float64).T)
    E = logits.shape[1]
    order = (E - 1) - np.argsort(-logits[:, ::-1], axis=1, kind="stable")
    idx = order[:, :k]
    sel = np.take_along_axis(logits, idx, axis=1)
    ex = np.exp(sel - sel[:, :1])
    return logits, idx.astype(np.int64), ex / ex.sum(axis=1, keepdims=True)


def router_gates_over_all(y, wr, k):   # gates from a softmax over every expert
    logits, idx, _ = om.__dict__["_orig_router_topk"](y, wr, k)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return logits, idx, np.take_along_axis(p, idx, axis=1)


def router_bottom_k(y, wr, k):         # the k smallest logits
    logits = om.f32(np.asarray(y, np.float64) @ np.asarray(wr, np.float64).T)
    idx = np.argsort(logits, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(logits, idx, axis=1)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    return logits, idx.astype(np.int64), ex / ex.sum(axis=1, keepdims=True)


def swiglu_swapped(yb, wg, wu, wd):    # silu on the up branch instead of the gate
    g = yb @ np.asarray(wg, np.float64).T
    u = yb @ np.asarray(wu, np.float64).T
    return (u / (1.0 + np.exp(-u)) * g) @ np.asarray(wd, np.float64).T


def swiglu_sigmoid(yb, wg, wu, wd):    # sigmoid instead of silu
    g = yb @ np.asarray(wg, np.float64).T
    u = yb @ np.asarray(wu, np.float64).T
    return (1.0 / (1.0 + np.exp(-g)) * u) @ np.asarray(wd, np.float64).T


def swiglu_down_transposed(yb, wg, wu, wd):
    g = yb @ np.asarray(wg, np.float64).T
    u = yb @ np.asarray(wu, np.float64).T
    return (g / (1.0 + np.exp(-g)) * u) @ np.asarray(wd, np.float64)


def moe_no_gates(y, experts, wr, k):   # expert outputs summed without their gates
    out, logits, idx, gates = om.__dict__["_orig_moe_ffn"](y, experts, wr, k)
    T = y.shape[0]
    yb = np.asarray(y, np.float64)
    plain = np.zeros_like(out)
    for e in range(len(experts)):
        tok, _ = np.nonzero(idx == e)
        if tok.size:
            np.add.at(plain, tok, om.swiglu_expert(yb[tok], *experts[e]))
    return plain, logits, idx, gates


def lm_head_keeps_mask(x, final_norm, head, mask_id, eps, return_logits=False):
    yb = om.rmsnorm(x, final_norm, eps)
    logits = om.f32(yb @ np.asarray(head, np.float64).T)
    m = logits.max(axis=1)
    arg = np.argmax(logits, axis=1)
    conf = np.asarray(1.0 / np.exp(logits - m[:, None]).sum(axis=1), np.float32)
    return (conf, arg, logits) if return_logits else (conf, arg)


def lm_head_last_max(x, final_norm, head, mask_id, eps, return_logits=False):   # ties to the highest id
    yb = om.rmsnorm(x, final_norm, eps)
    logits = om.f32(yb @ np.asarray(head, np.float64).T)
    logits[:, mask_id] = -np.inf
    m = logits.max(axis=1)
    arg = logits.shape[1] - 1 - np.argmax(logits[:, ::-1], axis=1)
    conf = np.asarray(1.0 / np.exp(logits - m[:, None]).sum(axis=1), np.float32)
    return (conf, arg, logits) if return_logits else (conf, arg)


def lm_head_conf_over_rest(x, final_norm, head, mask_id, eps, return_logits=False):   # 1 / (Z - 1)
    conf, arg, logits = om.__dict__["_orig_lm_head_conf"](x, final_norm, head, mask_id, eps, True)
    conf = np.asarray(1.0 / (1.0 / conf.astype(np.float64) - 1.0 + 1e-300), np.float32)
    return (conf, arg, logits) if return_logits else (conf, arg)


def commit_count_no_floor(R, n_above, policy, step, s_max):
    n = policy.k if policy.kind == "topk" else n_above
    return max(0, min(n, R))


def commit_count_floor_division(R, n_above, policy, step, s_max):
    if policy.kind == "topk":
        n = policy.k
    else:
        n = n_above
        if policy.floor:
            left = s_max - step
            n = max(n, R if left <= 0 else max(1, R // left))
    return max(0, min(n, R))


def commit_select_ties_high(conf, mask, policy, step, s_max):
    conf32 = np.asarray(conf, np.float32)
    masked = np.nonzero(np.asarray(mask, bool))[0]
    n_above = int(np.sum(conf32[masked] > np.float32(policy.tau))) if policy.kind != "topk" else 0
    n = om.commit_count(masked.size, n_above, policy, step, s_max)
    order = masked[np.lexsort((-masked, -conf32[masked].astype(np.float64)))]
    sel = np.zeros(np.asarray(mask).shape[0], bool)
    sel[order[:n]] = True
    return sel


def commit_select_at_or_above(conf, mask, policy, step, s_max):   # conf >= tau counts
    conf32 = np.asarray(conf, np.float32)
    masked = np.nonzero(np.asarray(mask, bool))[0]
    n_above = int(np.sum(conf32[masked] >= np.float32(policy.tau))) if policy.kind != "topk" else 0
    n = om.commit_count(masked.size, n_above, policy, step, s_max)
    order = masked[np.lexsort((masked, -conf32[masked].astype(np.float64)))]
    sel = np.zeros(np.asarray(mask).shape[0], bool)
    sel[order[:n]] = True
    return sel


def commit_select_ignores_mask(conf, mask, policy, step, s_max):   # committed positions compete again
    return om.__dict__["_orig_commit_select"](conf, np.ones_like(np.asarray(mask, bool)), policy, step, s_max)


def canvas_forward_rope_from_zero(self, req, canvas, mask, rec=None):   # canvas positions 0..C-1
    st = self.requests[req]
    P = st.P
    st.P = 0
    try:
        tokens = np.where(np.asarray(mask, bool), self.cfg.mask_id, np.asarray(canvas, np.int64))
        x = self.emb[tokens].astype(np.float64)
        pos = np.arange(tokens.size)
        ks, vs = [], []
        for l in range(self.cfg.n_layers):
            x, k, v = self.layer(l, x, pos, st.k[l], st.v[l], None, rec)
            ks.append(k)
            vs.append(v)
    finally:
        st.P = P
    return x, ks, vs


def canvas_forward_ignores_mask(self, req, canvas, mask, rec=None):   # [MASK] positions keep their token
    return om.OracleModel.__dict__["_orig_canvas_forward"](self, req, canvas, np.zeros_like(np.asarray(mask, bool)),
                                                          rec)


def append_keeps_prefix_length(self, req, canvas):
    st = self.requests[req]
    P = st.P
    om.OracleModel.__dict__["_orig_append"](self, req, canvas)
    st.P = P


def edit_select_masked_too(conf, argmax, canvas, mask, policy):   # edits masked positions as well
    if not policy.t2t:
        return np.zeros(np.asarray(mask).shape[0], dtype=bool)
    return (np.asarray(argmax) != np.asarray(canvas)) & (np.asarray(conf, np.float32) > np.float32(policy.edit_tau))


def edit_select_at_or_above(conf, argmax, canvas, mask, policy):   # conf >= edit_tau
    if not policy.t2t:
        return np.zeros(np.asarray(mask).shape[0], dtype=bool)
    committed = ~np.asarray(mask, bool)
    return committed & (np.asarray(argmax) != np.asarray(canvas)) & (
        np.asarray(conf, np.float32) >= np.float32(policy.edit_tau))


def edit_select_ignores_token(conf, argmax, canvas, mask, policy):   # re-writes even an equal token
    if not policy.t2t:
        return np.zeros(np.asarray(mask).shape[0], dtype=bool)
    return ~np.asarray(mask, bool) & (np.asarray(conf, np.float32) > np.float32(policy.edit_tau))


def append_approx_from_masked(self, req):   # K/V of the canvas as if every position were [MASK]
    st = self.requests[req]
    C = st.last_k[0].shape[0]
    _, ks, vs = om.OracleModel.__dict__["_canvas_forward"](self, req, np.full(C, self.cfg.mask_id),
                                                          np.ones(C, bool))
    st.last_k, st.last_v = ks, vs
    om.OracleModel.__dict__["_orig_append_approx"](self, req)


def fp8_exponents_plus_one(w, block=128):     # a scale twice the least one
    return om.__dict__["_orig_fp8_block_exponents"](w, block) + 1


def fp8_exponents_per_row(w, block=128):      # the first row's scale for its whole tile
    w = np.asarray(w, np.float64)
    ex = om.__dict__["_orig_fp8_block_exponents"](w, block)
    for bi in range(ex.shape[0]):
        ex[bi] = om.__dict__["_orig_fp8_block_exponents"](w[bi * block:bi * block + 1], block)[0]
    return ex


def e4m3_truncate(x):                         # rounds toward zero
    v = om.e4m3_values()
    x = np.asarray(x, np.float64)
    i = np.searchsorted(v, np.abs(x), side="right") - 1
    return np.sign(x) * v[i]


def e4m3_ties_up(x):                          # ties away from zero instead of to the even code
    v = om.e4m3_values()
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    i = np.clip(np.searchsorted(v, a), 1, v.size - 1)
    lo, hi = v[i - 1], v[i]
    return np.sign(x) * np.where(hi - a <= a - lo, hi, lo)


# ---------------------------------------------------------------- which pins guard what

P = pins
CASES = [
    ("rmsnorm", rmsnorm_sum, [P.test_rmsnorm_closed_forms]),
    ("rmsnorm", rmsnorm_eps_outside, [P.test_rmsnorm_closed_forms]),
    ("rmsnorm", rmsnorm_no_gain, [P.test_rmsnorm_closed_forms]),
    ("bf16", bf16_truncate, [P.test_bf16_rounding_ties_and_edges, P.test_bf16_rounding_matches_torch]),
    ("bf16", bf16_half_up, [P.test_bf16_rounding_ties_and_edges, P.test_bf16_rounding_matches_torch]),
    ("attention", attention_no_scale, [lambda: P.test_attention_matches_brute_force(4, 2),
                                       P.test_attention_closed_forms]),
    ("attention", attention_gqa_modulo, [P.test_attention_gqa_head_mapping,
                                         lambda: P.test_attention_matches_brute_force(4, 2)]),
    ("attention", attention_ignores_mask, [lambda: P.test_attention_matches_brute_force(4, 4),
                                           P.test_attention_closed_forms]),
    ("attention", attention_softmax_over_queries, [lambda: P.test_attention_matches_brute_force(4, 4)]),
    ("apply_rope", rope_sign_swapped, [P.test_rope_pairing_special_case]),
    ("apply_rope", rope_adjacent_pairs, [P.test_rope_pairing_special_case]),
    ("rope_cos_sin", rope_freq_wrong, [P.test_rope_pairing_special_case]),
    ("router_topk", router_ties_high, [P.test_router_ties_prefer_lower_expert]),
    ("router_topk", router_gates_over_all, [P.test_router_topk_brute_force_subsets]),
    ("router_topk", router_bottom_k, [P.test_router_topk_brute_force_subsets]),
    ("swiglu_expert", swiglu_swapped, [P.test_swiglu_expert_closed_form]),
    ("swiglu_expert", swiglu_sigmoid, [P.test_swiglu_expert_closed_form]),
    ("swiglu_expert", swiglu_down_transposed, [P.test_swiglu_expert_closed_form]),
    ("moe_ffn", moe_no_gates, [P.test_moe_reductions]),
    ("lm_head_conf", lm_head_keeps_mask, [P.test_lm_head_logsumexp_and_mask_exclusion,
                                          P.test_lm_head_zero_gain_closed_form]),
    ("lm_head_conf", lm_head_last_max, [P.test_lm_head_zero_gain_closed_form]),
    ("lm_head_conf", lm_head_conf_over_rest, [P.test_lm_head_zero_gain_closed_form]),
    ("commit_count", commit_count_no_floor, [P.test_threshold_floor_schedule_twelve_steps]),
    ("commit_count", commit_count_floor_division, [P.test_threshold_floor_schedule_twelve_steps]),
    ("commit_select", commit_select_ties_high, [P.test_topk_ties_go_to_lower_position]),
    ("commit_select", commit_select_at_or_above, [P.test_threshold_is_strictly_above_tau]),
    ("commit_select", commit_select_ignores_mask, [P.test_threshold_commits_everything_above_tau]),
    ("OracleModel._canvas_forward", canvas_forward_rope_from_zero,
     [lambda: P.test_cached_passes_equal_block_causal_sequence(P.MICRO)]),
    ("OracleModel._canvas_forward", canvas_forward_ignores_mask,
     [lambda: P.test_cached_passes_equal_block_causal_sequence(P.MICRO)]),
    ("OracleModel.append", append_keeps_prefix_length,
     [lambda: P.test_cached_passes_equal_block_causal_sequence(P.MICRO_DENSE)]),
    ("edit_select", edit_select_masked_too, [P.test_edit_select_rule]),
    ("edit_select", edit_select_at_or_above, [P.test_edit_select_rule]),
    ("edit_select", edit_select_ignores_token, [P.test_edit_select_rule, P.test_generate_block_t2t_invariants]),
    ("fp8_block_exponents", fp8_exponents_plus_one, [P.test_fp8_block_scales_and_round_trip]),
    ("fp8_block_exponents", fp8_exponents_per_row, [P.test_fp8_block_scales_and_round_trip]),
    ("e4m3_round", e4m3_truncate, [P.test_e4m3_rounding_ties_and_torch, P.test_fp8_block_scales_and_round_trip]),
    ("e4m3_round", e4m3_ties_up, [P.test_e4m3_rounding_ties_and_torch]),
    ("OracleModel.append_approx", append_approx_from_masked,
     [lambda: P.test_approximate_append_equals_exact_append_on_a_finished_pass(P.MICRO)]),
]


def _plant(monkeypatch, name, mutant):
    if name.startswith("OracleModel."):
        meth = name.split(".", 1)[1]
        monkeypatch.setattr(om.OracleModel, "_orig_" + meth.lstrip("_"), om.OracleModel.__dict__[meth],
                            raising=False)
        monkeypatch.setattr(om.OracleModel, meth, mutant)
        return
    monkeypatch.setitem(om.__dict__, "_orig_" + name, getattr(om, name))
    monkeypatch.setattr(om, name, mutant)
    for mod in (oracle, pins):
        if hasattr(mod, name):
            monkeypatch.setattr(mod, name, mutant)


@pytest.mark.parametrize("name,mutant,guards", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_planted_mistake_fails_a_pin(name, mutant, guards, monkeypatch):
    _plant(monkeypatch, name, mutant)
    caught = []
    for pin in guards:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            caught.append(pin)
    assert caught, f"no pin noticed the planted mistake {mutant.__name__} in {name}"


def test_pins_pass_on_the_real_oracle():
    """The guards above fail on the mutants, not on the oracle itself."""
    for _, _, guards in CASES:
        for pin in guards:
            pin()
