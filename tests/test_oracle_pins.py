"""Pins for the CPU oracle against what the pages and the mathematics fix.

No page prints a worked numeric example for this method, so every pin is a closed
form, an invariant, a brute-force count on tiny inputs or a reduction to a library
routine. A plausible mistake in the oracle (a dropped scale, a wrong GQA index, a
swapped RoPE sign, a wrong tie rule, a missing mask) fails at least one of them;
the planted-mistake tests at the end check that.
"""

import itertools
import math

import numpy as np
import pytest
import scipy.special

import oracle
from oracle import (OracleModel, Policy, apply_rope, attention, commit_count, commit_select,
                    lm_head_conf, moe_ffn, rope_cos_sin, router_topk, sequence_forward,
                    swiglu_expert)
from synth import gen_weights, prompt_tokens, uniform_f32
from synth.configs import ModelConfig

MICRO = ModelConfig("micro", n_layers=2, d_model=64, n_heads=4, n_kv_heads=2, head_dim=16,
                    n_experts=4, top_k=2, ffn_dim=64, vocab=64, canvas=8,
                    weight_dtype="bf16", weight_seed=77)
MICRO_DENSE = ModelConfig("micro-dense", n_layers=2, d_model=64, n_heads=4, n_kv_heads=4,
                          head_dim=16, n_experts=0, top_k=1, ffn_dim=64, vocab=64, canvas=8,
                          weight_dtype="f32", weight_seed=78)


def rnd(shape, tid, seed=5, scale=1.0):
    n = int(np.prod(shape))
    return (uniform_f32(seed, tid, n).astype(np.float64) * scale).reshape(shape)


# ---------------------------------------------------------------- attention

def brute_attention(q, k, v, allowed=None):
    Tq, H, hd = q.shape
    Tk, Hkv, _ = k.shape
    out = np.zeros_like(q)
    for i in range(Tq):
        for h in range(H):
            g = h // (H // Hkv)
            w = []
            for j in range(Tk):
                if allowed is None or allowed[i, j]:
                    w.append(math.exp(sum(q[i, h, t] * k[j, g, t] for t in range(hd)) / math.sqrt(hd)))
                else:
                    w.append(0.0)
            z = sum(w)
            for t in range(hd):
                out[i, h, t] = sum(w[j] * v[j, g, t] for j in range(Tk)) / z
    return out


@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (4, 1)])
def test_attention_matches_brute_force(H, Hkv):
    q, k, v = rnd((5, H, 8), 1), rnd((7, Hkv, 8), 2), rnd((7, Hkv, 8), 3)
    assert np.allclose(attention(q, k, v), brute_attention(q, k, v), rtol=1e-12, atol=1e-12)
    causal = np.arange(7)[None, :] <= np.arange(5)[:, None] + 2
    assert np.allclose(attention(q, k, v, causal), brute_attention(q, k, v, causal),
                       rtol=1e-12, atol=1e-12)


def test_attention_closed_forms():
    q, v = rnd((3, 2, 8), 4), rnd((6, 1, 8), 5)
    k_same = np.repeat(rnd((1, 1, 8), 6), 6, axis=0)
    # identical keys: uniform weights, output = mean of V for every head
    o = attention(q, k_same, v)
    assert np.allclose(o, np.broadcast_to(v.mean(axis=0)[None], o.shape), atol=1e-14)
    # one dominant score selects that value row
    k = np.zeros((6, 1, 8))
    k[4, 0, :] = 1e3 * np.sign(q[0, 0, :])
    o = attention(q[:1, :1], k, v)
    assert np.allclose(o[0, 0], v[4, 0], atol=1e-12)
    # a causal row 0 sees only key 0
    causal = np.arange(6)[None, :] <= np.arange(3)[:, None]
    o = attention(q, rnd((6, 1, 8), 7), v, causal)
    assert np.allclose(o[0, :, :], np.broadcast_to(v[0, 0], (2, 8)), atol=1e-14)


def test_attention_gqa_head_mapping():
    # Hkv = 2 with H = 4: heads 0,1 read KV head 0; heads 2,3 read KV head 1
    q = np.zeros((1, 4, 4))
    k = np.zeros((2, 2, 4))
    v = np.zeros((2, 2, 4))
    v[:, 0, :], v[:, 1, :] = 1.0, 2.0
    o = attention(q, k, v)
    assert np.allclose(o[0, :, 0], [1, 1, 2, 2])


# ---------------------------------------------------------------- RoPE

def test_rope_relative_position_and_norm():
    hd = 16
    q, k = rnd((1, 1, hd), 8), rnd((1, 1, hd), 9)
    dots = []
    for shift in (0, 5, 123, 4096):
        cq, sq = rope_cos_sin(np.array([7 + shift]), hd, 1e4)
        ck, sk = rope_cos_sin(np.array([3 + shift]), hd, 1e4)
        dots.append(float(np.sum(apply_rope(q, cq, sq) * apply_rope(k, ck, sk))))
    assert np.allclose(dots, dots[0], rtol=1e-10)
    c, s = rope_cos_sin(np.array([11]), hd, 1e4)
    assert np.isclose(np.linalg.norm(apply_rope(q, c, s)), np.linalg.norm(q), rtol=1e-12)
    c0, s0 = rope_cos_sin(np.array([0]), hd, 1e4)
    assert np.allclose(apply_rope(q, c0, s0), q)


def test_rope_pairing_special_case():
    # hd = 4, theta = 1e4: frequencies 1 and 1e-2; pair (0, 2) turns by pos radians
    x = np.array([[[1.0, 0.0, 0.0, 0.0]]])
    c, s = rope_cos_sin(np.array([1]), 4, 1e4)
    assert np.allclose(apply_rope(x, c, s)[0, 0], [math.cos(1), 0, math.sin(1), 0])
    y = np.array([[[0.0, 1.0, 0.0, 0.0]]])
    assert np.allclose(apply_rope(y, c, s)[0, 0], [0, math.cos(0.01), 0, math.sin(0.01)])


# ---------------------------------------------------------------- MoE

def test_router_topk_brute_force_subsets():
    E, k = 8, 2
    y, wr = rnd((40, 16), 10), rnd((E, 16), 11)
    logits, idx, gates = router_topk(y, wr, k)
    for t in range(40):
        best = max(itertools.combinations(range(E), k),
                   key=lambda sub: (sum(logits[t, list(sub)]), [-e for e in sub]))
        assert set(idx[t]) == set(best)
        assert logits[t, idx[t, 0]] >= logits[t, idx[t, 1]]
        sel = logits[t, idx[t]]
        assert np.allclose(gates[t], scipy.special.softmax(sel))


def test_router_ties_prefer_lower_expert():
    y = np.ones((1, 4))
    wr = np.array([[0.0] * 4, [1.0] * 4, [1.0] * 4, [1.0] * 4])
    _, idx, gates = router_topk(y, wr, 2)
    assert list(idx[0]) == [1, 2]
    assert np.allclose(gates[0], [0.5, 0.5])


def test_moe_reductions():
    d, F, T = 16, 32, 6
    y = rnd((T, d), 12)
    experts = [(rnd((F, d), 20 + e, scale=0.3), rnd((F, d), 30 + e, scale=0.3),
                rnd((d, F), 40 + e, scale=0.3)) for e in range(3)]
    wr = rnd((3, d), 13)
    # k = E: the softmax-weighted mixture of every expert
    out, logits, idx, gates = moe_ffn(y, experts, wr, 3)
    yb = y
    p = scipy.special.softmax(logits, axis=1)
    ref = sum(p[:, e:e + 1] * swiglu_expert(yb, *experts[e]) for e in range(3))
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    # dense = one expert with gate 1
    dense, _, _, g = moe_ffn(y, experts[:1], None, 1)
    assert np.allclose(g, 1.0)
    wg, wu, wd = experts[0]
    h = yb @ wg.T
    ref_dense = (h * scipy.special.expit(h) * (yb @ wu.T)) @ wd.T
    assert np.allclose(dense, ref_dense, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- LM head and confidence

def test_lm_head_zero_gain_closed_form():
    V, d = 64, 16
    x, head = rnd((5, d), 14), rnd((V, d), 15)
    conf, arg = lm_head_conf(x, np.zeros(d), head, V - 1, 1e-6)
    assert np.all(conf == np.float32(1.0 / (V - 1)))
    assert np.all(arg == 0)


def test_lm_head_logsumexp_and_mask_exclusion():
    V, d = 64, 16
    x, head = rnd((7, d), 16), rnd((V, d), 17)
    head[V - 1] = 50.0 * oracle.bf16(x[0]) / np.linalg.norm(x[0])   # [MASK] would win row 0
    head = oracle.bf16(head)
    conf, arg, logits = lm_head_conf(x, np.ones(d), head, V - 1, 1e-6, return_logits=True)
    y = oracle.rmsnorm(x, np.ones(d), 1e-6)
    raw = (y @ head.T)[:, : V - 1]
    assert np.all(arg != V - 1)
    assert np.array_equal(arg, np.argmax(raw, axis=1))
    lse = scipy.special.logsumexp(raw, axis=1)
    assert np.allclose(conf, np.exp(raw.max(axis=1) - lse), rtol=1e-6)


# ---------------------------------------------------------------- commit / sampler

def test_threshold_floor_schedule_twelve_steps():
    # flat confidences never pass tau = 0.9: the floor alone sets the schedule
    R, sched = 256, []
    for s in range(12):
        n = commit_count(R, 0, Policy("threshold", tau=0.9, floor=True), s, 12)
        sched.append(n)
        R -= n
    assert sched == [22] * 4 + [21] * 8 and R == 0


def test_threshold_commits_everything_above_tau():
    conf = np.array([0.95, 0.2, 0.91, 0.99, 0.5, 0.92], np.float32)
    mask = np.array([1, 1, 1, 0, 1, 1], bool)
    sel = commit_select(conf, mask, Policy("threshold", tau=0.9, floor=True), 0, 48)
    assert list(np.nonzero(sel)[0]) == [0, 2, 5]          # 0.99 is already committed
    sel = commit_select(conf, mask, Policy("threshold", tau=0.99, floor=False), 0, 48)
    assert not sel.any()
    # floor at the last step commits every remaining position
    sel = commit_select(conf, mask, Policy("threshold", tau=0.99, floor=True), 47, 48)
    assert sel.sum() == mask.sum()


def test_topk_ties_go_to_lower_position():
    conf = np.array([0.5, 0.7, 0.5, 0.7, 0.5], np.float32)
    mask = np.ones(5, bool)
    sel = commit_select(conf, mask, Policy("topk", k=3), 0, 8)
    assert list(np.nonzero(sel)[0]) == [0, 1, 3]


@pytest.mark.parametrize("cfg,policy,s_max", [
    (MICRO, Policy("topk", k=2), 4),
    (MICRO_DENSE, Policy("topk", k=1), 8),
    (MICRO, Policy("threshold", tau=0.9, floor=True), 3),
])
def test_generate_block_invariants(cfg, policy, s_max):
    m = OracleModel(cfg, gen_weights(cfg))
    m.prefill(0, prompt_tokens(cfg.vocab, 2000, 12))
    canvas, steps, tr = m.generate_block(0, policy, s_max, trace=True)
    C = cfg.canvas
    assert tr[0]["mask"].all()                                   # all-[MASK] start
    assert steps <= s_max and not np.any(canvas == cfg.mask_id)  # full within budget
    prev_R = C
    for e in tr:
        R = int(e["mask"].sum())
        assert R == prev_R
        committed = ~e["mask"]
        nxt = np.where(e["commit"], e["argmax"], e["canvas"])
        assert np.array_equal(nxt[committed], e["canvas"][committed])   # M2T: never revised
        assert not np.any(e["commit"] & committed)
        if policy.kind == "topk":
            assert e["commit"].sum() == min(policy.k, R)
        assert e["remaining"] < R                                # strictly decreasing
        prev_R = e["remaining"]
    assert prev_R == 0
    if policy.kind == "topk":
        assert steps == C // policy.k


# ---------------------------------------------------------------- KV cache

def block_causal(lengths):
    n = sum(lengths)
    blk = np.concatenate([[i] * L for i, L in enumerate(lengths)])
    pos = np.arange(n)
    allowed = blk[None, :] <= blk[:, None]
    # block 0 (the prompt) is causal inside itself
    allowed &= ~((blk[:, None] == 0) & (blk[None, :] == 0) & (pos[None, :] > pos[:, None]))
    return allowed


@pytest.mark.parametrize("cfg", [MICRO, MICRO_DENSE])
def test_cached_passes_equal_block_causal_sequence(cfg):
    m = OracleModel(cfg, gen_weights(cfg))
    P, C = 10, cfg.canvas
    prompt = prompt_tokens(cfg.vocab, 2001, P)
    m.prefill(0, prompt)
    c1 = prompt_tokens(cfg.vocab, 2002, C)
    mask = np.zeros(C, bool)
    mask[::3] = True
    x_cached, _, _ = m._canvas_forward(0, c1, mask)
    seq = np.concatenate([prompt, np.where(mask, cfg.mask_id, c1)])
    x_full = sequence_forward(m, seq, block_causal([P, C]))
    assert np.allclose(x_cached, x_full[P:], rtol=1e-9, atol=1e-9)
    # append c1, then a second canvas sees [prompt | c1 | c2]
    k0 = m.requests[0].k[0].copy()
    m.append(0, c1)
    assert m.requests[0].P == P + C
    assert np.array_equal(m.requests[0].k[0][:P], k0)        # prefix K/V untouched
    c2 = prompt_tokens(cfg.vocab, 2003, C)
    x2, _, _ = m._canvas_forward(0, c2, np.ones(C, bool))
    seq2 = np.concatenate([prompt, c1, np.full(C, cfg.mask_id)])
    x2_full = sequence_forward(m, seq2, block_causal([P, C, C]))
    assert np.allclose(x2, x2_full[P + C:], rtol=1e-9, atol=1e-9)


def test_prefix_kv_is_causal():
    cfg = MICRO
    m = OracleModel(cfg, gen_weights(cfg))
    p = prompt_tokens(cfg.vocab, 2004, 12)
    m.prefill(0, p)
    k_a = [a.copy() for a in m.requests[0].k]
    p2 = p.copy()
    p2[8:] = (p2[8:] + 1) % (cfg.vocab - 1)
    m.prefill(1, p2)
    for l in range(cfg.n_layers):
        assert np.array_equal(k_a[l][:8], m.requests[1].k[l][:8])
        assert not np.array_equal(k_a[l][8:], m.requests[1].k[l][8:])




# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_closed_forms():
    eps = 1e-6
    d = 8
    # a constant row c: mean(x^2) = c^2, so y = c / sqrt(c^2 + eps); at c = 1e-3 the
    # eps term is as large as c^2, so it must sit inside the square root
    for c in (1e-3, 0.5, 3.0, -2.0):
        y = oracle.rmsnorm(np.full((1, d), c), np.ones(d), eps)
        assert np.allclose(y, c / math.sqrt(c * c + eps), rtol=1e-13, atol=0)
    # a row of +-a: every entry keeps its sign and has magnitude a / sqrt(a^2 + eps)
    sgn = np.array([1, -1, 1, 1, -1, -1, 1, -1], np.float64)
    y = oracle.rmsnorm(0.25 * sgn[None], np.ones(d), eps)
    assert np.allclose(y[0], sgn * 0.25 / math.sqrt(0.0625 + eps), rtol=1e-13, atol=0)
    # by hand: x = (1, 2, 3, 4), mean(x^2) = 30 / 4 = 7.5, gains (1, 0.5, 2, -1)
    y = oracle.rmsnorm(np.array([[1.0, 2.0, 3.0, 4.0]]), np.array([1.0, 0.5, 2.0, -1.0]), eps)
    assert np.allclose(y[0], np.array([1.0, 1.0, 6.0, -4.0]) / math.sqrt(7.5 + eps), rtol=1e-13, atol=0)
    # scale invariance: with eps negligible against mean(x^2), y does not depend on |x|
    x = rnd((3, 16), 18)
    g = rnd((16,), 19)
    assert np.allclose(oracle.rmsnorm(1e3 * x, g, eps), oracle.rmsnorm(x, g, 0.0), rtol=1e-12)
    # rows are normalised independently
    two = oracle.rmsnorm(np.stack([np.full(d, 2.0), np.full(d, -0.5)]), np.ones(d), 0.0)
    assert np.allclose(two, np.stack([np.ones(d), -np.ones(d)]), rtol=1e-15)


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_ties_and_edges():
    # bf16 keeps 7 explicit mantissa bits: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    # and goes to the even neighbour 1; 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 (odd)
    # and 1 + 2^-6 (even)
    cases = {
        1.0 + 2.0 ** -8: 1.0,
        1.0 + 3 * 2.0 ** -8: 1.0 + 2.0 ** -6,
        -(1.0 + 2.0 ** -8): -1.0,
        1.0 + 2.0 ** -8 + 2.0 ** -20: 1.0 + 2.0 ** -7,     # just above the tie: up
        1.0 + 2.0 ** -8 - 2.0 ** -20: 1.0,                  # just below: down
        2.0 ** -133: 2.0 ** -133,                           # smallest bf16 subnormal
        3 * 2.0 ** -134: 2.0 ** -132,                       # subnormal tie, to even
        2.0 ** -149: 0.0,                                   # below half the smallest subnormal
        0.1: 0.10009765625,                                 # 0x3DCCCCCD -> 0x3DCD
        65504.0: 65536.0,
    }
    got = oracle.bf16(np.array(list(cases), np.float32))
    assert np.array_equal(got, np.array(list(cases.values()), np.float64))
    assert np.isinf(oracle.bf16(np.array([3.4e38], np.float32))[0])   # above the bf16 maximum


def test_bf16_rounding_matches_torch():
    import torch
    x = np.concatenate([uniform_f32(9, 1, 20000, -4, 4), uniform_f32(9, 2, 20000, -1e-3, 1e-3),
                        (uniform_f32(9, 3, 5000, -1, 1) * np.float32(2.0 ** -130)).astype(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16(x), ref)


# ---------------------------------------------------------------- SwiGLU expert

def test_swiglu_expert_closed_form():
    # sigmoid(ln 3) = 3/4, so silu(ln 3) = 0.75 ln 3 and silu(-ln 3) = -0.25 ln 3
    l3 = math.log(3.0)
    y = np.array([[l3, -l3]])
    wg, wu = np.eye(2), 2.0 * np.eye(2)
    wd = np.array([[1.0, 0.0], [1.0, 1.0]])
    # h = silu(Wg y) * (Wu y) = (0.75 l3 * 2 l3, -0.25 l3 * -2 l3) = (1.5, 0.5) l3^2
    # out = Wd h = (1.5, 2.0) l3^2
    out = swiglu_expert(y, wg, wu, wd)
    assert np.allclose(out[0], np.array([1.5, 2.0]) * l3 * l3, rtol=1e-14, atol=0)


def test_threshold_is_strictly_above_tau():
    # "above" the threshold: a confidence equal to tau is not committed
    conf = np.array([0.9, 0.95, 0.1], np.float32)
    sel = commit_select(conf, np.ones(3, bool), Policy("threshold", tau=0.9, floor=False), 0, 48)
    assert list(np.nonzero(sel)[0]) == [1]


# ---------------------------------------------------------------- T2T editing and approximate append

def test_edit_select_rule():
    M = 63
    canvas = np.array([5, 7, M, 3, 9])
    mask = np.array([0, 0, 1, 0, 0], bool)
    argmax = np.array([5, 8, 9, 4, 2])
    conf = np.array([0.95, 0.95, 0.99, 0.5, 0.9], np.float32)
    on = Policy("topk", k=1, t2t=True, edit_tau=0.9)
    # 0: same token; 1: edited; 2: masked (the commit's business); 3: below tau;
    # 4: exactly at tau (not above)
    assert list(oracle.edit_select(conf, argmax, canvas, mask, on)) == [False, True, False, False, False]
    assert not oracle.edit_select(conf, argmax, canvas, mask, Policy("topk", k=1)).any()


def test_generate_block_t2t_invariants():
    cfg = MICRO
    m = OracleModel(cfg, gen_weights(cfg))
    m.prefill(0, prompt_tokens(cfg.vocab, 2000, 12))
    pol = Policy("topk", k=2, t2t=True, edit_tau=0.02)
    canvas, steps, tr = m.generate_block(0, pol, 4, trace=True)
    assert steps == 4 and not np.any(canvas == cfg.mask_id)
    edits = 0
    prev_R = cfg.canvas
    for e in tr:
        assert int(e["mask"].sum()) == prev_R
        nxt = canvas if e is tr[-1] else tr[tr.index(e) + 1]["canvas"]
        committed = ~e["mask"]
        changed = committed & (nxt != e["canvas"])
        # a committed position changes only to the pass's argmax, with conf above edit_tau
        assert np.array_equal(changed, e["edit"])
        assert np.all(nxt[changed] == e["argmax"][changed])
        assert np.all(e["conf"][changed] > np.float32(pol.edit_tau))
        assert not np.any(nxt[committed] == cfg.mask_id)        # no mask comes back
        assert e["commit"].sum() == min(pol.k, prev_R)          # the commit count is unchanged
        edits += int(changed.sum())
        prev_R = e["remaining"]
    assert edits > 0


@pytest.mark.parametrize("cfg", [MICRO, MICRO_DENSE])
def test_approximate_append_equals_exact_append_on_a_finished_pass(cfg):
    """When the last denoising pass already saw the finished canvas (nothing masked),
    its K/V are exactly what the append pass computes: the approximate and exact caches
    agree. In general they differ by what the last commit changed."""
    W = gen_weights(cfg)
    a, b = OracleModel(cfg, W), OracleModel(cfg, W)
    p = prompt_tokens(cfg.vocab, 2005, 10)
    a.prefill(0, p)
    b.prefill(0, p)
    fin = prompt_tokens(cfg.vocab, 2006, cfg.canvas).astype(np.int64)
    a.denoise_pass(0, fin, np.zeros(cfg.canvas, bool))
    a.append_approx(0)
    b.append(0, fin)
    assert a.requests[0].P == b.requests[0].P == 10 + cfg.canvas
    for l in range(cfg.n_layers):
        assert np.array_equal(a.requests[0].k[l], b.requests[0].k[l])
        assert np.array_equal(a.requests[0].v[l], b.requests[0].v[l])
    # after a pass with masked positions, the approximate cache is not the exact one
    a2, b2 = OracleModel(cfg, W), OracleModel(cfg, W)
    a2.prefill(0, p)
    b2.prefill(0, p)
    mask = np.zeros(cfg.canvas, bool)
    mask[::2] = True
    a2.denoise_pass(0, np.where(mask, cfg.mask_id, fin), mask)
    a2.append_approx(0)
    b2.append(0, fin)
    assert not np.array_equal(a2.requests[0].k[0][10:], b2.requests[0].k[0][10:])


# ---------------------------------------------------------------- FP8 expert weights

def test_e4m3_value_set():
    v = oracle.model.e4m3_values()
    assert v.size == 127 and v[0] == 0.0 and v[-1] == 448.0
    assert v[1] == 2.0 ** -9 and v[8] == 2.0 ** -6            # smallest subnormal, smallest normal
    assert np.all(np.diff(v) > 0)
    # one binade holds 8 values, equally spaced by a 1/8 of its lower end
    b = v[(v >= 1.0) & (v < 2.0)]
    assert np.allclose(b, 1.0 + np.arange(8) / 8.0)


def test_e4m3_rounding_ties_and_torch():
    import torch
    cases = {0.53125: 0.5,            # halfway between 0.5 (code 48) and 0.5625 (49): even code
             0.59375: 0.625,          # halfway between 0.5625 (49) and 0.625 (50)
             -0.59375: -0.625,
             3 * 2.0 ** -10: 2.0 ** -8,   # subnormal tie between codes 1 and 2
             440.0: 448.0, 0.0: 0.0, 17.0: 16.0, 17.5: 18.0}
    got = oracle.model.e4m3_round(np.array(list(cases)))
    assert np.array_equal(got, np.array(list(cases.values())))
    x = np.concatenate([uniform_f32(11, 1, 20000, -448, 448), uniform_f32(11, 2, 20000, -0.05, 0.05)])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.model.e4m3_round(x.astype(np.float64)), ref)


def test_fp8_block_scales_and_round_trip():
    om = oracle.model
    # 200 x 300: tiles of 128 x 128 with a 72-row and a 44-column edge
    w = rnd((200, 300), 40, scale=0.05)
    w[130:140, 10] = 3.0                  # one tile with a large entry
    ex = om.fp8_block_exponents(w)
    assert ex.shape == (2, 3)
    for bi in range(2):
        for bj in range(3):
            t = w[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
            amax = np.abs(t).max()
            # the least power of two that brings the tile's largest entry within 448
            assert 224.0 < amax / 2.0 ** ex[bi, bj] <= 448.0
    assert ex[1, 0] > ex[0, 0]            # the large entry sets only its own tile's scale
    d = om.fp8_block_dequant(w)
    s = np.ldexp(1.0, np.repeat(np.repeat(ex, 128, 0), 128, 1)[:200, :300])
    q = d.astype(np.float64) / s
    # the stored values are E4M3 numbers times the tile scale, and bf16-exact
    assert np.array_equal(np.abs(q), om.e4m3_round(np.abs(q)))
    assert np.array_equal(d.astype(np.float64), oracle.bf16(d))
    # round trip: relative error <= 2^-4 in the normal range, absolute <= 2^-10 * s below it
    err = np.abs(d - w)
    normal = np.abs(w) / s >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(w[normal]))
    assert np.all(err[~normal] <= 2.0 ** -10 * s[~normal])
    # a tile whose entries are E4M3 numbers times a power of two is held exactly
    exact = np.ldexp(om.e4m3_values()[80:120], -12)
    assert np.array_equal(om.fp8_block_dequant(exact[None, :]).astype(np.float64), exact[None, :])
    assert np.all(om.fp8_block_dequant(np.zeros((4, 4))) == 0.0)


def test_fp8_expert_model_runs_on_the_dequantised_experts():
    cfg = MICRO
    W = gen_weights(cfg)
    m8 = OracleModel(cfg, W, expert_fp8=True)
    m = OracleModel(cfg, W)
    wg = W["layers.0.experts.1.wg"]
    assert np.array_equal(m8.layers[0]["experts"][1][0], oracle.model.fp8_block_dequant(wg))
    assert np.array_equal(m8.layers[0]["wq"], m.layers[0]["wq"])      # only the experts change
    # the FP8 model's pass equals the bf16 model's pass on weights replaced by their FP8 values
    W2 = dict(W)
    for l in range(cfg.n_layers):
        for e in range(cfg.n_experts):
            for n in ("wg", "wu", "wd"):
                key = f"layers.{l}.experts.{e}.{n}"
                W2[key] = oracle.model.fp8_block_dequant(W[key])
    m2 = OracleModel(cfg, W2)
    p = prompt_tokens(cfg.vocab, 2007, 9)
    m8.prefill(0, p)
    m2.prefill(0, p)
    c8, a8 = m8.denoise_pass(0, np.full(cfg.canvas, cfg.mask_id), np.ones(cfg.canvas, bool))
    c2, a2 = m2.denoise_pass(0, np.full(cfg.canvas, cfg.mask_id), np.ones(cfg.canvas, bool))
    assert np.array_equal(c8, c2) and np.array_equal(a8, a2)
