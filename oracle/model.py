"""Oracle: one masked block-diffusion denoising pass, written out plainly (TEST INFRASTRUCTURE).

Only tests/, the smoke check and the benchmark's CPU-baseline leg use this module.

What the pages fix (page titles abbreviated as "Distributed" = "Diffusion LLMs are
not a good fit for distributed inference", "DiffusionGemma" = "DiffusionGemma: 4x
Faster Text Generation via Parallel Diffusion", "What changes" = "Diffusion LLMs:
what changes when you stop generating one token at a time"):

* generation starts from an all-[MASK] block and repeatedly commits the positions
  the model is most confident about until none is masked (What changes, section 2,
  "Reverse (generation) process");
* attention within the block is bidirectional (What changes, section 2, property 1;
  DiffusionGemma, "Bi-directional Attention");
* several positions may be committed per pass (What changes, section 2, property 2);
* block decoding: a 256-token canvas is denoised in parallel, finished canvases are
  appended to the KV cache, prefill is causal and denoising bidirectional (What
  changes, section 4.2 "Block decoding"; section 4.1 Block Diffusion);
* at most 48 denoising steps, about 12 with adaptive stopping (What changes,
  section 4.2 "Few steps"; Distributed, canvas paragraph);
* commit by confidence threshold (What changes, section 5 "Quality vs steps");
* mask-to-token decoding: committed tokens are not revised (What changes,
  section 4.3, M2T versus T2T);
* a mixture-of-experts backbone (DiffusionGemma, "Memory Optimization"; What
  changes, section 4.2).

Readings where the pages are silent (all listed in the design notes):

1. pre-norm blocks: x += Attn(RMSNorm(x)); x += FFN(RMSNorm(x)); no other extras;
2. RMSNorm with eps 1e-6, gains from the weights (ones);
3. RoPE, theta 1e4, rotate-half pairs (i, i + hd/2), absolute positions: prompt
   0..P-1, canvas P..P+C-1;
4. attention scale 1/sqrt(hd); query head h reads KV head floor(h * Hkv / H);
5. router in fp32 on the un-rounded normalised activations, no bias; top-k by logit
   with ties to the lower expert index; gate = softmax over the k selected logits;
   expert = Wd (silu(Wg y) * (Wu y)); dense FFN = the same with one expert, gate 1;
6. append = one more bidirectional pass over the finished canvas, whose K/V go to
   the cache;
7. [MASK] = vocab - 1, excluded from argmax and from the softmax sum;
8. confidence = max softmax probability = 1 / sum_v exp(l_v - max); argmax ties go to
   the lowest token id;
9. commit: top-k: the min(k, R) most confident masked positions, ties to the lower
   position; threshold: every masked position with conf > tau, and at least
   n_min = max(1, ceil(R / (S_max - s))) of the most confident ones so that the
   canvas completes within the step budget;
10. precision: the task fixes bf16 operands with fp32 accumulation. The oracle
   applies that rounding to the operands the model hands from one operation to the
   next as data: the weights (the tiny model's fp32 weights enter every product as
   their bf16 roundings) and the attention operands Q, K and V, rounded after RoPE (K
   and V also stay in the KV cache from pass to pass). The operands formed inside an
   operation from fp32 arithmetic (normalised activations, softmax probabilities,
   attention output, SwiGLU output) are kept exact here; the kernels carry them as a
   bf16 (hi, lo) pair, and the QKV projection's input as three bf16 terms, more
   precisely than bf16 operands. Residual stream, router and
   softmax statistics are fp64; router and LM-head logits are rounded to fp32 before
   the top-k / argmax decision, and conf to fp32 before commit ranking;
11. token-to-token editing (What changes, section 4.3, LLaDA2.1: the model may revise
   tokens it already wrote; the pages give no rule, so the plainest one that mirrors
   the threshold commit): with T2T on, a position committed before the pass is
   re-written to the pass's argmax when that token differs from its own and the pass's
   confidence there is above edit_tau; a re-written position stays committed, and the
   masked count is the commit's alone;
12. approximate append (What changes, section 5 "KV caching": Fast-dLLM's
   training-free, block-wise approximate cache): the finished canvas's K/V are taken
   from its last denoising pass, computed while the positions that pass committed
   were still [MASK], instead of from one more pass over the finished canvas;
13. FP8 expert weights (What changes, section 4.2 "Speed": the measured setting runs
   FP8; DiffusionGemma names NVFP4 as the next step): optionally, the expert matrices
   Wg, Wu, Wd are held as FP8 E4M3 with one power-of-two scale 2^e per 128 x 128 tile
   of each matrix, e the least integer with the tile's max |w| <= 448 * 2^e, values
   rounded to nearest (ties to even); the pass then runs on those values exactly as on
   bf16 weights (they are bf16-exact).

Parity pins (tests/test_oracle_pins.py), one or more per function: RMSNorm against
closed forms (constant and +-a rows, a hand-worked row, scale invariance); bf16
rounding against its ties-to-even cases, subnormals and torch's conversion;
attention against brute force and closed forms; RoPE against a hand-worked pairing
case and relative-position invariance; the SwiGLU expert against a closed form at
sigmoid(ln 3) = 3/4; MoE top-k against brute force over all subsets and the k = E
reduction; LM-head confidence against a zero-gain closed form and log-sum-exp; commit
schedule, strict threshold, T2T edit rule and sampler invariants; the KV-cache pass
against an uncached block-causal sequence forward; the approximate append against the
last pass's own K/V and the exact append at a canvas without a final commit; FP8 E4M3
rounding against the format's value set, its ties and torch's float8_e4m3fn, and the
tile scales against their round trip. tests/test_oracle_mutations.py plants a plausible
mistake in each function in turn and checks that a pin fails. Values produced for random
weights beyond those properties are "parity unpinned": no page prints a worked example.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional

import numpy as np


# --------------------------------------------------------------------------------------
# precision helpers

def bf16(x) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as float64."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    r = ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def bf16_store(w) -> np.ndarray:
    """A weight matrix as its bf16 values, kept in float32 (exact); matmuls upcast to fp64."""
    w = np.asarray(w, dtype=np.float32)
    u = w.view(np.uint32)
    if not np.any(u & np.uint32(0xFFFF)):
        return w                      # already bf16-exact: no copy
    return bf16(w).astype(np.float32)


_bf16_store = bf16_store


# --------------------------------------------------------------------------------------
# FP8 expert weights (reading 13)

def e4m3_values() -> np.ndarray:
    """The non-negative finite values of FP8 E4M3 in code order: 1 sign bit, 4 exponent
    bits with bias 7, 3 mantissa bits, no infinities, code 0x7F is NaN. Code c = 8 e + m
    is m / 8 * 2^-6 for e = 0 (subnormal) and (1 + m / 8) * 2^(e - 7) otherwise; the
    largest finite value is 448."""
    vals = []
    for code in range(127):
        e, m = code >> 3, code & 7
        vals.append(m / 8.0 * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals)


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value to x (|x| <= 448), ties to the even code, sign kept."""
    v = e4m3_values()
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    i = np.clip(np.searchsorted(v, a), 1, v.size - 1)      # v[i - 1] < a <= v[i]
    lo, hi = v[i - 1], v[i]
    up = (hi - a < a - lo) | ((hi - a == a - lo) & (i % 2 == 0))
    return np.sign(x) * np.where(up, hi, lo)


def fp8_block_exponents(w: np.ndarray, block: int = 128) -> np.ndarray:
    """Per block x block tile of w (edge tiles smaller): the least integer e with
    max|w| <= 448 * 2^e over the tile (0 for an all-zero tile)."""
    w = np.asarray(w, dtype=np.float64)
    R, Cn = w.shape
    ex = np.zeros(((R + block - 1) // block, (Cn + block - 1) // block), dtype=np.int64)
    for bi in range(ex.shape[0]):
        for bj in range(ex.shape[1]):
            amax = float(np.max(np.abs(w[bi * block:(bi + 1) * block, bj * block:(bj + 1) * block])))
            if amax == 0.0:
                continue
            e = int(math.ceil(math.log2(amax / 448.0)))
            while amax > math.ldexp(448.0, e):
                e += 1
            while amax <= math.ldexp(448.0, e - 1):
                e -= 1
            ex[bi, bj] = e
    return ex


def fp8_block_dequant(w: np.ndarray, block: int = 128) -> np.ndarray:
    """The values an FP8 E4M3 copy of w holds with one power-of-two scale 2^e per
    block x block tile (e from fp8_block_exponents): q = e4m3_round(w / 2^e), returned
    as q * 2^e in float32 (exact: 4 significant bits times a power of two)."""
    w = np.asarray(w, dtype=np.float64)
    ex = fp8_block_exponents(w, block)
    s = np.repeat(np.repeat(np.ldexp(1.0, ex), block, axis=0), block, axis=1)[:w.shape[0], :w.shape[1]]
    return (e4m3_round(w / s) * s).astype(np.float32)


# --------------------------------------------------------------------------------------
# layer pieces

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) * g over the last axis (reading 2)."""
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * np.asarray(g, dtype=np.float64)


def rope_cos_sin(positions: np.ndarray, head_dim: int, theta: float):
    """cos/sin of pos * theta^(-2i/hd), i < hd/2 (reading 3)."""
    half = head_dim // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / head_dim)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE on x [T][heads][hd] with cos/sin [T][hd/2]."""
    half = x.shape[-1] // 2
    a, b = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
              allowed: Optional[np.ndarray] = None) -> np.ndarray:
    """softmax(q k^T / sqrt(hd)) v per query head; GQA by floor(h * Hkv / H) (reading 4).

    q [Tq][H][hd], k/v [Tk][Hkv][hd]; allowed [Tq][Tk] (None = every key visible,
    the bidirectional canvas case). Three-pass softmax: max, sum of exponentials,
    normalise.
    """
    Tq, H, hd = q.shape
    Hkv = k.shape[1]
    out = np.zeros((Tq, H, v.shape[2]), dtype=np.float64)
    scale = 1.0 / math.sqrt(hd)
    for h in range(H):
        g = (h * Hkv) // H
        s = (q[:, h, :] @ k[:, g, :].T) * scale
        if allowed is not None:
            s = np.where(allowed, s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        e = np.exp(s - m)
        z = np.sum(e, axis=1, keepdims=True)
        out[:, h, :] = (e / z) @ v[:, g, :]
    return out


def router_topk(y: np.ndarray, wr: np.ndarray, k: int):
    """Router logits (fp32 decision), top-k experts and their gates (reading 5).

    y [T][d] normalised activations (not rounded to bf16), wr [E][d].
    Returns logits fp32-valued [T][E], idx [T][k] (descending logit, ties to the
    lower expert), gates [T][k] = softmax of the selected logits.
    """
    logits = f32(np.asarray(y, np.float64) @ np.asarray(wr, np.float64).T)
    T, E = logits.shape
    # stable sort on -logit keeps the lower index first among equal logits
    order = np.argsort(-logits, axis=1, kind="stable")
    idx = order[:, :k]
    sel = np.take_along_axis(logits, idx, axis=1)
    ex = np.exp(sel - sel[:, :1])
    gates = ex / np.sum(ex, axis=1, keepdims=True)
    return logits, idx.astype(np.int64), gates


def swiglu_expert(yb: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """Wd (silu(Wg y) * (Wu y)) in fp64."""
    g = yb @ np.asarray(wg, np.float64).T
    u = yb @ np.asarray(wu, np.float64).T
    h = g / (1.0 + np.exp(-g)) * u
    return h @ np.asarray(wd, np.float64).T


def moe_ffn(y: np.ndarray, experts, wr: Optional[np.ndarray], k: int):
    """Mixture-of-experts FFN: sum_j gate_j * expert_{idx_j}(y).

    experts: list of (wg, wu, wd); wr None means the dense FFN (one expert, gate 1).
    Returns (delta [T][d], logits or None, idx [T][k], gates [T][k]).
    """
    T = y.shape[0]
    yb = np.asarray(y, dtype=np.float64)
    if wr is None:
        logits = None
        idx = np.zeros((T, 1), dtype=np.int64)
        gates = np.ones((T, 1), dtype=np.float64)
    else:
        logits, idx, gates = router_topk(y, wr, k)
    out = np.zeros((T, experts[0][2].shape[0]), dtype=np.float64)
    for e in range(len(experts)):
        tok, slot = np.nonzero(idx == e)
        if tok.size == 0:
            continue
        o = swiglu_expert(yb[tok], *experts[e])
        np.add.at(out, tok, gates[tok, slot][:, None] * o)
    return out, logits, idx, gates


def lm_head_conf(x: np.ndarray, final_norm: np.ndarray, head: np.ndarray, mask_id: int,
                 eps: float, return_logits: bool = False):
    """Per row: argmax token and conf = max softmax probability, [MASK] excluded (readings 7, 8)."""
    yb = rmsnorm(x, final_norm, eps)
    logits = f32(yb @ np.asarray(head, np.float64).T)
    logits[:, mask_id] = -np.inf
    m = np.max(logits, axis=1)
    arg = np.argmax(logits, axis=1)          # first maximum = lowest token id
    z = np.sum(np.exp(logits - m[:, None]), axis=1)
    conf = np.asarray(1.0 / z, dtype=np.float32)
    if return_logits:
        return conf, arg.astype(np.int64), logits
    return conf, arg.astype(np.int64)


# --------------------------------------------------------------------------------------
# sampler (commit)

@dataclass(frozen=True)
class Policy:
    kind: str = "topk"       # "topk" or "threshold"
    k: int = 1
    tau: float = 0.9
    floor: bool = True
    t2t: bool = False        # token-to-token editing of committed positions (reading 11)
    edit_tau: float = 0.9    # a committed token is re-written when the pass's conf exceeds it


def commit_count(R: int, n_above: int, policy: Policy, step: int, s_max: int) -> int:
    """How many masked positions step `step` commits (reading 9)."""
    if policy.kind == "topk":
        n = policy.k
    else:
        n = n_above
        if policy.floor:
            left = s_max - step
            n_min = R if left <= 0 else max(1, -(-R // left))
            n = max(n, n_min)
    return max(0, min(n, R))


def commit_select(conf: np.ndarray, mask: np.ndarray, policy: Policy, step: int,
                  s_max: int) -> np.ndarray:
    """Boolean [C]: the positions committed this step.

    The n most confident masked positions (fp32 conf, ties to the lower position),
    n from commit_count; for the threshold policy every masked position above tau
    is among them.
    """
    conf32 = np.asarray(conf, dtype=np.float32)
    masked = np.nonzero(np.asarray(mask, dtype=bool))[0]
    R = masked.size
    n_above = int(np.sum(conf32[masked] > np.float32(policy.tau))) if policy.kind != "topk" else 0
    n = commit_count(R, n_above, policy, step, s_max)
    order = masked[np.lexsort((masked, -conf32[masked].astype(np.float64)))]
    sel = np.zeros(np.asarray(mask).shape[0], dtype=bool)
    sel[order[:n]] = True
    return sel


def edit_select(conf: np.ndarray, argmax: np.ndarray, canvas: np.ndarray, mask: np.ndarray,
                policy: Policy) -> np.ndarray:
    """Boolean [C]: the committed positions this pass re-writes (T2T, reading 11).

    A position committed before the pass is re-written to the pass's argmax when that
    token differs from the one it holds and the pass's confidence there (fp32) is above
    edit_tau. Masked positions are the commit's business, never the edit's.
    """
    if not policy.t2t:
        return np.zeros(np.asarray(mask).shape[0], dtype=bool)
    conf32 = np.asarray(conf, dtype=np.float32)
    committed = ~np.asarray(mask, dtype=bool)
    differs = np.asarray(argmax) != np.asarray(canvas)
    return committed & differs & (conf32 > np.float32(policy.edit_tau))


# --------------------------------------------------------------------------------------
# the model

class _Request:
    def __init__(self, n_layers: int):
        self.k = [None] * n_layers      # per layer [P][Hkv][hd] (bf16 values)
        self.v = [None] * n_layers
        self.P = 0
        self.last_k = None              # K/V of the request's last canvas pass (per layer)
        self.last_v = None


class OracleModel:
    """The denoiser over named weights (float32 arrays, e.g. from synth.gen_weights)."""

    def __init__(self, cfg, weights: Dict[str, np.ndarray], f64_matrices: bool = False,
                 expert_fp8: bool = False):
        """f64_matrices keeps every matrix as float64 (the same bf16 values) instead of
        float32, so that the products do not convert their operands on every call: faster
        for repeated passes, twice the memory, identical results. expert_fp8 replaces the
        expert matrices (Wg, Wu, Wd of every MoE expert) by their FP8 block-scaled values
        (reading 13); everything else is unchanged."""
        self.cfg = cfg
        c = cfg
        # every matrix enters its products as a bf16 operand (reading 10); norm gains
        # stay as given
        if f64_matrices:
            bf16_store = lambda w: _bf16_store(w).astype(np.float64)   # noqa: E731
        else:
            bf16_store = _bf16_store
        self.emb = bf16_store(weights["emb"])
        self.layers = []
        for l in range(c.n_layers):
            p = f"layers.{l}."
            lw = {
                "attn_norm": np.asarray(weights[p + "attn_norm"], np.float64),
                "wq": bf16_store(weights[p + "wq"]),
                "wk": bf16_store(weights[p + "wk"]),
                "wv": bf16_store(weights[p + "wv"]),
                "wo": bf16_store(weights[p + "wo"]),
                "ffn_norm": np.asarray(weights[p + "ffn_norm"], np.float64),
            }
            if c.dense:
                lw["wr"] = None
                lw["experts"] = [(bf16_store(weights[p + "wg"]), bf16_store(weights[p + "wu"]),
                                  bf16_store(weights[p + "wd"]))]
            else:
                lw["wr"] = bf16_store(weights[p + "wr"])
                ex = (lambda w: bf16_store(fp8_block_dequant(_bf16_store(w)))) if expert_fp8 else bf16_store
                lw["experts"] = [(ex(weights[p + f"experts.{e}.wg"]),
                                  ex(weights[p + f"experts.{e}.wu"]),
                                  ex(weights[p + f"experts.{e}.wd"]))
                                 for e in range(c.n_experts)]
            self.layers.append(lw)
        self.final_norm = np.asarray(weights["final_norm"], np.float64)
        self.head = bf16_store(weights["head"])
        self.requests: Dict[int, _Request] = {}

    # ---- one transformer layer -------------------------------------------------------
    def layer(self, l: int, x: np.ndarray, positions: np.ndarray, k_prev, v_prev,
              allowed: Optional[np.ndarray], rec: Optional[dict] = None):
        """x [T][d] -> x', plus the layer's new K/V [T][Hkv][hd] (bf16 values)."""
        c, lw = self.cfg, self.layers[l]
        T = x.shape[0]
        y = rmsnorm(x, lw["attn_norm"], c.rms_eps)
        q = (y @ lw["wq"].T).reshape(T, c.n_heads, c.head_dim)
        k = (y @ lw["wk"].T).reshape(T, c.n_kv_heads, c.head_dim)
        v = (y @ lw["wv"].T).reshape(T, c.n_kv_heads, c.head_dim)
        cos, sin = rope_cos_sin(positions, c.head_dim, c.rope_theta)
        q = bf16(apply_rope(q, cos, sin))      # the attention operands are bf16 (reading 10)
        k = bf16(apply_rope(k, cos, sin))
        v = bf16(v)
        if k_prev is not None and k_prev.shape[0] > 0:
            kk = np.concatenate([k_prev, k], axis=0)
            vv = np.concatenate([v_prev, v], axis=0)
        else:
            kk, vv = k, v
        o = attention(q, kk, vv, allowed).reshape(T, c.q_dim)
        x = x + o @ lw["wo"].T
        y2 = rmsnorm(x, lw["ffn_norm"], c.rms_eps)
        delta, logits, idx, gates = moe_ffn(y2, lw["experts"], lw["wr"], c.top_k)
        x = x + delta
        if rec is not None:
            rec.setdefault("router_logits", []).append(logits)
            rec.setdefault("topk_idx", []).append(idx)
            rec.setdefault("gates", []).append(gates)
            rec.setdefault("x", []).append(x.copy())
        return x, k, v

    # ---- request lifecycle ------------------------------------------------------------
    def reset(self, req: int = 0):
        self.requests[req] = _Request(self.cfg.n_layers)

    def prefill(self, req: int, prompt: np.ndarray, rec: Optional[dict] = None):
        """Causal forward over the prompt; its K/V fill the cache at 0..n-1."""
        c = self.cfg
        prompt = np.asarray(prompt, dtype=np.int64)
        n = prompt.size
        st = _Request(c.n_layers)
        x = self.emb[prompt].astype(np.float64)
        pos = np.arange(n)
        allowed = pos[None, :] <= pos[:, None]
        for l in range(c.n_layers):
            x, k, v = self.layer(l, x, pos, None, None, allowed, rec)
            st.k[l], st.v[l] = k, v
        st.P = n
        self.requests[req] = st

    def _canvas_forward(self, req: int, canvas: np.ndarray, mask: np.ndarray,
                        rec: Optional[dict] = None):
        c = self.cfg
        st = self.requests[req]
        tokens = np.where(np.asarray(mask, bool), c.mask_id, np.asarray(canvas, np.int64))
        x = self.emb[tokens].astype(np.float64)
        C = tokens.size
        pos = st.P + np.arange(C)
        new_k, new_v = [], []
        for l in range(c.n_layers):
            x, k, v = self.layer(l, x, pos, st.k[l], st.v[l], None, rec)
            new_k.append(k)
            new_v.append(v)
        return x, new_k, new_v

    def denoise_pass(self, req: int, canvas: np.ndarray, mask: np.ndarray,
                     rec: Optional[dict] = None):
        """One pass: conf [C] (fp32) and argmax [C] for every canvas position."""
        x, ks, vs = self._canvas_forward(req, canvas, mask, rec)
        st = self.requests[req]
        st.last_k, st.last_v = ks, vs
        out = lm_head_conf(x, self.final_norm, self.head, self.cfg.mask_id, self.cfg.rms_eps,
                           return_logits=rec is not None)
        if rec is not None:
            conf, arg, logits = out
            top2 = np.partition(logits, -2, axis=1)[:, -2:]      # the two largest, either order
            rec["logit_margin"] = np.abs(top2[:, 1] - top2[:, 0])
            rec["final_x"] = x
            return conf, arg
        return out

    def append(self, req: int, canvas: np.ndarray, rec: Optional[dict] = None):
        """Bidirectional pass over the finished canvas; its K/V join the cache (reading 6).

        rec, if given, receives the pass's per-layer records (as in denoise_pass).
        """
        st = self.requests[req]
        C = np.asarray(canvas).size
        _, ks, vs = self._canvas_forward(req, canvas, np.zeros(C, dtype=bool), rec)
        for l in range(self.cfg.n_layers):
            st.k[l] = np.concatenate([st.k[l], ks[l]], axis=0) if st.k[l] is not None else ks[l]
            st.v[l] = np.concatenate([st.v[l], vs[l]], axis=0) if st.v[l] is not None else vs[l]
        st.P += C

    def append_approx(self, req: int):
        """Approximate append (Fast-dLLM-style reuse, reading 12): the finished canvas's
        K/V are those its last denoising pass computed, taken as they are; no extra pass."""
        st = self.requests[req]
        if st.last_k is None:
            raise ValueError("no canvas pass to reuse")
        C = st.last_k[0].shape[0]
        for l in range(self.cfg.n_layers):
            st.k[l] = np.concatenate([st.k[l], st.last_k[l]], axis=0) if st.k[l] is not None else st.last_k[l]
            st.v[l] = np.concatenate([st.v[l], st.last_v[l]], axis=0) if st.v[l] is not None else st.last_v[l]
        st.P += C
        st.last_k = st.last_v = None

    def generate_block(self, req: int, policy: Policy, s_max: int, trace: bool = False):
        """Denoise one all-[MASK] canvas until no position is masked or S_max passes ran.

        Returns (canvas, steps, trace list). Each trace entry holds the pass's input
        canvas/mask, conf, argmax, the commit set, the edit set (T2T) and the masked
        count after it.
        """
        c = self.cfg
        C = c.canvas
        canvas = np.full(C, c.mask_id, dtype=np.int64)
        mask = np.ones(C, dtype=bool)
        steps, tr = 0, []
        for s in range(s_max):
            if not mask.any():
                break
            rec = {} if trace else None
            conf, arg = self.denoise_pass(req, canvas, mask, rec)
            sel = commit_select(conf, mask, policy, s, s_max)
            edit = edit_select(conf, arg, canvas, mask, policy)
            if trace:
                tr.append(dict(step=s, canvas=canvas.copy(), mask=mask.copy(), conf=conf,
                               argmax=arg, commit=sel.copy(), edit=edit.copy(), rec=rec))
            canvas = np.where(sel | edit, arg, canvas)
            mask = mask & ~sel
            steps += 1
            if trace:
                tr[-1]["remaining"] = int(mask.sum())
        return canvas, steps, tr


def sequence_forward(model: OracleModel, tokens: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    """Uncached forward over a whole sequence with an explicit attention mask.

    Positions are 0..n-1. Used only to pin the cached path: a canvas pass over a
    cached prefix must equal this forward with a block-causal mask.
    """
    c = model.cfg
    tokens = np.asarray(tokens, dtype=np.int64)
    x = model.emb[tokens].astype(np.float64)
    pos = np.arange(tokens.size)
    for l in range(c.n_layers):
        x, _, _ = model.layer(l, x, pos, None, None, allowed)
    return x
