"""Counter-based, bit-reproducible generators for weights, prompts and test tensors.

Every value is a pure function of (seed, tensor id, element index):

    base  = splitmix64((seed << 32) | tensor_id)
    z_i   = splitmix64(base + i)                      (uint64 arithmetic, wraps)

splitmix64 is the published mixer of Steele, Lea and Flood ("Fast splittable
pseudorandom number generators", OOPSLA 2014): add the golden-ratio increment,
then two xor-shift-multiply rounds and a final xor-shift.

Weights are "N(0, 0.02)" (the workload list). To stay bit-identical between numpy
and the device generator, the normal deviate is an Irwin-Hall sum of the four
16-bit lanes of z_i, an integer:

    n_i = 2 * (u0 + u1 + u2 + u3) - 4 * 65535        (even integer, |n_i| <= 262140)
    w_i = fl32(n_i) * SCALE                          (one correctly rounded fp32 multiply)

with SCALE = 0.02 / sd(n), sd(n) = 2 * sqrt((65536^2 - 1) / 3). bf16 tensors are
w_i rounded to nearest-even bf16. RMSNorm gains are ones.

Prompt tokens are uniform over the vocabulary minus [MASK]: (z_i >> 32) mod (V - 1).
"""

from __future__ import annotations

import math
from typing import Dict, List, NamedTuple

import numpy as np

from .configs import ModelConfig

U64 = np.uint64
GOLDEN = U64(0x9E3779B97F4A7C15)
MIX1 = U64(0xBF58476D1CE4E5B9)
MIX2 = U64(0x94D049BB133111EB)

# fp32 bit pattern of 0.02 / (2 * sqrt((65536^2 - 1) / 3)); the device filler uses the same bits.
SCALE_BITS = 0x348DE3BD
SCALE = np.array([SCALE_BITS], dtype=np.uint32).view(np.float32)[0]
LANE_SUM_OFFSET = 4 * 65535

_CHUNK = 1 << 24


def splitmix64(z: np.ndarray) -> np.ndarray:
    """splitmix64 on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=U64)
    with np.errstate(over="ignore"):
        z = z + GOLDEN
        z = (z ^ (z >> U64(30))) * MIX1
        z = (z ^ (z >> U64(27))) * MIX2
        z = z ^ (z >> U64(31))
    return z


def stream_base(seed: int, tid: int) -> np.uint64:
    key = np.array([((seed & 0xFFFFFFFF) << 32) | (tid & 0xFFFFFFFF)], dtype=U64)
    return splitmix64(key)[0]


def _counter_words(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    base = stream_base(seed, tid)
    idx = np.arange(start, start + count, dtype=U64)
    with np.errstate(over="ignore"):
        return splitmix64(idx + base)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to the nearest bf16 (ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + U64(0x7FFF) + ((u >> U64(16)) & U64(1))) >> U64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_f32(seed: int, tid: int, n: int, start: int = 0) -> np.ndarray:
    """fp32 N(0, 0.02) deviates (Irwin-Hall, see module docstring)."""
    out = np.empty(n, dtype=np.float32)
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        z = _counter_words(seed, tid, start + s, c)
        lanes = ((z & U64(0xFFFF)) + ((z >> U64(16)) & U64(0xFFFF))
                 + ((z >> U64(32)) & U64(0xFFFF)) + (z >> U64(48)))
        ni = 2 * lanes.astype(np.int64) - LANE_SUM_OFFSET
        out[s:s + c] = ni.astype(np.float32) * SCALE
    return out


def uniform_f32(seed: int, tid: int, n: int, lo: float = -1.0, hi: float = 1.0) -> np.ndarray:
    """Uniform test values: 24-bit integer / 2^24 mapped to [lo, hi) (exact in fp64)."""
    z = _counter_words(seed, tid, 0, n)
    u = (z >> U64(40)).astype(np.float64) * (2.0 ** -24)
    return (lo + (hi - lo) * u).astype(np.float32)


def prompt_tokens(vocab: int, seed: int, n: int) -> np.ndarray:
    """n prompt tokens, uniform over [0, vocab - 2] (never [MASK] = vocab - 1)."""
    z = _counter_words(seed, 0, 0, n)
    return ((z >> U64(32)) % U64(vocab - 1)).astype(np.int32)


class TensorSpec(NamedTuple):
    name: str
    shape: tuple
    tid: int
    kind: str            # "normal" or "ones"


def tensor_specs(cfg: ModelConfig) -> List[TensorSpec]:
    """The weight blob's tensors, in blob order; all matrices are row-major [out][in]."""
    d, F = cfg.d_model, cfg.ffn_dim
    specs: List[TensorSpec] = []

    def add(name, shape, kind="normal"):
        specs.append(TensorSpec(name, tuple(shape), len(specs), kind))

    add("emb", (cfg.vocab, d))
    for l in range(cfg.n_layers):
        p = f"layers.{l}."
        add(p + "attn_norm", (d,), "ones")
        add(p + "wq", (cfg.q_dim, d))
        add(p + "wk", (cfg.kv_dim, d))
        add(p + "wv", (cfg.kv_dim, d))
        add(p + "wo", (d, cfg.q_dim))
        add(p + "ffn_norm", (d,), "ones")
        if cfg.dense:
            add(p + "wg", (F, d))
            add(p + "wu", (F, d))
            add(p + "wd", (d, F))
        else:
            add(p + "wr", (cfg.n_experts, d))
            for e in range(cfg.n_experts):
                q = p + f"experts.{e}."
                add(q + "wg", (F, d))
                add(q + "wu", (F, d))
                add(q + "wd", (d, F))
    add("final_norm", (d,), "ones")
    add("head", (cfg.vocab, d))
    return specs


def elem_bytes(cfg: ModelConfig) -> int:
    return 4 if cfg.weight_dtype == "f32" else 2


class BlobEntry(NamedTuple):
    spec: TensorSpec
    offset: int          # bytes from the blob start
    numel: int


def blob_layout(cfg: ModelConfig) -> List[BlobEntry]:
    """Byte offsets of each tensor; every tensor starts on a 256-byte boundary."""
    eb = elem_bytes(cfg)
    out, off = [], 0
    for s in tensor_specs(cfg):
        n = int(np.prod(s.shape))
        out.append(BlobEntry(s, off, n))
        off += n * eb
        off = (off + 255) // 256 * 256
    return out


def blob_bytes(cfg: ModelConfig) -> int:
    last = blob_layout(cfg)[-1]
    return last.offset + last.numel * elem_bytes(cfg)


def gen_tensor(cfg: ModelConfig, spec: TensorSpec, seed: int | None = None) -> np.ndarray:
    """One weight tensor as float32 values (bf16-exact for bf16 configs)."""
    seed = cfg.weight_seed if seed is None else seed
    n = int(np.prod(spec.shape))
    if spec.kind == "ones":
        return np.ones(spec.shape, dtype=np.float32)
    w = normal_f32(seed, spec.tid, n)
    if cfg.weight_dtype == "bf16":
        w = bf16_bits_to_f32(f32_to_bf16_bits(w))
    return w.reshape(spec.shape)


def gen_weights(cfg: ModelConfig, seed: int | None = None, threads: int = 0) -> Dict[str, np.ndarray]:
    """All tensors by name (host memory). threads > 1 generates tensors concurrently
    (numpy releases the GIL inside its array loops); values do not depend on it."""
    specs = tensor_specs(cfg)
    if threads <= 1:
        return {s.name: gen_tensor(cfg, s, seed) for s in specs}
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=threads) as ex:
        arrays = list(ex.map(lambda s: gen_tensor(cfg, s, seed), specs))
    return {s.name: a for s, a in zip(specs, arrays)}


def gen_blob(cfg: ModelConfig, seed: int | None = None) -> np.ndarray:
    """The weight blob as a uint8 host array in the documented order and dtype."""
    buf = np.zeros(blob_bytes(cfg), dtype=np.uint8)
    for ent in blob_layout(cfg):
        w = gen_tensor(cfg, ent.spec, seed).reshape(-1)
        if cfg.weight_dtype == "bf16":
            raw = f32_to_bf16_bits(w).view(np.uint8)
        else:
            raw = w.astype(np.float32).view(np.uint8)
        buf[ent.offset:ent.offset + raw.size] = raw
    return buf


def blob_from_weights(cfg: ModelConfig, weights: Dict[str, np.ndarray]) -> np.ndarray:
    """The blob holding already generated tensors (avoids generating them twice)."""
    buf = np.zeros(blob_bytes(cfg), dtype=np.uint8)
    for ent in blob_layout(cfg):
        w = np.asarray(weights[ent.spec.name], dtype=np.float32).reshape(-1)
        raw = f32_to_bf16_bits(w).view(np.uint8) if cfg.weight_dtype == "bf16" else w.view(np.uint8)
        buf[ent.offset:ent.offset + raw.size] = raw
    return buf
