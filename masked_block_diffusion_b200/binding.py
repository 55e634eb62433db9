"""ctypes binding of libdllm.so: the C ABI of include/dllm.h with the same names.

Argument marshalling only: every step of the denoising pass runs in the library's
CUDA kernels. Loading fails loudly when the library has not been built; there is no
fallback path.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdllm.so")

DLLM_OK = 0
DLLM_E_INVAL = -1
DLLM_E_OOM = -2
DLLM_E_CUDA = -3
DLLM_E_CTX_FULL = -4
DLLM_E_BUDGET = -5
DLLM_E_STATE = -6
DLLM_E_TIMEOUT = -7
ERROR_NAMES = {0: "DLLM_OK", -1: "DLLM_E_INVAL", -2: "DLLM_E_OOM", -3: "DLLM_E_CUDA", -4: "DLLM_E_CTX_FULL",
               -5: "DLLM_E_BUDGET", -6: "DLLM_E_STATE", -7: "DLLM_E_TIMEOUT"}

DLLM_WEIGHTS_F32 = 0
DLLM_WEIGHTS_BF16 = 1
DLLM_EXPERTS_BF16 = 0
DLLM_EXPERTS_FP8 = 1
DLLM_POLICY_TOPK = 0
DLLM_POLICY_THRESHOLD = 1

# every symbol include/dllm.h declares
EXPORTS = [
    "dllm_create", "dllm_prefill", "dllm_denoise_step", "dllm_generate_block", "dllm_append_kv",
    "dllm_generate", "dllm_reset", "dllm_prefix_len", "dllm_check", "dllm_launch_count",
    "dllm_set_debug", "dllm_debug_read", "dllm_debug_force_routing", "dllm_last_error", "dllm_destroy",
    "dllm_op_gemm_bf16", "dllm_op_lm_head_conf", "dllm_op_lm_head_conf_noalloc", "dllm_set_timing",
    "dllm_timing_read", "dllm_set_wait_limit", "dllm_append_kv_approx", "dllm_op_quantize_fp8",
]
DLLM_TIMING_GATE_UP = 0
DLLM_TIMING_DOWN = 1
DLLM_TIMING_ATTN = 2
DLLM_TIMING_QKV = 3
DLLM_TIMING_OPROJ = 4
DLLM_TIMING_ROUTE = 5
DLLM_TIMING_NORM = 6
DLLM_TIMING_HEAD = 7
DLLM_TIMING_KINDS = 8
DLLM_TIMING_STRIDE_SHIFT = 16   # bits 16..23 of the timing mask: bracket every S-th layer only
TIMING_NAMES = ["gate_up_gemm", "down_gemm", "attention", "qkv_gemm", "o_gemm", "routing", "norm_combine",
                "lm_head_commit"]


class dllm_config(ctypes.Structure):
    _fields_ = [
        ("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("n_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("n_experts", ctypes.c_int),
        ("top_k", ctypes.c_int), ("ffn_dim", ctypes.c_int), ("vocab", ctypes.c_int),
        ("mask_id", ctypes.c_int), ("canvas", ctypes.c_int), ("max_ctx", ctypes.c_int),
        ("max_batch", ctypes.c_int), ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
        ("weight_dtype", ctypes.c_int), ("expert_format", ctypes.c_int),
    ]


class dllm_policy(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("k", ctypes.c_int), ("tau", ctypes.c_float), ("floor", ctypes.c_int),
                ("t2t", ctypes.c_int), ("edit_tau", ctypes.c_float)]


class DllmError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str = ""):
        super().__init__(f"{where} failed: {ERROR_NAMES.get(code, code)} {msg}".strip())
        self.code = code


_lib: Optional[ctypes.CDLL] = None

_vp = ctypes.c_void_p
_i = ctypes.c_int


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libdllm.so (raises if it is missing: build it with masked_block_diffusion_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; run `python -m masked_block_diffusion_b200.build` first")
    lib = ctypes.CDLL(path)
    sig = {
        "dllm_create": (_i, [ctypes.POINTER(dllm_config), _vp, ctypes.c_size_t, _i, _vp, ctypes.POINTER(_vp)]),
        "dllm_prefill": (_i, [_vp, _i, _vp, _i]),
        "dllm_denoise_step": (_i, [_vp, _i, _vp, _vp, ctypes.POINTER(dllm_policy), _i, _i, _vp, _vp, _vp]),
        "dllm_generate_block": (_i, [_vp, _i, _i, ctypes.POINTER(dllm_policy), _vp, _vp]),
        "dllm_append_kv": (_i, [_vp, _i, _vp]),
        "dllm_generate": (_i, [_vp, _i, _vp, _i, _i, _i, ctypes.POINTER(dllm_policy), _vp, _vp]),
        "dllm_reset": (_i, [_vp, _i]),
        "dllm_prefix_len": (_i, [_vp, _i]),
        "dllm_check": (_i, [_vp]),
        "dllm_launch_count": (ctypes.c_longlong, [_vp]),
        "dllm_set_debug": (_i, [_vp, _i]),
        "dllm_debug_read": (_i, [_vp, _i, _i, _vp, ctypes.c_size_t]),
        "dllm_debug_force_routing": (_i, [_vp, _vp, _i]),
        "dllm_last_error": (ctypes.c_char_p, [_vp]),
        "dllm_destroy": (None, [_vp]),
        "dllm_op_gemm_bf16": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
        "dllm_op_lm_head_conf": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
        "dllm_op_lm_head_conf_noalloc": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
        "dllm_set_timing": (_i, [_vp, _i]),
        "dllm_timing_read": (_i, [_vp, _vp, _vp, _vp, _i]),
        "dllm_set_wait_limit": (_i, [_vp, ctypes.c_longlong]),
        "dllm_append_kv_approx": (_i, [_vp, _i]),
        "dllm_op_quantize_fp8": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def make_config(model, max_ctx: int, max_batch: int, expert_fp8: bool = False) -> dllm_config:
    """dllm_config from a model description with the fields of synth.ModelConfig."""
    return dllm_config(
        expert_format=DLLM_EXPERTS_FP8 if expert_fp8 else DLLM_EXPERTS_BF16,
        n_layers=model.n_layers, d_model=model.d_model, n_heads=model.n_heads,
        n_kv_heads=model.n_kv_heads, head_dim=model.head_dim, n_experts=model.n_experts,
        top_k=model.top_k, ffn_dim=model.ffn_dim, vocab=model.vocab, mask_id=model.vocab - 1,
        canvas=model.canvas, max_ctx=max_ctx, max_batch=max_batch, rms_eps=model.rms_eps,
        rope_theta=model.rope_theta,
        weight_dtype=DLLM_WEIGHTS_F32 if model.weight_dtype == "f32" else DLLM_WEIGHTS_BF16)


def make_policy(kind: str, k: int = 0, tau: float = 0.9, floor: bool = True, t2t: bool = False,
                edit_tau: float = 0.9) -> dllm_policy:
    return dllm_policy(kind=DLLM_POLICY_TOPK if kind == "topk" else DLLM_POLICY_THRESHOLD, k=int(k),
                       tau=float(tau), floor=1 if floor else 0, t2t=1 if t2t else 0, edit_tau=float(edit_tau))


def _check(code: int, where: str, handle=None):
    if code != DLLM_OK:
        msg = ""
        if handle:
            m = load().dllm_last_error(handle)
            msg = m.decode() if m else ""
        raise DllmError(code, where, msg)


# ---------------------------------------------------------------- same-name wrappers

def dllm_create(cfg: dllm_config, weights_ptr: int, weight_bytes: int, weights_on_device: bool,
                stream_ptr: int):
    h = _vp()
    _check(load().dllm_create(ctypes.byref(cfg), _vp(weights_ptr), weight_bytes, 1 if weights_on_device else 0,
                              _vp(stream_ptr), ctypes.byref(h)), "dllm_create")
    return h


def dllm_prefill(h, req: int, prompt_ptr: int, n: int):
    _check(load().dllm_prefill(h, req, _vp(prompt_ptr), n), "dllm_prefill", h)


def dllm_denoise_step(h, req_count, canvas_ptr, mask_ptr, policy: dllm_policy, step, max_steps,
                      conf_ptr=0, argmax_ptr=0, remaining_ptr=0):
    _check(load().dllm_denoise_step(h, req_count, _vp(canvas_ptr), _vp(mask_ptr), ctypes.byref(policy), step,
                                    max_steps, _vp(conf_ptr), _vp(argmax_ptr), _vp(remaining_ptr)),
           "dllm_denoise_step", h)


def dllm_generate_block(h, req_count, max_steps, policy: dllm_policy, canvas_ptr=0):
    steps = (ctypes.c_int * req_count)()
    code = load().dllm_generate_block(h, req_count, max_steps, ctypes.byref(policy), _vp(canvas_ptr), steps)
    return code, list(steps)


def dllm_append_kv(h, req_count, canvas_ptr=0):
    _check(load().dllm_append_kv(h, req_count, _vp(canvas_ptr)), "dllm_append_kv", h)


def dllm_append_kv_approx(h, req_count):
    _check(load().dllm_append_kv_approx(h, req_count), "dllm_append_kv_approx", h)


def dllm_generate(h, req_count, prompts_host_ptr, n_prompt, n_canvases, max_steps, policy: dllm_policy,
                  tokens_host_ptr, steps_host_ptr=0):
    _check(load().dllm_generate(h, req_count, _vp(prompts_host_ptr), n_prompt, n_canvases, max_steps,
                                ctypes.byref(policy), _vp(tokens_host_ptr), _vp(steps_host_ptr)),
           "dllm_generate", h)


def dllm_reset(h, req):
    _check(load().dllm_reset(h, req), "dllm_reset", h)


def dllm_prefix_len(h, req) -> int:
    return load().dllm_prefix_len(h, req)


def dllm_check(h) -> int:
    return load().dllm_check(h)


def dllm_launch_count(h) -> int:
    return load().dllm_launch_count(h)


def dllm_set_debug(h, on: bool):
    _check(load().dllm_set_debug(h, 1 if on else 0), "dllm_set_debug", h)


def dllm_debug_read(h, what: int, layer: int, dst_ptr: int, nbytes: int):
    _check(load().dllm_debug_read(h, what, layer, _vp(dst_ptr), nbytes), "dllm_debug_read", h)


def dllm_debug_force_routing(h, idx_host_ptr: int, T: int):
    _check(load().dllm_debug_force_routing(h, _vp(idx_host_ptr), T), "dllm_debug_force_routing", h)


def dllm_last_error(h) -> str:
    m = load().dllm_last_error(h)
    return m.decode() if m else ""


def dllm_destroy(h):
    load().dllm_destroy(h)


def dllm_op_gemm_bf16(a_ptr, b_ptr, d_ptr, M, N, K, stream_ptr):
    _check(load().dllm_op_gemm_bf16(_vp(a_ptr), _vp(b_ptr), _vp(d_ptr), M, N, K, _vp(stream_ptr)),
           "dllm_op_gemm_bf16")


def dllm_op_lm_head_conf(y_ptr, head_ptr, T, d, V, mask_id, conf_ptr, argmax_ptr, stream_ptr):
    _check(load().dllm_op_lm_head_conf(_vp(y_ptr), _vp(head_ptr), T, d, V, mask_id, _vp(conf_ptr),
                                       _vp(argmax_ptr), _vp(stream_ptr)), "dllm_op_lm_head_conf")


def dllm_set_timing(h, kinds: int):
    """kinds: bit mask of (1 << DLLM_TIMING_*), optionally | (S << DLLM_TIMING_STRIDE_SHIFT) to time
    every S-th layer only; 0 switches timing off."""
    _check(load().dllm_set_timing(h, int(kinds)), "dllm_set_timing", h)


def dllm_timing_read(h, reset: bool = False):
    ms = (ctypes.c_double * DLLM_TIMING_KINDS)()
    n = (ctypes.c_longlong * DLLM_TIMING_KINDS)()
    b = (ctypes.c_double * DLLM_TIMING_KINDS)()
    _check(load().dllm_timing_read(h, ms, n, b, 1 if reset else 0), "dllm_timing_read", h)
    return list(ms), list(n), list(b)


def dllm_op_lm_head_conf_noalloc(y_ptr, head_ptr, T, d, V, mask_id, conf_ptr, argmax_ptr, stream_ptr):
    """The fused LM head on a fixed in-library scratch array (no device allocation)."""
    _check(load().dllm_op_lm_head_conf_noalloc(_vp(y_ptr), _vp(head_ptr), T, d, V, mask_id, _vp(conf_ptr),
                                               _vp(argmax_ptr), _vp(stream_ptr)), "dllm_op_lm_head_conf_noalloc")


def dllm_set_wait_limit(h, ns: int):
    """Pipeline-wait limit of the kernels on this device in ns (<= 0: the 2 s default)."""
    _check(load().dllm_set_wait_limit(h, int(ns)), "dllm_set_wait_limit", h)


def dllm_op_quantize_fp8(w_ptr, rows, cols, q_ptr, exps_ptr, stream_ptr):
    """FP8 E4M3 codes and per-128x128-tile scale exponents of a bf16 matrix (device buffers)."""
    _check(load().dllm_op_quantize_fp8(_vp(w_ptr), rows, cols, _vp(q_ptr), _vp(exps_ptr), _vp(stream_ptr)),
           "dllm_op_quantize_fp8")
