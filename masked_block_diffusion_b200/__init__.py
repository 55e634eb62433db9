"""B200-native masked block-diffusion denoiser.

The denoising pass, prefill, append and the commit sampler run in libdllm.so
(hand-written sm_100a CUDA kernels behind the C ABI of include/dllm.h). This package
holds the ctypes binding (``binding``) and ``Denoiser``, a thin torch-facing wrapper
that only moves pointers, sizes and streams across the ABI.
"""

from __future__ import annotations

import ctypes

import numpy as np

from . import binding
from .binding import (DllmError, dllm_config, dllm_policy, make_config, make_policy)

__all__ = ["binding", "Denoiser", "DllmError", "dllm_config", "dllm_policy", "make_config", "make_policy"]


class Denoiser:
    """One libdllm handle on its own CUDA stream.

    Torch tensors passed in must live on the handle's device. Calls that return
    tensors synchronise the handle's stream first, so results are ready to use.
    """

    def __init__(self, model, weights, max_ctx: int, max_batch: int = 1, expert_fp8: bool = False):
        import torch
        self.torch = torch
        self.model = model
        self.C = model.canvas
        self.max_batch = max_batch
        self.stream = torch.cuda.Stream()
        self.cfg = make_config(model, max_ctx, max_batch, expert_fp8)
        if isinstance(weights, np.ndarray):
            buf = np.ascontiguousarray(weights)
            ptr, nbytes, on_dev = buf.ctypes.data, buf.nbytes, False
        else:
            torch.cuda.synchronize()
            ptr, nbytes, on_dev = weights.data_ptr(), weights.numel() * weights.element_size(), True
        self.h = binding.dllm_create(self.cfg, ptr, nbytes, on_dev, self.stream.cuda_stream)

    # ---- helpers
    def _sync_in(self):
        self.stream.wait_stream(self.torch.cuda.current_stream())

    def _sync_out(self):
        self.stream.synchronize()

    def close(self):
        if self.h:
            binding.dllm_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- the ABI calls
    def prefill(self, req: int, prompt):
        t = self.torch
        p = t.as_tensor(prompt, dtype=t.int32).to("cuda").contiguous()
        self._sync_in()
        binding.dllm_prefill(self.h, req, p.data_ptr(), p.numel())
        self._sync_out()

    def denoise_step(self, canvas, mask, policy: dllm_policy, step: int, max_steps: int):
        """canvas int32 [B][C], mask uint8 [B][C] (device, updated in place)."""
        t = self.torch
        B = canvas.shape[0]
        conf = t.empty((B, self.C), dtype=t.float32, device="cuda")
        arg = t.empty((B, self.C), dtype=t.int32, device="cuda")
        rem = t.empty((B,), dtype=t.int32, device="cuda")
        self._sync_in()
        binding.dllm_denoise_step(self.h, B, canvas.data_ptr(), mask.data_ptr(), policy, step, max_steps,
                                  conf.data_ptr(), arg.data_ptr(), rem.data_ptr())
        self._sync_out()
        return conf, arg, rem

    def generate_block(self, req_count: int, max_steps: int, policy: dllm_policy):
        t = self.torch
        out = t.empty((req_count, self.C), dtype=t.int32, device="cuda")
        self._sync_in()
        code, steps = binding.dllm_generate_block(self.h, req_count, max_steps, policy, out.data_ptr())
        self._sync_out()
        return code, out, steps

    def append_kv(self, req_count: int, canvas=None):
        self._sync_in()
        binding.dllm_append_kv(self.h, req_count, 0 if canvas is None else canvas.data_ptr())
        self._sync_out()

    def append_kv_approx(self, req_count: int):
        """Keeps the last canvas pass's K/V as the finished canvases' cache entries."""
        self._sync_in()
        binding.dllm_append_kv_approx(self.h, req_count)
        self._sync_out()

    def generate(self, prompts: np.ndarray, n_canvases: int, max_steps: int, policy: dllm_policy):
        """End to end with host buffers: prompts int32 [B][n] -> tokens int32 [B][n_canvases*C]."""
        prompts = np.ascontiguousarray(prompts, dtype=np.int32)
        B, n = prompts.shape
        tokens = np.zeros((B, n_canvases * self.C), dtype=np.int32)
        steps = np.zeros((B * n_canvases,), dtype=np.int32)
        binding.dllm_generate(self.h, B, prompts.ctypes.data, n, n_canvases, max_steps, policy,
                              tokens.ctypes.data, steps.ctypes.data)
        return tokens, steps.reshape(B, n_canvases)

    def reset(self, req: int):
        binding.dllm_reset(self.h, req)

    def prefix_len(self, req: int) -> int:
        return binding.dllm_prefix_len(self.h, req)

    def check(self) -> int:
        return binding.dllm_check(self.h)

    def launch_count(self) -> int:
        return binding.dllm_launch_count(self.h)

    def set_debug(self, on: bool):
        binding.dllm_set_debug(self.h, on)

    def force_routing(self, idx):
        """idx: int [n_layers][T][k] experts for the next canvas passes, or None to stop."""
        if idx is None:
            binding.dllm_debug_force_routing(self.h, 0, 0)
            return
        a = np.ascontiguousarray(idx, dtype=np.int32)
        binding.dllm_debug_force_routing(self.h, a.ctypes.data, a.shape[1])

    def debug_read(self, what: int, layer: int, shape, dtype) -> np.ndarray:
        out = np.zeros(shape, dtype=dtype)
        binding.dllm_debug_read(self.h, what, layer, out.ctypes.data, out.nbytes)
        return out
