"""Device-side generation of the synthetic weight blob (libsynth.so).

The blob of the 26B-parameter configuration is 48 GB; generating it on the host would
take minutes, so the device filler writes each tensor in place with the same integer
recipe as synth.gen (bit-identical values).
"""

from __future__ import annotations

import ctypes
import os

from .configs import ModelConfig
from .gen import blob_bytes, blob_layout, elem_bytes

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsynth.so")
_lib = None


def load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; run `python -m masked_block_diffusion_b200.build`")
        _lib = ctypes.CDLL(LIB_PATH)
        _lib.synth_fill.restype = ctypes.c_int
        _lib.synth_fill.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    return _lib


def fill_tensor(dst_ptr: int, numel: int, seed: int, tid: int, ones: bool, bf16: bool, stream_ptr: int = 0):
    r = load().synth_fill(ctypes.c_void_p(dst_ptr), numel, seed, tid, 1 if ones else 0, 1 if bf16 else 0,
                          ctypes.c_void_p(stream_ptr))
    if r != 0:
        raise RuntimeError(f"synth_fill failed with CUDA error {r}")


def device_blob(cfg: ModelConfig, seed: int | None = None):
    """The weight blob as a uint8 CUDA tensor (same bytes as synth.gen.gen_blob)."""
    import torch
    seed = cfg.weight_seed if seed is None else seed
    buf = torch.zeros(blob_bytes(cfg), dtype=torch.uint8, device="cuda")
    base = buf.data_ptr()
    bf16 = elem_bytes(cfg) == 2
    stream = torch.cuda.current_stream().cuda_stream
    for ent in blob_layout(cfg):
        fill_tensor(base + ent.offset, ent.numel, seed, ent.spec.tid, ent.spec.kind == "ones", bf16, stream)
    torch.cuda.synchronize()
    return buf
