"""The C-ABI library builds for sm_100a, loads and exports every declared symbol (no GPU needed)."""

import ctypes
import os
import re
import subprocess

import pytest

from masked_block_diffusion_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "dllm.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dllm_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib_path():
    return build.build_dllm()


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(binding.EXPORTS)


def test_binding_constants_match_header_defines():
    """Every integer #define of the header that the binding also names has the same value."""
    text = open(os.path.join(ROOT, "include", "dllm.h")).read()
    defines = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define\s+(DLLM_\w+)\s+\(?(-?\d+)\)?", text)}
    shared = [n for n in defines if hasattr(binding, n)]
    assert len(shared) >= 10, shared
    for n in shared:
        assert getattr(binding, n) == defines[n], n
    assert "DLLM_TIMING_STRIDE_SHIFT" in shared and "DLLM_E_OOM" in shared


def test_library_exports_every_declared_symbol(lib_path):
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\b(dllm_\w+)\b", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing


def test_library_loads_without_gpu(lib_path):
    lib = binding.load(lib_path)
    for s in declared_symbols():
        assert hasattr(lib, s)
    # argument validation runs on the host: no device work is queued
    assert lib.dllm_create(None, None, 0, 0, None, None) == binding.DLLM_E_INVAL
    assert lib.dllm_op_gemm_bf16(None, None, None, 0, 0, 0, None) == binding.DLLM_E_INVAL
    assert lib.dllm_launch_count(None) == -1


def test_config_validation_rejects_unsupported_shapes(lib_path):
    lib = binding.load(lib_path)
    from synth import CONFIGS
    cfg = binding.make_config(CONFIGS["tiny-dense"], max_ctx=256, max_batch=1)
    cfg.head_dim = 80                      # not a supported head size
    h = ctypes.c_void_p()
    dummy = (ctypes.c_uint8 * 16)()
    assert lib.dllm_create(ctypes.byref(cfg), dummy, 16, 0, None, ctypes.byref(h)) == binding.DLLM_E_INVAL
    assert not h.value
