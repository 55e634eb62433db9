"""The allocation-free LM head (dllm_op_lm_head_conf_noalloc) against the allocating one.

For callers that cannot allocate device memory while they run, the library offers a
variant of the fused LM head whose scratch is a fixed array inside the library. This
test calls it through the C ABI twice in a row, on different shapes (so the second
call runs on scratch the first one left behind), and checks each result against
dllm_op_lm_head_conf on the same inputs, with the tolerances of the other LM-head tests:
argmax equal wherever the top-2 logit margin exceeds 1e-3, conf within 2e-2 relative.
It also checks that sizes beyond the scratch limit are refused. The file name sorts last
so that a run stopping at the first failure has run every other test before this one.
"""

import numpy as np
import pytest
import torch

from masked_block_diffusion_b200 import DllmError, binding, build
from synth import bf16_bits_to_f32, f32_to_bf16_bits, normal_f32, uniform_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build_all()
    binding.load()


def _dev_bf16(vals):
    return torch.from_numpy(f32_to_bf16_bits(vals.astype(np.float32)).view(np.int16)).cuda()


def _case(T, d, V, seed):
    y = bf16_bits_to_f32(f32_to_bf16_bits(uniform_f32(seed, 1, T * d, -2, 2))).reshape(T, d)
    head = bf16_bits_to_f32(f32_to_bf16_bits(normal_f32(seed, 2, V * d))).reshape(V, d)
    logits = (y.astype(np.float64) @ head.astype(np.float64).T).astype(np.float32).astype(np.float64)
    logits[:, V - 1] = -np.inf
    srt = np.sort(logits, axis=1)
    return _dev_bf16(y), _dev_bf16(head), srt[:, -1] - srt[:, -2]


def _run(fn, Y, H, T, d, V):
    conf = torch.full((T,), -1.0, dtype=torch.float32, device="cuda")
    arg = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    fn(Y.data_ptr(), H.data_ptr(), T, d, V, V - 1, conf.data_ptr(), arg.data_ptr(),
       torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return conf.cpu().numpy(), arg.cpu().numpy()


def test_noalloc_lm_head_matches_allocating_entry_point_twice():
    # full-size canvas rows of the 26B model, then a ragged, smaller second call
    for T, d, V, seed in ((256, 2816, 65536, 61), (130, 1024, 32768, 62)):
        Y, H, margin = _case(T, d, V, seed)
        ref_conf, ref_arg = _run(binding.dllm_op_lm_head_conf, Y, H, T, d, V)
        conf, arg = _run(binding.dllm_op_lm_head_conf_noalloc, Y, H, T, d, V)
        sel = margin > 1e-3
        assert np.array_equal(arg[sel], ref_arg[sel])
        assert np.all(np.abs(conf / ref_conf - 1.0) <= 2e-2)
        assert np.all(arg >= 0) and np.all(arg < V - 1)


def test_noalloc_lm_head_rejects_sizes_beyond_its_scratch():
    Y = torch.zeros((1025, 256), dtype=torch.int16, device="cuda")
    H = torch.zeros((1024, 256), dtype=torch.int16, device="cuda")
    conf = torch.zeros(1025, dtype=torch.float32, device="cuda")
    arg = torch.zeros(1025, dtype=torch.int32, device="cuda")
    with pytest.raises(DllmError) as e:
        binding.dllm_op_lm_head_conf_noalloc(Y.data_ptr(), H.data_ptr(), 1025, 256, 1024, 1023, conf.data_ptr(),
                                             arg.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert e.value.code == binding.DLLM_E_INVAL


_FRESH_SCRIPT = """
import sys
sys.path.insert(0, {root!r})
import numpy as np
import torch
from masked_block_diffusion_b200 import binding
from synth import bf16_bits_to_f32, f32_to_bf16_bits, normal_f32, uniform_f32
T, d, V = 256, 1024, 32768
y = bf16_bits_to_f32(f32_to_bf16_bits(uniform_f32(63, 1, T * d, -2, 2))).reshape(T, d)
hd = bf16_bits_to_f32(f32_to_bf16_bits(normal_f32(63, 2, V * d))).reshape(V, d)
Y = torch.from_numpy(f32_to_bf16_bits(y).view(np.int16)).cuda()
H = torch.from_numpy(f32_to_bf16_bits(hd).view(np.int16)).cuda()
s = torch.cuda.current_stream().cuda_stream
out = []
# the library's first calls on this device are the allocation-free ones
for fn in (binding.dllm_op_lm_head_conf_noalloc, binding.dllm_op_lm_head_conf_noalloc, binding.dllm_op_lm_head_conf):
    conf = torch.full((T,), -1.0, dtype=torch.float32, device="cuda")
    arg = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    fn(Y.data_ptr(), H.data_ptr(), T, d, V, V - 1, conf.data_ptr(), arg.data_ptr(), s)
    torch.cuda.synchronize()
    out.append((conf.cpu().numpy(), arg.cpu().numpy()))
np.savez({path!r}, c0=out[0][0], a0=out[0][1], c1=out[1][0], a1=out[1][1], c2=out[2][0], a2=out[2][1])
print("OK")
"""


def test_noalloc_lm_head_as_the_first_call_in_a_fresh_process(tmp_path):
    """In a new process the allocation-free entry point is the library's first call on
    the device (it looks up its scratch array there itself); two such calls in a row
    agree with the allocating entry point made afterwards."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    path = str(tmp_path / "fresh.npz")
    r = subprocess.run([sys.executable, "-c", _FRESH_SCRIPT.format(root=root, path=path)], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "OK" in r.stdout, r.stderr[-3000:]
    z = np.load(path)
    T, d, V = 256, 1024, 32768
    _, _, margin = _case(T, d, V, 63)
    sel = margin > 1e-3
    for i in (0, 1):
        assert np.array_equal(z[f"a{i}"][sel], z["a2"][sel])
        assert np.all(np.abs(z[f"c{i}"] / z["c2"] - 1.0) <= 2e-2)
        assert np.all(z[f"a{i}"] >= 0) and np.all(z[f"a{i}"] < V - 1)
