"""Error paths of the C ABI on the GPU: the documented codes, and the timeout path.

- DLLM_E_STATE: a canvas pass on a slot that has no prefill;
- DLLM_E_CTX_FULL: a prompt that leaves no room for a canvas, and a canvas pass once
  appended canvases have filled the KV cache;
- DLLM_E_BUDGET: a threshold no confidence reaches, with the step-budget floor off;
- DLLM_E_INVAL: a policy the sampler does not know;
- DLLM_E_TIMEOUT: every pipeline wait of the kernels limited to 1 ns, so that waits
  give up. The passes then commit nothing and report -1 / NaN, the synchronising calls
  return DLLM_E_TIMEOUT, and with the default limit back the next pass on the same
  handle matches the oracle again (the context stays usable). No kernel faults, traps
  or hangs: a wait that runs out returns and the kernel exits through its drain path.
"""

import numpy as np
import pytest
import torch

from masked_block_diffusion_b200 import Denoiser, DllmError, binding, make_policy
from oracle import Policy
from parity_util import build_pair, compare_trace
from synth import WORKLOADS, blob_from_weights, gen_weights, prompt_tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    cfg = WORKLOADS["c1-tiny-dense"].model
    return cfg, blob_from_weights(cfg, gen_weights(cfg))


def _canvas(cfg, B=1):
    C = cfg.canvas
    cv = torch.full((B, C), cfg.mask_id, dtype=torch.int32, device="cuda")
    mk = torch.ones((B, C), dtype=torch.uint8, device="cuda")
    return cv, mk


def test_denoise_before_prefill_is_a_state_error(tiny):
    cfg, blob = tiny
    den = Denoiser(cfg, blob, max_ctx=256, max_batch=2)
    try:
        den.prefill(0, prompt_tokens(cfg.vocab, 2100, 64))
        cv, mk = _canvas(cfg, 2)            # slot 1 has no prefill
        with pytest.raises(DllmError) as e:
            den.denoise_step(cv, mk, make_policy("topk", 4), 0, 8)
        assert e.value.code == binding.DLLM_E_STATE
        code, _, _ = den.generate_block(2, 8, make_policy("topk", 4))
        assert code == binding.DLLM_E_STATE
        den.reset(0)                         # a reset slot needs a new prefill too
        with pytest.raises(DllmError) as e:
            den.denoise_step(*_canvas(cfg, 1), make_policy("topk", 4), 0, 8)
        assert e.value.code == binding.DLLM_E_STATE
    finally:
        den.close()


def test_kv_cache_capacity_errors(tiny):
    cfg, blob = tiny
    C = cfg.canvas
    den = Denoiser(cfg, blob, max_ctx=64 + 2 * C, max_batch=1)
    try:
        with pytest.raises(DllmError) as e:   # prompt + one canvas exceed max_ctx
            den.prefill(0, prompt_tokens(cfg.vocab, 2100, 64 + C + 1))
        assert e.value.code == binding.DLLM_E_CTX_FULL
        den.prefill(0, prompt_tokens(cfg.vocab, 2100, 64))
        pol = make_policy("topk", 4)
        assert den.generate_block(1, 8, pol)[0] == 0
        den.append_kv(1)                     # prefix 64 + 32: one more canvas fits
        assert den.prefix_len(0) == 64 + C
        assert den.generate_block(1, 8, pol)[0] == 0
        den.append_kv(1)                     # prefix 64 + 64 = max_ctx - 0: no room left
        assert den.prefix_len(0) == 64 + 2 * C
        with pytest.raises(DllmError) as e:
            den.denoise_step(*_canvas(cfg), pol, 0, 8)
        assert e.value.code == binding.DLLM_E_CTX_FULL
        assert den.generate_block(1, 8, pol)[0] == binding.DLLM_E_CTX_FULL
        with pytest.raises(DllmError) as e:
            den.append_kv(1)
        assert e.value.code == binding.DLLM_E_CTX_FULL
    finally:
        den.close()


def test_step_budget_and_policy_errors(tiny):
    cfg, blob = tiny
    den = Denoiser(cfg, blob, max_ctx=256, max_batch=1)
    try:
        den.prefill(0, prompt_tokens(cfg.vocab, 2100, 64))
        # no confidence exceeds +inf and the floor is off: nothing is ever committed
        never = make_policy("threshold", 0, float("inf"), floor=False)
        code, out, steps = den.generate_block(1, 5, never)
        assert code == binding.DLLM_E_BUDGET
        assert steps == [5]
        assert np.all(out.cpu().numpy() == cfg.mask_id)
        bad = binding.dllm_policy(kind=7, k=1, tau=0.5, floor=1)
        with pytest.raises(DllmError) as e:
            den.denoise_step(*_canvas(cfg), bad, 0, 8)
        assert e.value.code == binding.DLLM_E_INVAL
        with pytest.raises(DllmError) as e:
            den.denoise_step(*_canvas(cfg), make_policy("topk", 0), 0, 8)
        assert e.value.code == binding.DLLM_E_INVAL
        assert den.check() == 0              # host-side refusals leave no device error
        assert den.generate_block(1, 8, make_policy("topk", 4))[0] == 0
    finally:
        den.close()


def test_timeout_path_reports_and_keeps_the_context_usable():
    w = WORKLOADS["c2-small-moe"]
    cfg = w.model.with_layers(2)
    C = cfg.canvas
    pol = Policy("topk", k=32)
    orc, den, _ = build_pair(cfg, 512, w.prompt_seed + 11, 512 + 2 * C)
    try:
        binding.dllm_set_wait_limit(den.h, 1)
        try:
            code, _, steps = den.generate_block(1, 8, make_policy("topk", 32))
            assert code == binding.DLLM_E_TIMEOUT, code
            assert steps[0] <= 8
            # a single pass: queued without error, its outputs say it gave up
            cv, mk = _canvas(cfg)
            conf, arg, rem = den.denoise_step(cv, mk, make_policy("topk", 32), 0, 8)
            assert int(rem.cpu()[0]) == -1
            assert np.all(np.isnan(conf.cpu().numpy())) and np.all(arg.cpu().numpy() == -1)
            assert np.all(mk.cpu().numpy() == 1)          # nothing committed
            assert den.check() == binding.DLLM_E_TIMEOUT
            assert den.check() == 0                       # reported once, then cleared
        finally:
            binding.dllm_set_wait_limit(den.h, 0)
        # the same handle, default limit: the next passes match the oracle again
        _, _, trace = orc.generate_block(0, pol, 8, trace=True)
        compare_trace(cfg, trace[:2], den, pol, 8)
        assert den.check() == 0
    finally:
        den.close()


def test_single_ops_poison_their_outputs_on_timeout():
    # a wait first suspends for up to 256 ns before the limit counts, so the shapes are
    # large enough (44 k blocks per tile) that some wait of each launch takes longer
    from synth import bf16_bits_to_f32, f32_to_bf16_bits, normal_f32, uniform_f32
    T, d, V = 64, 2816, 4096
    y = bf16_bits_to_f32(f32_to_bf16_bits(uniform_f32(5, 1, T * d, -2, 2)))
    hd = bf16_bits_to_f32(f32_to_bf16_bits(normal_f32(5, 2, V * d)))
    Y = torch.from_numpy(f32_to_bf16_bits(y).view(np.int16)).cuda()
    H = torch.from_numpy(f32_to_bf16_bits(hd).view(np.int16)).cuda()
    cfg = WORKLOADS["c1-tiny-dense"].model
    den = Denoiser(cfg, blob_from_weights(cfg, gen_weights(cfg)), max_ctx=256, max_batch=1)
    s = torch.cuda.current_stream().cuda_stream
    try:
        binding.dllm_set_wait_limit(den.h, 1)
        try:
            for fn in (binding.dllm_op_lm_head_conf, binding.dllm_op_lm_head_conf_noalloc):
                conf = torch.zeros(T, dtype=torch.float32, device="cuda")
                arg = torch.zeros(T, dtype=torch.int32, device="cuda")
                fn(Y.data_ptr(), H.data_ptr(), T, d, V, V - 1, conf.data_ptr(), arg.data_ptr(), s)
                torch.cuda.synchronize()
                assert np.all(np.isnan(conf.cpu().numpy())) and np.all(arg.cpu().numpy() == -1)
            D = torch.zeros((T, V), dtype=torch.float32, device="cuda")
            binding.dllm_op_gemm_bf16(Y.data_ptr(), H.data_ptr(), D.data_ptr(), T, V, d, s)
            torch.cuda.synchronize()
            assert torch.isnan(D).all()
        finally:
            binding.dllm_set_wait_limit(den.h, 0)
        conf = torch.zeros(T, dtype=torch.float32, device="cuda")
        arg = torch.zeros(T, dtype=torch.int32, device="cuda")
        binding.dllm_op_lm_head_conf(Y.data_ptr(), H.data_ptr(), T, d, V, V - 1, conf.data_ptr(), arg.data_ptr(), s)
        torch.cuda.synchronize()
        assert np.all(np.isfinite(conf.cpu().numpy())) and np.all(arg.cpu().numpy() >= 0)
    finally:
        den.close()
