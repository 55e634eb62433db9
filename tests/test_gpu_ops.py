"""GPU checks of single operations through the C ABI: the tcgen05 GEMM core and the
fused LM head, against the oracle and plain fp32/fp64 references."""

import numpy as np
import pytest
import torch

from masked_block_diffusion_b200 import binding, build
from synth import bf16_bits_to_f32, f32_to_bf16_bits, normal_f32, uniform_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build_all()
    binding.load()


def dev_bf16(vals: np.ndarray) -> torch.Tensor:
    bits = f32_to_bf16_bits(vals.astype(np.float32))
    return torch.from_numpy(bits.view(np.int16)).cuda()


@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (256, 384, 512), (200, 256, 2816), (1, 128, 128),
                                   (1000, 640, 1024)])
def test_gemm_core_matches_fp64(M, N, K):
    a = uniform_f32(31, 1, M * K).reshape(M, K)
    b = uniform_f32(31, 2, N * K).reshape(N, K)
    ab = bf16_bits_to_f32(f32_to_bf16_bits(a)).astype(np.float64)
    bb = bf16_bits_to_f32(f32_to_bf16_bits(b)).astype(np.float64)
    ref = ab @ bb.T
    A, B = dev_bf16(a), dev_bf16(b)
    D = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    binding.dllm_op_gemm_bf16(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, K, s)
    torch.cuda.synchronize()
    got = D.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


def test_device_weight_filler_matches_numpy():
    from synth import device
    n = 1 << 20
    for bf16 in (True, False):
        buf = torch.zeros(n * (2 if bf16 else 4), dtype=torch.uint8, device="cuda")
        device.fill_tensor(buf.data_ptr(), n, 1003, 17, False, bf16)
        torch.cuda.synchronize()
        got = buf.cpu().numpy()
        ref = normal_f32(1003, 17, n)
        if bf16:
            assert np.array_equal(got.view(np.uint16), f32_to_bf16_bits(ref))
        else:
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def _lm_head_case(T, d, V, seed, rows=None):
    y = bf16_bits_to_f32(f32_to_bf16_bits(uniform_f32(seed, 1, T * d, -2, 2))).reshape(T, d)
    head = bf16_bits_to_f32(f32_to_bf16_bits(normal_f32(seed, 2, V * d))).reshape(V, d)
    Y, Hd = dev_bf16(y), dev_bf16(head)
    conf = torch.zeros(T, dtype=torch.float32, device="cuda")
    arg = torch.zeros(T, dtype=torch.int32, device="cuda")
    binding.dllm_op_lm_head_conf(Y.data_ptr(), Hd.data_ptr(), T, d, V, V - 1, conf.data_ptr(), arg.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    conf, arg = conf.cpu().numpy(), arg.cpu().numpy()
    rows = np.arange(T) if rows is None else rows
    # the definition on the sampled rows: fp32 logits, [MASK] excluded, first maximum,
    # conf = 1 / sum exp(l - max), in fp64 from the same bf16 operands
    yr = y[rows].astype(np.float64)
    ref_logits = yr @ head.astype(np.float64).T
    ref_logits = ref_logits.astype(np.float32).astype(np.float64)
    ref_logits[:, V - 1] = -np.inf
    m = ref_logits.max(axis=1)
    ref_arg = ref_logits.argmax(axis=1)
    ref_conf = 1.0 / np.exp(ref_logits - m[:, None]).sum(axis=1)
    srt = np.sort(ref_logits, axis=1)
    margin = srt[:, -1] - srt[:, -2]
    return conf[rows], arg[rows], ref_conf, ref_arg, margin


@pytest.mark.parametrize("T,d,V", [(32, 256, 1024), (130, 1024, 32768)])
def test_lm_head_conf_small(T, d, V):
    conf, arg, rc, ra, margin = _lm_head_case(T, d, V, seed=41)
    sel = margin > 1e-3
    assert sel.mean() > 0.9
    assert np.array_equal(arg[sel], ra[sel])
    assert np.all(np.abs(conf / rc - 1) < 2e-2)


def test_lm_head_conf_full_size_sampled():
    # full vocabulary and width of the 26B configuration, 256 canvas rows; 16 sampled rows
    T, d, V = 256, 2816, 65536
    rows = np.arange(0, T, 16)
    conf, arg, rc, ra, margin = _lm_head_case(T, d, V, seed=43, rows=rows)
    sel = margin > 1e-3
    assert np.array_equal(arg[sel], ra[sel])
    assert np.all(np.abs(conf / rc - 1) < 2e-2)


def test_fp8_block_quantiser_matches_the_oracle_bit_for_bit():
    """dllm_op_quantize_fp8 (the quantiser dllm_create applies to expert matrices) against
    the oracle's definition: the same tile exponents and the same E4M3 codes, on a matrix
    whose tiles have ragged edges, a large outlier and an all-zero tile."""
    import oracle.model as om
    rows, cols = 300, 400
    w = (uniform_f32(47, 1, rows * cols, -1, 1) * np.float32(0.05)).reshape(rows, cols)
    w[140, 7] = 2.5
    w[256:, 384:] = 0.0
    w = bf16_bits_to_f32(f32_to_bf16_bits(w))
    W = dev_bf16(w)
    q = torch.zeros((rows, cols), dtype=torch.uint8, device="cuda")
    ex = torch.zeros((3, 4), dtype=torch.int8, device="cuda")
    binding.dllm_op_quantize_fp8(W.data_ptr(), rows, cols, q.data_ptr(), ex.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ex_ref = om.fp8_block_exponents(w.astype(np.float64))
    assert np.array_equal(ex.cpu().numpy().astype(np.int64), ex_ref)
    codes = q.cpu().numpy()
    vals = om.e4m3_values()
    mag = vals[codes & 0x7F]
    sign = np.where(codes & 0x80, -1.0, 1.0)
    s = np.ldexp(1.0, np.repeat(np.repeat(ex_ref, 128, 0), 128, 1)[:rows, :cols])
    assert np.all((codes & 0x7F) != 0x7F)                       # no NaN code
    assert np.array_equal(sign * mag * s, om.fp8_block_dequant(w.astype(np.float64)).astype(np.float64))
